"""Plain fp64 CPU oracle of the MS-GLA layer forward pass.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module. The product (the CUDA library and its binding) never calls it, and it
shares no code with the product: it depends on numpy alone.

What it computes follows "MS-GLA: Multi-Scale Gated Linear Attention" as
summarised in the MS-GLA reading notes (arXiv 2609.35664v1):

* Sec. 2.1 (the paper's Eqs. (2), (5), (6)): the GLA recurrence in row-vector
  form, S_t = Diag(alpha_t) S_{t-1} + k_t^T v_t and o_t = q_t S_t, with
  q_t, k_t in R^{1 x d_k}, v_t in R^{1 x d_v}, S_t in R^{d_k x d_v}; alpha_t in
  (0,1)^{d_k} comes from a low-rank projection of the hidden state followed by
  a sigmoid-type map.
* Sec. 3.1, Eq. (8): non-overlapping mean pooling over s adjacent rows, pooled
  length ceil(L/s), each block averaged over its valid rows (token mask M, 1 =
  valid, 0 = padding; rows past L count as padding; the denominator is clamped
  to at least 1, so an all-padding block pools to zero). Without a mask every
  row inside L is valid. The formula is applied at every scale, s = 1 included,
  where it zeroes padded rows.
* Sec. 3.2, Eq. (9): the H heads are split over the scales (sum_s h_s = H);
  each branch has its own q/k/v/gate/output projections.
* Sec. 3.3: causal hold -- each coarse output is repeated s times and shifted
  right by s-1 with zero fill, i.e. position t reads pooled row
  floor((t+1)/s) - 1, or zero when that index is negative.
* Sec. 3.3, Eqs. (10)-(11): w_t = softmax(W_fuse x_t + b_fuse) from the
  unpooled row x_t, and O_t = sum_s w_{t,s} Yhat^(s)_t.
* token-by-token inference (the notes' item on training and per-token
  inference, after the authors' cache): each branch keeps its GLA state, the
  tokens of its unfinished block and its latest output; a branch steps once
  its block is full and otherwise repeats its latest output.

Readings where the notes leave a step open (each is also listed in the design
notes of this repository):
* gate form: log alpha = logsigmoid(g W_g2^T + b_g) / gate_normalizer with
  g = xbar W_g1^T of rank r (the notes only say "low-rank + sigmoid-like");
* output projection before the hold (the two orders are identical: the hold
  is a row gather);
* o_t = qk_scale * q_t S_t with qk_scale = 1 by default (the notes' equation
  has no scale);
* per-branch normalisation (Sec. 3.2 lists one per branch without defining
  it): off by default; when asked for, an RMS normalisation of each head's GLA
  output row before the output projection, o_h / sqrt(mean(o_h^2) + eps) times a
  per-channel weight (``head_rmsnorm``). No output gate;
* the mask enters the pooling only: the fusion weights of Eq. (10) read the
  unpooled row x_t whatever its mask.

Every step is written token by token or row by row; numpy's matmul is used as
a library primitive for the per-row projections only (and, in the gradients,
for their transposed products: dW = dYᵀ X and dX = dY W).

Parity pins (tests/test_oracle.py): brute-force quadratic form of the GLA
recurrence, alpha = 1 reducing to causal (Q K^T) V, the single-scale layer
reducing to plain GLA + W_o, the constant-input geometric closed form, the
worked s = 4 hold table and pooling example of Sec. 3.1/3.3, a masked s = 4
pooling example with an all-padding block, unit RMS per head and invariance to
the value scale of the optional head normalisation, causality,
half-life, the 11/16 update count and the simplex property of the fusion
weights. The gradients (``layer_backward``, for a backward pass that has no
GPU counterpart yet) are pinned by central finite differences of the forward.
"""
from __future__ import annotations

import numpy as np


# ---------------------------------------------------------------------------
# Sec. 3.1, Eq. (8): non-overlapping mean pooling with the valid-token mask M
# ---------------------------------------------------------------------------
def pool(X: np.ndarray, s: int, M: np.ndarray | None = None) -> np.ndarray:
    """Eq. (8): block i of s consecutive rows of X [L, d] -> [ceil(L/s), d].

    X_i = sum_j X_{is+j} M_{is+j} / max(1, sum_j M_{is+j}) over the rows j of the
    block that lie inside L (right padding past L counts as M = 0). Without a mask,
    M = 1 for every row inside L: the incomplete tail block is the mean of its
    valid rows.
    """
    L = X.shape[0]
    if M is None:
        M = np.ones(L)
    n = -(-L // s)
    out = np.zeros((n, X.shape[1]), dtype=np.float64)
    for i in range(n):
        rows = [i * s + j for j in range(s) if i * s + j < L]
        acc = np.zeros(X.shape[1], dtype=np.float64)
        cnt = 0.0
        for r in rows:
            acc += X[r] * M[r]
            cnt += M[r]
        out[i] = acc / max(1.0, cnt)
    return out


# ---------------------------------------------------------------------------
# Sec. 2.1 gate: low-rank projection + sigmoid-type map (form fixed above)
# ---------------------------------------------------------------------------
def logsigmoid(z: np.ndarray) -> np.ndarray:
    """log(1 / (1 + exp(-z))) evaluated without overflow."""
    return -np.logaddexp(0.0, -z)


def branch_projections(Xp: np.ndarray, br: dict, gate_normalizer: float):
    """q, k, v and log alpha of one branch from its pooled rows Xp [n, d].

    q = Xp W_q^T, k = Xp W_k^T, v = Xp W_v^T (heads side by side along the
    feature axis), log alpha = logsigmoid((Xp W_g1^T) W_g2^T + b_g) / normalizer.
    """
    q = Xp @ br["Wq"].T
    k = Xp @ br["Wk"].T
    v = Xp @ br["Wv"].T
    g = Xp @ br["Wg1"].T
    log_alpha = logsigmoid(g @ br["Wg2"].T + br["bg"]) / gate_normalizer
    return q, k, v, log_alpha


# ---------------------------------------------------------------------------
# Sec. 2.1: GLA recurrence, one head, token by token
# ---------------------------------------------------------------------------
def gla_recurrent(q: np.ndarray, k: np.ndarray, v: np.ndarray, log_alpha: np.ndarray,
                  qk_scale: float = 1.0, counter: list | None = None) -> np.ndarray:
    """S_0 = 0; for each step t: S_t = Diag(alpha_t) S_{t-1} + k_t^T v_t and
    o_t = qk_scale * q_t S_t. q, k, log_alpha are [n, d_k]; v is [n, d_v]."""
    n, dk = q.shape
    dv = v.shape[1]
    S = np.zeros((dk, dv), dtype=np.float64)
    o = np.zeros((n, dv), dtype=np.float64)
    alpha = np.exp(log_alpha)
    for t in range(n):
        S = alpha[t][:, None] * S + np.outer(k[t], v[t])
        o[t] = qk_scale * (q[t] @ S)
        if counter is not None:
            counter[0] += 1
    return o


# ---------------------------------------------------------------------------
# Sec. 3.2: per-branch normalisation (optional, read as a per-head RMS norm)
# ---------------------------------------------------------------------------
def head_rmsnorm(o: np.ndarray, weight: np.ndarray, eps: float) -> np.ndarray:
    """One head's output rows o [n, d_v]: each row divided by its root mean
    square over the head's d_v channels (with eps inside the root), then
    multiplied channel-wise by ``weight`` [d_v]."""
    out = np.zeros_like(o)
    for t in range(o.shape[0]):
        ms = float(np.dot(o[t], o[t])) / o.shape[1]
        out[t] = o[t] / np.sqrt(ms + eps) * weight
    return out


# ---------------------------------------------------------------------------
# Sec. 3.3: causal hold (repeat s times, shift right by s-1, zero fill)
# ---------------------------------------------------------------------------
def hold_index(t: int, s: int) -> int:
    """Pooled row read at original position t, or -1 for the zero fill."""
    return (t + 1) // s - 1


def hold(Y: np.ndarray, s: int, L: int) -> np.ndarray:
    """Yhat [L, d] from the pooled branch output Y [ceil(L/s), d]."""
    out = np.zeros((L, Y.shape[1]), dtype=np.float64)
    for t in range(L):
        i = hold_index(t, s)
        if i >= 0:
            out[t] = Y[i]
    return out


# ---------------------------------------------------------------------------
# Sec. 3.3, Eqs. (10)-(11): input-dependent fusion
# ---------------------------------------------------------------------------
def fusion_weights(X: np.ndarray, Wfuse: np.ndarray, bfuse: np.ndarray) -> np.ndarray:
    """w_t = softmax(W_fuse x_t + b_fuse) for every row of X [L, d]."""
    z = X @ Wfuse.T + bfuse
    z = z - z.max(axis=1, keepdims=True)
    e = np.exp(z)
    return e / e.sum(axis=1, keepdims=True)


# ---------------------------------------------------------------------------
# whole layer
# ---------------------------------------------------------------------------
def layer_forward(X: np.ndarray, weights: dict, scales, heads, d_k: int, d_v: int,
                  gate_normalizer: float = 16.0, qk_scale: float = 1.0,
                  intermediates: bool = False, counter: list | None = None,
                  mask: np.ndarray | None = None, head_norm_eps: float | None = None):
    """MS-GLA layer forward for X [B, L, d] (float64).

    ``mask`` [B, L] (1 = valid token, 0 = padding) enters only the pooling of
    Eq. (8); without it every row inside L is valid. ``head_norm_eps`` (None =
    off) turns on the per-head RMS normalisation of the GLA output with the
    branch's ``norm_w`` [h*d_v] (all ones when absent).

    ``weights`` holds ``branches`` (per scale: Wq, Wk, Wv, Wg1, Wg2, bg, Wo)
    and ``Wfuse``, ``bfuse``. Returns O [B, L, d]; with ``intermediates`` also a
    dict of per-branch pooled rows, q, k, v, log alpha, o and Y plus the fusion
    weights w, each with a leading batch axis.
    """
    X = np.asarray(X, dtype=np.float64)
    B, L, d = X.shape
    assert len(scales) == len(heads) == len(weights["branches"])
    O = np.zeros((B, L, d), dtype=np.float64)
    inter = {"w": [], "branches": [dict(Xp=[], q=[], k=[], v=[], log_alpha=[], o=[], Y=[])
                                   for _ in scales]}
    for b in range(B):
        w = fusion_weights(X[b], weights["Wfuse"], weights["bfuse"])
        inter["w"].append(w)
        for j, (s, h) in enumerate(zip(scales, heads)):
            br = weights["branches"][j]
            Xp = pool(X[b], s, None if mask is None else np.asarray(mask[b], dtype=np.float64))
            q, k, v, la = branch_projections(Xp, br, gate_normalizer)
            o = np.zeros((Xp.shape[0], h * d_v), dtype=np.float64)
            for hh in range(h):
                ck, cv = slice(hh * d_k, (hh + 1) * d_k), slice(hh * d_v, (hh + 1) * d_v)
                o[:, cv] = gla_recurrent(q[:, ck], k[:, ck], v[:, cv], la[:, ck],
                                         qk_scale=qk_scale, counter=counter)
                if head_norm_eps is not None:
                    nw = br.get("norm_w")
                    nw = np.ones(h * d_v) if nw is None else nw
                    o[:, cv] = head_rmsnorm(o[:, cv], nw[cv], head_norm_eps)
            Y = o @ br["Wo"].T
            O[b] += w[:, j:j + 1] * hold(Y, s, L)
            if intermediates:
                for name, val in (("Xp", Xp), ("q", q), ("k", k), ("v", v),
                                  ("log_alpha", la), ("o", o), ("Y", Y)):
                    inter["branches"][j][name].append(val)
    if not intermediates:
        return O
    inter["w"] = np.stack(inter["w"])
    for br in inter["branches"]:
        for name in list(br):
            br[name] = np.stack(br[name]) if br[name] else None
    return O, inter


# ---------------------------------------------------------------------------
# gradients (the backward pass of training; pinned by finite differences)
# ---------------------------------------------------------------------------
def gla_recurrent_backward(q: np.ndarray, k: np.ndarray, v: np.ndarray, log_alpha: np.ndarray,
                           do: np.ndarray, qk_scale: float = 1.0):
    """Adjoints of ``gla_recurrent`` for the output adjoint do [n, d_v]:
    returns dq, dk, dv, dlog_alpha.

    The forward keeps every state S_t. Walking back from the last step, G holds
    the adjoint of S_t: G_t = qk_scale q_t^T do_t + Diag(alpha_{t+1}) G_{t+1}.
    Then dq_t = qk_scale S_t do_t^T, dk_t = G_t v_t^T, dv_t = k_t G_t, and
    d alpha_t = rowsum(G_t * S_{t-1}) (elementwise), d log alpha_t = alpha_t *
    d alpha_t."""
    n, dk_ = q.shape
    dv_ = v.shape[1]
    alpha = np.exp(log_alpha)
    S = np.zeros((n + 1, dk_, dv_), dtype=np.float64)
    for t in range(n):
        S[t + 1] = alpha[t][:, None] * S[t] + np.outer(k[t], v[t])
    dq = np.zeros_like(q, dtype=np.float64)
    dkk = np.zeros_like(k, dtype=np.float64)
    dvv = np.zeros_like(v, dtype=np.float64)
    dla = np.zeros_like(log_alpha, dtype=np.float64)
    G = np.zeros((dk_, dv_), dtype=np.float64)
    for t in range(n - 1, -1, -1):
        G = G + qk_scale * np.outer(q[t], do[t])
        dq[t] = qk_scale * (S[t + 1] @ do[t])
        dkk[t] = G @ v[t]
        dvv[t] = k[t] @ G
        dla[t] = alpha[t] * (G * S[t]).sum(axis=1)
        G = alpha[t][:, None] * G
    return dq, dkk, dvv, dla


def _norm_weight(br: dict, h: int, d_v: int) -> np.ndarray:
    """The branch's per-channel head-norm weight [h*d_v] (all ones when absent)."""
    nw = br.get("norm_w")
    return np.ones(h * d_v) if nw is None else np.asarray(nw, dtype=np.float64)


def head_rmsnorm_backward(o: np.ndarray, weight: np.ndarray, eps: float, dy: np.ndarray):
    """Adjoints of ``head_rmsnorm`` for dy [n, d_v]: returns do and dweight.
    With r_t = sqrt(mean(o_t^2) + eps) and y_t = o_t / r_t * weight:
    do_t = (dy_t * weight) / r_t - o_t * sum(dy_t * weight * o_t) / (d_v r_t^3),
    dweight = sum_t dy_t * o_t / r_t."""
    n, dv_ = o.shape
    do = np.zeros_like(o, dtype=np.float64)
    dweight = np.zeros_like(weight, dtype=np.float64)
    for t in range(n):
        r = np.sqrt(float(np.dot(o[t], o[t])) / dv_ + eps)
        gw = dy[t] * weight
        do[t] = gw / r - o[t] * float(np.dot(gw, o[t])) / (dv_ * r ** 3)
        dweight += dy[t] * o[t] / r
    return do, dweight


def layer_backward(X: np.ndarray, weights: dict, scales, heads, d_k: int, d_v: int, dO: np.ndarray,
                   gate_normalizer: float = 16.0, qk_scale: float = 1.0, mask: np.ndarray | None = None,
                   head_norm_eps: float | None = None):
    """Gradients of sum(O * dO), O = layer_forward(X, ...) with the same
    arguments: returns dX [B, L, d] and a dict shaped like ``weights``
    (``branches`` with Wq, Wk, Wv, Wg1, Wg2, bg, Wo each, and norm_w when the
    per-head norm is on; ``Wfuse``, ``bfuse``).

    The steps of the forward in reverse: the fusion softmax (dz = w * (dw -
    sum_s w_s dw_s) with dw_{t,s} = dO_t . Yhat^(s)_t), the causal hold (dY_i
    sums dYhat_t over the positions t that read row i), W_o, the GLA recurrence
    per head (gla_recurrent_backward), the gate (d/du logsigmoid(u) =
    sigmoid(-u)), the projections, and the pooling of Eq. (8) (each valid row of
    block i receives dXbar_i / max(1, sum M)); with the per-head norm, its
    adjoint (head_rmsnorm_backward) sits between W_o and the recurrence."""
    X = np.asarray(X, dtype=np.float64)
    dO = np.asarray(dO, dtype=np.float64)
    B, L, d = X.shape
    names = ("Wq", "Wk", "Wv", "Wg1", "Wg2", "bg", "Wo")
    grads = {"branches": [{n_: np.zeros_like(np.asarray(br[n_], dtype=np.float64)) for n_ in names}
                          for br in weights["branches"]],
             "Wfuse": np.zeros_like(np.asarray(weights["Wfuse"], dtype=np.float64)),
             "bfuse": np.zeros_like(np.asarray(weights["bfuse"], dtype=np.float64))}
    dX = np.zeros_like(X)
    for b in range(B):
        M = None if mask is None else np.asarray(mask[b], dtype=np.float64)
        w = fusion_weights(X[b], weights["Wfuse"], weights["bfuse"])
        fwd = []
        for j, (s, h) in enumerate(zip(scales, heads)):
            br = weights["branches"][j]
            Xp = pool(X[b], s, M)
            q, k, v, la = branch_projections(Xp, br, gate_normalizer)
            o_raw = np.zeros((Xp.shape[0], h * d_v), dtype=np.float64)
            for hh in range(h):
                ck, cv = slice(hh * d_k, (hh + 1) * d_k), slice(hh * d_v, (hh + 1) * d_v)
                o_raw[:, cv] = gla_recurrent(q[:, ck], k[:, ck], v[:, cv], la[:, ck], qk_scale=qk_scale)
            o = o_raw.copy()
            if head_norm_eps is not None:
                for hh in range(h):
                    cv = slice(hh * d_v, (hh + 1) * d_v)
                    o[:, cv] = head_rmsnorm(o_raw[:, cv], _norm_weight(br, h, d_v)[cv], head_norm_eps)
            Y = o @ br["Wo"].T
            fwd.append((Xp, q, k, v, la, o_raw, o, Y, hold(Y, s, L)))
        # fusion: O_t = sum_s w_{t,s} Yhat^(s)_t, w_t = softmax(z_t), z_t = W_fuse x_t + b_fuse
        dw = np.stack([(dO[b] * f[8]).sum(axis=1) for f in fwd], axis=1)
        dz = w * (dw - (w * dw).sum(axis=1, keepdims=True))
        grads["Wfuse"] += dz.T @ X[b]
        grads["bfuse"] += dz.sum(axis=0)
        dX[b] += dz @ weights["Wfuse"]
        for j, (s, h) in enumerate(zip(scales, heads)):
            br, gb = weights["branches"][j], grads["branches"][j]
            Xp, q, k, v, la, o_raw, o, Y, _ = fwd[j]
            dYhat = w[:, j:j + 1] * dO[b]
            dY = np.zeros_like(Y)
            for t in range(L):
                i = hold_index(t, s)
                if i >= 0:
                    dY[i] += dYhat[t]
            gb["Wo"] += dY.T @ o
            do = dY @ br["Wo"]
            if head_norm_eps is not None:
                nw = _norm_weight(br, h, d_v)
                gb.setdefault("norm_w", np.zeros(h * d_v))
                for hh in range(h):
                    cv = slice(hh * d_v, (hh + 1) * d_v)
                    do[:, cv], dnw = head_rmsnorm_backward(o_raw[:, cv], nw[cv], head_norm_eps, do[:, cv])
                    gb["norm_w"][cv] += dnw
            dq, dk, dv, dla = (np.zeros_like(q), np.zeros_like(k), np.zeros_like(v), np.zeros_like(la))
            for hh in range(h):
                ck, cv = slice(hh * d_k, (hh + 1) * d_k), slice(hh * d_v, (hh + 1) * d_v)
                dq[:, ck], dk[:, ck], dv[:, cv], dla[:, ck] = gla_recurrent_backward(
                    q[:, ck], k[:, ck], v[:, cv], la[:, ck], do[:, cv], qk_scale=qk_scale)
            g = Xp @ br["Wg1"].T
            u = g @ br["Wg2"].T + br["bg"]
            du = dla / gate_normalizer * np.exp(-np.logaddexp(0.0, u))  # sigmoid(-u)
            gb["Wg2"] += du.T @ g
            gb["bg"] += du.sum(axis=0)
            dg = du @ br["Wg2"]
            gb["Wg1"] += dg.T @ Xp
            gb["Wq"] += dq.T @ Xp
            gb["Wk"] += dk.T @ Xp
            gb["Wv"] += dv.T @ Xp
            dXp = dq @ br["Wq"] + dk @ br["Wk"] + dv @ br["Wv"] + dg @ br["Wg1"]
            Mb = np.ones(L) if M is None else M
            for i in range(Xp.shape[0]):
                rows = [i * s + r for r in range(s) if i * s + r < L]
                cnt = max(1.0, sum(Mb[r] for r in rows))
                for r in rows:
                    dX[b, r] += Mb[r] * dXp[i] / cnt
    return dX, grads


# ---------------------------------------------------------------------------
# token-by-token inference (reading notes, method part, item 7 "training and
# token-by-token inference"): per-branch cache, one token at a time
# ---------------------------------------------------------------------------
def decode_init(B: int, d: int, scales, heads, d_k: int, d_v: int) -> dict:
    """Empty cache for B sequences. Per branch: the GLA state of every head
    (S [B, h, d_k, d_v]), the running sum of the tokens not yet forming a full
    block (buf [B, d]) with their count, and the branch output most recently
    produced (Y [B, d], zero before the first complete block). Its size does
    not depend on how many tokens have been consumed."""
    return {"branches": [dict(S=np.zeros((B, h, d_k, d_v)), buf=np.zeros((B, d)), n=0, Y=np.zeros((B, d)))
                         for s, h in zip(scales, heads)]}


def decode_step(cache: dict, x: np.ndarray, weights: dict, scales, heads, d_k: int, d_v: int,
                gate_normalizer: float = 16.0, qk_scale: float = 1.0,
                head_norm_eps: float | None = None) -> np.ndarray:
    """Consume one token x [B, d] of each sequence; return O_t [B, d].

    Each branch adds x to its buffer; once it holds s tokens, their mean is the
    next pooled row (Eq. (8)), which takes one GLA step per head (S = Diag(alpha)
    S + k^T v, o = qk_scale * q S), goes through W_o, replaces the cached output
    and empties the buffer. Otherwise the branch keeps its previous output. The
    output fuses the cached branch outputs with w = softmax(W_fuse x + b_fuse)."""
    x = np.asarray(x, dtype=np.float64)
    B = x.shape[0]
    w = fusion_weights(x, weights["Wfuse"], weights["bfuse"])
    O = np.zeros_like(x)
    for j, (s, h) in enumerate(zip(scales, heads)):
        br, c = weights["branches"][j], cache["branches"][j]
        c["buf"] = c["buf"] + x
        c["n"] += 1
        if c["n"] == s:
            xbar = c["buf"] / s
            q, k, v, la = branch_projections(xbar, br, gate_normalizer)
            alpha = np.exp(la)
            o = np.zeros((B, h * d_v))
            for b in range(B):
                for hh in range(h):
                    ck, cv = slice(hh * d_k, (hh + 1) * d_k), slice(hh * d_v, (hh + 1) * d_v)
                    S = alpha[b, ck][:, None] * c["S"][b, hh] + np.outer(k[b, ck], v[b, cv])
                    c["S"][b, hh] = S
                    o[b, cv] = qk_scale * (q[b, ck] @ S)
                    if head_norm_eps is not None:
                        nw = br.get("norm_w")
                        nw = np.ones(h * d_v) if nw is None else nw
                        o[b:b + 1, cv] = head_rmsnorm(o[b:b + 1, cv], nw[cv], head_norm_eps)
            c["Y"] = o @ br["Wo"].T
            c["buf"] = np.zeros_like(c["buf"])
            c["n"] = 0
        O += w[:, j:j + 1] * c["Y"]
    return O


def state_updates(L: int, scales, heads) -> int:
    """Number of per-head state updates the layer performs on one sequence of
    length L (each branch updates its h_s states once per pooled step)."""
    return sum(h * (-(-L // s)) for s, h in zip(scales, heads))
