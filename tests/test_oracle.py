"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Every check here is fixed by the MS-GLA reading notes (worked examples,
stated counts) or by mathematics (brute-force quadratic form, closed forms,
reductions to textbook linear attention, invariants). The mutation tests at
the end plant plausible mistakes in the oracle and check that some pin fails.
"""
import math
import os

import numpy as np
import pytest

import oracle
from oracle import msgla_oracle as om

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_table(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([float(x) for x in line.split()])
    return np.array(rows)


def _rand_weights(rng, d, scales, heads, dk, dv, r=4, gate_bias=0.0):
    brs = []
    for s, h in zip(scales, heads):
        brs.append(dict(
            Wq=rng.normal(0, 1 / math.sqrt(d), (h * dk, d)),
            Wk=rng.normal(0, 1 / math.sqrt(d), (h * dk, d)),
            Wv=rng.normal(0, 1 / math.sqrt(d), (h * dv, d)),
            Wg1=rng.normal(0, 1 / math.sqrt(d), (r, d)),
            Wg2=rng.normal(0, 1 / math.sqrt(r), (h * dk, r)),
            bg=np.full(h * dk, gate_bias),
            Wo=rng.normal(0, 1 / math.sqrt(h * dv), (d, h * dv)),
        ))
    return dict(branches=brs, Wfuse=rng.normal(0, 1 / math.sqrt(d), (len(scales), d)),
                bfuse=rng.normal(0, 0.5, len(scales)))


# --------------------------------------------------------------------------
# brute-force references written independently of the oracle's recurrence
# --------------------------------------------------------------------------
def gla_quadratic(q, k, v, log_alpha):
    """o_i = sum_{j<=i} sum_a q_ia k_ja prod_{m=j+1..i} alpha_ma v_j (pure loops):
    the unrolled GLA recurrence of Sec. 2.1."""
    n, dk = q.shape
    dv = v.shape[1]
    a = np.exp(log_alpha)
    o = np.zeros((n, dv))
    for i in range(n):
        for j in range(i + 1):
            coef = 0.0
            for c in range(dk):
                decay = 1.0
                for m in range(j + 1, i + 1):
                    decay *= a[m, c]
                coef += q[i, c] * k[j, c] * decay
            o[i] += coef * v[j]
    return o


def layer_bruteforce(X, W, scales, heads, dk, dv, normalizer):
    """Whole layer with pure loops: pooled rows summed directly, GLA in its
    quadratic form, hold via the notes' equivalent index floor((t-s+1)/s)
    for t >= s-1, softmax written out."""
    L, d = X.shape
    O = np.zeros((L, d))
    for t in range(L):
        z = [sum(W["Wfuse"][j, c] * X[t, c] for c in range(d)) + W["bfuse"][j]
             for j in range(len(scales))]
        zmax = max(z)
        e = [math.exp(zz - zmax) for zz in z]
        w = [ee / sum(e) for ee in e]
        for j, (s, h) in enumerate(zip(scales, heads)):
            if t < s - 1:
                continue
            i_read = (t - s + 1) // s
            br = W["branches"][j]
            n = i_read + 1
            Xp = np.zeros((n, d))
            for i in range(n):
                rows = [X[i * s + u] for u in range(s) if i * s + u < L]
                Xp[i] = sum(rows) / len(rows)
            q, k, v = Xp @ br["Wq"].T, Xp @ br["Wk"].T, Xp @ br["Wv"].T
            z_g = (Xp @ br["Wg1"].T) @ br["Wg2"].T + br["bg"]
            la = -np.log1p(np.exp(-z_g)) / normalizer
            o = np.zeros(h * dv)
            for hh in range(h):
                ck, cv = slice(hh * dk, (hh + 1) * dk), slice(hh * dv, (hh + 1) * dv)
                o[cv] = gla_quadratic(q[:, ck], k[:, ck], v[:, cv], la[:, ck])[i_read]
            O[t] += w[j] * (br["Wo"] @ o)
    return O


# --------------------------------------------------------------------------
# pins from the notes' worked examples
# --------------------------------------------------------------------------
def check_hold_table():
    tab = _read_table("hold_s4.txt")
    for t, expect in tab:
        assert om.hold_index(int(t), 4) == int(expect)
    Y = np.array([[10.0], [20.0]])
    Yh = om.hold(Y, 4, 8)[:, 0]
    want = [0.0 if e < 0 else Y[int(e), 0] for e in tab[:, 1]]
    np.testing.assert_array_equal(Yh, want)


def test_hold_table_s4():
    check_hold_table()


def test_hold_all_scales_matches_shift_form():
    # repeat s times then shift right by s-1 with zero fill (Sec. 3.3)
    for s in (1, 2, 4, 8):
        L = 37
        n = -(-L // s)
        Y = np.arange(1, n + 1, dtype=float)[:, None]
        rep = np.repeat(Y[:, 0], s)
        shifted = np.concatenate([np.zeros(s - 1), rep])[:L]
        np.testing.assert_array_equal(om.hold(Y, s, L)[:, 0], shifted)


def check_pool_example():
    tab = _read_table("pool_s4_first_row.txt")
    X = np.eye(8)
    P = om.pool(X, 4)
    for row in tab:
        np.testing.assert_allclose(P[int(row[0])], row[1:], rtol=0, atol=1e-15)


def test_pool_first_row_example():
    check_pool_example()


def check_pool_tail():
    # L = 10, s = 4: the tail block holds rows 8, 9 and is their mean (Eq. 8, M = 1
    # inside L, denominator = number of valid rows)
    X = np.arange(10, dtype=float)[:, None]
    P = om.pool(X, 4)
    np.testing.assert_array_equal(P[:, 0], [1.5, 5.5, 8.5])


def test_pool_tail_block():
    check_pool_tail()


def check_pool_mask():
    tab = _read_table("pool_mask_s4.txt")
    M = np.array([0, 1, 1, 0, 0, 0, 0, 0], dtype=float)
    P = om.pool(np.eye(8), 4, M)
    for row in tab:
        np.testing.assert_allclose(P[int(row[0])], row[1:], rtol=0, atol=1e-15)


def test_pool_mask_example():
    check_pool_mask()


def test_all_ones_mask_is_the_unmasked_layer():
    rng = np.random.default_rng(11)
    d, dk, dv, L = 6, 3, 2, 14
    W = _rand_weights(rng, d, (1, 2, 4), (2, 1, 1), dk, dv)
    X = rng.normal(size=(2, L, d))
    np.testing.assert_array_equal(om.layer_forward(X, W, (1, 2, 4), (2, 1, 1), dk, dv, mask=np.ones((2, L))),
                                  om.layer_forward(X, W, (1, 2, 4), (2, 1, 1), dk, dv))


def test_masked_rows_do_not_reach_pooled_rows():
    """Changing X at a masked position changes no pooled row (Eq. (8) weights it by 0)."""
    rng = np.random.default_rng(12)
    X = rng.normal(size=(12, 5))
    M = np.ones(12); M[[0, 1, 5, 11]] = 0
    X2 = X.copy(); X2[[0, 1, 5, 11]] += 7.0
    for s in (1, 2, 4):
        np.testing.assert_array_equal(om.pool(X, s, M), om.pool(X2, s, M))


def test_mask_at_scale_one_zeroes_padded_rows():
    """Eq. (8) at s = 1: x_t M_t / max(1, M_t) is x_t when valid and 0 when padded."""
    rng = np.random.default_rng(14)
    X = rng.normal(size=(6, 4))
    M = np.array([1, 0, 1, 1, 0, 1], dtype=float)
    np.testing.assert_array_equal(om.pool(X, 1, M), X * M[:, None])


def test_left_padding_changes_only_mixed_blocks():
    rng = np.random.default_rng(13)
    X = rng.normal(size=(8, 3))
    M = np.array([0, 0, 0, 1, 1, 1, 1, 1], dtype=float)
    P = om.pool(X, 4, M)
    np.testing.assert_allclose(P[0], X[3], rtol=1e-15)
    np.testing.assert_allclose(P[1], X[4:8].mean(0), rtol=1e-15)


# --------------------------------------------------------------------------
# optional per-head RMS normalisation (Sec. 3.2 reading)
# --------------------------------------------------------------------------
def check_head_norm_unit_rms(seed=21):
    """eps ~ 0, unit weight: every head's normalised output row has RMS 1."""
    rng = np.random.default_rng(seed)
    d, dk, dv, L = 8, 3, 5, 19
    W = _rand_weights(rng, d, (1, 2), (2, 1), dk, dv)
    X = rng.normal(size=(1, L, d))
    _, inter = om.layer_forward(X, W, (1, 2), (2, 1), dk, dv, intermediates=True, head_norm_eps=1e-30)
    for (s, h), br in zip(((1, 2), (2, 1)), inter["branches"]):
        o = br["o"][0]
        for hh in range(h):
            rms = np.sqrt((o[:, hh * dv:(hh + 1) * dv] ** 2).mean(axis=1))
            np.testing.assert_allclose(rms, 1.0, rtol=1e-12)


def check_head_norm_constant_row():
    """A constant row c of width n: c / sqrt(c^2 + eps) times the weight."""
    c, eps = 0.3, 0.05
    w = np.array([1.0, -2.0, 0.5, 3.0])
    got = om.head_rmsnorm(np.full((2, 4), c), w, eps)
    np.testing.assert_allclose(got, np.tile(c / math.sqrt(c * c + eps) * w, (2, 1)), rtol=1e-14)


def test_head_norm_unit_rms():
    check_head_norm_unit_rms()


def test_head_norm_constant_row():
    check_head_norm_constant_row()


def test_head_norm_is_invariant_to_value_scale():
    """eps = 0: o is linear in W_v, and the RMS norm is homogeneous of degree 0,
    so scaling every W_v by c > 0 leaves the layer output unchanged."""
    rng = np.random.default_rng(22)
    d, dk, dv = 6, 3, 4
    W = _rand_weights(rng, d, (1, 2, 4), (2, 1, 1), dk, dv)
    for br in W["branches"]:
        br["norm_w"] = rng.normal(1.0, 0.3, br["Wv"].shape[0])
    X = rng.normal(size=(2, 17, d))
    a = om.layer_forward(X, W, (1, 2, 4), (2, 1, 1), dk, dv, head_norm_eps=0.0)
    for br in W["branches"]:
        br["Wv"] = br["Wv"] * 3.7
    b = om.layer_forward(X, W, (1, 2, 4), (2, 1, 1), dk, dv, head_norm_eps=0.0)
    np.testing.assert_allclose(b, a, rtol=1e-10, atol=1e-12)
    c = om.layer_forward(X, W, (1, 2, 4), (2, 1, 1), dk, dv)
    assert np.abs(c).max() > 2 * np.abs(a).max() or not np.allclose(c, a)


def test_head_norm_off_by_default():
    rng = np.random.default_rng(23)
    W = _rand_weights(rng, 5, (1, 2), (1, 1), 2, 3)
    for br in W["branches"]:
        br["norm_w"] = np.full(3, 2.0)
    X = rng.normal(size=(1, 9, 5))
    _, inter = om.layer_forward(X, W, (1, 2), (1, 1), 2, 3, intermediates=True)
    q, k, v, la = om.branch_projections(inter["branches"][0]["Xp"][0], W["branches"][0], 16.0)
    np.testing.assert_array_equal(inter["branches"][0]["o"][0], om.gla_recurrent(q, k, v, la))


# --------------------------------------------------------------------------
# token-by-token inference against the whole-sequence layer
# --------------------------------------------------------------------------
def _decode_all(X, W, scales, heads, dk, dv, **kw):
    B, L, d = X.shape
    cache = om.decode_init(B, d, scales, heads, dk, dv)
    return np.stack([om.decode_step(cache, X[:, t], W, scales, heads, dk, dv, **kw) for t in range(L)], axis=1)


def check_decode_matches_parallel(seed=31):
    """Feeding a ragged sequence one token at a time gives, at every position,
    the layer output of Sec. 3 (the causal hold reads the block that ended last),
    for scale sets with and without the scale-1 branch."""
    rng = np.random.default_rng(seed)
    d, dk, dv, L = 7, 3, 4, 23
    for scales, heads in (((1, 2, 4), (2, 1, 1)), ((2, 3), (1, 2)), ((1, 5), (1, 1))):
        W = _rand_weights(rng, d, scales, heads, dk, dv, gate_bias=1.0)
        X = rng.normal(size=(2, L, d))
        np.testing.assert_allclose(_decode_all(X, W, scales, heads, dk, dv, qk_scale=0.7),
                                   om.layer_forward(X, W, scales, heads, dk, dv, qk_scale=0.7),
                                   rtol=1e-11, atol=1e-12)


def test_decode_matches_parallel():
    check_decode_matches_parallel()


def test_decode_with_head_norm_matches_parallel():
    rng = np.random.default_rng(32)
    d, dk, dv, L = 6, 2, 3, 17
    W = _rand_weights(rng, d, (1, 2, 4), (2, 1, 1), dk, dv)
    for br in W["branches"]:
        br["norm_w"] = rng.normal(1.0, 0.2, br["Wv"].shape[0])
    X = rng.normal(size=(1, L, d))
    np.testing.assert_allclose(_decode_all(X, W, (1, 2, 4), (2, 1, 1), dk, dv, head_norm_eps=1e-3),
                               om.layer_forward(X, W, (1, 2, 4), (2, 1, 1), dk, dv, head_norm_eps=1e-3),
                               rtol=1e-11, atol=1e-12)


def test_decode_cache_does_not_grow():
    rng = np.random.default_rng(33)
    W = _rand_weights(rng, 5, (1, 4), (1, 1), 2, 2)
    cache = om.decode_init(3, 5, (1, 4), (1, 1), 2, 2)
    shapes = [[v.shape for v in (c["S"], c["buf"], c["Y"])] for c in cache["branches"]]
    for t in range(41):
        om.decode_step(cache, rng.normal(size=(3, 5)), W, (1, 4), (1, 1), 2, 2)
    assert [[v.shape for v in (c["S"], c["buf"], c["Y"])] for c in cache["branches"]] == shapes
    assert cache["branches"][1]["n"] == 41 % 4


def test_update_ratio_11_16():
    num, den = _read_table("update_ratio.txt")[0]
    L = 256
    counter = [0]
    rng = np.random.default_rng(0)
    W = _rand_weights(rng, 8, (1, 2, 4), (2, 1, 1), 2, 2)
    om.layer_forward(rng.normal(size=(1, L, 8)), W, (1, 2, 4), (2, 1, 1), 2, 2, counter=counter)
    gla = om.state_updates(L, (1,), (4,))
    assert counter[0] == om.state_updates(L, (1, 2, 4), (2, 1, 1))
    assert counter[0] * den == gla * num


# --------------------------------------------------------------------------
# pins from mathematics
# --------------------------------------------------------------------------
def check_gla_bruteforce(seed=0):
    rng = np.random.default_rng(seed)
    n, dk, dv = 9, 3, 4
    q, k = rng.normal(size=(n, dk)), rng.normal(size=(n, dk))
    v = rng.normal(size=(n, dv))
    la = -rng.uniform(0.01, 1.5, size=(n, dk))
    np.testing.assert_allclose(om.gla_recurrent(q, k, v, la), gla_quadratic(q, k, v, la),
                               rtol=1e-12, atol=1e-12)


def test_gla_matches_quadratic_form():
    for seed in range(3):
        check_gla_bruteforce(seed)


def test_alpha_one_is_causal_linear_attention():
    rng = np.random.default_rng(1)
    n, dk, dv = 20, 5, 7
    q, k, v = rng.normal(size=(n, dk)), rng.normal(size=(n, dk)), rng.normal(size=(n, dv))
    want = np.tril(q @ k.T) @ v
    np.testing.assert_allclose(om.gla_recurrent(q, k, v, np.zeros((n, dk))), want,
                               rtol=1e-12, atol=1e-12)


def test_qk_scale_is_linear():
    rng = np.random.default_rng(2)
    n, dk, dv = 6, 3, 2
    q, k, v = rng.normal(size=(n, dk)), rng.normal(size=(n, dk)), rng.normal(size=(n, dv))
    la = -rng.uniform(0, 1, (n, dk))
    np.testing.assert_allclose(om.gla_recurrent(q, k, v, la, qk_scale=0.25),
                               0.25 * om.gla_recurrent(q, k, v, la), rtol=1e-14)


def check_layer_bruteforce(seed=3, L=13):
    rng = np.random.default_rng(seed)
    d, dk, dv = 6, 3, 2
    scales, heads = (1, 2, 4), (2, 1, 1)
    W = _rand_weights(rng, d, scales, heads, dk, dv, r=3, gate_bias=0.5)
    X = rng.normal(size=(1, L, d))
    O = om.layer_forward(X, W, scales, heads, dk, dv, gate_normalizer=4.0)
    np.testing.assert_allclose(O[0], layer_bruteforce(X[0], W, scales, heads, dk, dv, 4.0),
                               rtol=1e-10, atol=1e-11)


def test_layer_matches_bruteforce():
    check_layer_bruteforce(3, 13)
    check_layer_bruteforce(4, 8)


def test_single_scale_is_plain_gla():
    rng = np.random.default_rng(5)
    d, dk, dv, L = 8, 4, 3, 11
    W = _rand_weights(rng, d, (1,), (2,), dk, dv)
    X = rng.normal(size=(1, L, d))
    O, inter = om.layer_forward(X, W, (1,), (2,), dk, dv, intermediates=True)
    np.testing.assert_array_equal(inter["w"], np.ones((1, L, 1)))
    br = W["branches"][0]
    q, k, v = X[0] @ br["Wq"].T, X[0] @ br["Wk"].T, X[0] @ br["Wv"].T
    la = -np.logaddexp(0, -((X[0] @ br["Wg1"].T) @ br["Wg2"].T + br["bg"])) / 16.0
    o = np.concatenate([gla_quadratic(q[:, h * dk:(h + 1) * dk], k[:, h * dk:(h + 1) * dk],
                                      v[:, h * dv:(h + 1) * dv], la[:, h * dk:(h + 1) * dk])
                        for h in range(2)], axis=1)
    np.testing.assert_allclose(O[0], o @ br["Wo"].T, rtol=1e-11, atol=1e-12)


def check_constant_input_closed_form():
    """X_t = c: q, k, v, alpha are constant per branch, so
    o_n = sum_a q_a k_a (1 - alpha_a^(n+1)) / (1 - alpha_a) v (geometric sum)."""
    rng = np.random.default_rng(6)
    d, dk, dv, L = 8, 4, 3, 23
    scales, heads = (1, 2, 4), (2, 1, 1)
    W = _rand_weights(rng, d, scales, heads, dk, dv, gate_bias=1.0)
    c = rng.normal(size=d)
    X = np.tile(c, (1, L, 1))
    z = W["Wfuse"] @ c + W["bfuse"]
    w = np.exp(z - z.max()) / np.exp(z - z.max()).sum()
    want = np.zeros((L, d))
    for j, (s, h) in enumerate(zip(scales, heads)):
        br = W["branches"][j]
        q, k, v = br["Wq"] @ c, br["Wk"] @ c, br["Wv"] @ c
        alpha = 1.0 / (1.0 + np.exp(-(br["Wg2"] @ (br["Wg1"] @ c) + br["bg"]))) ** (1 / 16.0)
        for t in range(L):
            if t < s - 1:
                continue
            n = (t - s + 1) // s
            o = np.zeros(h * dv)
            for hh in range(h):
                ck, cv = slice(hh * dk, (hh + 1) * dk), slice(hh * dv, (hh + 1) * dv)
                geo = (1 - alpha[ck] ** (n + 1)) / (1 - alpha[ck])
                o[cv] = np.sum(q[ck] * k[ck] * geo) * v[cv]
            want[t] += w[j] * (br["Wo"] @ o)
    got = om.layer_forward(X, W, scales, heads, dk, dv)[0]
    np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-12)


def test_constant_input_closed_form():
    check_constant_input_closed_form()


def test_half_life():
    """A single write at pooled step 0 under constant alpha = a decays as a^i, so at
    original distance D = s*i it is a^(D/s): half-life s*ln(1/2)/ln(a) (Sec. 3.3)."""
    a, n = 0.9, 40
    q = np.ones((n, 1))
    k = np.zeros((n, 1)); k[0, 0] = 1.0
    v = np.ones((n, 1))
    o = om.gla_recurrent(q, k, v, np.full((n, 1), math.log(a)))[:, 0]
    np.testing.assert_allclose(o, a ** np.arange(n), rtol=1e-13)
    for s in (1, 2, 4):
        half = s * math.log(0.5) / math.log(a)
        i_half = half / s
        assert abs(a ** i_half - 0.5) < 1e-12


def test_coarse_gate_input_is_block_mean_of_row_projections():
    """Eq. (8) is linear, so a coarse branch's low-rank gate input xbar_i W_g1^T
    equals the mean over block i of x_j W_g1^T (a ragged tail block: over its
    rows inside L). log alpha rebuilt that way from the unpooled rows, with the
    sigmoid written out, agrees with the oracle's."""
    rng = np.random.default_rng(41)
    d, dk, dv, L = 8, 3, 5, 23  # 23 leaves ragged tail blocks at s = 2 and 4
    scales, heads = (1, 2, 4), (1, 1, 1)
    W = _rand_weights(rng, d, scales, heads, dk, dv, gate_bias=0.3)
    X = rng.normal(size=(1, L, d))
    _, inter = om.layer_forward(X, W, scales, heads, dk, dv, intermediates=True)
    for j, s in enumerate(scales):
        br = W["branches"][j]
        g_rows = X[0] @ br["Wg1"].T
        n = -(-L // s)
        g = np.stack([g_rows[i * s:min(L, (i + 1) * s)].mean(axis=0) for i in range(n)])
        z = g @ br["Wg2"].T + br["bg"]
        la = np.log(1.0 / (1.0 + np.exp(-z))) / 16.0
        np.testing.assert_allclose(inter["branches"][j]["log_alpha"][0], la, rtol=1e-10, atol=1e-14)


# --------------------------------------------------------------------------
# gradients (layer_backward): central finite differences of the forward
# --------------------------------------------------------------------------
def _check_gradients(X, W, scales, heads, dk, dv, mask=None, qk_scale=1.0, seed=0, eps=1e-6, rtol=1e-6,
                     head_norm_eps=None):
    dO = np.random.default_rng(seed).normal(size=X.shape)
    dX, g = om.layer_backward(X, W, scales, heads, dk, dv, dO, qk_scale=qk_scale, mask=mask,
                              head_norm_eps=head_norm_eps)

    def loss():
        return float((om.layer_forward(X, W, scales, heads, dk, dv, qk_scale=qk_scale, mask=mask,
                                       head_norm_eps=head_norm_eps) * dO).sum())

    def finite_difference(arr):
        out = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            keep = arr[idx]
            arr[idx] = keep + eps
            up = loss()
            arr[idx] = keep - eps
            down = loss()
            arr[idx] = keep
            out[idx] = (up - down) / (2 * eps)
        return out

    # central differences carry about |loss| * 2^-52 / eps ~ 1e-8 of rounding noise;
    # the 1e-7 floor is still ~1e-4 of the smallest gradient block checked
    def close(name, got, want):
        assert np.abs(got - want).max() <= rtol * np.abs(want).max() + 1e-7, name

    close("X", dX, finite_difference(X))
    for j, br in enumerate(W["branches"]):
        for name in ("Wq", "Wk", "Wv", "Wg1", "Wg2", "bg", "Wo") + (("norm_w",) if head_norm_eps else ()):
            close(f"{name} of branch {j}", g["branches"][j][name], finite_difference(br[name]))
    close("Wfuse", g["Wfuse"], finite_difference(W["Wfuse"]))
    close("bfuse", g["bfuse"], finite_difference(W["bfuse"]))


def check_gradients_plain():
    """Every gradient of layer_backward (input, all projections, gate factors
    and bias, output projections, fusion weights and bias) against central
    differences of layer_forward; ragged tail blocks at s = 2 and 4."""
    rng = np.random.default_rng(51)
    d, dk, dv, L = 5, 3, 2, 9
    W = _rand_weights(rng, d, (1, 2, 4), (1, 1, 1), dk, dv, gate_bias=0.5)
    W["bfuse"] = rng.normal(size=3)
    X = rng.normal(size=(2, L, d))
    _check_gradients(X, W, (1, 2, 4), (1, 1, 1), dk, dv, seed=52)


def check_gradients_masked():
    """The same with a padding mask in the pooling, qk_scale 0.7, two heads on
    one branch and no scale-1 branch (scales 2 and 3)."""
    rng = np.random.default_rng(53)
    d, dk, dv, L = 4, 2, 3, 8
    W = _rand_weights(rng, d, (2, 3), (2, 1), dk, dv, gate_bias=-0.3)
    X = rng.normal(size=(2, L, d))
    mask = np.ones((2, L))
    mask[1, :3] = 0.0  # left padding of the second sequence
    _check_gradients(X, W, (2, 3), (2, 1), dk, dv, mask=mask, qk_scale=0.7, seed=54)


def check_gradients_head_norm():
    """The same with the optional per-head RMS norm (and its weight) on."""
    rng = np.random.default_rng(55)
    d, dk, dv, L = 4, 2, 3, 7
    W = _rand_weights(rng, d, (1, 2), (1, 2), dk, dv)
    for j, h in enumerate((1, 2)):
        W["branches"][j]["norm_w"] = rng.normal(1.0, 0.3, size=h * dv)
    X = rng.normal(size=(1, L, d))
    _check_gradients(X, W, (1, 2), (1, 2), dk, dv, seed=56, head_norm_eps=1e-3)


def test_gradients_match_finite_differences():
    check_gradients_plain()


def test_gradients_with_head_norm():
    check_gradients_head_norm()


def test_gradients_with_mask_scale_and_no_fine_branch():
    check_gradients_masked()


def test_fusion_weights_simplex():
    rng = np.random.default_rng(7)
    X = rng.normal(size=(50, 16)) * 5
    w = om.fusion_weights(X, rng.normal(size=(3, 16)), rng.normal(size=3))
    assert (w >= 0).all()
    np.testing.assert_allclose(w.sum(1), 1.0, rtol=0, atol=1e-14)
    # invariant to a common shift of the logits
    Wf = rng.normal(size=(3, 16))
    np.testing.assert_allclose(om.fusion_weights(X, Wf, np.zeros(3)),
                               om.fusion_weights(X, Wf, np.full(3, 7.0)), rtol=1e-13)


def test_causality():
    rng = np.random.default_rng(8)
    d, dk, dv, L = 6, 3, 2, 21
    scales, heads = (1, 2, 4), (2, 1, 1)
    W = _rand_weights(rng, d, scales, heads, dk, dv)
    X = rng.normal(size=(1, L, d))
    O = om.layer_forward(X, W, scales, heads, dk, dv)
    for p in (0, 5, 11, 20):
        X2 = X.copy()
        X2[0, p] += rng.normal(size=d)
        O2 = om.layer_forward(X2, W, scales, heads, dk, dv)
        np.testing.assert_array_equal(O2[0, :p], O[0, :p])
        assert np.abs(O2[0, p] - O[0, p]).max() > 0


def test_incomplete_tail_block_never_read():
    # the pooled row of an incomplete tail block is first due at t = i*s + s - 1 >= L
    for s in (2, 4, 8):
        for L in (s + 1, 3 * s - 1, 5 * s + 3):
            n = -(-L // s)
            Y = np.zeros((n, 1)); Y[-1, 0] = 1.0
            held = om.hold(Y, s, L)
            assert held.sum() == (1.0 if L % s == 0 else 0.0)


def test_batch_independence():
    rng = np.random.default_rng(9)
    d, dk, dv, L = 6, 3, 2, 10
    W = _rand_weights(rng, d, (1, 2), (1, 1), dk, dv)
    X = rng.normal(size=(3, L, d))
    O = om.layer_forward(X, W, (1, 2), (1, 1), dk, dv)
    for b in range(3):
        np.testing.assert_array_equal(O[b], om.layer_forward(X[b:b + 1], W, (1, 2), (1, 1), dk, dv)[0])


# --------------------------------------------------------------------------
# mutation tests: a planted mistake in the oracle must trip a pin
# --------------------------------------------------------------------------
def _mutant_hold_shift_s(t, s):
    return t // s - 1                      # shift by s instead of s-1


def _mutant_gla_no_decay(q, k, v, log_alpha, qk_scale=1.0, counter=None):
    return np.tril(q @ k.T) @ v * qk_scale


def _mutant_gla_read_before_write(q, k, v, log_alpha, qk_scale=1.0, counter=None):
    S = np.zeros((q.shape[1], v.shape[1])); o = np.zeros((q.shape[0], v.shape[1]))
    for t in range(q.shape[0]):
        o[t] = q[t] @ S
        S = np.exp(log_alpha[t])[:, None] * S + np.outer(k[t], v[t])
    return o


def _mutant_gla_decay_after_write(q, k, v, log_alpha, qk_scale=1.0, counter=None):
    S = np.zeros((q.shape[1], v.shape[1])); o = np.zeros((q.shape[0], v.shape[1]))
    for t in range(q.shape[0]):
        S = np.exp(log_alpha[t])[:, None] * (S + np.outer(k[t], v[t]))
        o[t] = q[t] @ S
    return o


def _mutant_pool_divide_by_s(X, s, M=None):
    L = X.shape[0]; n = -(-L // s)
    Xp = np.zeros((n * s, X.shape[1])); Xp[:L] = X
    return Xp.reshape(n, s, -1).sum(1) / s


def _mutant_pool_mask_divide_by_block(X, s, M=None):
    L = X.shape[0]; n = -(-L // s)
    M = np.ones(L) if M is None else M
    out = np.zeros((n, X.shape[1]))
    for i in range(n):
        rows = [i * s + j for j in range(s) if i * s + j < L]
        out[i] = sum(X[r] * M[r] for r in rows) / len(rows)   # ignores the mask in the denominator
    return out


def _mutant_head_norm_no_sqrt(o, weight, eps):
    return o / ((o * o).mean(axis=1, keepdims=True) + eps) * weight


def _mutant_head_norm_sum_not_mean(o, weight, eps):
    return o / np.sqrt((o * o).sum(axis=1, keepdims=True) + eps) * weight


def _mutant_head_norm_eps_outside(o, weight, eps):
    return o / (np.sqrt((o * o).mean(axis=1, keepdims=True)) + eps) * weight


def _mutant_head_norm_no_weight(o, weight, eps):
    return o / np.sqrt((o * o).mean(axis=1, keepdims=True) + eps)


_real_decode_step = om.decode_step


def _mutant_decode_one_step_late(cache, x, weights, scales, heads, d_k, d_v, **kw):
    old = [c["Y"].copy() for c in cache["branches"]]
    _real_decode_step(cache, x, weights, scales, heads, d_k, d_v, **kw)
    w = om.fusion_weights(np.asarray(x, dtype=float), weights["Wfuse"], weights["bfuse"])
    return sum(w[:, j:j + 1] * old[j] for j in range(len(scales)))


def _mutant_decode_buffer_kept(cache, x, weights, scales, heads, d_k, d_v, **kw):
    before = [c["buf"].copy() for c in cache["branches"]]
    out = _real_decode_step(cache, x, weights, scales, heads, d_k, d_v, **kw)
    for c, b in zip(cache["branches"], before):
        if c["n"] == 0:          # the branch fired: keep the old tokens in its buffer
            c["buf"] = b + x
    return out


_real_gla_backward = om.gla_recurrent_backward


def _mutant_gla_backward_no_alpha(q, k, v, log_alpha, do, qk_scale=1.0):
    dq, dk, dv, dla = _real_gla_backward(q, k, v, log_alpha, do, qk_scale)
    return dq, dk, dv, dla / np.exp(log_alpha)          # d alpha instead of d log alpha


def _mutant_gla_backward_no_carry(q, k, v, log_alpha, do, qk_scale=1.0):
    n = q.shape[0]
    out = [np.zeros_like(a, dtype=float) for a in (q, k, v, log_alpha)]
    for t in range(n):                                  # drops the adjoint carried from later steps
        g = [np.zeros_like(do)]
        g[0][t] = do[t]
        parts = _real_gla_backward(q[:t + 1], k[:t + 1], v[:t + 1], log_alpha[:t + 1], g[0][:t + 1], qk_scale)
        for a, p in zip(out, parts):
            a[t] += p[t]
    return tuple(out)


def _mutant_gla_backward_k_for_v(q, k, v, log_alpha, do, qk_scale=1.0):
    dq, dk, dv, dla = _real_gla_backward(q, k, v, log_alpha, do, qk_scale)
    return dq, dk[:, ::-1], dv, dla                     # key adjoint channels reversed


def _mutant_softmax_wrong_axis(X, Wfuse, bfuse):
    z = X @ Wfuse.T + bfuse
    return np.exp(z) / np.exp(z).sum(axis=0, keepdims=True)


PINS = [check_hold_table, check_pool_example, check_pool_tail, check_pool_mask, check_gla_bruteforce,
        check_layer_bruteforce, check_constant_input_closed_form, check_head_norm_unit_rms,
        check_head_norm_constant_row, check_decode_matches_parallel, check_gradients_plain,
        check_gradients_masked, check_gradients_head_norm]


@pytest.mark.parametrize("name,mutant", [
    ("hold_index", _mutant_hold_shift_s),
    ("gla_recurrent", _mutant_gla_no_decay),
    ("gla_recurrent", _mutant_gla_read_before_write),
    ("gla_recurrent", _mutant_gla_decay_after_write),
    ("pool", _mutant_pool_divide_by_s),
    ("pool", _mutant_pool_mask_divide_by_block),
    ("fusion_weights", _mutant_softmax_wrong_axis),
    ("head_rmsnorm", _mutant_head_norm_no_sqrt),
    ("head_rmsnorm", _mutant_head_norm_sum_not_mean),
    ("head_rmsnorm", _mutant_head_norm_eps_outside),
    ("head_rmsnorm", _mutant_head_norm_no_weight),
    ("decode_step", _mutant_decode_one_step_late),
    ("decode_step", _mutant_decode_buffer_kept),
    ("gla_recurrent_backward", _mutant_gla_backward_no_alpha),
    ("gla_recurrent_backward", _mutant_gla_backward_no_carry),
    ("gla_recurrent_backward", _mutant_gla_backward_k_for_v),
])
def test_planted_mistake_is_caught(monkeypatch, name, mutant):
    monkeypatch.setattr(om, name, mutant)
    caught = 0
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught >= 1, f"no pin caught the mutant of {name}"
