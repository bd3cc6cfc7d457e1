/*
 * msgla.h -- C ABI of the MS-GLA (multi-scale gated linear attention) layer
 * forward pass on NVIDIA B200 (sm_100a).
 *
 * The layer (MS-GLA reading notes, arXiv 2609.35664v1, Secs. 2.1 and 3.1-3.3):
 *   for every scale s of the scale set S, with h_s heads (sum_s h_s = H, Eq. (9)):
 *     Xbar^(s)_i = mean of rows i*s .. i*s+s-1 of X        (Sec. 3.1, Eq. (8))
 *     q, k = Xbar W_q^T, Xbar W_k^T      [per head d_k wide]
 *     v    = Xbar W_v^T                  [per head d_v wide]
 *     log alpha = logsigmoid((Xbar W_g1^T) W_g2^T + b_g) / gate_normalizer
 *     S_t = Diag(alpha_t) S_{t-1} + k_t^T v_t,  o_t = qk_scale * q_t S_t  (Sec. 2.1)
 *     Y^(s) = o W_o^T                                        (Sec. 3.2)
 *     Yhat^(s)_t = Y^(s)_{floor((t+1)/s)-1}, zero when that index is < 0 (Sec. 3.3)
 *   w_t = softmax(W_fuse x_t + b_fuse),  O_t = sum_s w_{t,s} Yhat^(s)_t  (Eqs. (10)-(11))
 *
 * Conventions
 *   - Matrices are row-major with PyTorch Linear layout [out, in] (y = x W^T).
 *   - "device" pointers are CUDA global memory of the handle's device; "host"
 *     pointers are ordinary (preferably pinned) host memory.
 *   - bf16 = IEEE-754 bfloat16 stored as uint16; f32 = IEEE float.
 *   - Every call returns an msgla_status (0 = success, negative = error), except
 *     msgla_destroy and msgla_status_string. msgla_last_error() gives a message
 *     for the last failing call on the calling thread.
 *   - Calls are not thread-safe on one handle. A handle may be used with one
 *     stream at a time (its device-side error flags are per handle).
 */
#ifndef MSGLA_H_
#define MSGLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MSGLA_MAX_SCALES 8

typedef enum msgla_status {
  MSGLA_OK = 0,
  MSGLA_ERR_INVALID_ARG = -1,    /* null pointer, bad size, inconsistent config       */
  MSGLA_ERR_UNSUPPORTED = -2,    /* valid but outside what the kernels implement      */
  MSGLA_ERR_CUDA = -3,           /* a CUDA runtime/driver call failed                 */
  MSGLA_ERR_DEVICE_TIMEOUT = -4, /* a bounded wait inside a kernel gave up            */
  MSGLA_ERR_RANGE = -5,          /* a value left the fp16 range of an internal operand */
  MSGLA_ERR_WORKSPACE = -6       /* workspace missing, too small or misaligned        */
} msgla_status;

/* Layer configuration (Sec. 3.2 of the notes: scale set, head split, widths). */
typedef struct msgla_config {
  int d;                         /* model width; multiple of 64, 64..8192                 */
  int n_scales;                  /* |S|, 1..MSGLA_MAX_SCALES                              */
  int scales[MSGLA_MAX_SCALES];  /* pooling factors, strictly increasing, 1..64           */
  int heads[MSGLA_MAX_SCALES];   /* h_s >= 1 for each scale; H = sum of heads             */
  int d_k;                       /* key width per head, 1..256                            */
  int d_v;                       /* value width per head, 1..1024                         */
  int gate_rank;                 /* rank r of the gate projection, 1..32                  */
  int chunk;                     /* chunk length of the chunkwise GLA kernel: 0 or 128.
                                    A compute parameter with no effect on the result
                                    beyond rounding (Sec. 3.4 of the notes).             */
  float gate_normalizer;         /* log alpha = logsigmoid(.) / gate_normalizer (> 0)     */
  float qk_scale;                /* o_t = qk_scale * q_t S_t                              */
  int head_norm;                 /* per-branch normalisation (Sec. 3.2 lists one per branch
                                    without defining it): 0 = none (default), 1 = RMS norm
                                    of each head's GLA output row before W_o:
                                    o_h <- o_h / sqrt(mean_c o_hc^2 + eps) * norm_w        */
  float head_norm_eps;           /* eps of the RMS norm; finite and > 0 when head_norm = 1 */
} msgla_config;

/* Weights: DEVICE pointers on the handle's device, read during msgla_create only
 * (the handle keeps its own packed copies; the caller may free these after).
 * Per scale j (index into msgla_config.scales):
 *   Wq[j]  bf16 [h_j*d_k, d]     Wk[j] bf16 [h_j*d_k, d]    Wv[j] bf16 [h_j*d_v, d]
 *   Wg1[j] bf16 [gate_rank, d]   Wg2[j] f32 [h_j*d_k, gate_rank]   bg[j] f32 [h_j*d_k]
 *   Wo[j]  bf16 [d, h_j*d_v]
 * Heads are laid side by side: head h of scale j owns rows h*d_k..h*d_k+d_k-1 of
 * Wq/Wk/Wg2/bg, rows h*d_v.. of Wv and columns h*d_v.. of Wo.
 *   Wfuse  bf16 [n_scales, d]    bfuse f32 [n_scales] (NULL = zeros)
 *   norm_w[j] f32 [h_j*d_v]  per-channel weight of the head RMS norm (read only when
 *              msgla_config.head_norm = 1; NULL = ones)
 * bg[j] may be NULL (zeros). */
typedef struct msgla_weights {
  const void*  Wq[MSGLA_MAX_SCALES];
  const void*  Wk[MSGLA_MAX_SCALES];
  const void*  Wv[MSGLA_MAX_SCALES];
  const void*  Wg1[MSGLA_MAX_SCALES];
  const float* Wg2[MSGLA_MAX_SCALES];
  const float* bg[MSGLA_MAX_SCALES];
  const void*  Wo[MSGLA_MAX_SCALES];
  const void*  Wfuse;
  const float* bfuse;
  const float* norm_w[MSGLA_MAX_SCALES];
} msgla_weights;

typedef struct msgla_handle msgla_handle;

/* Create a layer on CUDA device `device`. Validates the configuration, packs the
 * weights into handle-owned device buffers (converted to fp16 where a tensor-core
 * operand pairs them with fp16 data; a weight whose magnitude exceeds 65504 is
 * rejected with MSGLA_ERR_RANGE) and synchronises the device.
 * On success *out owns device memory until msgla_destroy. On error *out = NULL. */
int msgla_create(msgla_handle** out, const msgla_config* cfg, const msgla_weights* w,
                 int device);

/* Free everything the handle owns (weights, counters, its second stream and
 * events). NULL-safe. Synchronises the handle's device. */
void msgla_destroy(msgla_handle* h);

/* Bytes of device workspace msgla_forward needs for a [B, L, d] input.
 * B >= 0, L >= 0 (B*L = 0 gives 0 bytes). */
int msgla_workspace_size(const msgla_handle* h, int B, int L, size_t* bytes);

/* Layer forward: O = MS-GLA(X).
 *   X  device bf16 [B, L, d], row-major, 16-byte aligned, not written.
 *   O  device bf16 [B, L, d], row-major, 16-byte aligned; may not alias X.
 *   workspace  device buffer of at least msgla_workspace_size bytes, 256-byte
 *              aligned, owned by the caller; its contents on entry do not matter.
 *   stream     cudaStream_t (NULL = legacy default stream).
 * Asynchronous: returns after enqueuing the kernels on `stream`. Errors found by
 * the kernels (timeouts, fp16 range) are latched in the handle and reported by
 * msgla_sync_status. B*L = 0 launches nothing.
 * With a scale-1 branch, the output projection of the coarse branches may run on
 * a second stream owned by the handle, concurrently with the GLA kernel (forked
 * after the gates, joined back before the final output projection), so all of
 * the forward's work is still ordered before what follows it on `stream`; the
 * fork and join use events, so the forward can be captured into a CUDA graph
 * and replayed any number of times (the cross-stream counters start from zero
 * at every launch and are cleared by the launch that waited on them).
 * The environment variable MSGLA_SERIAL=1 (read once per process) keeps every
 * kernel on `stream`: needed under profilers that run kernels one at a time,
 * where the concurrent GEMM's bounded wait for the GLA CTAs would time out.
 * The handle keeps per-forward counters: forwards on one handle must not run
 * concurrently (serialise calls from several host threads or streams). */
int msgla_forward(msgla_handle* h, const void* X, int B, int L, void* O,
                  void* workspace, size_t workspace_bytes, void* stream);

/* msgla_forward with a valid-token mask M in the pooling (Sec. 3.1, Eq. (8)):
 *   Xbar^(s)_i = sum_j x_{is+j} M_{is+j} / max(1, sum_j M_{is+j}),
 * the sums over the rows of block i that lie inside L. The formula applies at
 * every scale, so at s = 1 a padded row enters its branch as a zero row; an
 * all-padding block pools to zero. The fusion weights (Eq. (10)) read the
 * unpooled x_t whatever its mask.
 *   M  device uint8 [B, L], row-major; nonzero = valid token, 0 = padding; not
 *      written. NULL gives msgla_forward's result.
 *   X, O, workspace, stream and errors as for msgla_forward (same workspace size).
 * Padding anywhere (left, right or interior) is accepted. Outputs at padded
 * positions are computed like any other (they are not zeroed). */
int msgla_forward_masked(msgla_handle* h, const void* X, const void* M, int B, int L,
                         void* O, void* workspace, size_t workspace_bytes, void* stream);

/* msgla_forward without a caller workspace and without any device allocation:
 * for callers that cannot call cudaMalloc (or their framework's allocator) at the
 * point where they run the layer -- for instance code inside a fixed memory arena
 * or a runtime that forbids allocation after start-up. The pages describe no such
 * entry point; it has no counterpart in the paper.
 *   X, O, stream  as for msgla_forward (device bf16 [B, L, d], 16-byte aligned).
 * The intermediates live in one fixed scratch array of 32 MiB inside the library's
 * device image, which every GPU that loads the library holds until the process
 * exits. Sizes whose workspace (msgla_workspace_size) exceeds 32 MiB are rejected
 * with MSGLA_ERR_WORKSPACE; for the 340M-shaped layer (d = 1024, scales {1,2,4},
 * d_k = 256, d_v = 512) that admits one sequence of up to about 2300 tokens.
 * The first call on a device looks up the array's device address (a one-time
 * set-up); make that first call before any stream capture. All calls share the
 * array and it keeps the previous call's contents (every value a forward reads is
 * written earlier in the same forward, so nothing needs clearing). Calls that can
 * overlap on the GPU -- on different streams, or from different handles or
 * threads -- race on the array and must be serialised by the caller.
 * Asynchronous on `stream` like msgla_forward; device-side errors are reported by
 * msgla_sync_status. */
int msgla_forward_noalloc(msgla_handle* h, const void* X, int B, int L, void* O,
                          void* stream);

/* msgla_forward that also records CUDA events around its kernels, for timing each
 * kernel on `stream` with events. `events` holds caller-created cudaEvent_t
 * handles: events[0] is recorded before the first kernel and events[i+1] after
 * the i-th kernel; msgla_launch_plan lists the kernels in launch order. A NULL
 * entry skips that record: the kernels are launched so that each may start
 * while the previous one finishes, and an event recorded between two kernels
 * takes that overlap away, so time only the boundaries needed.
 * `max_events` is the length of `events` (it must be at least the number of
 * msgla_launch_plan entries + 1); *n_launches receives the number of kernels
 * launched, which includes the kernels run on the second stream (the coarse
 * output projection and the one-warp wait before it; no plan entries and no
 * events of their own). `M` is the optional
 * valid-token mask of msgla_forward_masked (NULL = every token valid). */
int msgla_forward_profiled(msgla_handle* h, const void* X, const void* M, int B, int L, void* O,
                           void* workspace, size_t workspace_bytes, void* stream,
                           void* const* events, int max_events, int* n_launches);

/* Workspace for msgla_forward_host: msgla_workspace_size plus room to stage X and O. */
int msgla_workspace_size_host(const msgla_handle* h, int B, int L, size_t* bytes);

/* Host-buffer forward: copies X (HOST bf16 [B, L, d]) to the device part of
 * `workspace`, runs the layer, copies O back to HOST bf16 [B, L, d] and
 * synchronises. The batch goes through in chunks of whole sequences (one
 * sequence first and last, max(2, ceil((B - 2) / 4)) in each chunk between): the
 * upload of the next chunk and the download of the previous one run
 * on two copy streams owned by the handle while the current chunk's forward runs
 * on `stream`, so PCIe transfers in both directions overlap each other and the
 * compute. Pinned host memory is needed for that overlap (pageable memory works,
 * with staged copies). Returns the status of the whole call, including
 * device-side errors. */
int msgla_forward_host(msgla_handle* h, const void* X_host, int B, int L, void* O_host,
                       void* workspace, size_t workspace_bytes, void* stream);

/* Synchronise the handle's device and return (then clear) the first device-side
 * error latched since the previous call: MSGLA_OK, MSGLA_ERR_DEVICE_TIMEOUT or
 * MSGLA_ERR_RANGE; MSGLA_ERR_CUDA if the synchronisation itself failed. */
int msgla_sync_status(msgla_handle* h);

/* Intermediate tensors inside the workspace of a forward with the same B and L
 * (for inspection by tests and tools; valid after the forward completes).
 * With b the cumulative sum of log alpha over the rows of a 128-row chunk (from
 * its first row) and m its value at the chunk's row 63, per key channel:
 * `which`: 0 pooled X (fp16 [B, n_s, d]; scales > 1 only),
 * 1 Qs = q e^{b - m} (fp16 [B, n_s, h*dkp]), 2 Ks = k e^{m - b} (same shape),
 * 3 v (fp16 [B, n_s, h*dvp]), 5 o (fp16 [B, n_s, h*dvp]), 6 Y (fp16 [B, n_s, d];
 * branches whose output is materialised), 7 fusion weights w (f32 [B, L, n_scales]),
 * 8 U = X Wu^T (f32 [B, L, ldu]): the fusion logits W_fuse x_t in columns
 * 0..n_scales-1 and the low-rank gate input x_t W_g1^T of scale index j in columns
 * 16 + j*rp .. (unpooled rows; a coarse branch uses their block means),
 * 9 gamma = e^{b_last - m} and 10 mid = e^{m} (f32 [B, n_chunks, h*dkp], n_chunks =
 * ceil(n_s / 128)). `scale_index` is ignored for 7 and 8. dkp, dvp and rp (the gate
 * rank rounded up to 16) are padded widths; dims[2] reports the columns. Padding
 * columns hold zeros. A tensor that does not exist gives MSGLA_ERR_INVALID_ARG. */
int msgla_workspace_tensor(const msgla_handle* h, int B, int L, int scale_index, int which,
                           size_t* offset, int dims[3]);

/* ---- token-by-token inference (the notes' item on per-token inference, after the
 * authors' cache): every branch keeps its GLA state, the sum of the tokens of its
 * unfinished block and its latest output; a branch steps once its block of s
 * tokens is complete (the block's mean is its next pooled row, Eq. (8)) and
 * otherwise repeats its latest output, which is the causal hold of Sec. 3.3. The
 * outputs equal those of msgla_forward position by position.
 *
 * Bytes of the decode cache of B sequences (B in [0, 65535]): per branch the state
 * f32 [B, h, dkp, dvp] (dkp = 128 or 256, dvp = d_v rounded up to 128) and, for
 * s > 1, the block sum f32 [B, d] and the latest output f16 [B, d]. The size does
 * not depend on how many tokens have been consumed. */
int msgla_cache_size(const msgla_handle* h, int B, size_t* bytes);

/* Empty the cache (the state before the first token): an asynchronous memset of
 * msgla_cache_size bytes on `stream`. `cache` is a device buffer owned by the
 * caller, 256-byte aligned. */
int msgla_cache_reset(msgla_handle* h, void* cache, int B, void* stream);

/* Bytes of device workspace msgla_step needs for B sequences. */
int msgla_step_workspace_size(const msgla_handle* h, int B, size_t* bytes);

/* Consume token t of each of B sequences and write the layer output at t.
 *   cache  device buffer of msgla_cache_size(h, B) bytes, 256-byte aligned; read
 *          and updated. After msgla_cache_reset it must be fed t = 0, 1, 2, ... in
 *          order: the position decides which branches step ((t + 1) % s == 0).
 *   x      device bf16 [B, d], 16-byte aligned (token t of every sequence).
 *   O      device bf16 [B, d], 16-byte aligned, not overlapping x.
 *   workspace  device buffer of at least msgla_step_workspace_size bytes, 256-byte
 *          aligned, owned by the caller.
 * Asynchronous on `stream`; kernel-side errors are reported by msgla_sync_status.
 * B = 0 launches nothing. A padding mask is not supported here. */
int msgla_step(msgla_handle* h, void* cache, const void* x, int B, long long t, void* O,
               void* workspace, size_t workspace_bytes, void* stream);

/* Kernels that msgla_forward launches for a [B, L, d] input, in launch order, as a
 * comma-separated list written to `names` (NUL-terminated, at most `len` bytes):
 * pool_u | (gate_inputs, [pool]), gate, proj_gemm, [gla_state, gla_scan], gla,
 * [head_norm], [out_gemm_coarse], out_gemm_fused | out_gemm_coarse, hold_fuse.
 * pool_u (one pass over X for the pooled rows, the fusion logits and the gate
 * inputs) runs when every coarse scale is a power of two up to 8; otherwise a
 * GEMM for the gate inputs and a pooling kernel do its work. gla_state and
 * gla_scan appear when long sequences are cut into segments (few sequences: the
 * GLA kernel would fill less than half of the GPU); head_norm when the config
 * enables the head RMS norm. out_gemm_coarse is absent when it runs on the
 * handle's second stream alongside gla (a scale-1 branch, no segments, no head
 * norm, and SMs left free by the GLA CTAs). msgla_forward_profiled records one
 * event per entry. */
int msgla_launch_plan(const msgla_handle* h, int B, int L, char* names, size_t len);

/* Failure-detection testing: with enable != 0, the next forward on this handle
 * runs its chunkwise-GLA kernel with one internal barrier arrival withheld in its
 * first CTA. The warp waiting on it gives up after its bounded wait (about 2 s),
 * the kernel exits normally and msgla_sync_status then returns
 * MSGLA_ERR_DEVICE_TIMEOUT; the output of that forward is undefined. The switch
 * resets itself after one forward; the handle stays usable. No counterpart in the
 * pages (it exercises this library's own bounded waits). */
int msgla_test_skip_arrival(msgla_handle* h, int enable);

/* Static description of an error code. */
const char* msgla_status_string(int status);

/* Message of the last failing call on this thread ("" if none). */
const char* msgla_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* MSGLA_H_ */
