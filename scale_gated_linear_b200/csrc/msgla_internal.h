// msgla_internal.h -- parameter blocks shared by the host side of the C ABI and
// the sm_100a kernels. Not part of the public interface.
#pragma once
#include <cstddef>
#include <cstdint>
#include <utility>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>

namespace msgla {

// Launch with programmatic stream serialisation (the kernel calls griddep_wait
// before reading what earlier kernels wrote): it may start while the previous
// kernel on the stream finishes.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Fixed tile constants.
constexpr int kGemmBM = 128;     // GEMM rows per tile (tcgen05 M)
constexpr int kGemmBK = 64;      // GEMM K per stage (one 128-byte swizzle atom of 16-bit data)
constexpr int kGlaChunk = 128;   // chunk length of the chunkwise GLA kernel
constexpr int kGlaTile = 128;    // value columns per GLA CTA (tcgen05 M of the output MMA)
constexpr int kMaxTasks = 8;     // GEMM tasks per grouped launch
constexpr int kMaxScales = 8;

enum EpiKind : int {
  kEpiProj = 0,      // split columns into q | k | v (fp16) | g (fp32)
  kEpiStoreF16 = 1,  // plain fp16 store
  kEpiFuse = 2,      // O = w_main * acc + sum_coarse w_s * held Y_s  (bf16)
  kEpiProjGate = 3,  // q|k tiles -> decay-scaled Qs | Ks (fp16) from the gate exponents; v tiles fp16
  kEpiStoreF32 = 4,  // plain fp32 store (gate inputs and fusion logits), optionally the fusion weights
};

// One GEMM D[rows x N] = A[rows x K] * B[N x K]^T per batch, tiled 128 x BN.
struct alignas(64) GemmTask {
  CUtensorMap tmA;  // 3D {K, rows, B}, box {64, 128, 1}, 128B swizzle
  CUtensorMap tmB;  // 2D {K, N}, box {64, 128}, 128B swizzle
  // 16-bit outputs, 3D {columns, rows, B}, box {64, 32, 1}, 128B swizzle (TMA stores
  // of 32 rows x 64 columns staged per epilogue warp): kEpiProj q, k, v;
  // kEpiStoreF16 y; kEpiFuse out
  CUtensorMap tmOut[3];
  // kEpiProjGate: Qs and Ks, 3D {nq, rows, B}, box {32, 32, 1}, 64B swizzle;
  // the gate exponents d, 2D {nq, B * rows} fp32, box {32, 32}, 128B swizzle
  CUtensorMap tmQK[2];
  CUtensorMap tmD;
  int rows, m_tiles, n_tiles, N, K, tile_begin, ab_bf16, epi;
  // kEpiProj (columns: q | k | v | g (ng) | fusion logits z (nz, scale-1 branch))
  int nq, nk, nv, ng, nz, ldz;
  __half* q;
  __half* k;
  __half* v;
  float* g;
  float* z;  // [B, rows, ldz] fp32
  const uint8_t* mask;  // [B, rows] valid-token mask of the scale-1 branch or null: padded rows
                        // get zero q | k | v | g (the logits z stay: Eq. (10) reads x_t)
  // kEpiStoreF16
  __half* y;
  // kEpiFuse (rows == L, the branch with scale 1)
  __nv_bfloat16* out;
  const float* zf;     // fusion logits [B, L, ldz] from the projection GEMM
  const float* bfuse;  // [n_scales]
  float* w;            // fusion weights [B, L, n_scales] (written by the n0 == 0 tiles)
  int n_scales, main_index, n_coarse, pad_;
  // A operand produced by a kernel running concurrently (the GLA of this branch
  // on the other stream): loads start once *dep >= dep_target (null: no wait)
  const unsigned long long* dep;
  unsigned long long dep_target;
  int coarse_scale[kMaxScales];
  int coarse_index[kMaxScales];
  int coarse_rows[kMaxScales];
  const __half* coarse_y[kMaxScales];
  // kEpiProjGate. Tiles [0, n_qk) of a batch row tile are q|k tiles: 128 key
  // channels c0.. of one head, the B rows of W_q (CTA rank 0 / columns 0..127)
  // and of W_k (rank 1 / columns 128..255) for the same channels, so that one
  // load of the gate exponents d scales both. Tiles from n_qk on cover the v
  // columns. Outputs: Qs = q 2^d (tmQK[0]), Ks = k 2^-d (tmQK[1]), v (tmOut[2]).
  int n_qk, dkp;
  const float* gd;        // [B, rows, nq] gate exponents d = b - m (launch_gate)
  // with GemmParams::rows_done: this task's counters start at rows_done[done_base],
  // one per (batch element, 128-row block): [done_base + b * ceil(rows / 128) + m0 / 128]
  int done_base, pad2_;
  // kEpiStoreF32: D -> f32 [B, rows, ldf]; with w set, also the fusion weights
  // w = softmax(D[:, 0:n_scales] + bfuse) (columns 0.. hold the fusion logits)
  float* f32;
  int ldf;
  // > 0: tiles from this local index on are 128-column halves of the 256-column
  // tiles that would make up a last, partial wave (two per full tile, half 0
  // then half 1), so that wave keeps up to twice as many CTA pairs busy
  int half_from;
};

// Rows of one 64-column box of held coarse rows staged by the fused output GEMM
// for a 128-row CTA tile and coarse scale s (at most 127 / s + 2 distinct rows,
// rounded up to 8 for the 128-byte swizzle), and whether the boxes of the given
// coarse scales fit the 60 KB region.
inline __host__ __device__ int held_box_rows(int s) { return ((127 / s + 2) + 7) / 8 * 8; }
inline __host__ __device__ bool held_rows_fit(const int* scales, int n) {
  int bytes = 0;
  for (int c = 0; c < n; ++c) bytes += 4 * held_box_rows(scales[c]) * 128;
  return bytes <= 60 * 1024;
}

struct GemmParams {
  GemmTask task[kMaxTasks];
  int n_tasks;
  int total_tiles;
  int* err;
  // non-null: CTA pairs take tiles dynamically from *tile_counter (zero at launch)
  unsigned int* tile_counter;
  // with tile_counter: every CTA adds 1 to *tile_exit when it leaves; the last one
  // sets *tile_counter, *tile_exit and reset64[0, n_reset64) (the counters its
  // tasks waited on) back to zero, so every launch starts from zero and a captured
  // launch replays with the same targets
  unsigned int* tile_exit;
  unsigned long long* reset64;
  int n_reset64;
  // non-null (the forward's projection): after its TMA stores of a kEpiProjGate
  // tile have completed, every epilogue warp adds 1 (release) to the counter of
  // the 128-row block it stored (GemmTask::done_base), so a block is complete at
  // n_tiles * 8 -- the GLA kernel starts on a chunk as soon as its block is
  // counted, instead of waiting for the whole launch
  unsigned long long* rows_done;
};

// Chunkwise GLA over one or more branches.
struct alignas(64) GlaTask {
  CUtensorMap tmQ;  // 3D {h*dkp, n_s, B}, box {64, 128, 1}
  CUtensorMap tmK;  // same shape as tmQ
  CUtensorMap tmV;  // 3D {h*dvp, n_s, B}, box {64, 128, 1}
  CUtensorMap tmO;  // output o: 3D {h*dvp, n_s, B}, box {64, 32, 1} (TMA store)
  const float* gamma;  // [B, n_chunks, h*dkp]: e^{b_last - m} per chunk
  const float* mid;    // [B, n_chunks, h*dkp]: e^{m}, m = b at the chunk's 64th row
  __half* o;           // [B, n_s, h*dvp]
  // sequence segments (long sequences): chunks [s*seg_chunks, (s+1)*seg_chunks)
  float* seg_state;    // [B, h, v_tiles, n_segs, dkp, 128]: end states, then initial states
  float* seg_decay;    // [B, h, v_tiles, n_segs, dkp]: product of the state factors
  int rows, n_chunks, heads, dkp, dvp, v_tiles, cta_begin, seg_chunks, n_segs;
  int signal_done;  // full pass: this task's CTAs add 1 to GlaParams::done[task] when stored
  // with GlaParams::rows_done: the projection's counters of this branch (one per
  // batch element and 128-row chunk, at done_base + b * n_chunks + c) and the
  // count at which a chunk's Qs, Ks and v are all stored
  int done_base;
  unsigned long long done_target;
};

struct GlaParams {
  GlaTask task[kMaxScales];
  int n_tasks;
  int total_ctas;
  float qk_scale;
  int mode;          // 0: full pass; 1: state pass over segments 0..n_segs-2
  int skip_arrival;  // failure-detection tests: CTA 0 omits one barrier arrival
  int* err;
  // full pass only: every CTA of a task with signal_done adds 1 to done[t] once
  // its outputs are stored (release), for a concurrent consumer; every CTA adds
  // 1 to *started when it begins and to *exited when it leaves (null: none)
  unsigned long long* done;
  unsigned long long* started;
  unsigned long long* exited;
  // full pass of an unsegmented forward: the projection's per-chunk counters
  // (GemmParams::rows_done). The kernel then does not wait for the projection
  // launch to finish (no griddepcontrol.wait): a CTA takes an SM as soon as the
  // projection's CTA there has left, and loads chunk c once its counter reaches
  // the task's done_target (bounded wait). Null: wait for the launch.
  const unsigned long long* rows_done;
};
// One warp on a second stream, ordered before a kernel that may only take SMs
// once every CTA of a running GLA launch is resident: waits (bounded) until
// *started reaches target. If that bound runs out -- some GLA CTAs could not be
// resident at once, as on a GPU shared with other work -- it waits instead
// (bounded) until every GLA CTA has left (*exited reaches target), which
// degrades the overlap to the serial order; only if that too runs out does it
// latch kDevTimeout.
cudaError_t launch_wait_started(const unsigned long long* started, const unsigned long long* exited,
                                unsigned long long target, int* err, cudaStream_t st);

// ---------------------------------------------------------------- launchers
// (each returns the cudaError_t of the launch)
// max_pairs > 0 caps the number of CTA pairs of the persistent grid.
cudaError_t launch_gemm(const GemmParams& p, int bn, cudaStream_t st, int max_pairs = 0);
// streaming multiprocessors of the current device
int sm_count();
cudaError_t launch_gla(const GlaParams& p, cudaStream_t st);
// initial state of every segment from the state pass's end states (sequential over segments)
cudaError_t launch_gla_scan(const GlaParams& p, int B, cudaStream_t st);

// pooled rows (fp16) for scales > 1 and fusion weights w = softmax(W_fuse x + b)
struct PoolParams {
  const __nv_bfloat16* X;  // [B, L, d]
  const uint8_t* M;        // [B, L] valid-token mask (nonzero = valid) or null (all valid)
  int B, L, d, n_scales;
  int scales[kMaxScales];
  __half* Xp[kMaxScales];  // [B, n_s, d] or null (scale 1)
  const __nv_bfloat16* Wfuse;  // [n_scales, d]
  const float* bfuse;          // [n_scales]
  float* w;                    // [B, L, n_scales]
  int block_rows;              // least common multiple of the scales > 1 (1 if none)
  int want_w;                  // 1: also the fusion weights (no scale-1 branch)
  int* err;
};
cudaError_t launch_pool_fuse(const PoolParams& p, cudaStream_t st);


// One pass over X per 128-row tile (k_pool.cu): U = X Wu^T (the fusion logits
// and every branch's gate input, fp32 [B, L, ldu]), the pooled rows of every
// coarse scale (powers of two dividing 128) and, with w set, the fusion weights.
constexpr int kPoolUMaxStages = 8;
constexpr int kPoolUBufs = 4;  // TMEM buffers of pooled sums (64 columns each)
struct PoolUParams {
  CUtensorMap tmX;       // X: 3D {d, L, B}, box {64, 128, 1}, bf16, 128B swizzle
  CUtensorMap tmW;       // Wu: 2D {d, ldu}, box {64, ldu}, bf16, 128B swizzle
  const __nv_bfloat16* X;  // [B, L, d] (the tensor map's memory; bulk L2 prefetch)
  const uint8_t* M;      // [B, L] valid-token mask of the pooling, or null
  float* U;              // [B, L, ldu]
  float* w;              // [B, L, n_scales] fusion weights, or null
  const float* bfuse;    // [n_scales]
  int B, L, d, m_tiles, ldu, tmem_cols, pool_col, stages, n_scales;
  int n_coarse;          // coarse branches (scales 2, 4, 8)
  int lvl_branch[4];     // coarse branch of scale 2^l (l = 1..3), or -1
  int slot_base[4];      // first pooling slot (TMEM lane) of scale 2^l
  int rows[kMaxScales];  // pooled rows of each coarse branch
  __half* Xp[kMaxScales];
  int* err;
};
int pool_u_smem_bytes(int ldu, int stages);
cudaError_t launch_pool_u(const PoolUParams& p, cudaStream_t st);

// The gate of Sec. 2.1 per pooled row and key channel, in the form the chunkwise
// GLA kernel takes: with l = log2 alpha = log2(e) logsigmoid(z) / normalizer,
// z = g W_g2^T + b_g (g: the row's low-rank gate input, a coarse branch's the
// mean over its block of the unpooled rows' inputs), b the cumulative sum of l
// over the rows of a 128-row chunk and m = b at its row 63: the exponents
// d = b - m (the projection stores Qs = q 2^d, Ks = k 2^-d), and per chunk
// gamma = 2^{b_127 - m}, mid = 2^{m}.
struct GateBranch {
  const float* Wg2;  // [ldk, rp]
  const float* bg;   // [ldk]
  float* d;          // [B, rows, ldk]
  float* gamma;      // [B, n_chunks, ldk]
  float* mid;        // [B, n_chunks, ldk]
  int rows, n_chunks, ldk, cblocks, ucol, scale, block_begin;
};
struct GateParams {
  GateBranch br[kMaxScales];
  const float* u;        // [B, L, ldu] gate inputs of the unpooled rows
  const uint8_t* mask;   // [B, L] valid-token mask of the pooled means, or null
  int n_branches, total_blocks, L, ldu, rp;
  float inv_normalizer;
  int* err;
  // set to zero before the forward's GLA launch (the GLA exit counter of the
  // overlapped coarse projection; null: none)
  unsigned long long* clear;
  // the projection's per-chunk counters (GemmParams::rows_done), zeroed before the
  // projection launch starts counting (null: none)
  unsigned long long* clear_rows;
  int n_clear_rows;
};
cudaError_t launch_gate(const GateParams& p, cudaStream_t st);

// optional per-head RMS norm of the GLA output, in place:
// o_h <- o_h / sqrt(sum_c o_hc^2 / dv + eps) * w_h (one warp per row and head)
struct HeadNormBranch {
  __half* o;            // [B * rows, heads * dvp]
  const float* w;       // [heads * dvp], zero in the padding columns
  long long rows;       // B * rows
  long long warp_begin;
  int heads;
};
struct HeadNormParams {
  HeadNormBranch br[kMaxScales];
  int n_branches, dvp, dv;
  long long total_warps;
  float eps;
  int* err;
};
cudaError_t launch_head_norm(const HeadNormParams& p, cudaStream_t st);

// hold + fuse from materialised branch outputs (used when no branch has scale 1)
struct HoldFuseParams {
  const __half* Y[kMaxScales];  // [B, n_s, d]
  int scales[kMaxScales];
  int shift[kMaxScales];        // log2(scale) for a power of two, else -1
  int rows[kMaxScales];
  const float* w;               // [B, L, n_scales]
  __nv_bfloat16* out;           // [B, L, d]
  int B, L, d, n_scales;
};
cudaError_t launch_hold_fuse(const HoldFuseParams& p, cudaStream_t st);

// ---------------------------------------------------------------- decode step
// One token of each of B sequences (all at the same position t).
// Coarse branches: buf += x; a branch whose block completes at t writes its fp16
// pooled row xbar = buf / s and clears buf.
struct DecPoolParams {
  const __nv_bfloat16* x;      // [B, d]
  float* buf[kMaxScales];      // [B, d] running sums (null for scale 1)
  __half* xbar[kMaxScales];    // [B, d] pooled row of a branch that steps at t, else null
  int scales[kMaxScales];
  int B, d, n_scales;
  int* err;
};
// One GLA step per (sequence, stepping branch, head, 128 value columns):
// alpha = exp(logsigmoid(g W_g2^T + b_g) / normalizer), S = Diag(alpha) S + k^T v,
// o = qk_scale * q S.
struct DecGlaBranch {
  const __half* q;   // [B, h*dkp]
  const __half* k;   // [B, h*dkp]
  const __half* v;   // [B, h*dvp]
  const float* g;    // [B, rp]
  const float* Wg2;  // [h*dkp, rp]
  const float* bg;   // [h*dkp]
  float* S;          // [B, h, dkp, dvp] state in the cache
  __half* o;         // [B, h*dvp]
  int heads, cta_begin;
};
struct DecGlaParams {
  DecGlaBranch br[kMaxScales];
  int n_branches, total_ctas, dkp, dvp, rp;
  float inv_normalizer, qk_scale;
  int* err;
};
// w = softmax(W_fuse x + b_fuse), O = sum_s w_s Y_s (one CTA per sequence)
struct DecFuseParams {
  const __nv_bfloat16* x;      // [B, d]
  const __nv_bfloat16* Wfuse;  // [n_scales, d]
  const float* bfuse;          // [n_scales]
  const __half* Y[kMaxScales]; // [B, d] latest output of each branch
  __nv_bfloat16* out;          // [B, d]
  int B, d, n_scales;
};
cudaError_t launch_dec_pool(const DecPoolParams& p, cudaStream_t st);
cudaError_t launch_dec_gla(const DecGlaParams& p, cudaStream_t st);
cudaError_t launch_dec_fuse(const DecFuseParams& p, cudaStream_t st);

// bf16 -> fp16 with an overflow count; bf16 -> bf16 copy into a strided block
cudaError_t launch_bf16_to_f16_rows(const __nv_bfloat16* src, int src_ld, int rows, int cols, __half* dst,
                                    int dst_ld, int* overflow, cudaStream_t st);
cudaError_t launch_bf16_copy_rows(const __nv_bfloat16* src, int src_ld, int rows, int cols, __nv_bfloat16* dst,
                                  int dst_ld, cudaStream_t st);

}  // namespace msgla
