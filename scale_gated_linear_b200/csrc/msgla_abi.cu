// msgla_abi.cu -- host side of the C ABI declared in include/msgla.h.
//
// Launch sequence of one forward (MS-GLA reading notes, Sec. 3):
//   1. pool_fuse   pooled rows for every scale s > 1 (fp16) and the fusion
//                  weights w (fp32), one pass over X
//   2. gemm        q | k | v | low-rank gate of every branch (grouped launch)
//   3. gate        log alpha, in-chunk cumulative sums, scaled q/k, chunk decays
//   4. gla         chunkwise GLA of every branch and head (grouped launch)
//   5. gemm        Y^(s) = o W_o^T of the coarse branches (fp16)
//   6. gemm        Y^(1) = o W_o^T of the scale-1 branch fused with the causal
//                  hold of the coarse Y^(s) and the fusion weights -> O (bf16)
//      (without a scale-1 branch: all Y^(s) in step 5, then hold_fuse)
#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/msgla.h"
#include "msgla_internal.h"
#include "sm100_ptx.cuh"

using namespace msgla;

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

#define CUDA_TRY(expr)                                                                                   \
  do {                                                                                                   \
    cudaError_t e_ = (expr);                                                                             \
    if (e_ != cudaSuccess) return fail(MSGLA_ERR_CUDA, "%s failed: %s", #expr, cudaGetErrorString(e_)); \
  } while (0)

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
int ceil_div(int a, int b) { return (a + b - 1) / b; }
int gcd(int a, int b) { return b == 0 ? a : gcd(b, a % b); }

// ---------------------------------------------------------------- tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 16-bit row-major [batch][rows][inner] with a {64, box_rows, 1} box and 128B swizzle.
bool encode_3d(CUtensorMap* m, bool bf16, const void* base, uint64_t inner, uint64_t rows, uint64_t batch,
               uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {inner, rows, batch};
  cuuint64_t strides[2] = {inner * 2, inner * rows * 2};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(base),
            dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
bool encode_2d(CUtensorMap* m, bool bf16, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base),
            dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Output map of the GEMM epilogue: 16-bit [batch][rows][inner], {64, 32, 1} box, 128B swizzle.
bool encode_out_3d(CUtensorMap* m, bool bf16, void* base, uint64_t inner, uint64_t rows, uint64_t batch) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {inner, rows, batch};
  cuuint64_t strides[2] = {inner * 2, inner * rows * 2};
  cuuint32_t box[3] = {64, 32, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, base, dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp16 [batch][rows][inner] with a {32, 32, 1} box and 64B swizzle (32-column
// TMA stores of the gated projection's Qs and Ks).
bool encode_out_3d_32(CUtensorMap* m, void* base, uint64_t inner, uint64_t rows, uint64_t batch) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {inner, rows, batch};
  cuuint64_t strides[2] = {inner * 2, inner * rows * 2};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 row-major [rows][inner] with a {32, 32} box and 128B swizzle (the gate
// exponents one epilogue warp of the gated projection reads).
bool encode_f32_2d_32(CUtensorMap* m, void* base, uint64_t inner, uint64_t rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * 4};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct DeviceGuard {
  int prev = -1;
  bool ok = false;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) == cudaSuccess && cudaSetDevice(dev) == cudaSuccess) ok = true;
  }
  ~DeviceGuard() {
    if (prev >= 0) cudaSetDevice(prev);
  }
};

}  // namespace

// ---------------------------------------------------------------- handle
struct Branch {
  int scale, heads;
  int np;             // packed projection rows: h(2 dkp + dvp) + rp
  void* Bproj;        // [np, d] bf16 (scale 1) or fp16
  float* Wg2p;        // [h dkp, rp]
  float* bgp;         // [h dkp]
  __half* Wop;        // [d, h dvp]
  float* normw;       // [h dvp] head RMS-norm weight (zero padding), when enabled
};

struct msgla_handle {
  msgla_config cfg;
  int device;
  int dkp, dvp, rp, n_scales, main_index, pool_rows;
  int sm_count;  // streaming multiprocessors of the device
  int nzp, ldz;  // fusion-logit rows in the scale-1 packed weights (16) and z row stride
  Branch br[MSGLA_MAX_SCALES];
  // gate inputs and fusion logits of the unpooled rows in one GEMM:
  // U = X Wu^T with Wu [ldu, d] bf16 = [W_fuse (rows 0..n_scales-1, zero to 16);
  // W_g1 of scale index j at rows 16 + j rp ..], ldu = 16 + n_scales rp
  __nv_bfloat16* Wu;
  int ldu;
  __nv_bfloat16* Wfuse;
  float* bfuse;
  int* d_err;  // device error word
  int test_skip_arrival;  // failure-detection tests (msgla_test_skip_arrival)
  // Coarse output projection overlapped with the GLA kernel: a second stream,
  // fork/join events, per-branch GLA completion counters and a GLA start counter
  // (all zero when a forward begins: the overlapped GEMM's last CTA clears them).
  cudaStream_t side;
  cudaEvent_t ev_fork, ev_join;
  unsigned long long* d_gla_done;  // [MSGLA_MAX_SCALES] completion, then the start and exit counters
  unsigned int* d_tiles;           // [2] dynamic tile and exit counters of the overlapped GEMM
  // host-buffer forward: copy streams and events of its pipeline
  cudaStream_t copy_in, copy_out;
  cudaEvent_t ev_start, ev_in, ev_done;
};

namespace {

struct Region {
  size_t off = 0, bytes = 0;
};
struct BranchWs {
  int rows, n_chunks, seg_chunks, n_segs;
  Region seg_state, seg_decay;
  Region Xp, qs, ks, v, gd, gamma, mid, o, Y;
};
struct Workspace {
  BranchWs br[MSGLA_MAX_SCALES];
  Region w, u;
  // the projection's per-chunk completion counters (u64): branch j's at
  // rows_base[j] + b * n_chunks + c
  Region rows_done;
  int rows_base[MSGLA_MAX_SCALES];
  int n_rows_done = 0;
  size_t total = 0;
};

void add(Region& r, size_t& cur, size_t bytes) {
  r.off = cur;
  r.bytes = bytes;
  cur = round_up(cur + bytes, 256);
}

// Chunks per sequence segment of the GLA kernel. One CTA runs each (sequence, head,
// value tile); when those CTAs fill less than half of the GPU, long sequences are
// cut into segments (state pass + scan + full pass) using the shortest segment
// length that still fits all segments of all branches in one wave.
int plan_seg_chunks(const msgla_handle* h, int B, int L) {
  const int vt = h->dvp / kGlaTile;
  long long base = 0;
  int max_nch = 0;
  for (int j = 0; j < h->n_scales; ++j) {
    base += static_cast<long long>(B) * h->br[j].heads * vt;
    max_nch = std::max(max_nch, ceil_div(ceil_div(L, h->br[j].scale), kGlaChunk));
  }
  const int no_split = std::max(max_nch, 1);
  if (2 * base > h->sm_count) return no_split;
  for (int seg = 2; seg < max_nch; ++seg) {
    long long ctas = 0;
    for (int j = 0; j < h->n_scales; ++j)
      ctas += static_cast<long long>(B) * h->br[j].heads * vt *
              ceil_div(ceil_div(ceil_div(L, h->br[j].scale), kGlaChunk), seg);
    if (ctas <= h->sm_count) return seg;
  }
  return no_split;
}

Workspace layout(const msgla_handle* h, int B, int L) {
  Workspace ws;
  size_t cur = 0;
  const int seg_chunks = plan_seg_chunks(h, B, L);
  const size_t BB = static_cast<size_t>(B);
  const int d = h->cfg.d;
  for (int j = 0; j < h->n_scales; ++j) {
    const Branch& b = h->br[j];
    BranchWs& w = ws.br[j];
    w.rows = ceil_div(L, b.scale);
    w.n_chunks = ceil_div(w.rows, kGlaChunk);
    w.seg_chunks = std::max(1, std::min(seg_chunks, w.n_chunks));
    w.n_segs = std::max(1, ceil_div(w.n_chunks, w.seg_chunks));
    const size_t n = BB * w.rows;
    if (b.scale > 1) add(w.Xp, cur, n * d * 2);
    add(w.qs, cur, n * b.heads * h->dkp * 2);
    add(w.ks, cur, n * b.heads * h->dkp * 2);
    add(w.v, cur, n * b.heads * h->dvp * 2);
    add(w.gd, cur, n * b.heads * h->dkp * 4);
    add(w.gamma, cur, BB * w.n_chunks * b.heads * h->dkp * 4);
    add(w.mid, cur, BB * w.n_chunks * b.heads * h->dkp * 4);
    add(w.o, cur, n * b.heads * h->dvp * 2);
    if (j != h->main_index) add(w.Y, cur, n * d * 2);
    if (w.n_segs > 1) {
      const size_t seqs = BB * b.heads * (h->dvp / kGlaTile) * w.n_segs;
      add(w.seg_state, cur, seqs * h->dkp * kGlaTile * 4);
      add(w.seg_decay, cur, seqs * h->dkp * 4);
    }
  }
  add(ws.w, cur, BB * L * h->n_scales * 4);
  add(ws.u, cur, BB * L * h->ldu * 4);
  for (int j = 0; j < h->n_scales; ++j) {
    ws.rows_base[j] = ws.n_rows_done;
    ws.n_rows_done += B * ws.br[j].n_chunks;
  }
  add(ws.rows_done, cur, static_cast<size_t>(ws.n_rows_done) * 8);
  ws.total = cur;
  return ws;
}

int validate(const msgla_config* c) {
  if (!c) return fail(MSGLA_ERR_INVALID_ARG, "config is NULL");
  if (c->d < 64 || c->d > 8192 || c->d % 64)
    return fail(MSGLA_ERR_UNSUPPORTED, "d=%d: must be a multiple of 64 in [64, 8192]", c->d);
  if (c->n_scales < 1 || c->n_scales > MSGLA_MAX_SCALES)
    return fail(MSGLA_ERR_INVALID_ARG, "n_scales=%d outside [1, %d]", c->n_scales, MSGLA_MAX_SCALES);
  int H = 0;
  for (int j = 0; j < c->n_scales; ++j) {
    if (c->scales[j] < 1 || c->scales[j] > 64)
      return fail(MSGLA_ERR_INVALID_ARG, "scales[%d]=%d outside [1, 64]", j, c->scales[j]);
    if (j > 0 && c->scales[j] <= c->scales[j - 1])
      return fail(MSGLA_ERR_INVALID_ARG, "scales must be strictly increasing");
    if (c->heads[j] < 1) return fail(MSGLA_ERR_INVALID_ARG, "heads[%d]=%d must be >= 1", j, c->heads[j]);
    H += c->heads[j];
  }
  if (H > 64) return fail(MSGLA_ERR_UNSUPPORTED, "H=%d heads: at most 64", H);
  if (c->d_k < 1 || c->d_k > 256) return fail(MSGLA_ERR_UNSUPPORTED, "d_k=%d outside [1, 256]", c->d_k);
  if (c->d_v < 1 || c->d_v > 1024) return fail(MSGLA_ERR_UNSUPPORTED, "d_v=%d outside [1, 1024]", c->d_v);
  if (c->gate_rank < 1 || c->gate_rank > 32)
    return fail(MSGLA_ERR_UNSUPPORTED, "gate_rank=%d outside [1, 32]", c->gate_rank);
  if (c->chunk != 0 && c->chunk != kGlaChunk)
    return fail(MSGLA_ERR_UNSUPPORTED, "chunk=%d: the GLA kernel runs 128-row chunks (pass 0 or 128)", c->chunk);
  if (!(c->gate_normalizer > 0.f) || !std::isfinite(c->gate_normalizer))
    return fail(MSGLA_ERR_INVALID_ARG, "gate_normalizer must be finite and > 0");
  if (!std::isfinite(c->qk_scale)) return fail(MSGLA_ERR_INVALID_ARG, "qk_scale must be finite");
  if (c->head_norm != 0 && c->head_norm != 1)
    return fail(MSGLA_ERR_INVALID_ARG, "head_norm=%d: 0 (none) or 1 (RMS norm)", c->head_norm);
  if (c->head_norm && !(c->head_norm_eps > 0.f && std::isfinite(c->head_norm_eps)))
    return fail(MSGLA_ERR_INVALID_ARG, "head_norm_eps must be finite and > 0");
  int lcm = 1;
  for (int j = 0; j < c->n_scales; ++j)
    if (c->scales[j] > 1) lcm = lcm / gcd(lcm, c->scales[j]) * c->scales[j];
  if (lcm > 64)
    return fail(MSGLA_ERR_UNSUPPORTED, "least common multiple of the scales is %d (at most 64)", lcm);
  return MSGLA_OK;
}

void free_handle(msgla_handle* h) {
  if (!h) return;
  for (int j = 0; j < MSGLA_MAX_SCALES; ++j) {
    cudaFree(h->br[j].Bproj);
    cudaFree(h->br[j].Wg2p);
    cudaFree(h->br[j].bgp);
    cudaFree(h->br[j].Wop);
    cudaFree(h->br[j].normw);
  }
  cudaFree(h->Wu);
  cudaFree(h->Wfuse);
  cudaFree(h->bfuse);
  cudaFree(h->d_err);
  cudaFree(h->d_gla_done);
  cudaFree(h->d_tiles);
  for (cudaEvent_t e : {h->ev_start, h->ev_in, h->ev_done})
    if (e) cudaEventDestroy(e);
  if (h->copy_in) cudaStreamDestroy(h->copy_in);
  if (h->copy_out) cudaStreamDestroy(h->copy_out);
  if (h->ev_fork) cudaEventDestroy(h->ev_fork);
  if (h->ev_join) cudaEventDestroy(h->ev_join);
  if (h->side) cudaStreamDestroy(h->side);
  delete h;
}

template <class T>
int dmalloc_zero(T** p, size_t bytes) {
  *p = nullptr;
  CUDA_TRY(cudaMalloc(reinterpret_cast<void**>(p), bytes));
  CUDA_TRY(cudaMemset(*p, 0, bytes));
  return MSGLA_OK;
}

int create_impl(msgla_handle* h, const msgla_weights* w) {
  const msgla_config& c = h->cfg;
  const int d = c.d, dk = c.d_k, dv = c.d_v, r = c.gate_rank;
  int* d_over = nullptr;
  int st = dmalloc_zero(&d_over, sizeof(int));
  if (st) return st;
  struct Free {
    int* p;
    ~Free() { cudaFree(p); }
  } free_over{d_over};
  for (int j = 0; j < h->n_scales; ++j) {
    Branch& b = h->br[j];
    if (!w->Wq[j] || !w->Wk[j] || !w->Wv[j] || !w->Wg1[j] || !w->Wg2[j] || !w->Wo[j])
      return fail(MSGLA_ERR_INVALID_ARG, "weights of scale index %d: NULL pointer", j);
    const int hh = b.heads;
    const bool bf = (b.scale == 1);
    const size_t esz = 2;
    if ((st = dmalloc_zero(&b.Bproj, static_cast<size_t>(b.np) * d * esz))) return st;
    if ((st = dmalloc_zero(&b.Wg2p, static_cast<size_t>(hh) * h->dkp * h->rp * 4))) return st;
    if ((st = dmalloc_zero(&b.bgp, static_cast<size_t>(hh) * h->dkp * 4))) return st;
    if ((st = dmalloc_zero(&b.Wop, static_cast<size_t>(d) * hh * h->dvp * 2))) return st;
    auto put_rows = [&](const void* src, int src_row0, int nrows, int dst_row0) -> cudaError_t {
      const __nv_bfloat16* s = static_cast<const __nv_bfloat16*>(src) + static_cast<size_t>(src_row0) * d;
      if (bf)
        return launch_bf16_copy_rows(s, d, nrows, d,
                                     static_cast<__nv_bfloat16*>(b.Bproj) + static_cast<size_t>(dst_row0) * d, d, 0);
      return launch_bf16_to_f16_rows(s, d, nrows, d, static_cast<__half*>(b.Bproj) + static_cast<size_t>(dst_row0) * d,
                                     d, d_over, 0);
    };
    for (int x = 0; x < hh; ++x) {
      CUDA_TRY(put_rows(w->Wq[j], x * dk, dk, x * h->dkp));
      CUDA_TRY(put_rows(w->Wk[j], x * dk, dk, hh * h->dkp + x * h->dkp));
      CUDA_TRY(put_rows(w->Wv[j], x * dv, dv, 2 * hh * h->dkp + x * h->dvp));
      CUDA_TRY(cudaMemcpy2D(b.Wg2p + static_cast<size_t>(x) * h->dkp * h->rp, h->rp * 4,
                            w->Wg2[j] + static_cast<size_t>(x) * dk * r, r * 4, r * 4, dk, cudaMemcpyDeviceToDevice));
      if (w->bg[j])
        CUDA_TRY(cudaMemcpy(b.bgp + static_cast<size_t>(x) * h->dkp, w->bg[j] + static_cast<size_t>(x) * dk, dk * 4,
                            cudaMemcpyDeviceToDevice));
      CUDA_TRY(launch_bf16_to_f16_rows(static_cast<const __nv_bfloat16*>(w->Wo[j]) + static_cast<size_t>(x) * dv,
                                       hh * dv, d, dv, b.Wop + static_cast<size_t>(x) * h->dvp, hh * h->dvp, d_over,
                                       0));
    }
    if (c.head_norm) {
      if ((st = dmalloc_zero(&b.normw, static_cast<size_t>(hh) * h->dvp * 4))) return st;
      if (w->norm_w[j]) {
        CUDA_TRY(cudaMemcpy2D(b.normw, h->dvp * 4, w->norm_w[j], dv * 4, dv * 4, hh, cudaMemcpyDeviceToDevice));
      } else {
        std::vector<float> ones(static_cast<size_t>(hh) * h->dvp, 0.f);
        for (int x = 0; x < hh; ++x)
          for (int e = 0; e < dv; ++e) ones[static_cast<size_t>(x) * h->dvp + e] = 1.f;
        CUDA_TRY(cudaMemcpy(b.normw, ones.data(), ones.size() * 4, cudaMemcpyHostToDevice));
      }
    }
    CUDA_TRY(put_rows(w->Wg1[j], 0, r, hh * (2 * h->dkp + h->dvp)));
    if (j == h->main_index) {
      if (!w->Wfuse) return fail(MSGLA_ERR_INVALID_ARG, "Wfuse is NULL");
      CUDA_TRY(put_rows(w->Wfuse, 0, h->n_scales, hh * (2 * h->dkp + h->dvp) + h->rp));
    }
  }
  if (!w->Wfuse) return fail(MSGLA_ERR_INVALID_ARG, "Wfuse is NULL");
  // gate inputs and fusion logits of the unpooled rows (one bf16 GEMM over X)
  if ((st = dmalloc_zero(&h->Wu, static_cast<size_t>(h->ldu) * d * 2))) return st;
  CUDA_TRY(launch_bf16_copy_rows(static_cast<const __nv_bfloat16*>(w->Wfuse), d, h->n_scales, d, h->Wu, d, 0));
  for (int j = 0; j < h->n_scales; ++j)
    CUDA_TRY(launch_bf16_copy_rows(static_cast<const __nv_bfloat16*>(w->Wg1[j]), d, r, d,
                                   h->Wu + static_cast<size_t>(16 + j * h->rp) * d, d, 0));
  if ((st = dmalloc_zero(&h->Wfuse, static_cast<size_t>(h->n_scales) * d * 2))) return st;
  if ((st = dmalloc_zero(&h->bfuse, static_cast<size_t>(h->n_scales) * 4))) return st;
  CUDA_TRY(cudaMemcpy(h->Wfuse, w->Wfuse, static_cast<size_t>(h->n_scales) * d * 2, cudaMemcpyDeviceToDevice));
  if (w->bfuse) CUDA_TRY(cudaMemcpy(h->bfuse, w->bfuse, h->n_scales * 4, cudaMemcpyDeviceToDevice));
  if ((st = dmalloc_zero(&h->d_err, sizeof(int)))) return st;
  if ((st = dmalloc_zero(&h->d_gla_done, (MSGLA_MAX_SCALES + 2) * sizeof(unsigned long long)))) return st;
  if ((st = dmalloc_zero(&h->d_tiles, 2 * sizeof(unsigned int)))) return st;
  CUDA_TRY(cudaStreamCreateWithFlags(&h->side, cudaStreamNonBlocking));
  CUDA_TRY(cudaEventCreateWithFlags(&h->ev_fork, cudaEventDisableTiming));
  CUDA_TRY(cudaEventCreateWithFlags(&h->ev_join, cudaEventDisableTiming));
  CUDA_TRY(cudaStreamCreateWithFlags(&h->copy_in, cudaStreamNonBlocking));
  CUDA_TRY(cudaStreamCreateWithFlags(&h->copy_out, cudaStreamNonBlocking));
  CUDA_TRY(cudaEventCreateWithFlags(&h->ev_start, cudaEventDisableTiming));
  CUDA_TRY(cudaEventCreateWithFlags(&h->ev_in, cudaEventDisableTiming));
  CUDA_TRY(cudaEventCreateWithFlags(&h->ev_done, cudaEventDisableTiming));
  CUDA_TRY(cudaDeviceSynchronize());
  int over = 0;
  CUDA_TRY(cudaMemcpy(&over, d_over, sizeof(int), cudaMemcpyDeviceToHost));
  if (over) return fail(MSGLA_ERR_RANGE, "%d weight values exceed the fp16 range (|w| > 65504)", over);
  return MSGLA_OK;
}

// Optional per-launch event recording (msgla_forward_profiled).
struct Recorder {
  void* const* events = nullptr;
  int max_events = 0;
  int n = 0;
  int unmarked = 0;  // launches on the second stream (no event of their own)
  cudaError_t mark(cudaStream_t st) {
    if (!events) return cudaSuccess;
    if (n + 1 >= max_events) return cudaErrorInvalidValue;
    ++n;
    return events[n] ? cudaEventRecord(static_cast<cudaEvent_t>(events[n]), st) : cudaSuccess;
  }
};

// Whether the coarse output projection runs concurrently with the GLA kernel on
// the second stream: with a scale-1 branch, no sequence segments, no head norm,
// and GLA CTAs (one per SM) that leave SMs free. The GEMM starts only once every
// GLA CTA is resident (launch_wait_started) and takes its tiles dynamically, so
// it runs on the SMs the GLA leaves free and on those its coarse-branch CTAs
// release, and it can never keep a GLA CTA from starting.
// MSGLA_SERIAL=1 in the environment keeps every kernel on the caller's stream
// (for profilers that run kernels one at a time, under which the GEMM's wait
// for the resident GLA CTAs could only time out).
bool coarse_overlap(const msgla_handle* h, const Workspace& ws, int B, long long* gla_ctas) {
  static const bool serial = [] {
    const char* e = getenv("MSGLA_SERIAL");
    return e && *e && *e != '0';
  }();
  *gla_ctas = 0;
  if (serial || h->main_index < 0 || h->n_scales < 2 || h->cfg.head_norm) return false;
  long long ctas = 0;
  for (int j = 0; j < h->n_scales; ++j) {
    if (ws.br[j].n_segs > 1) return false;
    ctas += static_cast<long long>(B) * h->br[j].heads * (h->dvp / kGlaTile);
  }
  *gla_ctas = ctas;
  return h->sm_count - ctas >= 2;
}

// Pooling and the gate inputs in one pass over X (k_pool.cu): every coarse scale
// a power of two up to 8 (pooled blocks inside the 128-row tiles) and U at most
// 256 columns wide (one TMA box of Wu).
bool fused_pool(const msgla_handle* h) {
  if (h->ldu > 256) return false;
  for (int j = 0; j < h->n_scales; ++j) {
    const int s = h->br[j].scale;
    if (s != 1 && s != 2 && s != 4 && s != 8) return false;
  }
  return true;
}

int forward_impl(msgla_handle* h, const void* X, int B, int L, void* O, void* wsp, size_t ws_bytes,
                 cudaStream_t st, Recorder* rec = nullptr, const uint8_t* M = nullptr) {
  Recorder none;
  if (!rec) rec = &none;
  if (rec->events) {
    if (rec->max_events < 1) return fail(MSGLA_ERR_INVALID_ARG, "max_events < 1");
    if (rec->events[0]) CUDA_TRY(cudaEventRecord(static_cast<cudaEvent_t>(rec->events[0]), st));
  }
  const msgla_config& c = h->cfg;
  const int d = c.d;
  const Workspace ws = layout(h, B, L);
  if (!wsp || ws_bytes < ws.total)
    return fail(MSGLA_ERR_WORKSPACE, "workspace of %zu bytes, %zu needed", ws_bytes, ws.total);
  if (reinterpret_cast<uintptr_t>(wsp) % 256) return fail(MSGLA_ERR_WORKSPACE, "workspace not 256-byte aligned");
  uint8_t* base = static_cast<uint8_t*>(wsp);
  auto at = [&](const Region& r) { return static_cast<void*>(base + r.off); };
  const int ns = h->n_scales;

  static thread_local GemmParams gp;
  // 1-2. gate inputs and fusion logits of the unpooled rows, U = X Wu^T (fp32
  // [B, L, ldu]): every branch's low-rank gate input is a column block of U (a
  // coarse branch's is the mean over its pooled block, pooling being linear),
  // and the fusion logits z_t = W_fuse x_t of Eq. (10) are its first columns;
  // without a scale-1 branch the fusion weights too. Pooled rows of the coarse
  // branches (Eq. (8)). One pass over X when every coarse scale is a power of two
  // up to 8 (pool_u); otherwise a GEMM for U and a pooling kernel.
  if (fused_pool(h)) {
    PoolUParams q{};
    if (!encode_3d(&q.tmX, true, X, d, L, B, 128) || !encode_2d(&q.tmW, true, h->Wu, d, h->ldu, h->ldu))
      return fail(MSGLA_ERR_CUDA, "cuTensorMapEncodeTiled failed (pooling and gate inputs)");
    q.X = static_cast<const __nv_bfloat16*>(X);
    q.M = M;
    q.U = static_cast<float*>(at(ws.u));
    q.w = h->main_index < 0 ? static_cast<float*>(at(ws.w)) : nullptr;
    q.bfuse = h->bfuse;
    q.B = B;
    q.L = L;
    q.d = d;
    q.m_tiles = ceil_div(L, 128);
    q.ldu = h->ldu;
    // TMEM: U in [0, ldu rounded up to a power of two), then two 64-column
    // buffers of pooled sums
    q.pool_col = 32;
    while (q.pool_col < h->ldu) q.pool_col *= 2;
    q.tmem_cols = 32;
    while (q.tmem_cols < q.pool_col + 64 * kPoolUBufs) q.tmem_cols *= 2;
    const int stage_bytes = 128 * 128 + h->ldu * 128;
    q.stages = std::min(kPoolUMaxStages, (192 * 1024 - 32 * 1024) / stage_bytes);
    q.n_scales = ns;
    for (int l = 0; l < 4; ++l) q.lvl_branch[l] = -1;
    int slot = 0;
    for (int l = 1; l <= 3; ++l) {
      for (int j = 0; j < ns; ++j) {
        if (h->br[j].scale != (1 << l)) continue;
        q.lvl_branch[l] = q.n_coarse;
        q.slot_base[l] = slot;
        slot += 128 >> l;
        q.rows[q.n_coarse] = ws.br[j].rows;
        q.Xp[q.n_coarse] = static_cast<__half*>(at(ws.br[j].Xp));
        ++q.n_coarse;
      }
    }
    q.err = h->d_err;
    CUDA_TRY(launch_pool_u(q, st));
    CUDA_TRY(rec->mark(st));
  } else {
    memset(&gp, 0, sizeof(gp));
    gp.err = h->d_err;
    GemmTask& t = gp.task[0];
    if (!encode_3d(&t.tmA, true, X, d, L, B, kGemmBM) || !encode_2d(&t.tmB, true, h->Wu, d, h->ldu, 128))
      return fail(MSGLA_ERR_CUDA, "cuTensorMapEncodeTiled failed (gate inputs)");
    t.rows = L;
    t.m_tiles = ceil_div(L, kGemmBM);
    t.n_tiles = ceil_div(h->ldu, 256);
    t.N = h->ldu;
    t.K = d;
    t.tile_begin = 0;
    t.ab_bf16 = 1;
    t.epi = kEpiStoreF32;
    t.f32 = static_cast<float*>(at(ws.u));
    t.ldf = h->ldu;
    t.n_scales = ns;
    t.bfuse = h->bfuse;
    t.w = h->main_index < 0 ? static_cast<float*>(at(ws.w)) : nullptr;
    gp.n_tasks = 1;
    gp.total_tiles = B * t.m_tiles * t.n_tiles;
    CUDA_TRY(launch_gemm(gp, 256, st));
    CUDA_TRY(rec->mark(st));
    PoolParams pp{};
    pp.X = static_cast<const __nv_bfloat16*>(X);
    pp.M = M;
    pp.B = B;
    pp.L = L;
    pp.d = d;
    pp.n_scales = ns;
    for (int j = 0; j < ns; ++j) {
      pp.scales[j] = h->br[j].scale;
      pp.Xp[j] = h->br[j].scale > 1 ? static_cast<__half*>(at(ws.br[j].Xp)) : nullptr;
    }
    pp.Wfuse = h->Wfuse;
    pp.bfuse = h->bfuse;
    pp.w = static_cast<float*>(at(ws.w));
    pp.block_rows = h->pool_rows;
    pp.want_w = 0;
    pp.err = h->d_err;
    if (h->pool_rows > 1) {
      CUDA_TRY(launch_pool_fuse(pp, st));
      CUDA_TRY(rec->mark(st));
    }
  }

  // 3. the gate (one launch over all branches): exponents d = b - m per pooled
  // row and key channel (b the cumulative sum of log2 alpha over a 128-row
  // chunk, m its value at row 63) and the chunk decays gamma, mid
  {
    GateParams g{};
    int blocks = 0;
    for (int j = 0; j < ns; ++j) {
      const Branch& b = h->br[j];
      const BranchWs& bw = ws.br[j];
      GateBranch& q = g.br[j];
      q.Wg2 = b.Wg2p;
      q.bg = b.bgp;
      q.d = static_cast<float*>(at(bw.gd));
      q.gamma = static_cast<float*>(at(bw.gamma));
      q.mid = static_cast<float*>(at(bw.mid));
      q.rows = bw.rows;
      q.n_chunks = bw.n_chunks;
      q.ldk = b.heads * h->dkp;
      q.cblocks = ceil_div(q.ldk, 256);
      q.ucol = 16 + j * h->rp;
      q.scale = b.scale;
      q.block_begin = blocks;
      blocks += B * bw.n_chunks * 2 * q.cblocks;
    }
    g.u = static_cast<const float*>(at(ws.u));
    g.mask = M;
    g.n_branches = ns;
    g.total_blocks = blocks;
    g.L = L;
    g.ldu = h->ldu;
    g.rp = h->rp;
    g.inv_normalizer = 1.f / c.gate_normalizer;
    g.err = h->d_err;
    g.clear = h->d_gla_done + MSGLA_MAX_SCALES + 1;  // GLA exit counter
    g.clear_rows = static_cast<unsigned long long*>(at(ws.rows_done));
    g.n_clear_rows = ws.n_rows_done;
    CUDA_TRY(launch_gate(g, st));
    CUDA_TRY(rec->mark(st));
  }

  // 4. projections (grouped over branches): Qs = q 2^d, Ks = k 2^-d and v (fp16)
  memset(&gp, 0, sizeof(gp));
  gp.err = h->d_err;
  int tiles = 0;
  for (int j = 0; j < ns; ++j) {
    const Branch& b = h->br[j];
    const BranchWs& bw = ws.br[j];
    GemmTask& t = gp.task[j];
    const bool bf = (b.scale == 1);
    if (!encode_3d(&t.tmA, bf, bf ? X : at(bw.Xp), d, bw.rows, B, kGemmBM) ||
        !encode_2d(&t.tmB, bf, b.Bproj, d, b.np, 128))
      return fail(MSGLA_ERR_CUDA, "cuTensorMapEncodeTiled failed (projection, scale %d)", b.scale);
    t.rows = bw.rows;
    t.nq = t.nk = b.heads * h->dkp;
    t.nv = b.heads * h->dvp;
    t.ng = h->rp;
    t.n_qk = b.heads * (h->dkp / 128);
    t.m_tiles = ceil_div(bw.rows, kGemmBM);
    t.N = t.nq + t.nk + t.nv;
    t.n_tiles = t.n_qk + ceil_div(t.nv, 256);
    t.K = d;
    t.tile_begin = tiles;
    t.ab_bf16 = bf ? 1 : 0;
    t.epi = kEpiProjGate;
    t.dkp = h->dkp;
    t.done_base = ws.rows_base[j];
    t.gd = static_cast<const float*>(at(bw.gd));
    t.mask = bf ? M : nullptr;
    if (!encode_f32_2d_32(&t.tmD, at(bw.gd), t.nq, static_cast<uint64_t>(B) * bw.rows) ||
        !encode_out_3d_32(&t.tmQK[0], at(bw.qs), t.nq, bw.rows, B) ||
        !encode_out_3d_32(&t.tmQK[1], at(bw.ks), t.nk, bw.rows, B) ||
        !encode_out_3d(&t.tmOut[2], false, at(bw.v), t.nv, bw.rows, B))
      return fail(MSGLA_ERR_CUDA, "cuTensorMapEncodeTiled failed (projection outputs, scale %d)", b.scale);
    tiles += B * t.m_tiles * t.n_tiles;
  }
  gp.n_tasks = ns;
  gp.total_tiles = tiles;
  // an unsegmented GLA starts each chunk once the projection has counted its rows
  bool any_seg = false;
  for (int j = 0; j < ns; ++j) any_seg |= ws.br[j].n_segs > 1;
  if (!any_seg) gp.rows_done = static_cast<unsigned long long*>(at(ws.rows_done));
  CUDA_TRY(launch_gemm(gp, 256, st));
  CUDA_TRY(rec->mark(st));

  // 5. chunkwise GLA (grouped over branches; longest sequences first). Long
  // sequences with few CTAs run as segments: a state pass over all but the last
  // segment, a scan for the segments' initial states, then the full pass.
  static thread_local GlaParams lp;
  memset(&lp, 0, sizeof(lp));
  lp.err = h->d_err;
  lp.qk_scale = c.qk_scale;
  bool segmented = false;
  for (int j = 0; j < ns; ++j) {
    const Branch& b = h->br[j];
    const BranchWs& bw = ws.br[j];
    GlaTask& t = lp.task[j];
    if (!encode_3d(&t.tmQ, false, at(bw.qs), b.heads * h->dkp, bw.rows, B, kGlaChunk) ||
        !encode_3d(&t.tmK, false, at(bw.ks), b.heads * h->dkp, bw.rows, B, kGlaChunk) ||
        !encode_3d(&t.tmV, false, at(bw.v), b.heads * h->dvp, bw.rows, B, kGlaChunk) ||
        !encode_out_3d(&t.tmO, false, at(bw.o), b.heads * h->dvp, bw.rows, B))
      return fail(MSGLA_ERR_CUDA, "cuTensorMapEncodeTiled failed (gla, scale %d)", b.scale);
    t.gamma = static_cast<const float*>(at(bw.gamma));
    t.mid = static_cast<const float*>(at(bw.mid));
    t.o = static_cast<__half*>(at(bw.o));
    t.rows = bw.rows;
    t.n_chunks = bw.n_chunks;
    t.heads = b.heads;
    t.dkp = h->dkp;
    t.dvp = h->dvp;
    t.v_tiles = h->dvp / kGlaTile;
    t.seg_chunks = bw.seg_chunks;
    t.n_segs = bw.n_segs;
    t.done_base = ws.rows_base[j];
    t.done_target = 8ull * gp.task[j].n_tiles;  // every epilogue warp of every N tile
    if (bw.n_segs > 1) {
      t.seg_state = static_cast<float*>(at(bw.seg_state));
      t.seg_decay = static_cast<float*>(at(bw.seg_decay));
      segmented = true;
    }
  }
  lp.n_tasks = ns;
  if (segmented) {
    static thread_local GlaParams sp;
    sp = lp;
    sp.mode = 1;
    int nt = 0, sctas = 0;
    for (int j = 0; j < ns; ++j) {
      if (lp.task[j].n_segs < 2) continue;
      sp.task[nt] = lp.task[j];
      sp.task[nt].cta_begin = sctas;
      sctas += B * lp.task[j].heads * lp.task[j].v_tiles * (lp.task[j].n_segs - 1);
      ++nt;
    }
    sp.n_tasks = nt;
    sp.total_ctas = sctas;
    CUDA_TRY(launch_gla(sp, st));
    CUDA_TRY(rec->mark(st));
    CUDA_TRY(launch_gla_scan(sp, B, st));
    CUDA_TRY(rec->mark(st));
  }
  int ctas = 0;
  for (int j = 0; j < ns; ++j) {
    lp.task[j].cta_begin = ctas;
    ctas += B * lp.task[j].heads * lp.task[j].v_tiles * lp.task[j].n_segs;
  }
  lp.total_ctas = ctas;
  lp.mode = 0;
  lp.rows_done = gp.rows_done;
  lp.skip_arrival = h->test_skip_arrival;
  h->test_skip_arrival = 0;
  long long gla_ctas = 0;
  const bool overlap = coarse_overlap(h, ws, B, &gla_ctas);
  if (overlap) {
    // the second stream starts once the projection is done, alongside the GLA; the
    // coarse branches' CTAs signal their stored outputs to it. It cannot fork
    // earlier: its first kernel (one warp waiting for the GLA's CTAs) would hold an
    // SM that one of the projection's CTA pairs needs (they take every SM), and
    // that pair would run its tiles alone after the GLA had started
    lp.done = h->d_gla_done;
    lp.started = h->d_gla_done + MSGLA_MAX_SCALES;
    lp.exited = h->d_gla_done + MSGLA_MAX_SCALES + 1;
    for (int j = 0; j < ns; ++j) lp.task[j].signal_done = j != h->main_index;
    CUDA_TRY(cudaEventRecord(h->ev_fork, st));
  }
  CUDA_TRY(launch_gla(lp, st));
  CUDA_TRY(rec->mark(st));

  // 5b. optional per-head RMS norm of the GLA output (in place)
  if (c.head_norm) {
    HeadNormParams np{};
    long long warps = 0;
    for (int j = 0; j < ns; ++j) {
      HeadNormBranch& q = np.br[j];
      q.o = static_cast<__half*>(at(ws.br[j].o));
      q.w = h->br[j].normw;
      q.rows = static_cast<long long>(B) * ws.br[j].rows;
      q.heads = h->br[j].heads;
      q.warp_begin = warps;
      warps += q.rows * q.heads;
    }
    np.n_branches = ns;
    np.total_warps = warps;
    np.dvp = h->dvp;
    np.dv = c.d_v;
    np.eps = c.head_norm_eps;
    np.err = h->d_err;
    CUDA_TRY(launch_head_norm(np, st));
    CUDA_TRY(rec->mark(st));
  }

  // 6. coarse branches: Y^(s) = o W_o^T (fp16). Overlapped with the GLA, the
  // branches with the fewest chunks (largest scale) come first: their GLA CTAs
  // finish first.
  memset(&gp, 0, sizeof(gp));
  gp.err = h->d_err;
  tiles = 0;
  int nt = 0;
  for (int jj = 0; jj < ns; ++jj) {
    const int j = overlap ? ns - 1 - jj : jj;
    if (j == h->main_index) continue;
    const Branch& b = h->br[j];
    const BranchWs& bw = ws.br[j];
    GemmTask& t = gp.task[nt++];
    if (!encode_3d(&t.tmA, false, at(bw.o), b.heads * h->dvp, bw.rows, B, kGemmBM) ||
        !encode_2d(&t.tmB, false, b.Wop, b.heads * h->dvp, d, 128))
      return fail(MSGLA_ERR_CUDA, "cuTensorMapEncodeTiled failed (output, scale %d)", b.scale);
    t.rows = bw.rows;
    t.m_tiles = ceil_div(bw.rows, kGemmBM);
    t.n_tiles = ceil_div(d, 256);
    t.N = d;
    t.K = b.heads * h->dvp;
    t.tile_begin = tiles;
    t.ab_bf16 = 0;
    t.epi = kEpiStoreF16;
    t.y = static_cast<__half*>(at(bw.Y));
    if (!encode_out_3d(&t.tmOut[0], false, t.y, d, bw.rows, B))
      return fail(MSGLA_ERR_CUDA, "cuTensorMapEncodeTiled failed (output store, scale %d)", b.scale);
    if (overlap) {
      t.dep = h->d_gla_done + j;
      t.dep_target = static_cast<unsigned long long>(B) * b.heads * (h->dvp / kGlaTile);  // its GLA CTAs
    }
    tiles += B * t.m_tiles * t.n_tiles;
  }
  if (nt > 0) {
    gp.n_tasks = nt;
    gp.total_tiles = tiles;
    if (overlap) {
      CUDA_TRY(cudaStreamWaitEvent(h->side, h->ev_fork, 0));
      CUDA_TRY(launch_wait_started(h->d_gla_done + MSGLA_MAX_SCALES, h->d_gla_done + MSGLA_MAX_SCALES + 1,
                                   static_cast<unsigned long long>(gla_ctas),
                                   h->d_err, h->side));
      // the GEMM's last CTA clears the tile, start and completion counters (the
      // scale-1 GLA CTAs may still be running then: their exit counter is
      // cleared by the next forward's gate kernel instead)
      gp.tile_counter = h->d_tiles;
      gp.tile_exit = h->d_tiles + 1;
      gp.reset64 = h->d_gla_done;
      gp.n_reset64 = MSGLA_MAX_SCALES + 1;
      CUDA_TRY(launch_gemm(gp, 256, h->side));
      rec->unmarked += 2;
      CUDA_TRY(cudaEventRecord(h->ev_join, h->side));
      CUDA_TRY(cudaStreamWaitEvent(st, h->ev_join, 0));
    } else {
      CUDA_TRY(launch_gemm(gp, 256, st));
      CUDA_TRY(rec->mark(st));
    }
  }

  // 7. scale-1 branch fused with hold + fusion, or the stand-alone hold + fusion
  if (h->main_index >= 0) {
    memset(&gp, 0, sizeof(gp));
    gp.err = h->d_err;
    const int j = h->main_index;
    const Branch& b = h->br[j];
    const BranchWs& bw = ws.br[j];
    GemmTask& t = gp.task[0];
    if (!encode_3d(&t.tmA, false, at(bw.o), b.heads * h->dvp, bw.rows, B, kGemmBM) ||
        !encode_2d(&t.tmB, false, b.Wop, b.heads * h->dvp, d, 128))
      return fail(MSGLA_ERR_CUDA, "cuTensorMapEncodeTiled failed (output, scale 1)");
    t.rows = bw.rows;
    t.m_tiles = ceil_div(bw.rows, kGemmBM);
    t.n_tiles = ceil_div(d, 256);
    t.N = d;
    t.K = b.heads * h->dvp;
    t.tile_begin = 0;
    t.ab_bf16 = 0;
    t.epi = kEpiFuse;
    t.out = static_cast<__nv_bfloat16*>(O);
    if (!encode_out_3d(&t.tmOut[0], true, O, d, L, B))
      return fail(MSGLA_ERR_CUDA, "cuTensorMapEncodeTiled failed (layer output)");
    t.zf = static_cast<const float*>(at(ws.u));  // fusion logits: columns 0.. of U
    t.ldz = h->ldu;
    t.bfuse = h->bfuse;
    t.w = static_cast<float*>(at(ws.w));
    t.n_scales = ns;
    t.main_index = j;
    int nc = 0;
    for (int q = 0; q < ns; ++q) {
      if (q == j) continue;
      t.coarse_scale[nc] = h->br[q].scale;
      t.coarse_index[nc] = q;
      t.coarse_rows[nc] = ws.br[q].rows;
      t.coarse_y[nc] = static_cast<const __half*>(at(ws.br[q].Y));
      ++nc;
    }
    t.n_coarse = nc;
    // held coarse rows of a CTA tile, staged by TMA in the fused GEMM: one
    // 64-column box of held_box_rows(s) rows per load (rows before the first
    // block and past the end read as zero)
    if (nc >= 1 && nc <= 2 && held_rows_fit(t.coarse_scale, nc)) {
      for (int c = 0; c < nc; ++c) {
        EncodeTiledFn fn = encode_fn();
        cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(t.coarse_rows[c]),
                              static_cast<cuuint64_t>(B)};
        cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(d) * t.coarse_rows[c] * 2};
        cuuint32_t box[3] = {64, static_cast<cuuint32_t>(held_box_rows(t.coarse_scale[c])), 1};
        cuuint32_t es[3] = {1, 1, 1};
        if (!fn || fn(&t.tmOut[1 + c], CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<__half*>(t.coarse_y[c]), dims,
                      strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
          return fail(MSGLA_ERR_CUDA, "cuTensorMapEncodeTiled failed (held coarse rows, scale %d)", t.coarse_scale[c]);
      }
    }
    gp.n_tasks = 1;
    gp.total_tiles = B * t.m_tiles * t.n_tiles;
    CUDA_TRY(launch_gemm(gp, 256, st));
    CUDA_TRY(rec->mark(st));
  } else {
    HoldFuseParams hp{};
    for (int j = 0; j < ns; ++j) {
      hp.Y[j] = static_cast<const __half*>(at(ws.br[j].Y));
      hp.scales[j] = h->br[j].scale;
      hp.shift[j] = -1;
      for (int k = 0; k < 31; ++k)
        if ((1 << k) == hp.scales[j]) hp.shift[j] = k;
      hp.rows[j] = ws.br[j].rows;
    }
    hp.w = static_cast<const float*>(at(ws.w));
    hp.out = static_cast<__nv_bfloat16*>(O);
    hp.B = B;
    hp.L = L;
    hp.d = d;
    hp.n_scales = ns;
    CUDA_TRY(launch_hold_fuse(hp, st));
    CUDA_TRY(rec->mark(st));
  }
  return MSGLA_OK;
}

// ---------------------------------------------------------------- decode step
// Cache (caller-owned, zeroed by msgla_cache_reset), per branch j:
//   S fp32 [B, h, dkp, dvp] GLA state; for s > 1 also buf fp32 [B, d] (sum of the
//   tokens of the unfinished block) and Y fp16 [B, d] (latest branch output).
struct CacheLayout {
  Region S[MSGLA_MAX_SCALES], buf[MSGLA_MAX_SCALES], Y[MSGLA_MAX_SCALES];
  size_t total = 0;
};
CacheLayout cache_layout(const msgla_handle* h, int B) {
  CacheLayout c;
  size_t cur = 0;
  const size_t BB = static_cast<size_t>(B);
  for (int j = 0; j < h->n_scales; ++j) {
    add(c.S[j], cur, BB * h->br[j].heads * h->dkp * h->dvp * 4);
    if (h->br[j].scale > 1) {
      add(c.buf[j], cur, BB * h->cfg.d * 4);
      add(c.Y[j], cur, BB * h->cfg.d * 2);
    }
  }
  c.total = cur;
  return c;
}

// Step workspace: per branch the pooled row (s > 1), q, k, v, g, o; Y of the scale-1 branch.
struct StepLayout {
  Region xbar[MSGLA_MAX_SCALES], q[MSGLA_MAX_SCALES], k[MSGLA_MAX_SCALES], v[MSGLA_MAX_SCALES],
      g[MSGLA_MAX_SCALES], o[MSGLA_MAX_SCALES];
  Region Y1;
  size_t total = 0;
};
StepLayout step_layout(const msgla_handle* h, int B) {
  StepLayout w;
  size_t cur = 0;
  const size_t BB = static_cast<size_t>(B);
  for (int j = 0; j < h->n_scales; ++j) {
    const int hh = h->br[j].heads;
    if (h->br[j].scale > 1) add(w.xbar[j], cur, BB * h->cfg.d * 2);
    add(w.q[j], cur, BB * hh * h->dkp * 2);
    add(w.k[j], cur, BB * hh * h->dkp * 2);
    add(w.v[j], cur, BB * hh * h->dvp * 2);
    add(w.g[j], cur, BB * h->rp * 4);
    add(w.o[j], cur, BB * hh * h->dvp * 2);
  }
  if (h->main_index >= 0) add(w.Y1, cur, BB * h->cfg.d * 2);
  w.total = cur;
  return w;
}

int step_impl(msgla_handle* h, void* cache, const void* x, int B, long long t, void* O, void* wsp,
              cudaStream_t st) {
  const msgla_config& c = h->cfg;
  const int d = c.d, ns = h->n_scales;
  const CacheLayout cl = cache_layout(h, B);
  const StepLayout sl = step_layout(h, B);
  uint8_t* cb = static_cast<uint8_t*>(cache);
  uint8_t* wb = static_cast<uint8_t*>(wsp);
  auto cat = [&](const Region& r) { return static_cast<void*>(cb + r.off); };
  auto wat = [&](const Region& r) { return static_cast<void*>(wb + r.off); };
  bool fires[MSGLA_MAX_SCALES];
  bool any_fires = false;
  for (int j = 0; j < ns; ++j) {
    fires[j] = (t + 1) % h->br[j].scale == 0;  // the branch's block ends at this token
    any_fires |= fires[j];
  }

  // 1. running block sums of the coarse branches; pooled rows of those that step
  if (h->main_index < 0 || ns > 1) {
    DecPoolParams pp{};
    pp.x = static_cast<const __nv_bfloat16*>(x);
    pp.B = B;
    pp.d = d;
    pp.n_scales = ns;
    pp.err = h->d_err;
    for (int j = 0; j < ns; ++j) {
      pp.scales[j] = h->br[j].scale;
      if (h->br[j].scale == 1) continue;
      pp.buf[j] = static_cast<float*>(cat(cl.buf[j]));
      pp.xbar[j] = fires[j] ? static_cast<__half*>(wat(sl.xbar[j])) : nullptr;
    }
    CUDA_TRY(launch_dec_pool(pp, st));
  }

  if (any_fires) {
    // 2. projections of the stepping branches (grouped GEMM, the B sequences as rows)
    static thread_local GemmParams gp;
    memset(&gp, 0, sizeof(gp));
    gp.err = h->d_err;
    int tiles = 0, nt = 0;
    for (int j = 0; j < ns; ++j) {
      if (!fires[j]) continue;
      const Branch& b = h->br[j];
      const bool bf = (b.scale == 1);
      GemmTask& tk = gp.task[nt++];
      if (!encode_3d(&tk.tmA, bf, bf ? x : wat(sl.xbar[j]), d, B, 1, kGemmBM) ||
          !encode_2d(&tk.tmB, bf, b.Bproj, d, b.np, 128))
        return fail(MSGLA_ERR_CUDA, "cuTensorMapEncodeTiled failed (step projection, scale %d)", b.scale);
      tk.rows = B;
      tk.m_tiles = ceil_div(B, kGemmBM);
      tk.n_tiles = ceil_div(b.np, 256);
      tk.N = b.np;
      tk.K = d;
      tk.tile_begin = tiles;
      tk.ab_bf16 = bf ? 1 : 0;
      tk.epi = kEpiProj;
      tk.nq = tk.nk = b.heads * h->dkp;
      tk.nv = b.heads * h->dvp;
      tk.ng = h->rp;
      tk.nz = 0;  // the step forms the fusion logits itself
      tk.ldz = h->ldz;
      tk.q = static_cast<__half*>(wat(sl.q[j]));
      tk.k = static_cast<__half*>(wat(sl.k[j]));
      tk.v = static_cast<__half*>(wat(sl.v[j]));
      tk.g = static_cast<float*>(wat(sl.g[j]));
      if (!encode_out_3d(&tk.tmOut[0], false, tk.q, tk.nq, B, 1) ||
          !encode_out_3d(&tk.tmOut[1], false, tk.k, tk.nk, B, 1) ||
          !encode_out_3d(&tk.tmOut[2], false, tk.v, tk.nv, B, 1))
        return fail(MSGLA_ERR_CUDA, "cuTensorMapEncodeTiled failed (step projection outputs, scale %d)", b.scale);
      tiles += tk.m_tiles * tk.n_tiles;
    }
    gp.n_tasks = nt;
    gp.total_tiles = tiles;
    CUDA_TRY(launch_gemm(gp, 256, st));

    // 3. one GLA step per stepping branch and head
    DecGlaParams dp{};
    int ctas = 0, nb = 0;
    for (int j = 0; j < ns; ++j) {
      if (!fires[j]) continue;
      const Branch& b = h->br[j];
      DecGlaBranch& q = dp.br[nb++];
      q.q = static_cast<const __half*>(wat(sl.q[j]));
      q.k = static_cast<const __half*>(wat(sl.k[j]));
      q.v = static_cast<const __half*>(wat(sl.v[j]));
      q.g = static_cast<const float*>(wat(sl.g[j]));
      q.Wg2 = b.Wg2p;
      q.bg = b.bgp;
      q.S = static_cast<float*>(cat(cl.S[j]));
      q.o = static_cast<__half*>(wat(sl.o[j]));
      q.heads = b.heads;
      q.cta_begin = ctas;
      ctas += B * b.heads * (h->dvp / kGlaTile);
    }
    dp.n_branches = nb;
    dp.total_ctas = ctas;
    dp.dkp = h->dkp;
    dp.dvp = h->dvp;
    dp.rp = h->rp;
    dp.inv_normalizer = 1.f / c.gate_normalizer;
    dp.qk_scale = c.qk_scale;
    dp.err = h->d_err;
    CUDA_TRY(launch_dec_gla(dp, st));

    // 3b. optional per-head RMS norm of o
    if (c.head_norm) {
      HeadNormParams np{};
      long long warps = 0;
      int n = 0;
      for (int j = 0; j < ns; ++j) {
        if (!fires[j]) continue;
        HeadNormBranch& q = np.br[n++];
        q.o = static_cast<__half*>(wat(sl.o[j]));
        q.w = h->br[j].normw;
        q.rows = B;
        q.heads = h->br[j].heads;
        q.warp_begin = warps;
        warps += q.rows * q.heads;
      }
      np.n_branches = n;
      np.total_warps = warps;
      np.dvp = h->dvp;
      np.dv = c.d_v;
      np.eps = c.head_norm_eps;
      np.err = h->d_err;
      CUDA_TRY(launch_head_norm(np, st));
    }

    // 4. output projections: coarse outputs replace the cached ones
    memset(&gp, 0, sizeof(gp));
    gp.err = h->d_err;
    tiles = nt = 0;
    for (int j = 0; j < ns; ++j) {
      if (!fires[j]) continue;
      const Branch& b = h->br[j];
      GemmTask& tk = gp.task[nt++];
      if (!encode_3d(&tk.tmA, false, wat(sl.o[j]), b.heads * h->dvp, B, 1, kGemmBM) ||
          !encode_2d(&tk.tmB, false, b.Wop, b.heads * h->dvp, d, 128))
        return fail(MSGLA_ERR_CUDA, "cuTensorMapEncodeTiled failed (step output, scale %d)", b.scale);
      tk.rows = B;
      tk.m_tiles = ceil_div(B, kGemmBM);
      tk.n_tiles = ceil_div(d, 256);
      tk.N = d;
      tk.K = b.heads * h->dvp;
      tk.tile_begin = tiles;
      tk.ab_bf16 = 0;
      tk.epi = kEpiStoreF16;
      tk.y = static_cast<__half*>(b.scale == 1 ? wat(sl.Y1) : cat(cl.Y[j]));
      if (!encode_out_3d(&tk.tmOut[0], false, tk.y, d, B, 1))
        return fail(MSGLA_ERR_CUDA, "cuTensorMapEncodeTiled failed (step output store, scale %d)", b.scale);
      tiles += tk.m_tiles * tk.n_tiles;
    }
    gp.n_tasks = nt;
    gp.total_tiles = tiles;
    CUDA_TRY(launch_gemm(gp, 256, st));
  }

  // 5. fusion of the branches' latest outputs
  DecFuseParams fp{};
  fp.x = static_cast<const __nv_bfloat16*>(x);
  fp.Wfuse = h->Wfuse;
  fp.bfuse = h->bfuse;
  for (int j = 0; j < ns; ++j)
    fp.Y[j] = static_cast<const __half*>(h->br[j].scale == 1 ? wat(sl.Y1) : cat(cl.Y[j]));
  fp.out = static_cast<__nv_bfloat16*>(O);
  fp.B = B;
  fp.d = d;
  fp.n_scales = ns;
  CUDA_TRY(launch_dec_fuse(fp, st));
  return MSGLA_OK;
}

int check_forward_args(const msgla_handle* h, int B, int L) {
  if (!h) return fail(MSGLA_ERR_INVALID_ARG, "handle is NULL");
  if (B < 0 || L < 0) return fail(MSGLA_ERR_INVALID_ARG, "B=%d, L=%d must be >= 0", B, L);
  if (static_cast<long long>(B) * L * h->cfg.d > (1ll << 34))
    return fail(MSGLA_ERR_UNSUPPORTED, "B*L*d = %lld elements is beyond the supported size",
                static_cast<long long>(B) * L * h->cfg.d);
  if (L > (1 << 24)) return fail(MSGLA_ERR_UNSUPPORTED, "L=%d beyond 2^24", L);
  if (B > 65535) return fail(MSGLA_ERR_UNSUPPORTED, "B=%d beyond 65535", B);
  return MSGLA_OK;
}

}  // namespace

// ---------------------------------------------------------------- fixed scratch
// Scratch of msgla_forward_noalloc: a file-scope device array. It is part of the
// library's device image, so every GPU that loads the library holds these bytes
// until the process exits. Host code must not pass `g_noalloc_scratch` itself to
// a kernel (in host code the name is only a stand-in for the device symbol); the
// device address comes from cudaGetSymbolAddress, once per device.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (set-up on first use).
int noalloc_scratch(int device, void** out) {
  if (device < 0 || device >= kMaxDevices) return fail(MSGLA_ERR_UNSUPPORTED, "device index %d", device);
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (!g_noalloc_addr[device]) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p)
      return fail(MSGLA_ERR_CUDA, "cudaGetSymbolAddress(scratch) failed: %s", cudaGetErrorString(e));
    g_noalloc_addr[device] = p;
  }
  *out = g_noalloc_addr[device];
  return MSGLA_OK;
}
}  // namespace

// ---------------------------------------------------------------- C ABI
extern "C" {

int msgla_create(msgla_handle** out, const msgla_config* cfg, const msgla_weights* w, int device) {
  if (!out) return fail(MSGLA_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  int st = validate(cfg);
  if (st) return st;
  if (!w) return fail(MSGLA_ERR_INVALID_ARG, "weights are NULL");
  int ndev = 0;
  CUDA_TRY(cudaGetDeviceCount(&ndev));
  if (device < 0 || device >= ndev) return fail(MSGLA_ERR_INVALID_ARG, "device %d of %d", device, ndev);
  cudaDeviceProp prop;
  CUDA_TRY(cudaGetDeviceProperties(&prop, device));
  if (prop.major != 10 || prop.minor != 0)
    return fail(MSGLA_ERR_UNSUPPORTED, "device %d is sm_%d%d; the kernels are built for sm_100a", device, prop.major,
                prop.minor);
  if (!encode_fn()) return fail(MSGLA_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  DeviceGuard guard(device);
  if (!guard.ok) return fail(MSGLA_ERR_CUDA, "cudaSetDevice(%d) failed", device);
  msgla_handle* h = new msgla_handle();
  memset(h->br, 0, sizeof(h->br));
  h->side = nullptr;
  h->ev_fork = h->ev_join = nullptr;
  h->d_gla_done = nullptr;
  h->d_tiles = nullptr;
  h->copy_in = h->copy_out = nullptr;
  h->ev_start = h->ev_in = h->ev_done = nullptr;
  h->Wu = nullptr;
  h->Wfuse = nullptr;
  h->bfuse = nullptr;
  h->d_err = nullptr;
  h->test_skip_arrival = 0;
  h->cfg = *cfg;
  h->device = device;
  h->n_scales = cfg->n_scales;
  h->dkp = cfg->d_k <= 128 ? 128 : 256;
  h->dvp = static_cast<int>(round_up(cfg->d_v, kGlaTile));
  h->rp = static_cast<int>(round_up(cfg->gate_rank, 16));
  h->main_index = -1;
  h->sm_count = prop.multiProcessorCount;
  h->nzp = 16;
  h->ldz = cfg->n_scales <= 4 ? 4 : 8;
  h->ldu = 16 + cfg->n_scales * h->rp;
  int lcm = 1;
  for (int j = 0; j < h->n_scales; ++j) {
    h->br[j].scale = cfg->scales[j];
    h->br[j].heads = cfg->heads[j];
    h->br[j].np = cfg->heads[j] * (2 * h->dkp + h->dvp) + h->rp;
    if (cfg->scales[j] == 1) {
      h->main_index = j;
      h->br[j].np += 16;  // fusion logits W_fuse x (n_scales <= 8 rows, zero padded)
    }
    else lcm = lcm / gcd(lcm, cfg->scales[j]) * cfg->scales[j];
  }
  h->pool_rows = lcm;  // least common multiple of the coarse scales
  st = create_impl(h, w);
  if (st) {
    const std::string msg = g_last_error;
    free_handle(h);
    g_last_error = msg;
    return st;
  }
  *out = h;
  return MSGLA_OK;
}

void msgla_destroy(msgla_handle* h) {
  if (!h) return;
  DeviceGuard guard(h->device);
  cudaDeviceSynchronize();
  free_handle(h);
}

int msgla_workspace_size(const msgla_handle* h, int B, int L, size_t* bytes) {
  if (!bytes) return fail(MSGLA_ERR_INVALID_ARG, "bytes is NULL");
  int st = check_forward_args(h, B, L);
  if (st) return st;
  *bytes = (B == 0 || L == 0) ? 0 : layout(h, B, L).total;
  return MSGLA_OK;
}

int msgla_workspace_size_host(const msgla_handle* h, int B, int L, size_t* bytes) {
  int st = msgla_workspace_size(h, B, L, bytes);
  if (st) return st;
  if (B > 0 && L > 0) *bytes += 2 * round_up(static_cast<size_t>(B) * L * h->cfg.d * 2, 256);
  return MSGLA_OK;
}

int msgla_forward(msgla_handle* h, const void* X, int B, int L, void* O, void* workspace, size_t workspace_bytes,
                  void* stream) {
  int st = check_forward_args(h, B, L);
  if (st) return st;
  if (B == 0 || L == 0) return MSGLA_OK;
  if (!X || !O) return fail(MSGLA_ERR_INVALID_ARG, "X or O is NULL");
  if (reinterpret_cast<uintptr_t>(X) % 16 || reinterpret_cast<uintptr_t>(O) % 16)
    return fail(MSGLA_ERR_INVALID_ARG, "X and O must be 16-byte aligned");
  const size_t nbytes = static_cast<size_t>(B) * L * h->cfg.d * 2;
  const uint8_t* x0 = static_cast<const uint8_t*>(X);
  const uint8_t* o0 = static_cast<const uint8_t*>(O);
  if (x0 < o0 + nbytes && o0 < x0 + nbytes) return fail(MSGLA_ERR_INVALID_ARG, "O overlaps X");
  DeviceGuard guard(h->device);
  if (!guard.ok) return fail(MSGLA_ERR_CUDA, "cudaSetDevice(%d) failed", h->device);
  return forward_impl(h, X, B, L, O, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

int msgla_forward_masked(msgla_handle* h, const void* X, const void* M, int B, int L, void* O, void* workspace,
                         size_t workspace_bytes, void* stream) {
  int st = check_forward_args(h, B, L);
  if (st) return st;
  if (B == 0 || L == 0) return MSGLA_OK;
  if (!X || !O) return fail(MSGLA_ERR_INVALID_ARG, "X or O is NULL");
  if (reinterpret_cast<uintptr_t>(X) % 16 || reinterpret_cast<uintptr_t>(O) % 16)
    return fail(MSGLA_ERR_INVALID_ARG, "X and O must be 16-byte aligned");
  const size_t nbytes = static_cast<size_t>(B) * L * h->cfg.d * 2;
  const uint8_t* x0 = static_cast<const uint8_t*>(X);
  const uint8_t* o0 = static_cast<const uint8_t*>(O);
  if (x0 < o0 + nbytes && o0 < x0 + nbytes) return fail(MSGLA_ERR_INVALID_ARG, "O overlaps X");
  const uint8_t* m0 = static_cast<const uint8_t*>(M);
  if (m0 && m0 < o0 + nbytes && o0 < m0 + static_cast<size_t>(B) * L)
    return fail(MSGLA_ERR_INVALID_ARG, "O overlaps M");
  DeviceGuard guard(h->device);
  if (!guard.ok) return fail(MSGLA_ERR_CUDA, "cudaSetDevice(%d) failed", h->device);
  return forward_impl(h, X, B, L, O, workspace, workspace_bytes, static_cast<cudaStream_t>(stream), nullptr, m0);
}

int msgla_forward_noalloc(msgla_handle* h, const void* X, int B, int L, void* O, void* stream) {
  int st = check_forward_args(h, B, L);
  if (st) return st;
  if (B == 0 || L == 0) return MSGLA_OK;
  if (!X || !O) return fail(MSGLA_ERR_INVALID_ARG, "X or O is NULL");
  if (reinterpret_cast<uintptr_t>(X) % 16 || reinterpret_cast<uintptr_t>(O) % 16)
    return fail(MSGLA_ERR_INVALID_ARG, "X and O must be 16-byte aligned");
  const size_t nbytes = static_cast<size_t>(B) * L * h->cfg.d * 2;
  const uint8_t* x0 = static_cast<const uint8_t*>(X);
  const uint8_t* o0 = static_cast<const uint8_t*>(O);
  if (x0 < o0 + nbytes && o0 < x0 + nbytes) return fail(MSGLA_ERR_INVALID_ARG, "O overlaps X");
  const size_t need = layout(h, B, L).total;
  if (need > kNoAllocScratchBytes)
    return fail(MSGLA_ERR_WORKSPACE,
                "B=%d, L=%d needs %zu bytes of scratch; the fixed scratch of msgla_forward_noalloc holds %zu "
                "(use msgla_forward with a workspace)",
                B, L, need, kNoAllocScratchBytes);
  DeviceGuard guard(h->device);
  if (!guard.ok) return fail(MSGLA_ERR_CUDA, "cudaSetDevice(%d) failed", h->device);
  void* scratch = nullptr;
  st = noalloc_scratch(h->device, &scratch);
  if (st) return st;
  // Every intermediate the kernels read is written earlier in the same forward, so
  // the scratch needs no clearing between calls.
  return forward_impl(h, X, B, L, O, scratch, kNoAllocScratchBytes, static_cast<cudaStream_t>(stream));
}

int msgla_forward_profiled(msgla_handle* h, const void* X, const void* M, int B, int L, void* O, void* workspace,
                           size_t workspace_bytes, void* stream, void* const* events, int max_events,
                           int* n_launches) {
  if (!events || !n_launches) return fail(MSGLA_ERR_INVALID_ARG, "events or n_launches is NULL");
  *n_launches = 0;
  int st = check_forward_args(h, B, L);
  if (st) return st;
  if (B == 0 || L == 0) return MSGLA_OK;
  if (!X || !O) return fail(MSGLA_ERR_INVALID_ARG, "X or O is NULL");
  if (reinterpret_cast<uintptr_t>(X) % 16 || reinterpret_cast<uintptr_t>(O) % 16)
    return fail(MSGLA_ERR_INVALID_ARG, "X and O must be 16-byte aligned");
  const size_t nbytes = static_cast<size_t>(B) * L * h->cfg.d * 2;
  const uint8_t* x0 = static_cast<const uint8_t*>(X);
  const uint8_t* o0 = static_cast<const uint8_t*>(O);
  if (x0 < o0 + nbytes && o0 < x0 + nbytes) return fail(MSGLA_ERR_INVALID_ARG, "O overlaps X");
  const uint8_t* m0 = static_cast<const uint8_t*>(M);
  if (m0 && m0 < o0 + nbytes && o0 < m0 + static_cast<size_t>(B) * L)
    return fail(MSGLA_ERR_INVALID_ARG, "O overlaps M");
  DeviceGuard guard(h->device);
  if (!guard.ok) return fail(MSGLA_ERR_CUDA, "cudaSetDevice(%d) failed", h->device);
  Recorder rec;
  rec.events = events;
  rec.max_events = max_events;
  st = forward_impl(h, X, B, L, O, workspace, workspace_bytes, static_cast<cudaStream_t>(stream), &rec,
                    static_cast<const uint8_t*>(M));
  *n_launches = rec.n + rec.unmarked;
  return st;
}

int msgla_forward_host(msgla_handle* h, const void* X_host, int B, int L, void* O_host, void* workspace,
                       size_t workspace_bytes, void* stream) {
  int st = check_forward_args(h, B, L);
  if (st) return st;
  if (B == 0 || L == 0) return MSGLA_OK;
  if (!X_host || !O_host) return fail(MSGLA_ERR_INVALID_ARG, "X or O is NULL");
  size_t need = 0;
  msgla_workspace_size_host(h, B, L, &need);
  if (!workspace || workspace_bytes < need)
    return fail(MSGLA_ERR_WORKSPACE, "workspace of %zu bytes, %zu needed", workspace_bytes, need);
  if (reinterpret_cast<uintptr_t>(workspace) % 256)
    return fail(MSGLA_ERR_WORKSPACE, "workspace not 256-byte aligned");
  DeviceGuard guard(h->device);
  if (!guard.ok) return fail(MSGLA_ERR_CUDA, "cudaSetDevice(%d) failed", h->device);
  const size_t nbytes = static_cast<size_t>(B) * L * h->cfg.d * 2;
  const size_t core = layout(h, B, L).total;
  uint8_t* Xd = static_cast<uint8_t*>(workspace) + core;
  uint8_t* Od = Xd + round_up(nbytes, 256);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // Pipeline over chunks of whole sequences: the upload of chunk c + 1 (copy_in)
  // and the download of chunk c - 1 (copy_out) overlap the forward of chunk c on
  // `stream`; the chunks' forwards run one after another in the workspace's core
  // region (sized for all B sequences). One sequence first and last keeps the
  // pipeline's fill and drain short; the chunks between hold
  // max(2, ceil((B - 2) / 4)) sequences, so their forwards stay efficient
  // enough to hide under the copies.
  const int mid = B <= 2 ? 1 : std::max(2, (B - 2 + 3) / 4);
  const size_t row_bytes = static_cast<size_t>(L) * h->cfg.d * 2;  // one sequence
  const uint8_t* Xh = static_cast<const uint8_t*>(X_host);
  uint8_t* Oh = static_cast<uint8_t*>(O_host);
  CUDA_TRY(cudaEventRecord(h->ev_start, s));
  CUDA_TRY(cudaStreamWaitEvent(h->copy_in, h->ev_start, 0));
  for (int b0 = 0; b0 < B;) {
    const int bc = (b0 == 0 || B - b0 <= 1) ? 1 : std::min(mid, B - b0 - 1);
    const size_t off = static_cast<size_t>(b0) * row_bytes, bytes = static_cast<size_t>(bc) * row_bytes;
    CUDA_TRY(cudaMemcpyAsync(Xd + off, Xh + off, bytes, cudaMemcpyHostToDevice, h->copy_in));
    CUDA_TRY(cudaEventRecord(h->ev_in, h->copy_in));
    CUDA_TRY(cudaStreamWaitEvent(s, h->ev_in, 0));
    st = forward_impl(h, Xd + off, bc, L, Od + off, workspace, core, s);
    if (st) {
      cudaStreamSynchronize(h->copy_in);
      cudaStreamSynchronize(h->copy_out);
      return st;
    }
    CUDA_TRY(cudaEventRecord(h->ev_done, s));
    CUDA_TRY(cudaStreamWaitEvent(h->copy_out, h->ev_done, 0));
    CUDA_TRY(cudaMemcpyAsync(Oh + off, Od + off, bytes, cudaMemcpyDeviceToHost, h->copy_out));
    b0 += bc;
  }
  CUDA_TRY(cudaStreamSynchronize(h->copy_out));
  CUDA_TRY(cudaStreamSynchronize(s));
  int err = 0;
  CUDA_TRY(cudaMemcpy(&err, h->d_err, sizeof(int), cudaMemcpyDeviceToHost));
  if (err) {
    CUDA_TRY(cudaMemset(h->d_err, 0, sizeof(int)));
    return err == kDevTimeout ? fail(MSGLA_ERR_DEVICE_TIMEOUT, "a bounded wait inside a kernel timed out")
                              : fail(MSGLA_ERR_RANGE, "an internal fp16 operand overflowed");
  }
  return MSGLA_OK;
}

int msgla_sync_status(msgla_handle* h) {
  if (!h) return fail(MSGLA_ERR_INVALID_ARG, "handle is NULL");
  DeviceGuard guard(h->device);
  CUDA_TRY(cudaDeviceSynchronize());
  int err = 0;
  CUDA_TRY(cudaMemcpy(&err, h->d_err, sizeof(int), cudaMemcpyDeviceToHost));
  if (!err) return MSGLA_OK;
  CUDA_TRY(cudaMemset(h->d_err, 0, sizeof(int)));
  if (err == kDevTimeout) return fail(MSGLA_ERR_DEVICE_TIMEOUT, "a bounded wait inside a kernel timed out");
  return fail(MSGLA_ERR_RANGE, "an internal fp16 operand overflowed");
}

int msgla_workspace_tensor(const msgla_handle* h, int B, int L, int scale_index, int which, size_t* offset,
                           int dims[3]) {
  if (!h || !offset || !dims) return fail(MSGLA_ERR_INVALID_ARG, "NULL argument");
  int st = check_forward_args(h, B, L);
  if (st) return st;
  if (B == 0 || L == 0) return fail(MSGLA_ERR_INVALID_ARG, "empty input has no workspace");
  const Workspace ws = layout(h, B, L);
  if (which == 7 || which == 8) {
    *offset = which == 7 ? ws.w.off : ws.u.off;
    dims[0] = B;
    dims[1] = L;
    dims[2] = which == 7 ? h->n_scales : h->ldu;
    return MSGLA_OK;
  }
  if (scale_index < 0 || scale_index >= h->n_scales) return fail(MSGLA_ERR_INVALID_ARG, "scale_index out of range");
  const BranchWs& bw = ws.br[scale_index];
  const Branch& b = h->br[scale_index];
  const Region* r = nullptr;
  int cols = 0;
  switch (which) {
    case 0: r = &bw.Xp; cols = h->cfg.d; break;
    case 1: r = &bw.qs; cols = b.heads * h->dkp; break;
    case 2: r = &bw.ks; cols = b.heads * h->dkp; break;
    case 3: r = &bw.v; cols = b.heads * h->dvp; break;
    case 5: r = &bw.o; cols = b.heads * h->dvp; break;
    case 6: r = &bw.Y; cols = h->cfg.d; break;
    case 9: r = &bw.gamma; cols = b.heads * h->dkp; break;
    case 10: r = &bw.mid; cols = b.heads * h->dkp; break;
    default: return fail(MSGLA_ERR_INVALID_ARG, "which=%d unknown", which);
  }
  if (r->bytes == 0) return fail(MSGLA_ERR_INVALID_ARG, "tensor %d does not exist for scale index %d", which,
                                 scale_index);
  *offset = r->off;
  dims[0] = B;
  dims[1] = (which == 9 || which == 10) ? bw.n_chunks : bw.rows;
  dims[2] = cols;
  return MSGLA_OK;
}

int msgla_cache_size(const msgla_handle* h, int B, size_t* bytes) {
  if (!h || !bytes) return fail(MSGLA_ERR_INVALID_ARG, "NULL argument");
  if (B < 0 || B > 65535) return fail(MSGLA_ERR_INVALID_ARG, "B=%d outside [0, 65535]", B);
  *bytes = cache_layout(h, B).total;
  return MSGLA_OK;
}

int msgla_cache_reset(msgla_handle* h, void* cache, int B, void* stream) {
  if (!h) return fail(MSGLA_ERR_INVALID_ARG, "handle is NULL");
  if (B < 0 || B > 65535) return fail(MSGLA_ERR_INVALID_ARG, "B=%d outside [0, 65535]", B);
  const size_t n = cache_layout(h, B).total;
  if (n == 0) return MSGLA_OK;
  if (!cache || reinterpret_cast<uintptr_t>(cache) % 256)
    return fail(MSGLA_ERR_INVALID_ARG, "cache is NULL or not 256-byte aligned");
  DeviceGuard guard(h->device);
  if (!guard.ok) return fail(MSGLA_ERR_CUDA, "cudaSetDevice(%d) failed", h->device);
  CUDA_TRY(cudaMemsetAsync(cache, 0, n, static_cast<cudaStream_t>(stream)));
  return MSGLA_OK;
}

int msgla_step_workspace_size(const msgla_handle* h, int B, size_t* bytes) {
  if (!h || !bytes) return fail(MSGLA_ERR_INVALID_ARG, "NULL argument");
  if (B < 0 || B > 65535) return fail(MSGLA_ERR_INVALID_ARG, "B=%d outside [0, 65535]", B);
  *bytes = step_layout(h, B).total;
  return MSGLA_OK;
}

int msgla_step(msgla_handle* h, void* cache, const void* x, int B, long long t, void* O, void* workspace,
               size_t workspace_bytes, void* stream) {
  if (!h) return fail(MSGLA_ERR_INVALID_ARG, "handle is NULL");
  if (B < 0 || B > 65535) return fail(MSGLA_ERR_INVALID_ARG, "B=%d outside [0, 65535]", B);
  if (t < 0) return fail(MSGLA_ERR_INVALID_ARG, "t=%lld must be >= 0", t);
  if (B == 0) return MSGLA_OK;
  if (!cache || !x || !O) return fail(MSGLA_ERR_INVALID_ARG, "cache, x or O is NULL");
  if (reinterpret_cast<uintptr_t>(x) % 16 || reinterpret_cast<uintptr_t>(O) % 16)
    return fail(MSGLA_ERR_INVALID_ARG, "x and O must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(cache) % 256) return fail(MSGLA_ERR_INVALID_ARG, "cache not 256-byte aligned");
  const size_t need = step_layout(h, B).total;
  if (!workspace || workspace_bytes < need)
    return fail(MSGLA_ERR_WORKSPACE, "step workspace of %zu bytes, %zu needed", workspace_bytes, need);
  if (reinterpret_cast<uintptr_t>(workspace) % 256) return fail(MSGLA_ERR_WORKSPACE, "workspace not 256-byte aligned");
  const size_t nb = static_cast<size_t>(B) * h->cfg.d * 2;
  const uint8_t* x0 = static_cast<const uint8_t*>(x);
  const uint8_t* o0 = static_cast<const uint8_t*>(O);
  if (x0 < o0 + nb && o0 < x0 + nb) return fail(MSGLA_ERR_INVALID_ARG, "O overlaps x");
  DeviceGuard guard(h->device);
  if (!guard.ok) return fail(MSGLA_ERR_CUDA, "cudaSetDevice(%d) failed", h->device);
  return step_impl(h, cache, x, B, t, O, workspace, static_cast<cudaStream_t>(stream));
}

int msgla_launch_plan(const msgla_handle* h, int B, int L, char* names, size_t len) {
  if (!h || !names || len == 0) return fail(MSGLA_ERR_INVALID_ARG, "NULL argument");
  int st = check_forward_args(h, B, L);
  if (st) return st;
  std::string out;
  auto add_name = [&](const char* n) {
    if (!out.empty()) out += ",";
    out += n;
  };
  if (B > 0 && L > 0) {
    if (fused_pool(h)) {
      add_name("pool_u");
    } else {
      add_name("gate_inputs");
      if (h->pool_rows > 1) add_name("pool");
    }
    add_name("gate");
    add_name("proj_gemm");
    const Workspace ws = layout(h, B, L);
    bool segmented = false;
    for (int j = 0; j < h->n_scales; ++j) segmented |= ws.br[j].n_segs > 1;
    if (segmented) {
      add_name("gla_state");
      add_name("gla_scan");
    }
    add_name("gla");
    if (h->cfg.head_norm) add_name("head_norm");
    long long gla_ctas = 0;
    const bool overlap = coarse_overlap(h, ws, B, &gla_ctas);
    if (h->main_index >= 0) {
      // overlapped with the GLA on the second stream, the coarse output GEMM has
      // no interval of its own on the caller's stream
      if (h->n_scales > 1 && !overlap) add_name("out_gemm_coarse");
      add_name("out_gemm_fused");
    } else {
      add_name("out_gemm_coarse");
      add_name("hold_fuse");
    }
  }
  if (out.size() + 1 > len) return fail(MSGLA_ERR_INVALID_ARG, "names buffer of %zu bytes is too small", len);
  memcpy(names, out.c_str(), out.size() + 1);
  return MSGLA_OK;
}

int msgla_test_skip_arrival(msgla_handle* h, int enable) {
  if (!h) return fail(MSGLA_ERR_INVALID_ARG, "handle is NULL");
  h->test_skip_arrival = enable ? 1 : 0;
  return MSGLA_OK;
}

const char* msgla_status_string(int status) {
  switch (status) {
    case MSGLA_OK: return "ok";
    case MSGLA_ERR_INVALID_ARG: return "invalid argument";
    case MSGLA_ERR_UNSUPPORTED: return "unsupported configuration";
    case MSGLA_ERR_CUDA: return "CUDA error";
    case MSGLA_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case MSGLA_ERR_RANGE: return "value outside the fp16 range of an internal operand";
    case MSGLA_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
    default: return "unknown status";
  }
}

const char* msgla_last_error(void) { return g_last_error.c_str(); }

}  // extern "C"
