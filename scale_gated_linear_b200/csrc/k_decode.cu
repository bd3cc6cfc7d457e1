// k_decode.cu -- one token per sequence through the per-branch cache
// (token-by-token inference of the MS-GLA reading notes, the item on training
// and per-token inference, after the authors' cache):
//   dec_pool_kernel  coarse branches add the token to their running block sums;
//                    a branch whose block of s tokens completes emits the mean
//                    (Eq. (8)) as an fp16 row for its projection and clears it.
//   dec_gla_kernel   one GLA step (Sec. 2.1) of a stepping branch: the gate
//                    alpha from the low-rank projection, S = Diag(alpha) S + k^T v
//                    on the fp32 state in the cache, o = qk_scale * q S.
//   dec_fuse_kernel  w = softmax(W_fuse x + b_fuse) from the token itself
//                    (Eq. (10)) and O = sum_s w_s Y_s over the branches' latest
//                    outputs (Eq. (11); a coarse branch repeats its output until
//                    its next block completes, which is the causal hold).
// The projections and output projections of the stepping branches run on the
// grouped tcgen05 GEMM with the B sequences as rows.
#include "msgla_internal.h"
#include "sm100_ptx.cuh"

namespace msgla {
namespace {

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 t = __bfloat1622float2(h[e]);
    f[2 * e] = t.x;
    f[2 * e + 1] = t.y;
  }
}

// one thread per (sequence, 8 columns)
__global__ void __launch_bounds__(256) dec_pool_kernel(const DecPoolParams p) {
  griddep_wait();
  griddep_launch();
  const int groups = p.d / 8;
  const size_t gid = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  if (gid >= static_cast<size_t>(p.B) * groups) return;
  const size_t off = gid * 8;  // = b * d + 8 * column group
  float x[8];
  bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(p.x + off)), x);
  bool bad = false;
  for (int j = 0; j < p.n_scales; ++j) {
    float* buf = p.buf[j];
    if (!buf) continue;
    float4* b4 = reinterpret_cast<float4*>(buf + off);
    const float4 u0 = b4[0], u1 = b4[1];
    const float s[8] = {u0.x + x[0], u0.y + x[1], u0.z + x[2], u0.w + x[3],
                        u1.x + x[4], u1.y + x[5], u1.z + x[6], u1.w + x[7]};
    if (p.xbar[j]) {
      const float inv = 1.f / static_cast<float>(p.scales[j]);
      uint4 o;
      uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float a0 = s[2 * e] * inv, a1 = s[2 * e + 1] * inv;
        bad |= !(fabsf(a0) <= 65504.f) || !(fabsf(a1) <= 65504.f);
        ow[e] = pack_half2(a0, a1);
      }
      *reinterpret_cast<uint4*>(p.xbar[j] + off) = o;
      b4[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      b4[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    } else {
      b4[0] = make_float4(s[0], s[1], s[2], s[3]);
      b4[1] = make_float4(s[4], s[5], s[6], s[7]);
    }
  }
  if (bad) atomicCAS(p.err, 0, kDevRange);
}

constexpr int kDecTile = 128;  // value columns per CTA
constexpr int kDecMaxDk = 256;
constexpr int kDecThreads = 512;
constexpr int kDecGroups = kDecThreads / 32;  // key-channel groups; a warp covers the 128 columns

// One CTA (512 threads) per (sequence, stepping branch, head, 128 value columns).
// Warp g handles key channels [g*dkp/16, (g+1)*dkp/16), lane l value columns
// [4l, 4l+4): each key channel's state row segment (512 bytes) is one coalesced
// warp access, and all of a thread's state (16 x 16 bytes) is loaded before any
// of it is used, so the whole 128 KB tile is in flight at once. The partial
// o = q S of the 16 channel groups are summed through shared memory.
__global__ void __launch_bounds__(kDecThreads) dec_gla_kernel(const __grid_constant__ DecGlaParams p) {
  griddep_wait();
  griddep_launch();
  __shared__ float alpha_s[kDecMaxDk], q_s[kDecMaxDk], k_s[kDecMaxDk];
  __shared__ __align__(16) float v_s[kDecTile];
  __shared__ __align__(16) float red[kDecGroups][kDecTile];
  int bi = 0;
#pragma unroll 1
  for (int j = 1; j < p.n_branches; ++j)
    if (static_cast<int>(blockIdx.x) >= p.br[j].cta_begin) bi = j;
  const DecGlaBranch& P = p.br[bi];
  const int v_tiles = p.dvp / kDecTile;
  int local = blockIdx.x - P.cta_begin;
  const int vt = local % v_tiles;
  local /= v_tiles;
  const int head = local % P.heads;
  const int b = local / P.heads;
  const int dkp = p.dkp, rp = p.rp;
  const size_t qk_row = static_cast<size_t>(b) * P.heads * dkp + static_cast<size_t>(head) * dkp;
  const size_t v_row = static_cast<size_t>(b) * P.heads * p.dvp + static_cast<size_t>(head) * p.dvp + vt * kDecTile;
  const int grp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per = dkp / kDecGroups;  // 16 (dkp = 256) or 8 (dkp = 128)
  const int c0 = grp * per;
  float* S = P.S + ((static_cast<size_t>(b) * P.heads + head) * dkp + c0) * p.dvp + vt * kDecTile + 4 * lane;

  // issue the state loads first; the gate and the small operands follow
  float4 s[16];
#pragma unroll
  for (int e = 0; e < 16; ++e)
    if (e < per) s[e] = *reinterpret_cast<const float4*>(S + static_cast<size_t>(e) * p.dvp);

  for (int c = threadIdx.x; c < dkp; c += blockDim.x) {
    const float* w = P.Wg2 + (static_cast<size_t>(head) * dkp + c) * rp;
    const float* g = P.g + static_cast<size_t>(b) * rp;
    float z = __ldg(P.bg + head * dkp + c);
    for (int r = 0; r < rp; ++r) z = fmaf(__ldg(g + r), __ldg(w + r), z);
    // logsigmoid(z) = min(z, 0) - log(1 + e^{-|z|})
    const float la = (fminf(z, 0.f) - __logf(1.f + __expf(-fabsf(z)))) * p.inv_normalizer;
    alpha_s[c] = __expf(la);
    q_s[c] = __half2float(P.q[qk_row + c]);
    k_s[c] = __half2float(P.k[qk_row + c]);
  }
  if (threadIdx.x < kDecTile) v_s[threadIdx.x] = __half2float(P.v[v_row + threadIdx.x]);
  __syncthreads();

  const float4 v4 = *reinterpret_cast<const float4*>(&v_s[4 * lane]);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    if (e >= per) break;
    const int ch = c0 + e;
    const float a = alpha_s[ch], kk = k_s[ch], qq = q_s[ch];
    float4 t = s[e];
    t.x = fmaf(a, t.x, kk * v4.x);
    t.y = fmaf(a, t.y, kk * v4.y);
    t.z = fmaf(a, t.z, kk * v4.z);
    t.w = fmaf(a, t.w, kk * v4.w);
    acc.x = fmaf(qq, t.x, acc.x);
    acc.y = fmaf(qq, t.y, acc.y);
    acc.z = fmaf(qq, t.z, acc.z);
    acc.w = fmaf(qq, t.w, acc.w);
    *reinterpret_cast<float4*>(S + static_cast<size_t>(e) * p.dvp) = t;
  }
  *reinterpret_cast<float4*>(&red[grp][4 * lane]) = acc;
  __syncthreads();
  if (threadIdx.x < kDecTile) {
    float o = 0.f;
#pragma unroll
    for (int g2 = 0; g2 < kDecGroups; ++g2) o += red[g2][threadIdx.x];
    o *= p.qk_scale;
    if (!(fabsf(o) <= 65504.f)) atomicCAS(p.err, 0, kDevRange);
    P.o[v_row + threadIdx.x] = __float2half_rn(o);
  }
}

// One CTA (256 threads) per sequence: fusion logits from the token, softmax,
// then the weighted sum of the branches' latest outputs, 8 columns per thread.
__global__ void __launch_bounds__(256) dec_fuse_kernel(const DecFuseParams p) {
  griddep_wait();
  griddep_launch();
  __shared__ float red[8][kMaxScales];
  __shared__ float w_s[kMaxScales];
  const int b = blockIdx.x;
  const int groups = p.d / 8;
  const int ns = p.n_scales;
  const __nv_bfloat16* xb = p.x + static_cast<size_t>(b) * p.d;
  float part[kMaxScales];
#pragma unroll
  for (int j = 0; j < kMaxScales; ++j) part[j] = 0.f;
  for (int cg = threadIdx.x; cg < groups; cg += blockDim.x) {
    float x[8];
    bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(xb) + cg), x);
#pragma unroll
    for (int j = 0; j < kMaxScales; ++j) {
      if (j >= ns) break;
      float w[8];
      bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(p.Wfuse + static_cast<size_t>(j) * p.d) + cg), w);
#pragma unroll
      for (int e = 0; e < 8; ++e) part[j] = fmaf(x[e], w[e], part[j]);
    }
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int j = 0; j < kMaxScales; ++j) {
    float v = part[j];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if (lane == 0) red[warp][j] = v;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float z[kMaxScales], zmax = -INFINITY;
    for (int j = 0; j < ns; ++j) {
      z[j] = (p.bfuse ? p.bfuse[j] : 0.f);
      for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) z[j] += red[w][j];
      zmax = fmaxf(zmax, z[j]);
    }
    float sum = 0.f;
    for (int j = 0; j < ns; ++j) {
      z[j] = __expf(z[j] - zmax);
      sum += z[j];
    }
    for (int j = 0; j < ns; ++j) w_s[j] = z[j] / sum;
  }
  __syncthreads();
  for (int cg = threadIdx.x; cg < groups; cg += blockDim.x) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < ns; ++j) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(p.Y[j] + static_cast<size_t>(b) * p.d) + cg);
      const __half2* h = reinterpret_cast<const __half2*>(&u);
      const float wj = w_s[j];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(h[e]);
        acc[2 * e] = fmaf(wj, f.x, acc[2 * e]);
        acc[2 * e + 1] = fmaf(wj, f.y, acc[2 * e + 1]);
      }
    }
    uint4 o;
    o.x = pack_bf162(acc[0], acc[1]);
    o.y = pack_bf162(acc[2], acc[3]);
    o.z = pack_bf162(acc[4], acc[5]);
    o.w = pack_bf162(acc[6], acc[7]);
    reinterpret_cast<uint4*>(p.out + static_cast<size_t>(b) * p.d)[cg] = o;
  }
}

}  // namespace

cudaError_t launch_dec_pool(const DecPoolParams& p, cudaStream_t st) {
  const size_t n = static_cast<size_t>(p.B) * (p.d / 8);
  if (n == 0) return cudaSuccess;
  return launch_pdl(dec_pool_kernel, dim3(static_cast<unsigned>((n + 255) / 256)), dim3(256), 0, st, p);
}

cudaError_t launch_dec_gla(const DecGlaParams& p, cudaStream_t st) {
  if (p.total_ctas <= 0) return cudaSuccess;
  if ((p.dkp != 128 && p.dkp != 256) || p.dvp % kDecTile) return cudaErrorInvalidValue;
  return launch_pdl(dec_gla_kernel, dim3(p.total_ctas), dim3(kDecThreads), 0, st, p);
}

cudaError_t launch_dec_fuse(const DecFuseParams& p, cudaStream_t st) {
  if (p.B <= 0) return cudaSuccess;
  return launch_pdl(dec_fuse_kernel, dim3(p.B), dim3(256), 0, st, p);
}

}  // namespace msgla
