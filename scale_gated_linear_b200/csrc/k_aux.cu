// k_aux.cu -- the CUDA-core kernels of the MS-GLA path:
//   pool_fuse_kernel  one pass over X: mean pooling of s adjacent rows for every
//                     scale s > 1 (reading notes Sec. 3.1, Eq. (8)) and the
//                     fusion weights w_t = softmax(W_fuse x_t + b_fuse) from the
//                     unpooled rows (Sec. 3.3, Eq. (10)); pool_fuse_rows_kernel
//                     does both per row block when there is no scale-1 branch,
//                     pool_rows_kernel and pool_rows_flat_kernel pool only (with
//                     a scale-1 branch the fusion logits come from its
//                     projection GEMM).
//   gate_kernel       log alpha = logsigmoid(g W_g2^T + b_g) / normalizer (the
//                     low-rank gate of Sec. 2.1), its cumulative sum b inside
//                     each 128-row GLA chunk referenced to the chunk's 64th
//                     row (m): Qs = q e^{b - m}, Ks = k e^{m - b}, and per chunk
//                     gamma = e^{b_last - m}, mid = e^{m}.
//   head_norm_kernel  optional per-branch normalisation (Sec. 3.2), read as an
//                     RMS norm of each head's GLA output row, in place.
//   hold_fuse_kernel  O_t = sum_s w_{t,s} Y^(s)_{floor((t+1)/s)-1} (Sec. 3.3,
//                     Eq. (11)) when no branch has scale 1.
//   weight converters used once by msgla_create.
#include <algorithm>

#include "msgla_internal.h"
#include "sm100_ptx.cuh"

namespace msgla {
namespace {

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&f)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    float2 t = __bfloat1622float2(h[e]);
    f[2 * e] = t.x;
    f[2 * e + 1] = t.y;
  }
}

constexpr int kPoolThreads = 128;

// grid (ceil(L / block_rows), B); each thread owns 8 consecutive columns at a time.
__global__ void __launch_bounds__(kPoolThreads) pool_fuse_kernel(const PoolParams p) {
  griddep_wait();
  griddep_launch();
  __shared__ float logit[64 * kMaxScales];
  const int b = blockIdx.y;
  const int row0 = blockIdx.x * p.block_rows;
  const int nrows = min(p.block_rows, p.L - row0);
  const int ns = p.n_scales;
  for (int i = threadIdx.x; i < nrows * ns; i += blockDim.x) logit[i] = 0.f;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int ngroups = p.d / 8;
  const __nv_bfloat16* Xb = p.X + static_cast<size_t>(b) * p.L * p.d;
  // loop count is the same for all threads of a warp (required by the shuffles)
  const int iters = (ngroups + blockDim.x - 1) / blockDim.x;
  for (int it = 0; it < iters; ++it) {
    const int cg = it * blockDim.x + threadIdx.x;
    const bool active = cg < ngroups;
    float wf[kMaxScales][8];
#pragma unroll
    for (int j = 0; j < kMaxScales; ++j) {
      if (j < ns && active) {
        uint4 u = __ldg(reinterpret_cast<const uint4*>(p.Wfuse + static_cast<size_t>(j) * p.d) + cg);
        bf16x8_to_f32(u, wf[j]);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) wf[j][e] = 0.f;
      }
    }
    float acc[kMaxScales][8];
    int nvalid[kMaxScales];
#pragma unroll
    for (int j = 0; j < kMaxScales; ++j) {
      nvalid[j] = 0;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[j][e] = 0.f;
    }
    for (int r = 0; r < nrows; ++r) {
      const int t = row0 + r;
      const bool keep = !p.M || p.M[static_cast<size_t>(b) * p.L + t];
      float x[8];
      if (active) {
        uint4 u = __ldg(reinterpret_cast<const uint4*>(Xb + static_cast<size_t>(t) * p.d) + cg);
        bf16x8_to_f32(u, x);
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = 0.f;
      }
#pragma unroll
      for (int j = 0; j < kMaxScales; ++j) {
        if (j >= ns) break;
        float part = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) part = fmaf(x[e], wf[j][e], part);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
        if (lane == 0) atomicAdd(&logit[r * ns + j], part);
        const int s = p.scales[j];
        if (s > 1) {
          if (keep) {
            ++nvalid[j];
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[j][e] += x[e];
          }
          const bool block_end = ((t + 1) % s == 0) || (t == p.L - 1);
          if (block_end) {
            if (active) {
              const int i = t / s;
              const float inv = 1.f / static_cast<float>(max(1, nvalid[j]));
              uint4 o;
              uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
              bool bad = false;
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float a0 = acc[j][2 * e] * inv, a1 = acc[j][2 * e + 1] * inv;
                bad |= fabsf(a0) > 65504.f || fabsf(a1) > 65504.f;
                ow[e] = pack_half2(a0, a1);
              }
              if (bad) atomicCAS(p.err, 0, kDevRange);
              const int ns_rows = (p.L + s - 1) / s;
              reinterpret_cast<uint4*>(p.Xp[j] + (static_cast<size_t>(b) * ns_rows + i) * p.d)[cg] = o;
            }
            nvalid[j] = 0;
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[j][e] = 0.f;
          }
        }
      }
    }
  }
  __syncthreads();
  for (int r = threadIdx.x; r < nrows; r += blockDim.x) {
    float z[kMaxScales];
    float zmax = -INFINITY;
    for (int j = 0; j < ns; ++j) {
      z[j] = logit[r * ns + j] + (p.bfuse ? p.bfuse[j] : 0.f);
      zmax = fmaxf(zmax, z[j]);
    }
    float sum = 0.f;
    for (int j = 0; j < ns; ++j) {
      z[j] = __expf(z[j] - zmax);
      sum += z[j];
    }
    const float inv = 1.f / sum;
    float* wr = p.w + (static_cast<size_t>(b) * p.L + row0 + r) * ns;
    for (int j = 0; j < ns; ++j) wr[j] = z[j] * inv;
  }
}

// Streaming form for scale sets whose coarse scales all divide P (P <= 8): one
// warp per block of P rows of one sequence. Per pass each lane first issues the
// loads of GPL column groups (8 columns each) for all P rows (GPL * P * 16 bytes
// in flight per lane), then forms the pooled rows of every coarse scale and the
// partial fusion logits; the logits are reduced across the warp once per row at
// the end. NS bounds the number of scales held in registers.
template <int P, int GPL, int NS, int MB>
__global__ void __launch_bounds__(256, MB) pool_fuse_rows_kernel(const PoolParams p) {
  griddep_wait();
  griddep_launch();
  extern __shared__ float wf_s[];  // [n_scales][d] fp32
  const int ns = p.n_scales;
  for (int i = threadIdx.x; i < ns * p.d; i += blockDim.x) wf_s[i] = __bfloat162float(p.Wfuse[i]);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int blocks_per_seq = (p.L + P - 1) / P;
  const size_t gw = blockIdx.x * static_cast<size_t>(blockDim.x >> 5) + (threadIdx.x >> 5);
  if (gw >= static_cast<size_t>(p.B) * blocks_per_seq) return;
  const int b = static_cast<int>(gw / blocks_per_seq);
  const int row0 = static_cast<int>(gw % blocks_per_seq) * P;
  const int nrows = min(P, p.L - row0);
  const __nv_bfloat16* Xb = p.X + (static_cast<size_t>(b) * p.L + row0) * p.d;
  // rows of this block that enter the pooled means (bit r = row0 + r)
  uint32_t vm = (1u << nrows) - 1u;
  if (p.M)
#pragma unroll
    for (int r = 0; r < P; ++r)
      if (r < nrows && !p.M[static_cast<size_t>(b) * p.L + row0 + r]) vm &= ~(1u << r);
  float part[P][NS];
#pragma unroll
  for (int r = 0; r < P; ++r)
#pragma unroll
    for (int j = 0; j < NS; ++j) part[r][j] = 0.f;
  const int groups = p.d / 8;
  for (int base = 0; base < groups; base += 32 * GPL) {
    uint4 raw[GPL][P];
#pragma unroll
    for (int gi = 0; gi < GPL; ++gi) {
      const int cg = base + gi * 32 + lane;
#pragma unroll
      for (int r = 0; r < P; ++r)
        raw[gi][r] = (cg < groups && r < nrows)
                         ? __ldg(reinterpret_cast<const uint4*>(Xb + static_cast<size_t>(r) * p.d) + cg)
                         : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int gi = 0; gi < GPL; ++gi) {
      const int cg = base + gi * 32 + lane;
      if (cg >= groups) continue;
      float x[P][8];
#pragma unroll
      for (int r = 0; r < P; ++r) bf16x8_to_f32(raw[gi][r], x[r]);
#pragma unroll
      for (int j = 0; j < NS; ++j) {
        if (j >= ns) break;
        const float4 wa = *reinterpret_cast<const float4*>(wf_s + j * p.d + cg * 8);
        const float4 wb = *reinterpret_cast<const float4*>(wf_s + j * p.d + cg * 8 + 4);
#pragma unroll
        for (int r = 0; r < P; ++r)
          part[r][j] += x[r][0] * wa.x + x[r][1] * wa.y + x[r][2] * wa.z + x[r][3] * wa.w + x[r][4] * wb.x +
                        x[r][5] * wb.y + x[r][6] * wb.z + x[r][7] * wb.w;
        const int s = p.scales[j];
        if (s == 1) continue;
        const int n_s = (p.L + s - 1) / s;
        for (int i0 = 0; i0 < P; i0 += s) {
          if (i0 >= nrows) break;
          const int cnt = min(s, nrows - i0);
          float m[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) m[e] = 0.f;
#pragma unroll
          for (int r = 0; r < P; ++r)
            if (r >= i0 && r < i0 + cnt && ((vm >> r) & 1u))
#pragma unroll
              for (int e = 0; e < 8; ++e) m[e] += x[r][e];
          const float inv = 1.f / static_cast<float>(max(1, __popc((vm >> i0) & ((1u << cnt) - 1u))));
          uint4 o;
          uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
          bool bad = false;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float a0 = m[2 * e] * inv, a1 = m[2 * e + 1] * inv;
            bad |= !(fabsf(a0) <= 65504.f) || !(fabsf(a1) <= 65504.f);
            ow[e] = pack_half2(a0, a1);
          }
          if (bad) atomicCAS(p.err, 0, kDevRange);
          const int i = (row0 + i0) / s;
          reinterpret_cast<uint4*>(p.Xp[j] + (static_cast<size_t>(b) * n_s + i) * p.d)[cg] = o;
        }
      }
    }
  }
#pragma unroll
  for (int r = 0; r < P; ++r) {
    float z[NS];
    float zmax = -INFINITY;
#pragma unroll
    for (int j = 0; j < NS; ++j) {
      float v = part[r][j];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      z[j] = v + ((j < ns && p.bfuse) ? p.bfuse[j] : 0.f);
      if (j < ns) zmax = fmaxf(zmax, z[j]);
    }
    if (lane == 0 && r < nrows) {
      float sum = 0.f;
#pragma unroll
      for (int j = 0; j < NS; ++j) {
        z[j] = j < ns ? __expf(z[j] - zmax) : 0.f;
        sum += z[j];
      }
      float* wr = p.w + (static_cast<size_t>(b) * p.L + row0 + r) * ns;
      for (int j = 0; j < ns; ++j) wr[j] = z[j] / sum;
    }
  }
}

// Pooling only (the fusion logits come from the projection GEMM): one thread per
// (sequence, block of P rows, 8 columns); all P row loads are issued together.
template <int P>
__global__ void __launch_bounds__(256) pool_rows_kernel(const PoolParams p) {
  griddep_wait();
  griddep_launch();
  const int groups = p.d / 8;
  const int nblk = (p.L + P - 1) / P;
  const size_t gid = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  if (gid >= static_cast<size_t>(p.B) * nblk * groups) return;
  const int cg = static_cast<int>(gid % groups);
  const size_t rest = gid / groups;
  const int blk = static_cast<int>(rest % nblk), b = static_cast<int>(rest / nblk);
  const int row0 = blk * P;
  const int nrows = min(P, p.L - row0);
  const __nv_bfloat16* Xb = p.X + (static_cast<size_t>(b) * p.L + row0) * p.d;
  // rows of this block that enter the means (bit r = row0 + r); padded rows are not read
  uint32_t vm = (1u << nrows) - 1u;
  if (p.M)
#pragma unroll
    for (int r = 0; r < P; ++r)
      if (r < nrows && !p.M[static_cast<size_t>(b) * p.L + row0 + r]) vm &= ~(1u << r);
  uint4 raw[P];
#pragma unroll
  for (int r = 0; r < P; ++r)
    raw[r] = ((vm >> r) & 1u) ? __ldg(reinterpret_cast<const uint4*>(Xb + static_cast<size_t>(r) * p.d) + cg)
                              : make_uint4(0, 0, 0, 0);
  float x[P][8];
#pragma unroll
  for (int r = 0; r < P; ++r) bf16x8_to_f32(raw[r], x[r]);
  bool bad = false;
  auto put = [&](int j, int s, int i0, const float (&m)[8], float inv) {
    uint4 o;
    uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float a0 = m[2 * e] * inv, a1 = m[2 * e + 1] * inv;
      bad |= !(fabsf(a0) <= 65504.f) || !(fabsf(a1) <= 65504.f);
      ow[e] = pack_half2(a0, a1);
    }
    const int n_s = (p.L + s - 1) / s;
    reinterpret_cast<uint4*>(p.Xp[j] + (static_cast<size_t>(b) * n_s + (row0 + i0) / s) * p.d)[cg] = o;
  };
  if (nrows == P) {
    // complete block: sums over aligned groups of 2, 4, ... rows as a pairwise tree
    float lv[P][8];
#pragma unroll
    for (int r = 0; r < P; ++r)
#pragma unroll
      for (int e = 0; e < 8; ++e) lv[r][e] = x[r][e];
    int width = 1;
#pragma unroll
    for (int level = 0; (1 << level) < P; ++level) {
      // lv[i] holds the sum of rows [i*width, (i+1)*width)
      const int n = P >> level;
#pragma unroll
      for (int i = 0; i < P / 2; ++i)
        if (i < n / 2)
#pragma unroll
          for (int e = 0; e < 8; ++e) lv[i][e] = lv[2 * i][e] + lv[2 * i + 1][e];
      width <<= 1;
      for (int j = 0; j < p.n_scales; ++j) {
        if (p.scales[j] != width) continue;
#pragma unroll
        for (int i = 0; i < P / 2; ++i)
          if (i < n / 2)
            put(j, width, i * width, lv[i],
                1.f / static_cast<float>(max(1, __popc((vm >> (i * width)) & ((1u << width) - 1u)))));
      }
    }
  }
  for (int j = 0; j < p.n_scales; ++j) {
    const int s = p.scales[j];
    if (s == 1 || (nrows == P && (s & (s - 1)) == 0)) continue;  // done above
    for (int i0 = 0; i0 < nrows; i0 += s) {
      const int cnt = min(s, nrows - i0);
      float m[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) m[e] = 0.f;
#pragma unroll
      for (int r = 0; r < P; ++r)
        if (r >= i0 && r < i0 + cnt)
#pragma unroll
          for (int e = 0; e < 8; ++e) m[e] += x[r][e];
      put(j, s, i0, m, 1.f / static_cast<float>(max(1, __popc((vm >> i0) & ((1u << cnt) - 1u)))));
    }
  }
  if (bad) atomicCAS(p.err, 0, kDevRange);
}

// Pooling only, with no mask, coarse scales that are powers of two dividing P,
// and every sequence a whole number of P-row blocks: blocks are numbered flat
// over the batch (block f starts at token f P, and its pooled row for scale s is
// (f P + i0) / s), so the loop does no integer division. Thread (r, cg) of a CTA
// of R x (d / 8) threads takes 8 columns of blocks f = R blockIdx.x + r, then
// f + R gridDim.x, ..., U blocks' loads in flight per step.
template <int P, int U>
__global__ void __launch_bounds__(256) pool_rows_flat_kernel(const PoolParams p, int n_blocks, int R) {
  griddep_wait();
  griddep_launch();
  const int groups = p.d >> 3;
  const int cg = static_cast<int>(threadIdx.x) % groups, r = static_cast<int>(threadIdx.x) / groups;
  if (r >= R) return;
  const uint4* X4 = reinterpret_cast<const uint4*>(p.X) + cg;
  const int fstep = R * static_cast<int>(gridDim.x);
  bool bad = false;
  for (int f0 = R * static_cast<int>(blockIdx.x) + r; f0 < n_blocks; f0 += U * fstep) {
    uint4 raw[U][P];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int f = f0 + u * fstep;
      if (f < n_blocks)
#pragma unroll
        for (int q = 0; q < P; ++q) raw[u][q] = __ldg(X4 + (static_cast<size_t>(f) * P + q) * groups);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int f = f0 + u * fstep;
      if (f >= n_blocks) break;
      float lv[P][8];
#pragma unroll
      for (int q = 0; q < P; ++q) bf16x8_to_f32(raw[u][q], lv[q]);
#pragma unroll
      for (int level = 0; (1 << level) < P; ++level) {
        // lv[i] holds the sum of rows [i*width, (i+1)*width)
        const int n = P >> level;
        const int width = 2 << level;
#pragma unroll
        for (int i = 0; i < P / 2; ++i)
          if (i < n / 2)
#pragma unroll
            for (int e = 0; e < 8; ++e) lv[i][e] = lv[2 * i][e] + lv[2 * i + 1][e];
        for (int j = 0; j < p.n_scales; ++j) {
          if (p.scales[j] != width) continue;
          const float inv = 1.f / static_cast<float>(width);  // exact: width is a power of two
#pragma unroll
          for (int i = 0; i < P / 2; ++i) {
            if (i >= n / 2) break;
            uint4 o;
            uint32_t* ow = reinterpret_cast<uint32_t*>(&o);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float a0 = lv[i][2 * e] * inv, a1 = lv[i][2 * e + 1] * inv;
              bad |= !(fabsf(a0) <= 65504.f) || !(fabsf(a1) <= 65504.f);
              ow[e] = pack_half2(a0, a1);
            }
            reinterpret_cast<uint4*>(p.Xp[j] + (static_cast<size_t>(f) * (P / width) + i) * p.d)[cg] = o;
          }
        }
      }
    }
  }
  if (bad) atomicCAS(p.err, 0, kDevRange);
}

// One warp per (row, head): the head's dvp fp16 values (dvp <= 1024, a multiple
// of 128) are read once into registers, 8 per 16-byte load, and written back
// scaled; the padding columns are zero and stay zero (their weight is zero).
constexpr int kNormMaxLoads = 4;  // 16-byte loads per lane: 4 * 32 * 8 = 1024 values
__global__ void __launch_bounds__(256) head_norm_kernel(const HeadNormParams p) {
  griddep_wait();
  griddep_launch();
  const long long gw = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (gw >= p.total_warps) return;
  int j = 0;
  while (j + 1 < p.n_branches && gw >= p.br[j + 1].warp_begin) ++j;
  const HeadNormBranch& br = p.br[j];
  const long long local = gw - br.warp_begin;
  const long long row = local / br.heads;
  const int head = static_cast<int>(local % br.heads);
  __half* o = br.o + (row * br.heads + head) * p.dvp;
  const float* w = br.w + static_cast<size_t>(head) * p.dvp;
  const int lane = threadIdx.x & 31;
  uint4 u[kNormMaxLoads];
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < kNormMaxLoads; ++i) {
    const int c = (i * 32 + lane) * 8;
    u[i] = c < p.dvp ? *reinterpret_cast<const uint4*>(o + c) : make_uint4(0, 0, 0, 0);
    const __half2* h2 = reinterpret_cast<const __half2*>(&u[i]);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __half22float2(h2[e]);
      ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  const float inv = rsqrtf(ss / static_cast<float>(p.dv) + p.eps);
  bool bad = false;
#pragma unroll
  for (int i = 0; i < kNormMaxLoads; ++i) {
    const int c = (i * 32 + lane) * 8;
    if (c >= p.dvp) break;
    const __half2* h2 = reinterpret_cast<const __half2*>(&u[i]);
    const float4 wa = *reinterpret_cast<const float4*>(w + c);
    const float4 wb = *reinterpret_cast<const float4*>(w + c + 4);
    const float ws[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
    uint4 out;
    uint32_t* ow = reinterpret_cast<uint32_t*>(&out);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __half22float2(h2[e]);
      const float a0 = f.x * inv * ws[2 * e], a1 = f.y * inv * ws[2 * e + 1];
      bad |= !(fabsf(a0) <= 65504.f) || !(fabsf(a1) <= 65504.f);
      ow[e] = pack_half2(a0, a1);
    }
    *reinterpret_cast<uint4*>(o + c) = out;
  }
  if (bad) atomicCAS(p.err, 0, kDevRange);
}

constexpr int kGateThreads = 256;
constexpr int kGateChannels = 128;  // key channels per CTA

// 2^x by the hardware approximation (relative error about 2^-22, far below the
// fp16 rounding of the scaled q and k it feeds)
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// log2(x) by the hardware approximation (absolute error about 2^-22 for x in (1, 2])
__device__ __forceinline__ float lg2_approx(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Accumulates a packed fp16 pair's exponents into `acc` so that bit 15 or bit 31
// of acc ends up set iff some half seen was inf or nan (exponent all ones: adding
// one to the exponent field then carries into that half's sign position).
__device__ __forceinline__ void half2_track_nonfinite(uint32_t& acc, uint32_t h) {
  acc |= (h & 0x7c007c00u) + 0x04000400u;
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}

// tf32 split of an fp32 value: hi has the top 10 mantissa bits, lo the rest.
__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
  uint32_t h;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(h) : "f"(x));
  float r = x - __uint_as_float(h);
  uint32_t l;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(l) : "f"(r));
  hi = h;
  lo = l;
}

__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// One CTA per (branch, batch, head, 64-row half of a 128-row GLA chunk, 128 key
// channels), 256 threads.
//  0. cp.async stages the half chunk's low-rank gate rows g [64 x RP] and its q
//     and k rows [64 x 128] (fp16; the 16-byte chunks of a row are XOR-swizzled
//     by (row / 4) mod 8 so that phase 2 reads them without bank conflicts).
//  1. z = g W_g2^T for the 64 x 128 block on tensor cores (mma.sync m16n8k8 tf32;
//     each operand split into tf32 hi + lo parts, three products, so z keeps
//     fp32-level accuracy), then log alpha = logsigmoid(z + b_g) / normalizer,
//     kept in base-2 units (times log2 e) in shared memory; rows past the end of
//     the sequence get 0.
//  2. Thread (channel group cg of 8 channels, row group rg of 4 rows): the
//     cumulative sum of log alpha over its 4 rows, the exclusive prefix over the
//     16 row groups by a 16-lane shuffle scan, and Qs = q 2^{b - m},
//     Ks = k 2^{m - b} stored 16 bytes at a time. With b_loc the cumulative sum
//     from the half's first row and T its total: in the first half b - m =
//     b_loc - T, in the second half b - m = b_loc (m is the first half's total),
//     so each half needs only its own rows. Per chunk: gamma = e^{b_last - m},
//     mid = e^{m}.
constexpr int kGateBlk = 36;  // floats per (channel group, row group) block of log alpha: 4 x 8 + 4 padding

template <int RP>
struct GateSmem {
  static constexpr int kQK = 2 * kChunk * kGateChannels * 2;              // q, k rows (fp16)
  static constexpr int kLA = (kGateChannels / 8) * (kChunk / 4) * kGateBlk * 4;
  static constexpr int kGS = RP + 4;                                      // padded g row (floats)
  static constexpr int kG = kChunk * kGS * 4;
  static constexpr int kBytes = kQK + kLA + kG;
};

template <int RP>
__global__ void __launch_bounds__(kGateThreads, 3) gate_kernel(const __grid_constant__ GateParams p) {
  griddep_wait();
  griddep_launch();
  using L = GateSmem<RP>;
  extern __shared__ __align__(16) uint8_t gate_smem[];
  __half* qk_s = reinterpret_cast<__half*>(gate_smem);
  float* la_s = reinterpret_cast<float*>(gate_smem + L::kQK);
  float* g_s = reinterpret_cast<float*>(gate_smem + L::kQK + L::kLA);
  const int dkp = p.dkp;
  const int cblocks = dkp / kGateChannels;
  int bi = 0;
#pragma unroll 1
  for (int j = 1; j < p.n_branches; ++j)
    if (static_cast<int>(blockIdx.x) >= p.br[j].block_begin) bi = j;
  const GateBranch& P = p.br[bi];
  int local = blockIdx.x - P.block_begin;
  const int cb = local % cblocks;
  local /= cblocks;
  const int hc = local % P.n_halves;
  const int head = (local / P.n_halves) % P.heads;
  const int b = local / (P.n_halves * P.heads);
  const int ci = hc >> 1, second = hc & 1;
  const int n_chunks = (P.n_halves + 1) >> 1;
  const int t0 = hc * kChunk;
  const int nrows = min(kChunk, P.rows - t0);
  const int ldk = P.heads * dkp;
  const int cbase = head * dkp + cb * kGateChannels;  // first channel of this CTA
  const size_t row_base = static_cast<size_t>(b) * P.rows + t0;
  const int tid = threadIdx.x;

  // ---- phase 0: g rows (group 0), then q and k rows (group 1)
  constexpr int kGChunks = kChunk * RP / 4;
  for (int i = tid; i < kGChunks; i += kGateThreads) {
    const int row = i / (RP / 4), seg = i % (RP / 4);
    float* dst = g_s + row * L::kGS + seg * 4;
    if (row < nrows)
      cp_async16(dst, P.g + (row_base + row) * RP + seg * 4);
    else
      *reinterpret_cast<float4*>(dst) = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
#pragma unroll
  for (int it = 0; it < 2 * kChunk * 16 / kGateThreads; ++it) {
    const int flat = tid + it * kGateThreads;
    const int tsel = flat >> 10, row = (flat >> 4) & (kChunk - 1), seg = flat & 15;
    if (row < nrows) {
      const __half* src = (tsel ? P.k : P.q) + (row_base + row) * ldk + cbase + seg * 8;
      cp_async16(qk_s + (tsel * kChunk + row) * kGateChannels + ((seg ^ ((row >> 2) & 7)) * 8), src);
    }
  }
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 1;" ::: "memory");
  __syncthreads();

  // ---- phase 1: z = g W^T on tensor cores. Warp w owns channels [16w, 16w+16)
  // (two n8 tiles) for all 64 rows (four m16 tiles); K = RP in steps of 8.
  {
    const int warp = tid >> 5, lane = tid & 31;
    const int gq = lane >> 2, tq = lane & 3;
    float acc[4][2][4];
#pragma unroll
    for (int mt = 0; mt < 4; ++mt)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;
#pragma unroll
    for (int k8 = 0; k8 < RP / 8; ++k8) {
      // B fragments: W[channel][k]; b0 = (k = tq, n = gq), b1 = (k = tq + 4, n = gq)
      uint32_t bh[2][2], bl[2][2];
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const float* wr = P.Wg2 + static_cast<size_t>(cbase + warp * 16 + nt * 8 + gq) * RP + k8 * 8;
        split_tf32(__ldg(wr + tq), bh[nt][0], bl[nt][0]);
        split_tf32(__ldg(wr + tq + 4), bh[nt][1], bl[nt][1]);
      }
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        // A fragments: g[row][k]; a0 = (gq, tq), a1 = (gq + 8, tq), a2 = (gq, tq + 4), a3 = (gq + 8, tq + 4)
        const float* g0 = g_s + (mt * 16 + gq) * L::kGS + k8 * 8;
        const float* g1 = g0 + 8 * L::kGS;
        uint32_t ah[4], al[4];
        split_tf32(g0[tq], ah[0], al[0]);
        split_tf32(g1[tq], ah[1], al[1]);
        split_tf32(g0[tq + 4], ah[2], al[2]);
        split_tf32(g1[tq + 4], ah[3], al[3]);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          mma_tf32(acc[mt][nt], al, bh[nt]);
          mma_tf32(acc[mt][nt], ah, bl[nt]);
          mma_tf32(acc[mt][nt], ah, bh[nt]);
        }
      }
    }
    // log alpha (base 2) into the blocked layout; D fragment: d0 = (gq, 2tq),
    // d1 = (gq, 2tq+1), d2 = (gq+8, 2tq), d3 = (gq+8, 2tq+1). With z2 = z log2(e),
    // log2 alpha = (min(z2, 0) - log2(1 + 2^{-|z2|})) / normalizer, the base-2
    // form of logsigmoid(z) / normalizer (the log argument lies in (1, 2]).
    constexpr float kLog2e = 1.4426950408889634f;
    const float inv_norm = p.inv_normalizer;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int chl = warp * 16 + nt * 8 + 2 * tq;
      const float bias0 = __ldg(P.bg + cbase + chl) * kLog2e, bias1 = __ldg(P.bg + cbase + chl + 1) * kLog2e;
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int row = mt * 16 + gq + ((e & 2) ? 8 : 0), ch = chl + (e & 1);
          const float z2 = fmaf(acc[mt][nt][e], kLog2e, (e & 1) ? bias1 : bias0);
          const float la = (fminf(z2, 0.f) - lg2_approx(1.f + ex2_approx(-fabsf(z2)))) * inv_norm;
          la_s[((ch >> 3) * (kChunk / 4) + (row >> 2)) * kGateBlk + (row & 3) * 8 + (ch & 7)] = la;
        }
      }
    }
    if (nrows < kChunk) {
      // rows past the end of the sequence contribute nothing to the sums
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        const int chl = warp * 16 + nt * 8 + 2 * tq;
#pragma unroll
        for (int mt = 0; mt < 4; ++mt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int row = mt * 16 + gq + ((e & 2) ? 8 : 0), ch = chl + (e & 1);
            if (row >= nrows) la_s[((ch >> 3) * (kChunk / 4) + (row >> 2)) * kGateBlk + (row & 3) * 8 + (ch & 7)] = 0.f;
          }
      }
    }
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncthreads();

  // ---- phase 2: warp w holds channel groups 2w (lanes 0-15) and 2w+1 (lanes
  // 16-31); lane rg of a 16-lane segment holds rows [4rg, 4rg+4).
  const int lane = tid & 31;
  const int cg = 2 * (tid >> 5) + (lane >> 4), rg = lane & 15;
  const float* blk = la_s + (cg * (kChunk / 4) + rg) * kGateBlk;
  float c[4][8];
  float run[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) run[e] = 0.f;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const float4 x0 = *reinterpret_cast<const float4*>(blk + r * 8);
    const float4 x1 = *reinterpret_cast<const float4*>(blk + r * 8 + 4);
    const float x[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      run[e] += x[e];
      c[r][e] = run[e];
    }
  }
  // exclusive prefix over the row groups before this one, and the half's total
  float pre[8], tot[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    float v = run[e];
#pragma unroll
    for (int off = 1; off < 16; off <<= 1) {
      const float u = __shfl_up_sync(0xffffffffu, v, off, 16);
      if (rg >= off) v += u;
    }
    pre[e] = v - run[e];
    tot[e] = __shfl_sync(0xffffffffu, v, 15, 16);
  }
  // reference: b - m = b_loc - T in the first half, b_loc in the second
#pragma unroll
  for (int e = 0; e < 8; ++e) pre[e] -= second ? 0.f : tot[e];

  // A scaled value can leave the fp16 range only where its factor exceeds 1: b
  // does not increase along the chunk (log alpha <= 0), so in the first half
  // (rows up to m's) Qs = q 2^{b-m} can grow and Ks cannot, and in the second
  // half the reverse. Only the growing side is checked.
  uint32_t over = 0;
  const int sw = rg & 7;  // (row >> 2) & 7 for all four rows of this thread
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int row = 4 * rg + r;
    if (row >= nrows) break;
    const uint4 qv = *reinterpret_cast<const uint4*>(qk_s + row * kGateChannels + ((cg ^ sw) * 8));
    const uint4 kv = *reinterpret_cast<const uint4*>(qk_s + (kChunk + row) * kGateChannels + ((cg ^ sw) * 8));
    const __half2* qh = reinterpret_cast<const __half2*>(&qv);
    const __half2* kh = reinterpret_cast<const __half2*>(&kv);
    uint4 qo, ko;
    uint32_t* qw = reinterpret_cast<uint32_t*>(&qo);
    uint32_t* kw = reinterpret_cast<uint32_t*>(&ko);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float b0 = pre[2 * e] + c[r][2 * e], b1 = pre[2 * e + 1] + c[r][2 * e + 1];
      const float2 qf = __half22float2(qh[e]), kf = __half22float2(kh[e]);
      qw[e] = pack_half2(qf.x * ex2_approx(b0), qf.y * ex2_approx(b1));
      kw[e] = pack_half2(kf.x * ex2_approx(-b0), kf.y * ex2_approx(-b1));
      half2_track_nonfinite(over, second ? kw[e] : qw[e]);
    }
    const size_t go = (row_base + row) * ldk + cbase + cg * 8;
    *reinterpret_cast<uint4*>(P.qs + go) = qo;
    *reinterpret_cast<uint4*>(P.ks + go) = ko;
  }
  if (over & 0x80008000u) atomicCAS(p.err, 0, kDevRange);
  if (rg == 15) {
    const size_t gi = (static_cast<size_t>(b) * n_chunks + ci) * ldk + cbase + cg * 8;
    float* dst = second ? P.gamma : P.mid;
#pragma unroll
    for (int e = 0; e < 8; ++e) dst[gi + e] = exp2f(tot[e]);
    if (!second && hc + 1 >= P.n_halves)  // chunk without a second half: b_last = m
#pragma unroll
      for (int e = 0; e < 8; ++e) P.gamma[gi + e] = 1.f;
  }
}

template <int RP>
cudaError_t launch_gate_t(const GateParams& p, cudaStream_t st) {
  const int smem = GateSmem<RP>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(gate_kernel<RP>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(gate_kernel<RP>, dim3(p.total_blocks), dim3(kGateThreads), smem, st, p);
}

// O_t = sum_s w_{t,s} Y^(s)_{floor((t+1)/s)-1} (Eq. (11) with the causal hold of
// Sec. 3.3) when no branch has scale 1. One CTA per (sequence, tile of
// kHoldRows rows, block of up to 256 column groups): thread (r, cg) takes 8
// columns of rows t0 + r, t0 + r + R, ...; no division in the loop (the held
// row index is a shift for power-of-two scales).
constexpr int kHoldRows = 32;
__global__ void __launch_bounds__(256) hold_fuse_kernel(const HoldFuseParams p, int CG, int R) {
  griddep_wait();
  griddep_launch();
  const int groups = p.d >> 3;
  const int cgl = static_cast<int>(threadIdx.x) % CG, r = static_cast<int>(threadIdx.x) / CG;
  const int cg = static_cast<int>(blockIdx.z) * CG + cgl;
  if (r >= R || cg >= groups) return;
  const int b = blockIdx.y;
  const int t0 = blockIdx.x * kHoldRows, t1 = min(p.L, t0 + kHoldRows);
  uint4* ob = reinterpret_cast<uint4*>(p.out + static_cast<size_t>(b) * p.L * p.d) + cg;
  const float* wb = p.w + static_cast<size_t>(b) * p.L * p.n_scales;
#pragma unroll 4
  for (int t = t0 + r; t < t1; t += R) {
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
    for (int j = 0; j < kMaxScales; ++j) {
      if (j >= p.n_scales) break;
      const int i = (p.shift[j] >= 0 ? ((t + 1) >> p.shift[j]) : (t + 1) / p.scales[j]) - 1;
      if (i < 0) continue;
      const uint4 u =
          __ldg(reinterpret_cast<const uint4*>(p.Y[j] + (static_cast<size_t>(b) * p.rows[j] + i) * p.d) + cg);
      const __half2* h = reinterpret_cast<const __half2*>(&u);
      const float wj = __ldg(wb + static_cast<size_t>(t) * p.n_scales + j);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(h[e]);
        acc[2 * e] = fmaf(wj, f.x, acc[2 * e]);
        acc[2 * e + 1] = fmaf(wj, f.y, acc[2 * e + 1]);
      }
    }
    ob[static_cast<size_t>(t) * groups] =
        make_uint4(pack_bf162(acc[0], acc[1]), pack_bf162(acc[2], acc[3]), pack_bf162(acc[4], acc[5]),
                   pack_bf162(acc[6], acc[7]));
  }
}

__global__ void bf16_to_f16_rows_kernel(const __nv_bfloat16* src, int src_ld, int rows, int cols, __half* dst,
                                        int dst_ld, int* overflow) {
  const size_t n = static_cast<size_t>(rows) * cols;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int r = static_cast<int>(i / cols), c = static_cast<int>(i % cols);
    const float f = __bfloat162float(src[static_cast<size_t>(r) * src_ld + c]);
    if (!(fabsf(f) <= 65504.f)) atomicAdd(overflow, 1);
    dst[static_cast<size_t>(r) * dst_ld + c] = __float2half_rn(f);
  }
}

__global__ void bf16_copy_rows_kernel(const __nv_bfloat16* src, int src_ld, int rows, int cols, __nv_bfloat16* dst,
                                      int dst_ld) {
  const size_t n = static_cast<size_t>(rows) * cols;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int r = static_cast<int>(i / cols), c = static_cast<int>(i % cols);
    dst[static_cast<size_t>(r) * dst_ld + c] = src[static_cast<size_t>(r) * src_ld + c];
  }
}

}  // namespace

// MB: resident CTAs per SM the registers are fitted to (2 for 4-row blocks)
template <int P, int GPL, int NS>
cudaError_t launch_pool_rows(const PoolParams& p, cudaStream_t st) {
  constexpr int MB = P == 4 ? 2 : 1;
  const int smem = p.n_scales * p.d * static_cast<int>(sizeof(float));
  cudaError_t e = cudaFuncSetAttribute(pool_fuse_rows_kernel<P, GPL, NS, MB>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const size_t warps = static_cast<size_t>(p.B) * ((p.L + P - 1) / P);
  return launch_pdl(pool_fuse_rows_kernel<P, GPL, NS, MB>, dim3(static_cast<unsigned>((warps + 7) / 8)), dim3(256),
                    smem, st, p);
}

template <int P, int U>
cudaError_t launch_pool_flat(const PoolParams& p, cudaStream_t st) {
  const int groups = p.d / 8;
  const int R = 256 / groups;
  const long long n_blocks = static_cast<long long>(p.B) * p.L / P;
  const long long ctas = (n_blocks + static_cast<long long>(R) * U - 1) / (static_cast<long long>(R) * U);
  const long long resident = (P == 8 ? 2LL : 3LL) * sm_count();  // CTAs of 256 threads per SM at its registers
  const int grid = static_cast<int>(std::min<long long>(ctas, resident));
  return launch_pdl(pool_rows_flat_kernel<P, U>, dim3(grid), dim3(R * groups), 0, st, p, static_cast<int>(n_blocks),
                    R);
}

template <int P>
cudaError_t launch_pool_only(const PoolParams& p, cudaStream_t st) {
  const size_t n = static_cast<size_t>(p.B) * ((p.L + P - 1) / P) * (p.d / 8);
  return launch_pdl(pool_rows_kernel<P>, dim3(static_cast<unsigned>((n + 255) / 256)), dim3(256), 0, st, p);
}

cudaError_t launch_pool_fuse(const PoolParams& p, cudaStream_t st) {
  if (p.B * p.L == 0) return cudaSuccess;
  // block_rows carries the least common multiple of the coarse scales (1 if none);
  // the row-block kernels take P rows at a time, so every scale must divide P
  const int lcm = p.block_rows;
  if (!p.want_w) {
    // flat kernel: no mask, power-of-two coarse scales, whole blocks, d <= 2048
    const bool flat = !p.M && p.d <= 2048 && static_cast<long long>(p.B) * p.L < (1LL << 30);
    if (flat && lcm <= 2 && p.L % 2 == 0) return launch_pool_flat<2, 4>(p, st);
    if (flat && lcm == 4 && p.L % 4 == 0) return launch_pool_flat<4, 2>(p, st);
    if (flat && lcm == 8 && p.L % 8 == 0) return launch_pool_flat<8, 1>(p, st);
    if (2 % lcm == 0) return launch_pool_only<2>(p, st);
    if (4 % lcm == 0) return launch_pool_only<4>(p, st);
    if (6 % lcm == 0) return launch_pool_only<6>(p, st);
    if (8 % lcm == 0) return launch_pool_only<8>(p, st);
  }
  if (p.n_scales * p.d * 4 <= 160 * 1024) {
    if (4 % lcm == 0)
      return p.n_scales <= 4 ? launch_pool_rows<4, 2, 4>(p, st) : launch_pool_rows<4, 2, 8>(p, st);
    if (6 % lcm == 0)
      return p.n_scales <= 4 ? launch_pool_rows<6, 2, 4>(p, st) : launch_pool_rows<6, 2, 8>(p, st);
    if (8 % lcm == 0)
      return p.n_scales <= 4 ? launch_pool_rows<8, 2, 4>(p, st) : launch_pool_rows<8, 2, 8>(p, st);
  }
  PoolParams q = p;
  while (q.block_rows < 32) q.block_rows *= 2;
  dim3 grid((p.L + q.block_rows - 1) / q.block_rows, p.B);
  return launch_pdl(pool_fuse_kernel, grid, dim3(kPoolThreads), 0, st, q);
}

cudaError_t launch_head_norm(const HeadNormParams& p, cudaStream_t st) {
  if (p.total_warps <= 0) return cudaSuccess;
  if (p.dvp % 128 || p.dvp > kNormMaxLoads * 32 * 8) return cudaErrorInvalidValue;
  return launch_pdl(head_norm_kernel, dim3(static_cast<unsigned>((p.total_warps + 7) / 8)), dim3(256), 0, st, p);
}

cudaError_t launch_gate(const GateParams& p, cudaStream_t st) {
  if (p.total_blocks <= 0) return cudaSuccess;
  if (p.dkp % kGateChannels) return cudaErrorInvalidValue;
  return p.rp == 16 ? launch_gate_t<16>(p, st) : launch_gate_t<32>(p, st);
}

cudaError_t launch_hold_fuse(const HoldFuseParams& p, cudaStream_t st) {
  if (p.B * p.L == 0) return cudaSuccess;
  const int groups = p.d / 8;
  const int CG = std::min(groups, 256), R = 256 / CG;
  const dim3 grid((p.L + kHoldRows - 1) / kHoldRows, p.B, (groups + CG - 1) / CG);
  return launch_pdl(hold_fuse_kernel, grid, dim3(CG * R), 0, st, p, CG, R);
}

cudaError_t launch_bf16_to_f16_rows(const __nv_bfloat16* src, int src_ld, int rows, int cols, __half* dst,
                                    int dst_ld, int* overflow, cudaStream_t st) {
  if (rows * cols == 0) return cudaSuccess;
  bf16_to_f16_rows_kernel<<<256, 256, 0, st>>>(src, src_ld, rows, cols, dst, dst_ld, overflow);
  return cudaGetLastError();
}

cudaError_t launch_bf16_copy_rows(const __nv_bfloat16* src, int src_ld, int rows, int cols, __nv_bfloat16* dst,
                                  int dst_ld, cudaStream_t st) {
  if (rows * cols == 0) return cudaSuccess;
  bf16_copy_rows_kernel<<<256, 256, 0, st>>>(src, src_ld, rows, cols, dst, dst_ld);
  return cudaGetLastError();
}

}  // namespace msgla
