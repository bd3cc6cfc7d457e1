// k_aux.cu -- the CUDA-core kernels of the MS-GLA path:
//   pool_fuse_kernel  one pass over X: mean pooling of s adjacent rows for every
//                     scale s > 1 (reading notes Sec. 3.1, Eq. (8)) and the
//                     fusion weights w_t = softmax(W_fuse x_t + b_fuse) from the
//                     unpooled rows (Sec. 3.3, Eq. (10)); pool_fuse_rows_kernel
//                     does both per row block when there is no scale-1 branch,
//                     pool_rows_kernel and pool_rows_flat_kernel pool only (with
//                     a scale-1 branch the fusion logits come from its
//                     projection GEMM).
//   gate_kernel       the gate of Sec. 2.1 in the chunkwise GLA form: with b the
//                     cumulative sum of log2 alpha over a 128-row chunk and m
//                     its value at the chunk's row 63, the exponents d = b - m
//                     per row and key channel (the projection scales q and k by
//                     2^{+-d}), and per chunk gamma = 2^{b_127 - m}, mid = 2^{m}.
//   head_norm_kernel  optional per-branch normalisation (Sec. 3.2), read as an
//                     RMS norm of each head's GLA output row, in place.
//   hold_fuse_kernel  O_t = sum_s w_{t,s} Y^(s)_{floor((t+1)/s)-1} (Sec. 3.3,
//                     Eq. (11)) when no branch has scale 1.
//   weight converters used once by msgla_create.
#include <algorithm>
#include <type_traits>

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

// O_t = sum_s w_{t,s} Y^(s)_{floor((t+1)/s)-1} (Eq. (11) with the causal hold of
// Sec. 3.3) when no branch has scale 1. One CTA per (sequence, tile of
// kHoldRows rows, block of up to 256 column groups): thread (r, cg) takes 8
// columns of rows t0 + r, t0 + r + R, ...; no division in the loop (the held
// row index is a shift for power-of-two scales).
// One item per (branch, sequence, half of a 128-row chunk, block of 256 key
// channels), a CTA of 128 threads; thread t owns channels c0 + 2t, c0 + 2t + 1.
//  1. The half's 64 gate inputs g (rank RP) go to shared memory: a scale-1
//     row's are its columns of U, a coarse row's the mean of its block's valid
//     unpooled rows' columns (Eq. (8), pooling being linear).
//  2. Per row z2 = log2(e) (g W_g2[c]^T + b_g[c]) (packed fp32 pairs over the
//     rank) and l = log2 alpha = (min(z2, 0) - log2(1 + 2^{-|z2|})) /
//     normalizer: logsigmoid in base 2 with the hardware 2^x and log2
//     approximations (relative errors near 2^-22).
//  3. The first half walks its rows backwards: d(r) = b(r) - m = -(sum of l over
//     rows r+1..63), and its total is m (mid = 2^m); the second half walks
//     forwards: d(r) = sum of l over rows 64..r, its total giving gamma =
//     2^{b_127 - m}. The projection GEMM scales q and k of the row by 2^{+-d}.
//     Rows past the sequence's end add nothing (a chunk without a second half
//     gets gamma = 1).
constexpr int kGateThreads = 128;
constexpr int kGateRows = 64;
constexpr int kGateChannels = 2 * kGateThreads;

template <int RP>
__device__ __forceinline__ void gate_item(const GateParams& p, int item, float* gs);

// Persistent over the items (a grid of whole waves): CTA x takes items x,
// x + gridDim.x, ...
template <int RP>
__global__ void __launch_bounds__(kGateThreads) gate_kernel(const __grid_constant__ GateParams p) {
  __shared__ __align__(16) float gs[kGateRows * RP];
  griddep_wait();
  griddep_launch();
  if (p.clear && blockIdx.x == 0 && threadIdx.x == 0) *p.clear = 0ull;
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < p.n_clear_rows; i += blockDim.x) p.clear_rows[i] = 0ull;
#pragma unroll 1
  for (int item = blockIdx.x; item < p.total_blocks; item += gridDim.x) {
    gate_item<RP>(p, item, gs);
    __syncthreads();  // the next item overwrites gs
  }
}

template <int RP>
__device__ __forceinline__ void gate_item(const GateParams& p, int item, float* gs) {
  int bi = 0;
#pragma unroll 1
  for (int j = 1; j < p.n_branches; ++j)
    if (item >= p.br[j].block_begin) bi = j;
  const GateBranch& P = p.br[bi];
  int local = item - P.block_begin;
  const int cblk = local % P.cblocks;
  local /= P.cblocks;
  const int half = local & 1;
  local >>= 1;
  const int chunk = local % P.n_chunks;
  const int b = local / P.n_chunks;
  const int r0 = chunk * 2 * kGateRows + half * kGateRows;  // first pooled row of the half
  const int nr = min(kGateRows, P.rows - r0);               // its rows inside the sequence
  const int tid = threadIdx.x;
  const size_t ubase = static_cast<size_t>(b) * p.L;
  // 1. gate inputs of the half's rows
  for (int idx = tid; idx < kGateRows * RP / 4; idx += kGateThreads) {
    const int row = idx / (RP / 4), k4 = idx % (RP / 4);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (row < nr) {
      const int t0 = (r0 + row) * P.scale, t1 = min(t0 + P.scale, p.L);
      float cnt = 0.f;
      for (int t = t0; t < t1; ++t) {
        if (p.mask && !__ldg(p.mask + ubase + t)) continue;
        const float4 x = __ldg(reinterpret_cast<const float4*>(p.u + (ubase + t) * p.ldu + P.ucol) + k4);
        acc.x += x.x;
        acc.y += x.y;
        acc.z += x.z;
        acc.w += x.w;
        cnt += 1.f;
      }
      if (P.scale > 1) {
        const float inv = 1.f / fmaxf(cnt, 1.f);
        acc.x *= inv;
        acc.y *= inv;
        acc.z *= inv;
        acc.w *= inv;
      }
    }
    *reinterpret_cast<float4*>(gs + row * RP + 4 * k4) = acc;
  }
  __syncthreads();
  const int c0 = cblk * kGateChannels + 2 * tid;
  if (c0 >= P.ldk || nr <= 0) return;
  // 2. this thread's two rows of W_g2 and biases, in log2 units, as pairs over the rank
  constexpr float kLog2e = 1.4426950408889634f;
  uint64_t w0[RP / 2], w1[RP / 2];
  {
    const float4* a = reinterpret_cast<const float4*>(P.Wg2 + static_cast<size_t>(c0) * RP);
#pragma unroll
    for (int j = 0; j < RP / 4; ++j) {
      const float4 x = __ldg(a + j), y = __ldg(a + RP / 4 + j);
      w0[2 * j] = f2_pack(x.x * kLog2e, x.y * kLog2e);
      w0[2 * j + 1] = f2_pack(x.z * kLog2e, x.w * kLog2e);
      w1[2 * j] = f2_pack(y.x * kLog2e, y.y * kLog2e);
      w1[2 * j + 1] = f2_pack(y.z * kLog2e, y.w * kLog2e);
    }
  }
  const float2 bb = __ldg(reinterpret_cast<const float2*>(P.bg + c0));
  const float bias0 = bb.x * kLog2e, bias1 = bb.y * kLog2e;
  const float inv_norm = p.inv_normalizer;
  // log2 alpha of row r for both channels (two packed partial sums per channel)
  auto log2_alpha = [&](const float* g_row, float& l0, float& l1) {
    const uint64_t zero = f2_pack(0.f, 0.f);
    uint64_t a0 = zero, b0 = zero, a1 = zero, b1 = zero;
    const float4* g4 = reinterpret_cast<const float4*>(g_row);
#pragma unroll
    for (int j = 0; j < RP / 4; ++j) {
      const float4 g = g4[j];
      const uint64_t g01 = f2_pack(g.x, g.y), g23 = f2_pack(g.z, g.w);
      a0 = f2_fma(g01, w0[2 * j], a0);
      b0 = f2_fma(g23, w0[2 * j + 1], b0);
      a1 = f2_fma(g01, w1[2 * j], a1);
      b1 = f2_fma(g23, w1[2 * j + 1], b1);
    }
    const float2 pa0 = f2_unpack(a0), pb0 = f2_unpack(b0), pa1 = f2_unpack(a1), pb1 = f2_unpack(b1);
    const float z0 = bias0 + ((pa0.x + pa0.y) + (pb0.x + pb0.y));
    const float z1 = bias1 + ((pa1.x + pa1.y) + (pb1.x + pb1.y));
    l0 = fminf(z0, 0.f) - lg2_approx(1.f + ex2_approx(-fabsf(z0)));
    l1 = fminf(z1, 0.f) - lg2_approx(1.f + ex2_approx(-fabsf(z1)));
  };
  // Rows go in batches of kBatch, walked by a pointer stepping one row (backwards
  // in the first half): first the batch's log2 alpha (independent of each
  // other), then in row order d (first half: the sum of the rows after it,
  // negated, taken before its own l is added; second half: the running sum
  // including l), stored as soon as it is known. Full batches run without
  // bounds checks; the rows of a last, short batch one at a time.
  const int rstride = P.ldk / 2;  // float2 per row
  const int first = half == 0 ? nr - 1 : 0;
  float2* dp = reinterpret_cast<float2*>(P.d + (static_cast<size_t>(b) * P.rows + r0 + first) * P.ldk + c0);
  const float* gp = gs + first * RP;
  float acc0 = 0.f, acc1 = 0.f;
  auto walk = [&](auto dir) {
    constexpr int kDir = decltype(dir)::value;  // -1: first half (backwards), +1: second half
    constexpr int kBatch = 8;
    const float sgn = kDir < 0 ? -inv_norm : inv_norm;
    const int nfull = nr / kBatch;
#pragma unroll 1
    for (int bt = 0; bt < nfull; ++bt) {
      float l0[kBatch], l1[kBatch];
#pragma unroll
      for (int i = 0; i < kBatch; ++i) log2_alpha(gp + kDir * i * RP, l0[i], l1[i]);
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        const float a0 = acc0 + l0[i], a1 = acc1 + l1[i];
        dp[kDir * i * rstride] = kDir < 0 ? make_float2(acc0 * sgn, acc1 * sgn) : make_float2(a0 * sgn, a1 * sgn);
        acc0 = a0;
        acc1 = a1;
      }
      dp += kDir * kBatch * rstride;
      gp += kDir * kBatch * RP;
    }
#pragma unroll 1
    for (int r = nfull * kBatch; r < nr; ++r) {
      float l0, l1;
      log2_alpha(gp, l0, l1);
      const float a0 = acc0 + l0, a1 = acc1 + l1;
      *dp = kDir < 0 ? make_float2(acc0 * sgn, acc1 * sgn) : make_float2(a0 * sgn, a1 * sgn);
      acc0 = a0;
      acc1 = a1;
      dp += kDir * rstride;
      gp += kDir * RP;
    }
  };
  if (half == 0)
    walk(std::integral_constant<int, -1>());
  else
    walk(std::integral_constant<int, 1>());
  const size_t gi = (static_cast<size_t>(b) * P.n_chunks + chunk) * P.ldk + c0;
  if (half == 0) {
    *reinterpret_cast<float2*>(P.mid + gi) = make_float2(ex2_approx(acc0 * inv_norm), ex2_approx(acc1 * inv_norm));
    if (P.rows - r0 <= kGateRows)  // no second half: b_127 = m
      *reinterpret_cast<float2*>(P.gamma + gi) = make_float2(1.f, 1.f);
  } else {
    *reinterpret_cast<float2*>(P.gamma + gi) = make_float2(ex2_approx(acc0 * inv_norm), ex2_approx(acc1 * inv_norm));
  }
}

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


// whole waves of resident CTAs, no more than there are items
template <int RP>
cudaError_t launch_gate_t(const GateParams& p, cudaStream_t st) {
  static int per_sm = 0;
  if (per_sm == 0 && (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, gate_kernel<RP>, kGateThreads, 0) !=
                          cudaSuccess || per_sm < 1))
    per_sm = 1;
  const int grid = std::min(p.total_blocks, per_sm * sm_count());
  return launch_pdl(gate_kernel<RP>, dim3(grid), dim3(kGateThreads), 0, st, p);
}

cudaError_t launch_gate(const GateParams& p, cudaStream_t st) {
  if (p.total_blocks <= 0) return cudaSuccess;
  if (p.rp == 16) return launch_gate_t<16>(p, st);
  if (p.rp == 32) return launch_gate_t<32>(p, st);
  return cudaErrorInvalidValue;
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
