// k_aux.cu -- the CUDA-core kernels of the MS-GLA path:
//   pool_fuse_kernel  one pass over X: mean pooling of s adjacent rows for every
//                     scale s > 1 (reading notes Sec. 3.1, Eq. (8)) and the
//                     fusion weights w_t = softmax(W_fuse x_t + b_fuse) from the
//                     unpooled rows (Sec. 3.3, Eq. (10)).
//   gate_kernel       log alpha = logsigmoid(g W_g2^T + b_g) / normalizer (the
//                     low-rank gate of Sec. 2.1), its cumulative sum b inside
//                     each 64-row chunk, Qs = q e^{b}, Ks = k e^{-b} and the
//                     chunk decay gamma = e^{b_last} used by the GLA kernel.
//   hold_fuse_kernel  O_t = sum_s w_{t,s} Y^(s)_{floor((t+1)/s)-1} (Sec. 3.3,
//                     Eq. (11)) when no branch has scale 1.
//   weight converters used once by msgla_create.
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
#pragma unroll
    for (int j = 0; j < kMaxScales; ++j)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[j][e] = 0.f;
    for (int r = 0; r < nrows; ++r) {
      const int t = row0 + r;
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
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[j][e] += x[e];
          const bool block_end = ((t + 1) % s == 0) || (t == p.L - 1);
          if (block_end) {
            if (active) {
              const int i = t / s;
              const float inv = 1.f / static_cast<float>(t - i * s + 1);
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

constexpr int kGateRows = kChunk;

// grid (n_chunks, heads, B); block dkp/2 threads, two channels per thread.
__global__ void gate_kernel(const GateParams p) {
  extern __shared__ float gsm[];
  float* g_s = gsm;                       // [64][rp]
  float* w_s = gsm + kGateRows * p.rp;    // [dkp][rp]
  const int c = blockIdx.x, head = blockIdx.y, b = blockIdx.z;
  const int t0 = c * kGateRows;
  const int nrows = min(kGateRows, p.rows - t0);
  const int ldk = p.heads * p.dkp;
  for (int i = threadIdx.x; i < nrows * p.rp; i += blockDim.x)
    g_s[i] = p.g[(static_cast<size_t>(b) * p.rows + t0) * p.rp + i];
  for (int i = threadIdx.x; i < p.dkp * p.rp; i += blockDim.x)
    w_s[i] = p.Wg2[static_cast<size_t>(head) * p.dkp * p.rp + i];
  __syncthreads();
  const int a0 = 2 * threadIdx.x;
  const int ch = head * p.dkp + a0;
  const float bias0 = p.bg[ch], bias1 = p.bg[ch + 1];
  const float* w0 = w_s + a0 * p.rp;
  const float* w1 = w0 + p.rp;
  float b0 = 0.f, b1 = 0.f;
  bool bad = false;
  for (int i = 0; i < nrows; ++i) {
    float z0 = bias0, z1 = bias1;
    const float* gi = g_s + i * p.rp;
    for (int r = 0; r < p.rp; ++r) {
      z0 = fmaf(gi[r], w0[r], z0);
      z1 = fmaf(gi[r], w1[r], z1);
    }
    // logsigmoid(z) = min(z, 0) - log(1 + e^{-|z|})
    b0 += (fminf(z0, 0.f) - log1pf(__expf(-fabsf(z0)))) * p.inv_normalizer;
    b1 += (fminf(z1, 0.f) - log1pf(__expf(-fabsf(z1)))) * p.inv_normalizer;
    const size_t idx = (static_cast<size_t>(b) * p.rows + t0 + i) * ldk + ch;
    const float2 qf = __half22float2(*reinterpret_cast<const __half2*>(p.q + idx));
    const float2 kf = __half22float2(*reinterpret_cast<const __half2*>(p.k + idx));
    const float e0 = __expf(b0), e1 = __expf(b1);
    const float ks0 = kf.x * __expf(-b0), ks1 = kf.y * __expf(-b1);
    bad |= !(fabsf(ks0) <= 65504.f) || !(fabsf(ks1) <= 65504.f);
    *reinterpret_cast<__half2*>(p.qs + idx) = __floats2half2_rn(qf.x * e0, qf.y * e1);
    *reinterpret_cast<__half2*>(p.ks + idx) = __floats2half2_rn(ks0, ks1);
  }
  float* gm = p.gamma + (static_cast<size_t>(b) * p.n_chunks + c) * ldk + ch;
  gm[0] = __expf(b0);
  gm[1] = __expf(b1);
  if (bad) atomicCAS(p.err, 0, kDevRange);
}

// one thread per 8 output columns of one row; flat grid over B*L*(d/8)
__global__ void hold_fuse_kernel(const HoldFuseParams p) {
  const int groups = p.d / 8;
  const size_t gid = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  if (gid >= static_cast<size_t>(p.B) * p.L * groups) return;
  const int cg = static_cast<int>(gid % groups);
  const size_t bt = gid / groups;
  const int t = static_cast<int>(bt % p.L), b = static_cast<int>(bt / p.L);
  float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  const float* w = p.w + bt * p.n_scales;
  for (int j = 0; j < p.n_scales; ++j) {
    const int s = p.scales[j];
    const int i = (t + 1) / s - 1;
    if (i < 0) continue;
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p.Y[j] + (static_cast<size_t>(b) * p.rows[j] + i) * p.d) + cg);
    const __half2* h = reinterpret_cast<const __half2*>(&u);
    const float wj = w[j];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float2 f = __half22float2(h[e]);
      acc[2 * e] = fmaf(wj, f.x, acc[2 * e]);
      acc[2 * e + 1] = fmaf(wj, f.y, acc[2 * e + 1]);
    }
  }
  uint4 o;
  o.x = pack_bf162(acc[0], acc[1]);
  o.y = pack_bf162(acc[2], acc[3]);
  o.z = pack_bf162(acc[4], acc[5]);
  o.w = pack_bf162(acc[6], acc[7]);
  reinterpret_cast<uint4*>(p.out + bt * p.d)[cg] = o;
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

cudaError_t launch_pool_fuse(const PoolParams& p, cudaStream_t st) {
  if (p.B * p.L == 0) return cudaSuccess;
  dim3 grid((p.L + p.block_rows - 1) / p.block_rows, p.B);
  pool_fuse_kernel<<<grid, kPoolThreads, 0, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_gate(const GateParams& p, cudaStream_t st) {
  if (p.B * p.rows == 0) return cudaSuccess;
  const int smem = (kGateRows + p.dkp) * p.rp * static_cast<int>(sizeof(float));
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(gate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
  }
  dim3 grid(p.n_chunks, p.heads, p.B);
  gate_kernel<<<grid, p.dkp / 2, smem, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_hold_fuse(const HoldFuseParams& p, cudaStream_t st) {
  if (p.B * p.L == 0) return cudaSuccess;
  const size_t n = static_cast<size_t>(p.B) * p.L * (p.d / 8);
  hold_fuse_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, st>>>(p);
  return cudaGetLastError();
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
