// k_gemm.cu -- grouped tcgen05 GEMM for the MS-GLA projections.
//
// D[rows x N] = A[rows x K] * B[N x K]^T for each batch element and each task,
// with A and B K-major in global memory (PyTorch Linear layout), both bf16 or
// both fp16, fp32 accumulation in TMEM. Persistent: one CTA per SM walks the
// 128 x BN tiles round-robin (consecutive tiles share their A rows in L2):
//   warp 0      TMA producer (4-stage ring of 128B-swizzled A/B tiles, running
//               ahead across tile boundaries)
//   warp 1      TMEM allocation + single-thread tcgen05.mma issue into one of two
//               accumulators (2 x BN columns)
//   warps 2..5  epilogue of the other accumulator (tcgen05.ld, one row per thread),
//               overlapping the next tile's main loop
// Epilogues (MS-GLA reading notes, Secs. 3.2-3.3):
//   kEpiProj      q | k | v columns to fp16, the low-rank gate columns to fp32
//   kEpiStoreF16  a coarse branch's Y^(s) = o W_o^T to fp16
//   kEpiFuse      the scale-1 branch's Y^(1) fused with the causal hold of the
//                 coarse branches and the fusion softmax weights (Eq. (11)):
//                 O_t = w_{t,1} Y^(1)_t + sum_s w_{t,s} Y^(s)_{floor((t+1)/s)-1}
#include "msgla_internal.h"
#include "sm100_ptx.cuh"

namespace msgla {
namespace {

constexpr int kStages = 4;
constexpr int kThreads = 192;

template <int BN>
struct GemmLayout {
  static constexpr int kABytes = kGemmBM * kGemmBK * 2;
  static constexpr int kBBytes = BN * kGemmBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kBarOffset = kStages * kStageBytes;
  static constexpr int kSmemBytes = kBarOffset + 256 + 1024;  // barriers + 1024 B alignment slack
};

__device__ __forceinline__ void cvt_store_f16x32(__half* dst, const uint32_t (&r)[32]) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint4 u;
    u.x = pack_half2(__uint_as_float(r[8 * j + 0]), __uint_as_float(r[8 * j + 1]));
    u.y = pack_half2(__uint_as_float(r[8 * j + 2]), __uint_as_float(r[8 * j + 3]));
    u.z = pack_half2(__uint_as_float(r[8 * j + 4]), __uint_as_float(r[8 * j + 5]));
    u.w = pack_half2(__uint_as_float(r[8 * j + 6]), __uint_as_float(r[8 * j + 7]));
    d4[j] = u;
  }
}

__device__ __forceinline__ void store_f32(float* dst, const uint32_t* r, int n) {
  // n is a multiple of 4 and dst is 16-byte aligned
  float4* d4 = reinterpret_cast<float4*>(dst);
  for (int j = 0; j < n / 4; ++j)
    d4[j] = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]), __uint_as_float(r[4 * j + 2]),
                        __uint_as_float(r[4 * j + 3]));
}

__device__ __forceinline__ void add_scaled_f16x32(float (&acc)[32], const __half* src, float wgt) {
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    uint4 u = __ldg(s4 + j);
    const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float2 f = __half22float2(h[e]);
      acc[8 * j + 2 * e] = fmaf(wgt, f.x, acc[8 * j + 2 * e]);
      acc[8 * j + 2 * e + 1] = fmaf(wgt, f.y, acc[8 * j + 2 * e + 1]);
    }
  }
}

struct TileCoord {
  int task, b, m0, n0, n_eff, kblocks;
};

__device__ __forceinline__ TileCoord decode_tile(const GemmParams& p, int tile, int bn) {
  TileCoord c;
  int ti = 0;
#pragma unroll 1
  for (int t = 1; t < p.n_tasks; ++t)
    if (tile >= p.task[t].tile_begin) ti = t;
  const GemmTask& T = p.task[ti];
  const int local = tile - T.tile_begin;
  const int n_tile = local % T.n_tiles;
  const int m_tile = (local / T.n_tiles) % T.m_tiles;
  c.task = ti;
  c.b = local / (T.n_tiles * T.m_tiles);
  c.m0 = m_tile * kGemmBM;
  c.n0 = n_tile * bn;
  const int n_rem = T.N - c.n0;
  c.n_eff = n_rem >= bn ? bn : ((n_rem + 15) / 16) * 16;
  c.kblocks = (T.K + kGemmBK - 1) / kGemmBK;
  return c;
}

template <int BN>
__device__ __forceinline__ void epilogue_tile(const GemmParams& p, const TileCoord& tc, uint32_t tacc, int quad,
                                              int lane) {
  const GemmTask& T = p.task[tc.task];
  const int r = quad * 32 + lane;
  const int row = tc.m0 + r;
  const bool valid = row < T.rows;
  const size_t grow = static_cast<size_t>(tc.b) * T.rows + row;
  float wts[kMaxScales];
  if (T.epi == kEpiFuse && valid) {
    // w = softmax(W_fuse x + b_fuse) from the logits of the projection GEMM (Eq. (10))
    float zmax = -INFINITY;
    for (int j = 0; j < T.n_scales; ++j) {
      wts[j] = __ldg(T.zf + grow * T.ldz + j) + __ldg(T.bfuse + j);
      zmax = fmaxf(zmax, wts[j]);
    }
    float sum = 0.f;
    for (int j = 0; j < T.n_scales; ++j) {
      wts[j] = __expf(wts[j] - zmax);
      sum += wts[j];
    }
    const float inv = 1.f / sum;
    for (int j = 0; j < T.n_scales; ++j) wts[j] *= inv;
    if (tc.n0 == 0)
      for (int j = 0; j < T.n_scales; ++j) T.w[grow * T.n_scales + j] = wts[j];
  }
  const float wmain = (T.epi == kEpiFuse && valid) ? wts[T.main_index] : 0.f;
  for (int c0 = 0; c0 < tc.n_eff; c0 += 32) {
    uint32_t v[32];
    tmem_ld32(tmem_addr(tacc, quad * 32, c0), v);
    tmem_wait_ld();
    if (!valid) continue;
    const int col = tc.n0 + c0;
    if (T.epi == kEpiProj) {
      if (col < T.nq) {
        cvt_store_f16x32(T.q + grow * T.nq + col, v);
      } else if (col < T.nq + T.nk) {
        cvt_store_f16x32(T.k + grow * T.nk + (col - T.nq), v);
      } else if (col < T.nq + T.nk + T.nv) {
        cvt_store_f16x32(T.v + grow * T.nv + (col - T.nq - T.nk), v);
      } else {
        const int gc = col - T.nq - T.nk - T.nv;
        if (gc < T.ng) store_f32(T.g + grow * T.ng + gc, v, (T.ng - gc) < 32 ? (T.ng - gc) : 32);
        const int zs = (gc > T.ng ? gc : T.ng);  // first z column in this chunk (in gc units)
        const int zc = zs - T.ng;
        if (T.nz > 0 && zc < T.ldz && zs - gc < 32) {
          const int n = (T.ldz - zc) < (32 - (zs - gc)) ? (T.ldz - zc) : (32 - (zs - gc));
          store_f32(T.z + grow * T.ldz + zc, v + (zs - gc), n);
        }
      }
    } else if (T.epi == kEpiStoreF16) {
      cvt_store_f16x32(T.y + grow * T.N + col, v);
    } else {
      float acc[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) acc[j] = wmain * __uint_as_float(v[j]);
      for (int c = 0; c < T.n_coarse; ++c) {
        const int s = T.coarse_scale[c];
        const int i = (row + 1) / s - 1;
        if (i < 0) continue;
        const float wc = wts[T.coarse_index[c]];
        const __half* src = T.coarse_y[c] + (static_cast<size_t>(tc.b) * T.coarse_rows[c] + i) * T.N + col;
        add_scaled_f16x32(acc, src, wc);
      }
      uint4* d4 = reinterpret_cast<uint4*>(T.out + grow * T.N + col);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint4 u;
        u.x = pack_bf162(acc[8 * j + 0], acc[8 * j + 1]);
        u.y = pack_bf162(acc[8 * j + 2], acc[8 * j + 3]);
        u.z = pack_bf162(acc[8 * j + 4], acc[8 * j + 5]);
        u.w = pack_bf162(acc[8 * j + 6], acc[8 * j + 7]);
        d4[j] = u;
      }
    }
  }
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1) gemm_kernel(const __grid_constant__ GemmParams p) {
  using Lay = GemmLayout<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + Lay::kBarOffset);
  uint64_t* empty_bar = full_bar + kStages;
  uint64_t* acc_full = empty_bar + kStages;  // [2]
  uint64_t* acc_empty = acc_full + 2;        // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 128);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 2 * BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int ntiles = p.total_tiles;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer (runs ahead across tiles)
    for (int t = 0; t < p.n_tasks; ++t) {
      prefetch_tmap(&p.task[t].tmA);
      prefetch_tmap(&p.task[t].tmB);
    }
    uint32_t kbg = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
      const TileCoord tc = decode_tile(p, tile, BN);
      const GemmTask& T = p.task[tc.task];
      for (int kb = 0; kb < tc.kblocks; ++kb, ++kbg) {
        const uint32_t s = kbg % kStages;
        if (kbg >= kStages && !mbar_wait(&empty_bar[s], ((kbg / kStages) - 1) & 1, abort_flag, p.err)) {
          ok = false;
          break;
        }
        uint8_t* sa = smem + s * Lay::kStageBytes;
        uint8_t* sb = sa + Lay::kABytes;
        mbar_arrive_expect_tx(&full_bar[s], Lay::kStageBytes);
        tma_load_3d(&T.tmA, &full_bar[s], sa, kb * kGemmBK, tc.m0, tc.b);
        tma_load_2d(&T.tmB, &full_bar[s], sb, kb * kGemmBK, tc.n0);
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    uint32_t kbg = 0, it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x, ++it) {
      const TileCoord tc = decode_tile(p, tile, BN);
      const uint32_t buf = it & 1;
      if (it >= 2 && !mbar_wait(&acc_empty[buf], ((it >> 1) - 1) & 1, abort_flag, p.err)) break;
      tc_fence_after();
      const uint32_t idesc = idesc_f16(kGemmBM, tc.n_eff, p.task[tc.task].ab_bf16, 0, 0);
      const uint32_t tacc = tmem + buf * BN;
      for (int kb = 0; kb < tc.kblocks; ++kb, ++kbg) {
        const uint32_t s = kbg % kStages;
        if (!mbar_wait(&full_bar[s], (kbg / kStages) & 1, abort_flag, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + s * Lay::kStageBytes);
        const uint32_t sb = sa + Lay::kABytes;
#pragma unroll
        for (int kk = 0; kk < kGemmBK / 16; ++kk)
          umma_f16(tacc, sdesc_sw128(sa + kk * 32, 16, 1024), sdesc_sw128(sb + kk * 32, 16, 1024), idesc,
                   (kb | kk) != 0);
        umma_commit(&empty_bar[s]);
      }
      if (ok) umma_commit(&acc_full[buf]);
    }
  } else if (warp >= 2) {
    // ---------------- epilogue: one accumulator row per thread
    const int quad = warp & 3;
    uint32_t it = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
      const TileCoord tc = decode_tile(p, tile, BN);
      const uint32_t buf = it & 1;
      if (!mbar_wait(&acc_full[buf], (it >> 1) & 1, abort_flag, p.err)) break;
      tc_fence_after();
      epilogue_tile<BN>(p, tc, tmem + buf * BN, quad, lane);
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * BN);
  }
}

}  // namespace

int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      n = 148;
  }
  return n;
}

cudaError_t launch_gemm(const GemmParams& p, int bn, cudaStream_t st) {
  if (p.total_tiles <= 0) return cudaSuccess;
  const int grid = p.total_tiles < sm_count() ? p.total_tiles : sm_count();
  if (bn == 256) {
    const int smem = GemmLayout<256>::kSmemBytes;
    cudaError_t e = cudaFuncSetAttribute(gemm_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    gemm_kernel<256><<<grid, kThreads, smem, st>>>(p);
  } else if (bn == 128) {
    const int smem = GemmLayout<128>::kSmemBytes;
    cudaError_t e = cudaFuncSetAttribute(gemm_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    gemm_kernel<128><<<grid, kThreads, smem, st>>>(p);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace msgla
