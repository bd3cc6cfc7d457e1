// k_gemm.cu -- grouped tcgen05 GEMM for the MS-GLA projections.
//
// D[rows x N] = A[rows x K] * B[N x K]^T for each batch element and each task,
// with A and B K-major in global memory (PyTorch Linear layout), both bf16 or
// both fp16, fp32 accumulation in TMEM. One CTA computes one 128 x BN tile:
//   warp 0      TMA producer (4-stage ring of 128B-swizzled A/B tiles)
//   warp 1      TMEM allocation + single-thread tcgen05.mma issue
//   warps 2..5  epilogue: tcgen05.ld of the accumulator, one row per thread
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

template <int BN>
__global__ void __launch_bounds__(kThreads, 1) gemm_kernel(const __grid_constant__ GemmParams p) {
  using Lay = GemmLayout<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + Lay::kBarOffset);
  uint64_t* empty_bar = full_bar + kStages;
  uint64_t* accum_bar = empty_bar + kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  // ---- locate the tile
  int ti = 0;
#pragma unroll 1
  for (int t = 1; t < p.n_tasks; ++t)
    if (static_cast<int>(blockIdx.x) >= p.task[t].tile_begin) ti = t;
  const GemmTask& T = p.task[ti];
  const int local = blockIdx.x - T.tile_begin;
  const int n_tile = local % T.n_tiles;
  const int m_tile = (local / T.n_tiles) % T.m_tiles;
  const int b = local / (T.n_tiles * T.m_tiles);
  const int m0 = m_tile * kGemmBM;
  const int n0 = n_tile * BN;
  const int n_rem = T.N - n0;
  const int n_eff = n_rem >= BN ? BN : ((n_rem + 15) / 16) * 16;
  const int kblocks = (T.K + kGemmBK - 1) / kGemmBK;

  const int warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    mbar_init(accum_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, BN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer
    prefetch_tmap(&T.tmA);
    prefetch_tmap(&T.tmB);
    for (int kb = 0; kb < kblocks; ++kb) {
      const int s = kb % kStages;
      if (kb >= kStages && !mbar_wait(&empty_bar[s], ((kb / kStages) - 1) & 1, abort_flag, p.err)) break;
      uint8_t* sa = smem + s * Lay::kStageBytes;
      uint8_t* sb = sa + Lay::kABytes;
      mbar_arrive_expect_tx(&full_bar[s], Lay::kStageBytes);
      tma_load_3d(&T.tmA, &full_bar[s], sa, kb * kGemmBK, m0, b);
      tma_load_2d(&T.tmB, &full_bar[s], sb, kb * kGemmBK, n0);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer
    const uint32_t idesc = idesc_f16(kGemmBM, n_eff, T.ab_bf16, 0, 0);
    bool ok = true;
    for (int kb = 0; kb < kblocks && ok; ++kb) {
      const int s = kb % kStages;
      if (!mbar_wait(&full_bar[s], (kb / kStages) & 1, abort_flag, p.err)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t sa = smem_u32(smem + s * Lay::kStageBytes);
      const uint32_t sb = sa + Lay::kABytes;
#pragma unroll
      for (int kk = 0; kk < kGemmBK / 16; ++kk) {
        const uint64_t ad = sdesc_sw128(sa + kk * 32, 16, 1024);
        const uint64_t bd = sdesc_sw128(sb + kk * 32, 16, 1024);
        umma_f16(tmem, ad, bd, idesc, (kb | kk) != 0);
      }
      umma_commit(&empty_bar[s]);
    }
    if (ok) umma_commit(accum_bar);
  } else if (warp >= 2) {
    // ---------------- epilogue: one accumulator row per thread
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int row = m0 + r;
    const bool valid = row < T.rows;
    if (mbar_wait(accum_bar, 0, abort_flag, p.err)) {
      tc_fence_after();
      const size_t grow = static_cast<size_t>(b) * T.rows + row;
      float wmain = 0.f;
      if (T.epi == kEpiFuse && valid) wmain = __ldg(T.w + grow * T.n_scales + T.main_index);
      for (int c0 = 0; c0 < n_eff; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem_addr(tmem, quad * 32, c0), v);
        tmem_wait_ld();
        if (!valid) continue;
        const int col = n0 + c0;
        if (T.epi == kEpiProj) {
          if (col < T.nq) {
            cvt_store_f16x32(T.q + grow * T.nq + col, v);
          } else if (col < T.nq + T.nk) {
            cvt_store_f16x32(T.k + grow * T.nk + (col - T.nq), v);
          } else if (col < T.nq + T.nk + T.nv) {
            cvt_store_f16x32(T.v + grow * T.nv + (col - T.nq - T.nk), v);
          } else {
            const int gc = col - T.nq - T.nk - T.nv;
            const int n = (T.ng - gc) < 32 ? (T.ng - gc) : 32;
            store_f32(T.g + grow * T.ng + gc, v, n);
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
            const float wc = __ldg(T.w + grow * T.n_scales + T.coarse_index[c]);
            const __half* src = T.coarse_y[c] + (static_cast<size_t>(b) * T.coarse_rows[c] + i) * T.N + col;
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
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, BN);
  }
}

}  // namespace

cudaError_t launch_gemm(const GemmParams& p, int bn, cudaStream_t st) {
  if (p.total_tiles <= 0) return cudaSuccess;
  if (bn == 256) {
    const int smem = GemmLayout<256>::kSmemBytes;
    cudaError_t e = cudaFuncSetAttribute(gemm_kernel<256>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    gemm_kernel<256><<<p.total_tiles, kThreads, smem, st>>>(p);
  } else if (bn == 128) {
    const int smem = GemmLayout<128>::kSmemBytes;
    cudaError_t e = cudaFuncSetAttribute(gemm_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    gemm_kernel<128><<<p.total_tiles, kThreads, smem, st>>>(p);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace msgla
