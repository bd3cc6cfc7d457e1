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
//   warps 2..9  epilogue of the other accumulator (tcgen05.ld, one row per thread,
//               two warps per TMEM lane quadrant splitting the columns),
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
constexpr int kThreads = 320;  // warp 0 TMA, warp 1 MMA, warps 2..9 epilogue
constexpr int kEpiThreads = 256;

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

__device__ __forceinline__ TileCoord decode_tile(const GemmParams& p, int tile, int bn, int bm = kGemmBM) {
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
  c.m0 = m_tile * bm;
  c.n0 = n_tile * bn;
  const int n_rem = T.N - c.n0;
  c.n_eff = n_rem >= bn ? bn : ((n_rem + 15) / 16) * 16;
  c.kblocks = (T.K + kGemmBK - 1) / kGemmBK;
  return c;
}

// kEpiFuse with one or two coarse branches: the held rows of the next 32-column
// chunk are loaded while the current chunk is combined, so the L2 latency of the
// gather overlaps the arithmetic and the stores.
__device__ __forceinline__ void epilogue_fuse_prefetch(const GemmTask& T, const TileCoord& tc, uint32_t tacc,
                                                       int quad, int row, bool valid, size_t grow,
                                                       const float (&wts)[kMaxScales], int c_lo, int c_hi) {
  const uint4* base[2] = {nullptr, nullptr};
  float wc[2] = {0.f, 0.f};
  for (int c = 0; c < T.n_coarse; ++c) {
    const int s = T.coarse_scale[c];
    const int i = (row + 1) / s - 1;
    if (valid && i >= 0) {
      base[c] = reinterpret_cast<const uint4*>(T.coarse_y[c] +
                                               (static_cast<size_t>(tc.b) * T.coarse_rows[c] + i) * T.N + tc.n0);
      wc[c] = wts[T.coarse_index[c]];
    }
  }
  const float wmain = valid ? wts[T.main_index] : 0.f;
  uint4 cur[2][4], nxt[2][4];
  auto load = [&](uint4 (&dst)[2][4], int c0) {
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
      for (int j = 0; j < 4; ++j) dst[c][j] = base[c] ? __ldg(base[c] + (c0 >> 3) + j) : make_uint4(0, 0, 0, 0);
  };
  load(cur, c_lo);
  for (int c0 = c_lo; c0 < c_hi; c0 += 32) {
    if (c0 + 32 < c_hi) load(nxt, c0 + 32);
    uint32_t v[32];
    tmem_ld32(tmem_addr(tacc, quad * 32, c0), v);
    tmem_wait_ld();
    if (valid) {
      float acc[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) acc[j] = wmain * __uint_as_float(v[j]);
#pragma unroll
      for (int c = 0; c < 2; ++c)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const __half2* h = reinterpret_cast<const __half2*>(&cur[c][j]);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __half22float2(h[e]);
            acc[8 * j + 2 * e] = fmaf(wc[c], f.x, acc[8 * j + 2 * e]);
            acc[8 * j + 2 * e + 1] = fmaf(wc[c], f.y, acc[8 * j + 2 * e + 1]);
          }
        }
      uint4* d4 = reinterpret_cast<uint4*>(T.out + grow * T.N + tc.n0 + c0);
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
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
      for (int j = 0; j < 4; ++j) cur[c][j] = nxt[c][j];
  }
}

// Whether this thread's accumulator row is a padded token of a masked scale-1
// projection. Read before the wait for the accumulator so that the load's latency
// hides behind the MMAs.
__device__ __forceinline__ bool row_is_padded(const GemmParams& p, const TileCoord& tc, int quad, int lane) {
  const GemmTask& T = p.task[tc.task];
  if (T.epi != kEpiProj || !T.mask) return false;
  const int row = tc.m0 + quad * 32 + lane;
  return row < T.rows && !__ldg(T.mask + static_cast<size_t>(tc.b) * T.rows + row);
}

// Columns [c_lo, c_hi) of the tile (multiples of 32 from 0) for the accumulator
// rows of TMEM lane quadrant `quad`.
template <int BN>
__device__ __forceinline__ void epilogue_tile(const GemmParams& p, const TileCoord& tc, uint32_t tacc, int quad,
                                              int lane, int c_lo, int c_hi, bool padded) {
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
    if (tc.n0 == 0 && c_lo == 0)
      for (int j = 0; j < T.n_scales; ++j) T.w[grow * T.n_scales + j] = wts[j];
  }
  if (T.epi == kEpiFuse && T.n_coarse >= 1 && T.n_coarse <= 2) {
    epilogue_fuse_prefetch(T, tc, tacc, quad, row, valid, grow, wts, c_lo, c_hi);
    return;
  }
  const float wmain = (T.epi == kEpiFuse && valid) ? wts[T.main_index] : 0.f;
  // Eq. (8) at scale 1 zeroes a padded row; the projections have no bias, so its
  // q | k | v | g columns are zero (the fusion logits read x_t and are kept)
  const int n_zeroed = T.nq + T.nk + T.nv + T.ng;
  for (int c0 = c_lo; c0 < c_hi; c0 += 32) {
    uint32_t v[32];
    tmem_ld32(tmem_addr(tacc, quad * 32, c0), v);
    tmem_wait_ld();
    if (!valid) continue;
    const int col = tc.n0 + c0;
    if (T.epi == kEpiProj) {
      if (padded)
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (col + j < n_zeroed) v[j] = 0u;
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

// Two epilogue warps share each TMEM lane quadrant and split the tile's columns.
__device__ __forceinline__ void epi_columns(int warp, int n_eff, int& lo, int& hi) {
  const int mid = min(n_eff, ((n_eff / 2 + 31) / 32) * 32);
  const bool second = (warp - 2) >= 4;
  lo = second ? mid : 0;
  hi = second ? n_eff : mid;
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
      mbar_init(&acc_empty[a], kEpiThreads);
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
        // B tensor maps carry a 128-row box: BN / 128 loads fill the stage's B slot
#pragma unroll
        for (int h = 0; h < BN / 128; ++h)
          tma_load_2d(&T.tmB, &full_bar[s], sb + h * 128 * kGemmBK * 2, kb * kGemmBK, tc.n0 + h * 128);
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
      const bool padded = row_is_padded(p, tc, quad, lane);
      if (!mbar_wait(&acc_full[buf], (it >> 1) & 1, abort_flag, p.err)) break;
      tc_fence_after();
      int lo, hi;
      epi_columns(warp, tc.n_eff, lo, hi);
      epilogue_tile<BN>(p, tc, tmem + buf * BN, quad, lane, lo, hi, padded);
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

// ---------------------------------------------------------------- CTA-pair GEMM
// Same contraction on 256 x 256 tiles computed by a cluster of two CTAs with
// tcgen05.mma.cta_group::2: CTA r of the pair stages A rows [m0 + 128 r, +128)
// and B rows [n0 + r N/2, +N/2) (N = the tile's width), so each CTA moves
// 32 KB per 64-deep K step for 4 MFLOP of pair work -- two thirds of the
// 128 x 256 single-CTA tile's bytes per FLOP. The leader (rank 0) issues the
// MMAs; each CTA holds its 128 rows of the accumulator in its own TMEM and runs
// its own epilogue. Loads carry no multicast: both CTAs fetch their own halves
// and signal the leader's full barrier; the leader's commits reach both CTAs.
constexpr int kPairStages = 7;
constexpr int kPairStageBytes = 2 * kGemmBM * kGemmBK * 2;  // A half + B half = 32 KB
constexpr int kPairBarOffset = kPairStages * kPairStageBytes;
constexpr int kPairSmemBytes = kPairBarOffset + 256 + 1024;
constexpr int kPairBN = 256, kPairBM = 256;

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + kPairBarOffset);
  uint64_t* empty_bar = full_bar + kPairStages;
  uint64_t* acc_full = empty_bar + kPairStages;  // [2]
  uint64_t* acc_empty = acc_full + 2;            // [2] (used in the leader)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = warp_id(), lane = lane_id();
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 2 * kEpiThreads);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 2 * kPairBN);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int ntiles = p.total_tiles;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer of this CTA's halves
    for (int t = 0; t < p.n_tasks; ++t) {
      prefetch_tmap(&p.task[t].tmA);
      prefetch_tmap(&p.task[t].tmB);
    }
    uint32_t kbg = 0;
    bool ok = true;
    for (int tile = pair; tile < ntiles && ok; tile += npairs) {
      const TileCoord tc = decode_tile(p, tile, kPairBN, kPairBM);
      const GemmTask& T = p.task[tc.task];
      const int arow = tc.m0 + 128 * static_cast<int>(rank);
      const int brow = tc.n0 + static_cast<int>(rank) * (tc.n_eff >> 1);
      for (int kb = 0; kb < tc.kblocks; ++kb, ++kbg) {
        const uint32_t s = kbg % kPairStages;
        if (kbg >= kPairStages && !mbar_wait(&empty_bar[s], ((kbg / kPairStages) - 1) & 1, abort_flag, p.err)) {
          ok = false;
          break;
        }
        uint8_t* sa = smem + s * kPairStageBytes;
        uint8_t* sb = sa + kGemmBM * kGemmBK * 2;
        const uint32_t lead_full = mapa_shared(smem_u32(&full_bar[s]), 0);
        if (rank == 0) mbar_arrive_expect_tx(&full_bar[s], 2 * kPairStageBytes);
        tma_load_3d_pair(&T.tmA, lead_full, sa, kb * kGemmBK, arow, tc.b);
        tma_load_2d_pair(&T.tmB, lead_full, sb, kb * kGemmBK, brow);
      }
    }
  } else if (warp == 1 && lane == 0 && rank == 0) {
    // ---------------- MMA issuer (leader only)
    uint32_t kbg = 0, it = 0;
    bool ok = true;
    for (int tile = pair; tile < ntiles && ok; tile += npairs, ++it) {
      const TileCoord tc = decode_tile(p, tile, kPairBN, kPairBM);
      const uint32_t buf = it & 1;
      if (it >= 2 && !mbar_wait(&acc_empty[buf], ((it >> 1) - 1) & 1, abort_flag, p.err)) break;
      tc_fence_after();
      const uint32_t idesc = idesc_f16(kPairBM, tc.n_eff, p.task[tc.task].ab_bf16, 0, 0);
      const uint32_t tacc = tmem + buf * kPairBN;
      for (int kb = 0; kb < tc.kblocks; ++kb, ++kbg) {
        const uint32_t s = kbg % kPairStages;
        if (!mbar_wait(&full_bar[s], (kbg / kPairStages) & 1, abort_flag, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + s * kPairStageBytes);
        const uint32_t sb = sa + kGemmBM * kGemmBK * 2;
#pragma unroll
        for (int kk = 0; kk < kGemmBK / 16; ++kk)
          umma_f16_pair(tacc, sdesc_sw128(sa + kk * 32, 16, 1024), sdesc_sw128(sb + kk * 32, 16, 1024), idesc,
                        (kb | kk) != 0);
        umma_commit_pair(&empty_bar[s], 0x3);
      }
      if (ok) umma_commit_pair(&acc_full[buf], 0x3);
    }
  } else if (warp >= 2) {
    // ---------------- epilogue of this CTA's 128 accumulator rows
    const int quad = warp & 3;
    const uint32_t lead_empty0 = mapa_shared(smem_u32(&acc_empty[0]), 0);
    const uint32_t lead_empty1 = mapa_shared(smem_u32(&acc_empty[1]), 0);
    uint32_t it = 0;
    for (int tile = pair; tile < ntiles; tile += npairs, ++it) {
      TileCoord tc = decode_tile(p, tile, kPairBN, kPairBM);
      tc.m0 += 128 * static_cast<int>(rank);
      const uint32_t buf = it & 1;
      const bool padded = row_is_padded(p, tc, quad, lane);
      if (!mbar_wait(&acc_full[buf], (it >> 1) & 1, abort_flag, p.err)) break;
      tc_fence_after();
      int lo, hi;
      epi_columns(warp, tc.n_eff, lo, hi);
      epilogue_tile<kPairBN>(p, tc, tmem + buf * kPairBN, quad, lane, lo, hi, padded);
      tc_fence_before();
      mbar_arrive_cluster(buf ? lead_empty1 : lead_empty0);
    }
  }
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 2 * kPairBN);
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

// Pairs of CTAs that can be resident at once (0 if the pair kernel cannot run).
int max_active_pairs() {
  static int n = -1;
  if (n < 0) {
    n = 0;
    if (cudaFuncSetAttribute(gemm_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kPairSmemBytes) ==
        cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2 * sm_count(), 1, 1);
      cfg.blockDim = dim3(kThreads, 1, 1);
      cfg.dynamicSmemBytes = kPairSmemBytes;
      cudaLaunchAttribute attr;
      attr.id = cudaLaunchAttributeClusterDimension;
      attr.val.clusterDim.x = 2;
      attr.val.clusterDim.y = 1;
      attr.val.clusterDim.z = 1;
      cfg.attrs = &attr;
      cfg.numAttrs = 1;
      int c = 0;
      if (cudaOccupancyMaxActiveClusters(&c, gemm_pair_kernel, &cfg) == cudaSuccess) n = c;
    }
    cudaGetLastError();  // clear a failed query
  }
  return n;
}

cudaError_t launch_gemm(const GemmParams& p, int bn, cudaStream_t st) {
  if (p.total_tiles <= 0) return cudaSuccess;
  const int pairs = (bn == 256) ? max_active_pairs() : 0;
  if (pairs > 0) {
    // re-tile every task in 256 x 256 pair tiles
    static thread_local GemmParams q;
    q = p;
    int tiles = 0;
    for (int t = 0; t < p.n_tasks; ++t) {
      GemmTask& T = q.task[t];
      const int end = (t + 1 < p.n_tasks) ? p.task[t + 1].tile_begin : p.total_tiles;
      const int batches = (end - p.task[t].tile_begin) / (p.task[t].m_tiles * p.task[t].n_tiles);
      T.m_tiles = (T.rows + kPairBM - 1) / kPairBM;
      T.n_tiles = (T.N + kPairBN - 1) / kPairBN;
      T.tile_begin = tiles;
      tiles += batches * T.m_tiles * T.n_tiles;
    }
    q.total_tiles = tiles;
    const int grid_pairs = tiles < pairs ? tiles : pairs;
    gemm_pair_kernel<<<2 * grid_pairs, kThreads, kPairSmemBytes, st>>>(q);
    return cudaGetLastError();
  }
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
