// k_gla.cu -- chunkwise gated linear attention on tcgen05 (sm_100a).
//
// Computes, for every (batch, branch, head), the GLA recurrence of the MS-GLA
// reading notes, Sec. 2.1:  S_t = Diag(alpha_t) S_{t-1} + k_t^T v_t,
// o_t = qk_scale * q_t S_t,  in its chunkwise form (Sec. 3.4: each branch is a
// contiguous pooled sequence, so GLA's chunk algorithm applies unchanged).
// With b_i the cumulative log forget gate inside a chunk (from its first row),
// the gate kernel supplies Qs = q e^{b}, Ks = k e^{-b} and gamma = e^{b_last};
// then for chunk c with state S (entering the chunk):
//   A^T   = Ks Qs^T, masked to j <= i                 (intra-chunk scores)
//   o^T   = S^T Qs^T + V^T A^T                        (inter + intra output)
//   S    <- Diag(gamma) (S + Ks^T V)                  (state carried in TMEM)
// Orientation: o is produced transposed (value column on the TMEM lane) so that
// every MMA has M = 128; the 64-row score matrix uses an M = 128 MMA whose upper
// 64 rows are ignored.
//
// One CTA = (batch, branch, head, 128-column value tile), looping over chunks:
//   warp 0        TMA loads of Qs, Ks (64 x dkp, double-buffered: chunk c+1 is
//                 fetched while chunk c computes) and V (64 x 128) per chunk
//   warp 1        TMEM allocation (512 columns) + tcgen05.mma issue
//   warps 4..7    score epilogue (mask, fp16 into shared memory) and the o store
//   warps 8..15   state epilogue: S <- gamma * S in TMEM, fp16 copy of S for the
//                 next chunk's S^T Qs^T product (rows 0..127 / 128..255 of d_k)
// TMEM columns: [0,256) state (two 128-lane halves of d_k), [256,320) o^T,
// [320,384) A^T.
#include "msgla_internal.h"
#include "sm100_ptx.cuh"

namespace msgla {
namespace {

constexpr int kThreads = 512;
constexpr int kAtom = 64 * 128;  // one 64-row x 128-byte swizzle block (8 KB)
// shared memory map (bytes from the 1024-aligned base). The score MMA reads 128
// rows of Ks, i.e. up to 8 KB past a stage's last atom: that lands in the next
// buffer, never outside the allocation.
constexpr int kStageQK = 8 * kAtom;           // Qs (4 atoms) + Ks (4 atoms), d_k <= 256
constexpr int kOffQK = 0;                     // 2 stages
constexpr int kOffV = kOffQK + 2 * kStageQK;  // V: 2 atoms (128 value columns)
constexpr int kOffS = kOffV + 2 * kAtom;      // S^T fp16: 2 MN blocks x 256 rows x 128 B
constexpr int kOffA = kOffS + 2 * 256 * 128;  // A^T fp16: 64 rows x 128 B
constexpr int kOffBar = kOffA + kAtom;
constexpr int kSmemBytes = kOffBar + 256 + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

constexpr uint32_t kColS = 0, kColO = 256, kColA = 320;

enum {
  B_QK_FULL0 = 0, B_QK_FULL1, B_QK_EMPTY0, B_QK_EMPTY1, B_V_FULL, B_V_EMPTY,
  B_A_FULL, B_A_SMEM, B_O_FULL, B_O_EMPTY, B_S_FULL, B_S_DONE, B_COUNT
};

__global__ void __launch_bounds__(kThreads, 1) gla_chunk_kernel(const __grid_constant__ GlaParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + B_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  int ti = 0;
#pragma unroll 1
  for (int t = 1; t < p.n_tasks; ++t)
    if (static_cast<int>(blockIdx.x) >= p.task[t].cta_begin) ti = t;
  const GlaTask& T = p.task[ti];
  const int local = blockIdx.x - T.cta_begin;
  const int vt = local % T.v_tiles;
  const int head = (local / T.v_tiles) % T.heads;
  const int b = local / (T.v_tiles * T.heads);
  const int dkp = T.dkp;
  const int n_half = dkp / 128;  // 1 or 2 state halves
  const int nch = T.n_chunks;

  const int warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    mbar_init(&bar[B_QK_FULL0], 1);
    mbar_init(&bar[B_QK_FULL1], 1);
    mbar_init(&bar[B_QK_EMPTY0], 1);
    mbar_init(&bar[B_QK_EMPTY1], 1);
    mbar_init(&bar[B_V_FULL], 1);
    mbar_init(&bar[B_V_EMPTY], 1);
    mbar_init(&bar[B_A_FULL], 1);
    mbar_init(&bar[B_A_SMEM], 128);
    mbar_init(&bar[B_O_FULL], 1);
    mbar_init(&bar[B_O_EMPTY], 128);
    mbar_init(&bar[B_S_FULL], 1);
    mbar_init(&bar[B_S_DONE], 128 * n_half);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sbase = smem_u32(smem);

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer: Qs/Ks of chunk c into stage c&1, V of chunk c
      prefetch_tmap(&T.tmQ);
      prefetch_tmap(&T.tmK);
      prefetch_tmap(&T.tmV);
      const uint32_t qk_bytes = static_cast<uint32_t>(2 * (dkp / 64) * kAtom);
      for (int c = 0; c < nch; ++c) {
        const int st = c & 1;
        if (c >= 2 && !mbar_wait(&bar[B_QK_EMPTY0 + st], ((c >> 1) - 1) & 1, abort_flag, p.err)) break;
        uint8_t* sq = smem + kOffQK + st * kStageQK;
        mbar_arrive_expect_tx(&bar[B_QK_FULL0 + st], qk_bytes);
        for (int ka = 0; ka < dkp / 64; ++ka) {
          tma_load_3d(&T.tmQ, &bar[B_QK_FULL0 + st], sq + ka * kAtom, head * dkp + ka * 64, c * kChunk, b);
          tma_load_3d(&T.tmK, &bar[B_QK_FULL0 + st], sq + (4 + ka) * kAtom, head * dkp + ka * 64, c * kChunk, b);
        }
        if (c >= 1 && !mbar_wait(&bar[B_V_EMPTY], (c - 1) & 1, abort_flag, p.err)) break;
        mbar_arrive_expect_tx(&bar[B_V_FULL], 2 * kAtom);
        for (int mb = 0; mb < 2; ++mb)
          tma_load_3d(&T.tmV, &bar[B_V_FULL], smem + kOffV + mb * kAtom, head * T.dvp + vt * kGlaTile + mb * 64,
                      c * kChunk, b);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer. Per chunk: o^T(c), S update(c), scores(c+1).
      const uint32_t id_at = idesc_f16(128, 64, 0, 0, 0);   // Ks (K-major) x Qs (K-major)
      const uint32_t id_os = idesc_f16(128, 64, 0, 1, 0);   // S^T (MN-major) x Qs (K-major)
      const uint32_t id_ov = idesc_f16(128, 64, 0, 1, 1);   // V^T (MN-major) x A^T rows (MN-major)
      const uint32_t id_ds = idesc_f16(128, 128, 0, 1, 1);  // Ks^T (MN-major) x V (MN-major)
      const uint32_t sV = sbase + kOffV, sS = sbase + kOffS, sA = sbase + kOffA;
      const uint32_t lbo_s = static_cast<uint32_t>(dkp) * 128;
      auto scores = [&](int c) {
        // A^T[j][i] = sum_a Ks[j][a] Qs[i][a]
        const uint32_t sQ = sbase + kOffQK + (c & 1) * kStageQK, sK = sQ + 4 * kAtom;
        for (int ka = 0; ka < dkp / 64; ++ka)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_f16(tmem + kColA, sdesc_sw128(sK + ka * kAtom + kk * 32, 16, 1024),
                     sdesc_sw128(sQ + ka * kAtom + kk * 32, 16, 1024), id_at, (ka | kk) != 0);
        umma_commit(&bar[B_A_FULL]);
      };
      bool ok = mbar_wait(&bar[B_QK_FULL0], 0, abort_flag, p.err);
      if (ok) {
        tc_fence_after();
        scores(0);
      }
      for (int c = 0; c < nch && ok; ++c) {
        const int st = c & 1;
        const uint32_t sQ = sbase + kOffQK + st * kStageQK, sK = sQ + 4 * kAtom;
        if (!mbar_wait(&bar[B_A_SMEM], c & 1, abort_flag, p.err)) break;
        if (!mbar_wait(&bar[B_V_FULL], c & 1, abort_flag, p.err)) break;
        if (c > 0) {
          if (!mbar_wait(&bar[B_S_DONE], (c - 1) & 1, abort_flag, p.err)) break;
          if (!mbar_wait(&bar[B_O_EMPTY], (c - 1) & 1, abort_flag, p.err)) break;
        }
        tc_fence_after();
        uint32_t acc = 0;
        if (c > 0) {
          // o^T += S^T Qs^T  (K = d_k)
          for (int ks = 0; ks < dkp / 16; ++ks) {
            umma_f16(tmem + kColO, sdesc_sw128(sS + ks * 2048, lbo_s, 1024),
                     sdesc_sw128(sQ + (ks >> 2) * kAtom + (ks & 3) * 32, 16, 1024), id_os, acc);
            acc = 1;
          }
        }
        // o^T += V^T A^T  (K = chunk rows j)
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
          umma_f16(tmem + kColO, sdesc_sw128(sV + ks * 2048, kAtom, 1024), sdesc_sw128(sA + ks * 2048, kAtom, 1024),
                   id_ov, acc);
          acc = 1;
        }
        umma_commit(&bar[B_O_FULL]);
        // S += Ks^T V, per 128-row half of d_k
        for (int h = 0; h < n_half; ++h)
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            umma_f16(tmem + kColS + h * 128, sdesc_sw128(sK + 2 * h * kAtom + ks * 2048, kAtom, 1024),
                     sdesc_sw128(sV + ks * 2048, kAtom, 1024), id_ds, (c > 0 || ks > 0) ? 1u : 0u);
        umma_commit(&bar[B_S_FULL]);
        umma_commit(&bar[B_V_EMPTY]);
        umma_commit(&bar[B_QK_EMPTY0 + st]);
        if (c + 1 < nch) {
          if (!mbar_wait(&bar[B_QK_FULL0 + ((c + 1) & 1)], ((c + 1) >> 1) & 1, abort_flag, p.err)) break;
          tc_fence_after();
          scores(c + 1);
        }
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // ---------------- scores (mask + fp16 into smem) and output store
    const int quad = warp & 3;
    const int j = quad * 32 + lane;  // TMEM lane: chunk row j for A^T, value column for o^T
    uint8_t* sA = smem + kOffA;
    const size_t ld_o = static_cast<size_t>(T.heads) * T.dvp;
    for (int c = 0; c < nch; ++c) {
      if (!mbar_wait(&bar[B_A_FULL], c & 1, abort_flag, p.err)) break;
      tc_fence_after();
      uint32_t r0[32], r1[32];
      tmem_ld32(tmem_addr(tmem, quad * 32, kColA), r0);
      tmem_ld32(tmem_addr(tmem, quad * 32, kColA + 32), r1);
      tmem_wait_ld();
      if (j < kChunk) {
        // A^T[j][i] kept for i >= j (causal within the chunk)
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          float f[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int i = cc * 8 + e;
            const float x = __uint_as_float(i < 32 ? r0[i & 31] : r1[i & 31]);
            f[e] = (i >= j) ? x : 0.f;
          }
          st_shared_v4(smem_u32(sA + j * 128 + ((cc ^ (j & 7)) << 4)), pack_half2(f[0], f[1]),
                       pack_half2(f[2], f[3]), pack_half2(f[4], f[5]), pack_half2(f[6], f[7]));
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&bar[B_A_SMEM]);

      if (!mbar_wait(&bar[B_O_FULL], c & 1, abort_flag, p.err)) break;
      tc_fence_after();
      tmem_ld32(tmem_addr(tmem, quad * 32, kColO), r0);
      tmem_ld32(tmem_addr(tmem, quad * 32, kColO + 32), r1);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&bar[B_O_EMPTY]);
      const int col = head * T.dvp + vt * kGlaTile + j;
      const int t0 = c * kChunk;
      __half* dst = T.o + (static_cast<size_t>(b) * T.rows + t0) * ld_o + col;
      const int nvalid = min(kChunk, T.rows - t0);
#pragma unroll
      for (int i = 0; i < kChunk; ++i) {
        if (i < nvalid) {
          const float x = __uint_as_float(i < 32 ? r0[i & 31] : r1[i & 31]);
          dst[static_cast<size_t>(i) * ld_o] = __float2half_rn(p.qk_scale * x);
        }
      }
    }
  } else if (warp >= 8) {
    // ---------------- state epilogue: S <- gamma * S, fp16 copy for the next chunk
    const int g = (warp - 8) >> 2;  // d_k half
    const int quad = warp & 3;
    if (g < n_half) {
      const int a = g * 128 + quad * 32 + lane;  // d_k row
      uint8_t* sS = smem + kOffS;
      const size_t ld_g = static_cast<size_t>(T.heads) * dkp;
      const float* gp = T.gamma + static_cast<size_t>(b) * nch * ld_g + head * dkp + a;
      float gam = __ldg(gp);
      for (int c = 0; c < nch; ++c) {
        const float gam_next = (c + 1 < nch) ? __ldg(gp + (c + 1) * ld_g) : 0.f;
        if (!mbar_wait(&bar[B_S_FULL], c & 1, abort_flag, p.err)) break;
        tc_fence_after();
#pragma unroll 1
        for (int q2 = 0; q2 < 2; ++q2) {
          uint32_t ra[32], rb[32];
          const uint32_t ta = tmem_addr(tmem, quad * 32, kColS + g * 128 + q2 * 64);
          tmem_ld32(ta, ra);
          tmem_ld32(ta + 32, rb);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            ra[e] = __float_as_uint(gam * __uint_as_float(ra[e]));
            rb[e] = __float_as_uint(gam * __uint_as_float(rb[e]));
          }
          tmem_st32(ta, ra);
          tmem_st32(ta + 32, rb);
          // value columns q2*64 .. q2*64+63 -> MN block q2, 16-byte chunks 0..7
          uint8_t* row = sS + q2 * dkp * 128 + a * 128;
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            const uint32_t* r = e4 < 4 ? ra + 8 * e4 : rb + 8 * (e4 - 4);
            st_shared_v4(smem_u32(row + ((e4 ^ (a & 7)) << 4)),
                         pack_half2(__uint_as_float(r[0]), __uint_as_float(r[1])),
                         pack_half2(__uint_as_float(r[2]), __uint_as_float(r[3])),
                         pack_half2(__uint_as_float(r[4]), __uint_as_float(r[5])),
                         pack_half2(__uint_as_float(r[6]), __uint_as_float(r[7])));
          }
        }
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bar[B_S_DONE]);
        gam = gam_next;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

cudaError_t launch_gla(const GlaParams& p, cudaStream_t st) {
  if (p.total_ctas <= 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(gla_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  gla_chunk_kernel<<<p.total_ctas, kThreads, kSmemBytes, st>>>(p);
  return cudaGetLastError();
}

}  // namespace msgla
