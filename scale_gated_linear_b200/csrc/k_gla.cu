// k_gla.cu -- chunkwise gated linear attention on tcgen05 (sm_100a).
//
// Computes, for every (batch, branch, head), the GLA recurrence of the MS-GLA
// reading notes, Sec. 2.1:  S_t = Diag(alpha_t) S_{t-1} + k_t^T v_t,
// o_t = qk_scale * q_t S_t,  in its chunkwise form (Sec. 3.4: each branch is a
// contiguous pooled sequence, so GLA's chunk algorithm applies unchanged).
//
// Chunks hold C = 128 rows. With b_i the cumulative log forget gate from the
// chunk's first row and m = b at its 64th row (the reference point), the gate
// kernel supplies Qs = q e^{b - m}, Ks = k e^{m - b}, gamma = e^{b_last - m} and
// mid = e^{m} per chunk and key channel. TMEM holds the transposed scaled state
// T = S'^T, S' = Diag(e^{m_c}) S_{c-1}, on entry to chunk c (value columns on
// the TMEM lanes, key channels on the columns); per chunk:
//   [A | o] = Qs [Ks ; T]^T                 one N = 256 product: the scores
//                                            A = Qs Ks^T (masked to j <= i) and
//                                            o = Qs S', reading Qs once
//   T      += V^T Ks                         per 128-channel half of d_k
//   o      += A V                            (A converted to fp16 in TMEM)
//   T      <- T Diag(gamma_c mid_{c+1})      (epilogue, in TMEM)
// so every exponent stays within half a chunk's decay. The tensor cores read
// their shared-memory operands at about 64 bytes per clock, which bounds the
// chunk loop; the fused product and the transposed state keep those reads at
// 352 KB per chunk (Qs 64, [Ks ; T] 128, V^T 2 x 32, Ks 64, V 32).
//
// One CTA = (batch, branch, head, 128-column value tile), looping over chunks:
//   warp 0        TMA loads of Qs, Ks (128 x dkp) and V (128 x 128)
//   warp 1        TMEM allocation (512 columns) + tcgen05.mma issue
//   warps 4..7    score epilogue (mask, fp16 back into TMEM) and the o store
//                 (staged in the V buffer once V is read, TMA tile stores)
//   warps 8..15   state epilogue: T <- T * factor in TMEM and its fp16 copy,
//                 which sits right after each Ks atom in shared memory so that
//                 [Ks ; T] is one K-major operand (d_k half 0 / half 1)
// TMEM columns: [0,256) T (d_k channels), [256,384) A (fp32; its fp16 form
// occupies [256,320)), [384,512) o.
#include "msgla_internal.h"
#include "sm100_ptx.cuh"

namespace msgla {
namespace {

constexpr int kThreads = 512;
constexpr int kC = kGlaChunk;                 // 128 rows per chunk
constexpr int kAtom = kC * 128;               // 128 rows x 128 bytes = 16 KB (64 16-bit columns)
constexpr int kOffQ = 0;                      // Qs: up to 4 atoms (d_k <= 256)
constexpr int kOffKT = kOffQ + 4 * kAtom;     // per 64-channel block ka: Ks atom, then the T atom
constexpr int kOffV = kOffKT + 8 * kAtom;     // V: 2 atoms (128 value columns)
constexpr int kOffBar = kOffV + 2 * kAtom;
constexpr int kOffF = kOffBar + 256;          // the chunk's 256 state factors
constexpr int kSmemBytes = kOffF + 256 * 4 + 1024;
static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");

constexpr uint32_t kColS = 0, kColA = 256, kColO = 384;

// Ks, T and the state epilogue are split by 128-channel half h of d_k (the
// barrier + h), so the refill of a Ks half and the epilogue of a state half
// start as soon as that half's update has completed.
enum {
  B_Q_FULL = 0, B_Q_EMPTY, B_K_FULL, B_K_FULL1, B_K_EMPTY, B_K_EMPTY1, B_V_FULL, B_V_EMPTY,
  B_A_FULL, B_A_READY, B_O_FULL, B_O_EMPTY, B_S_FULL, B_S_FULL1, B_S_DONE, B_S_DONE1,
  B_F_READY, B_F_READY1, B_F_FREE, B_F_FREE1, B_V_FREE, B_COUNT
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
  const bool state_pass = p.mode == 1;
  const int segs = state_pass ? T.n_segs - 1 : T.n_segs;  // segments launched per sequence
  int local = blockIdx.x - T.cta_begin;
  const int seg = local % segs;
  local /= segs;
  const int vt = local % T.v_tiles;
  const int head = (local / T.v_tiles) % T.heads;
  const int b = local / (T.v_tiles * T.heads);
  const int dkp = T.dkp;
  const int n_half = dkp / 128;  // 1 or 2 halves of d_k
  const int nch_all = T.n_chunks;
  const int c_begin = seg * T.seg_chunks;
  const int nch = min(T.seg_chunks, nch_all - c_begin);  // chunks of this CTA
  const bool has_init = !state_pass && seg > 0;          // starts from a carried state
  const size_t seq_slot = ((static_cast<size_t>(b) * T.heads + head) * T.v_tiles + vt) * T.n_segs;

  const int warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0 && p.started && !state_pass) atomicAdd(p.started, 1ull);
  if (threadIdx.x == 0) {
    for (int i = 0; i < B_COUNT; ++i) mbar_init(&bar[i], 1);
    mbar_init(&bar[B_A_READY], 128);
    mbar_init(&bar[B_O_EMPTY], 128);
    for (int h = 0; h < 2; ++h) {
      mbar_init(&bar[B_S_DONE + h], 128);
      mbar_init(&bar[B_F_READY + h], 128);
      mbar_init(&bar[B_F_FREE + h], 128);
    }
    // full pass: the four output warps release V once their staged o tile is read
    mbar_init(&bar[B_V_EMPTY], state_pass ? 1 : 4);
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
  // with per-chunk counters the producer waits for each chunk's operands itself
  const bool chunk_waits = p.rows_done && !state_pass;
  if (!chunk_waits) griddep_wait();
  griddep_launch();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sbase = smem_u32(smem);

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer; each buffer is refilled once the MMAs of the
      // previous chunk that read it have completed.
      prefetch_tmap(&T.tmQ);
      prefetch_tmap(&T.tmK);
      prefetch_tmap(&T.tmV);
      const uint32_t qk_bytes = static_cast<uint32_t>((dkp / 64) * kAtom);
      for (int c = 0; c < nch; ++c) {
        const int row = (c_begin + c) * kC;
        if (chunk_waits) {
          // Qs, Ks and v of the chunk's rows are stored by the projection
          if (!wait_count(p.rows_done + T.done_base + static_cast<size_t>(b) * nch_all + c_begin + c, T.done_target,
                          abort_flag, p.err))
            break;
          fence_proxy_async_global();
        }
        if (!state_pass) {  // the state pass reads only Ks and V
          if (c > 0 && !mbar_wait(&bar[B_Q_EMPTY], (c - 1) & 1, abort_flag, p.err)) break;
          mbar_arrive_expect_tx(&bar[B_Q_FULL], qk_bytes);
          for (int ka = 0; ka < dkp / 64; ++ka)
            tma_load_3d(&T.tmQ, &bar[B_Q_FULL], smem + kOffQ + ka * kAtom, head * dkp + ka * 64, row, b);
        }
        bool ok = true;
        for (int h = 0; h < n_half && ok; ++h) {
          if (c > 0 && !mbar_wait(&bar[B_K_EMPTY + h], (c - 1) & 1, abort_flag, p.err)) ok = false;
          if (!ok) break;
          mbar_arrive_expect_tx(&bar[B_K_FULL + h], 2 * kAtom);
          for (int ka = 2 * h; ka < 2 * h + 2; ++ka)
            tma_load_3d(&T.tmK, &bar[B_K_FULL + h], smem + kOffKT + ka * 2 * kAtom, head * dkp + ka * 64, row, b);
        }
        if (!ok) break;
        if (c > 0 && !mbar_wait(&bar[B_V_EMPTY], (c - 1) & 1, abort_flag, p.err)) break;
        mbar_arrive_expect_tx(&bar[B_V_FULL], 2 * kAtom);
        for (int mb = 0; mb < 2; ++mb)
          tma_load_3d(&T.tmV, &bar[B_V_FULL], smem + kOffV + mb * kAtom, head * T.dvp + vt * kGlaTile + mb * 64, row,
                      b);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer
      const uint32_t id_fused = idesc_f16(128, 256, 0, 0, 0);  // [A | o] = Qs [Ks ; T]^T
      const uint32_t id_score = idesc_f16(128, 128, 0, 0, 0);  // A = Qs Ks^T (no state yet)
      const uint32_t id_mm = idesc_f16(128, 128, 0, 1, 1);     // T += V^T Ks: both MN-major
      const uint32_t id_km = idesc_f16(128, 128, 0, 0, 1);     // o += A V: A in TMEM, V MN-major
      const uint32_t sQ = sbase + kOffQ, sKT = sbase + kOffKT, sV = sbase + kOffV;
      const uint32_t sd0 = has_init ? 1u : 0u;  // state-epilogue completions before chunk 0
      // T += V^T Ks for the channels of half h (K = chunk rows j); releases that
      // Ks half and hands the half to the state epilogue
      auto state_update = [&](int h, bool acc) {
        for (int ks = 0; ks < kC / 16; ++ks)
          umma_f16(tmem + kColS + h * 128, sdesc_sw128(sV + ks * 2048, kAtom, 1024),
                   sdesc_sw128(sKT + h * 4 * kAtom + ks * 2048, 2 * kAtom, 1024), id_mm, (acc || ks > 0) ? 1u : 0u);
        umma_commit(&bar[B_K_EMPTY + h]);
        umma_commit(&bar[B_S_FULL + h]);
      };
      for (int c = 0; c < nch && state_pass; ++c) {
        // state pass: the state update and the state epilogue only
        const uint32_t ph = c & 1;
        if (!mbar_wait(&bar[B_V_FULL], ph, abort_flag, p.err)) break;
        bool ok = true;
        for (int h = 0; h < n_half && ok; ++h) {
          ok = mbar_wait(&bar[B_K_FULL + h], ph, abort_flag, p.err) &&
               (c == 0 || mbar_wait(&bar[B_S_DONE + h], (c - 1) & 1, abort_flag, p.err));
          if (!ok) break;
          tc_fence_after();
          state_update(h, c > 0);
        }
        if (!ok) break;
        umma_commit(&bar[B_V_EMPTY]);
      }
      // Full pass, per chunk c in pipe order: the fused scores + Qs S' product
      // (first d_k half while the second half of Ks may still be loading), the
      // state update of d_k half 0, A V, then the update of half 1. The score
      // conversion overlaps the first update, the o drain the second, and the
      // state epilogue of each half what follows it, so the next chunk's fused
      // product finds its inputs ready.
      for (int c = 0; c < nch && !state_pass; ++c) {
        const uint32_t ph = c & 1;
        const bool carried = c > 0 || has_init;  // a state enters this chunk
        if (!mbar_wait(&bar[B_Q_FULL], ph, abort_flag, p.err)) break;
        if (c > 0 && !mbar_wait(&bar[B_O_EMPTY], (c - 1) & 1, abort_flag, p.err)) break;
        bool ok = true;
        for (int h = 0; h < n_half && ok; ++h) {
          ok = mbar_wait(&bar[B_K_FULL + h], ph, abort_flag, p.err) &&
               (!carried || mbar_wait(&bar[B_S_DONE + h], (c - 1 + sd0) & 1, abort_flag, p.err));
          if (!ok) break;
          tc_fence_after();
          for (int ks = 8 * h; ks < 8 * h + 8; ++ks)
            umma_f16(tmem + kColA, sdesc_sw128(sQ + (ks >> 2) * kAtom + (ks & 3) * 32, 16, 1024),
                     sdesc_sw128(sKT + (ks >> 2) * 2 * kAtom + (ks & 3) * 32, 16, 1024),
                     carried ? id_fused : id_score, ks > 0 ? 1u : 0u);
        }
        if (!ok) break;
        umma_commit(&bar[B_Q_EMPTY]);
        umma_commit(&bar[B_A_FULL]);
        if (!mbar_wait(&bar[B_V_FULL], ph, abort_flag, p.err)) break;
        tc_fence_after();
        state_update(0, carried);
        if (!mbar_wait(&bar[B_A_READY], ph, abort_flag, p.err)) break;
        tc_fence_after();
        // o += A V  (A fp16 in TMEM, 8 columns per 16 rows j)
        for (int ks = 0; ks < kC / 16; ++ks)
          umma_f16_ts(tmem + kColO, tmem + kColA + ks * 8, sdesc_sw128(sV + ks * 2048, kAtom, 1024), id_km,
                      (carried || ks > 0) ? 1u : 0u);
        umma_commit(&bar[B_O_FULL]);
        for (int h = 1; h < n_half; ++h) state_update(h, carried);
        umma_commit(&bar[B_V_FREE]);  // V is read: the o rows may be staged there
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // ---------------- scores -> fp16 in TMEM, then the output rows
    const int quad = warp & 3;
    const int i = quad * 32 + lane;  // chunk row (TMEM lane)
    if (lane == 0 && !state_pass) prefetch_tmap(&T.tmO);
    for (int c = 0; c < nch && !state_pass; ++c) {
      if (!mbar_wait(&bar[B_A_FULL], c & 1, abort_flag, p.err)) break;
      tc_fence_after();
#pragma unroll 1
      for (int h2 = 0; h2 < 2; ++h2) {
        uint32_t ra[32], rb[32], pk[32];
        const uint32_t src = tmem_addr(tmem, quad * 32, kColA + h2 * 64);
        tmem_ld32(src, ra);
        tmem_ld32(src + 32, rb);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int j0 = h2 * 64 + 2 * e;
          pk[e] = pack_half2(j0 <= i ? __uint_as_float(ra[2 * e]) : 0.f,
                             j0 + 1 <= i ? __uint_as_float(ra[2 * e + 1]) : 0.f);
          const int j1 = j0 + 32;
          pk[16 + e] = pack_half2(j1 <= i ? __uint_as_float(rb[2 * e]) : 0.f,
                                  j1 + 1 <= i ? __uint_as_float(rb[2 * e + 1]) : 0.f);
        }
        tmem_st32(tmem_addr(tmem, quad * 32, kColA + h2 * 32), pk);
      }
      tmem_wait_st();
      tc_fence_before();
      // failure-detection tests: CTA 0 may withhold its first arrival, so the MMA
      // warp's bounded wait runs out and the launch reports a device timeout
      if (!(p.skip_arrival && blockIdx.x == 0 && c == 0)) mbar_arrive(&bar[B_A_READY]);

      if (!mbar_wait(&bar[B_O_FULL], c & 1, abort_flag, p.err)) break;
      tc_fence_after();
      // o row i, scaled and rounded to fp16 in registers; the o columns are
      // released at once, then the rows are staged in the V buffer (once the
      // state update has read it) with the 128-byte swizzle of the TMA store,
      // which writes whole 128-byte rows
      uint32_t po[64];
      const float qs = p.qk_scale;
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        uint32_t ra[32], rb[32];
        const uint32_t src = tmem_addr(tmem, quad * 32, kColO + h2 * 64);
        tmem_ld32(src, ra);
        tmem_ld32(src + 32, rb);
        tmem_wait_ld(ra);
        tmem_wait_ld(rb);
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          po[32 * h2 + e] = half2_of_mul(ra[2 * e], ra[2 * e + 1], qs, qs);
          po[32 * h2 + 16 + e] = half2_of_mul(rb[2 * e], rb[2 * e + 1], qs, qs);
        }
      }
      tc_fence_before();
      mbar_arrive(&bar[B_O_EMPTY]);
      if (!mbar_wait(&bar[B_V_FREE], c & 1, abort_flag, p.err)) break;
      uint8_t* stage = smem + kOffV + quad * 8192;
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        uint8_t* row = stage + h2 * 4096 + lane * 128;
#pragma unroll
        for (int q = 0; q < 8; ++q)
          st_shared_v4(smem_u32(row + ((q ^ (lane & 7)) << 4)), po[32 * h2 + 4 * q], po[32 * h2 + 4 * q + 1],
                       po[32 * h2 + 4 * q + 2], po[32 * h2 + 4 * q + 3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        // rows past the sequence end are clipped by the tensor map
        const int x = head * T.dvp + vt * kGlaTile, y = (c_begin + c) * kC + quad * 32;
        tma_store_3d(&T.tmO, stage, x, y, b);
        tma_store_3d(&T.tmO, stage + 4096, x + 64, y, b);
        bulk_commit();
        bulk_wait_read0();
        mbar_arrive(&bar[B_V_EMPTY]);  // the next V tile may overwrite the staging
      }
    }
    if (lane == 0 && !state_pass) {
      // the o rows are in global memory before the CTA reports them done
      bulk_wait0();
      fence_proxy_async_global();
    }
  } else if (warp >= 8) {
    // ---------------- state epilogue of d_k half g: T <- T Diag(gamma_c mid_{c+1})
    // for channels [128 g, 128 g + 128) of value row v, and the fp16 copy of
    // those T entries after the matching Ks atoms
    const int g = (warp - 8) >> 2;
    const int quad = warp & 3;
    if (g < n_half) {
      const int v = quad * 32 + lane;            // value column of the tile (TMEM lane)
      const int a_own = g * 128 + quad * 32 + lane;  // channel whose factor this thread supplies
      float* fac = reinterpret_cast<float*>(smem + kOffF);
      const size_t ld_g = static_cast<size_t>(T.heads) * dkp;
      const float* gp = T.gamma + static_cast<size_t>(b) * nch_all * ld_g + head * dkp + a_own;
      const float* mp = T.mid + static_cast<size_t>(b) * nch_all * ld_g + head * dkp + a_own;
      // factor of global chunk cg: gamma_cg * mid_{cg+1} (1 past the sequence's end)
      auto factor = [&](int cg) {
        return __ldg(gp + static_cast<size_t>(cg) * ld_g) *
               (cg + 1 < nch_all ? __ldg(mp + static_cast<size_t>(cg + 1) * ld_g) : 1.f);
      };
      // fp16 copy of 64 channels (block ka) of row v: the rows 128..255 of the
      // K-major [Ks ; T] operand, with the 128-byte swizzle of the Ks atoms
      auto put_f16 = [&](int ka, const uint32_t (&ra)[32], const uint32_t (&rb)[32]) {
        uint8_t* row = smem + kOffKT + ka * 2 * kAtom + kAtom + v * 128;
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const uint32_t* r = e4 < 4 ? ra + 8 * e4 : rb + 8 * (e4 - 4);
          st_shared_v4(smem_u32(row + ((e4 ^ (v & 7)) << 4)), pack_half2(__uint_as_float(r[0]), __uint_as_float(r[1])),
                       pack_half2(__uint_as_float(r[2]), __uint_as_float(r[3])),
                       pack_half2(__uint_as_float(r[4]), __uint_as_float(r[5])),
                       pack_half2(__uint_as_float(r[6]), __uint_as_float(r[7])));
        }
      };
      // segment states are stored [channel a][value column v]
      float* seg_base = state_pass || has_init ? T.seg_state + (seq_slot + seg - (has_init ? 1 : 0)) * dkp * kGlaTile + v
                                               : nullptr;
      if (has_init) {
        // carried state of this segment (written by the scan) into TMEM and smem
#pragma unroll 1
        for (int q2 = 0; q2 < 2; ++q2) {
          uint32_t ra[32], rb[32];
          const float* src = seg_base + static_cast<size_t>(g * 128 + q2 * 64) * kGlaTile;
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            ra[e] = __float_as_uint(__ldg(src + e * kGlaTile));
            rb[e] = __float_as_uint(__ldg(src + (32 + e) * kGlaTile));
          }
          const uint32_t ta = tmem_addr(tmem, quad * 32, kColS + g * 128 + q2 * 64);
          tmem_st32(ta, ra);
          tmem_st32(ta + 32, rb);
          put_f16(2 * g + q2, ra, rb);
        }
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bar[B_S_DONE + g]);
      }
      float decay = 1.f;  // product of this segment's factors of channel a_own (state pass)
      float f = factor(c_begin);
      int c = 0;
      for (; c < nch; ++c) {
        const float f_next = (c + 1 < nch) ? factor(c_begin + c + 1) : 0.f;
        // publish this chunk's factors once every thread of the half has read the last ones
        if (c > 0 && !mbar_wait(&bar[B_F_FREE + g], (c - 1) & 1, abort_flag, p.err)) break;
        fac[a_own] = f;
        mbar_arrive(&bar[B_F_READY + g]);
        if (!mbar_wait(&bar[B_F_READY + g], c & 1, abort_flag, p.err)) break;
        if (!mbar_wait(&bar[B_S_FULL + g], c & 1, abort_flag, p.err)) break;
        tc_fence_after();
#pragma unroll 1
        for (int q2 = 0; q2 < 2; ++q2) {
          uint32_t ra[32], rb[32];
          const uint32_t ta = tmem_addr(tmem, quad * 32, kColS + g * 128 + q2 * 64);
          tmem_ld32(ta, ra);
          tmem_ld32(ta + 32, rb);
          tmem_wait_ld();
          const float4* fr = reinterpret_cast<const float4*>(fac + g * 128 + q2 * 64);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float4 x = fr[e], y = fr[8 + e];
            ra[4 * e] = __float_as_uint(x.x * __uint_as_float(ra[4 * e]));
            ra[4 * e + 1] = __float_as_uint(x.y * __uint_as_float(ra[4 * e + 1]));
            ra[4 * e + 2] = __float_as_uint(x.z * __uint_as_float(ra[4 * e + 2]));
            ra[4 * e + 3] = __float_as_uint(x.w * __uint_as_float(ra[4 * e + 3]));
            rb[4 * e] = __float_as_uint(y.x * __uint_as_float(rb[4 * e]));
            rb[4 * e + 1] = __float_as_uint(y.y * __uint_as_float(rb[4 * e + 1]));
            rb[4 * e + 2] = __float_as_uint(y.z * __uint_as_float(rb[4 * e + 2]));
            rb[4 * e + 3] = __float_as_uint(y.w * __uint_as_float(rb[4 * e + 3]));
          }
          tmem_st32(ta, ra);
          tmem_st32(ta + 32, rb);
          if (!state_pass) put_f16(2 * g + q2, ra, rb);
        }
        mbar_arrive(&bar[B_F_FREE + g]);
        decay *= f;
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bar[B_S_DONE + g]);
        f = f_next;
      }
      if (state_pass && c == nch) {
        // end state of this segment (from zero) and its decay, for the scan
#pragma unroll 1
        for (int q2 = 0; q2 < 2; ++q2) {
          uint32_t ra[32], rb[32];
          const uint32_t ta = tmem_addr(tmem, quad * 32, kColS + g * 128 + q2 * 64);
          tmem_ld32(ta, ra);
          tmem_ld32(ta + 32, rb);
          tmem_wait_ld();
          float* dst = seg_base + static_cast<size_t>(g * 128 + q2 * 64) * kGlaTile;
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            dst[e * kGlaTile] = __uint_as_float(ra[e]);
            dst[(32 + e) * kGlaTile] = __uint_as_float(rb[e]);
          }
        }
        T.seg_decay[(seq_slot + seg) * dkp + a_own] = decay;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0 && p.done && !state_pass && T.signal_done) {
    // every o row of this CTA is stored (the barrier above orders the stores of
    // all its threads before this release)
    __threadfence();
    atomicAdd(p.done + ti, 1ull);
  }
  if (threadIdx.x == 0 && p.exited && !state_pass) {
    __threadfence();
    atomicAdd(p.exited, 1ull);
  }
}

// Initial state of every segment: S'_init(s+1) = G_s * S'_init(s) + A_s with
// S'_init(0) = 0, written over A_s. One thread per state element of a sequence.
__global__ void gla_scan_kernel(const __grid_constant__ GlaParams p, int B) {
  griddep_wait();
  griddep_launch();
  size_t gid = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  for (int t = 0; t < p.n_tasks; ++t) {
    const GlaTask& T = p.task[t];
    const size_t per_seq = static_cast<size_t>(T.dkp) * kGlaTile;
    const size_t n = static_cast<size_t>(B) * T.heads * T.v_tiles * per_seq;
    if (gid >= n) {
      gid -= n;
      continue;
    }
    const size_t sq = gid / per_seq, e = gid % per_seq;
    const int a = static_cast<int>(e / kGlaTile);
    float x = 0.f;
    for (int s = 0; s + 1 < T.n_segs; ++s) {
      float* slot = T.seg_state + (sq * T.n_segs + s) * per_seq + e;
      x = T.seg_decay[(sq * T.n_segs + s) * T.dkp + a] * x + *slot;
      *slot = x;
    }
    return;
  }
}

__global__ void wait_started_kernel(const unsigned long long* started, const unsigned long long* exited,
                                    unsigned long long target, int* err) {
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    if (!wait_count_quiet(started, target)) wait_count(exited, target, &abort_flag, err);
  }
}

}  // namespace

cudaError_t launch_wait_started(const unsigned long long* started, const unsigned long long* exited,
                                unsigned long long target, int* err, cudaStream_t st) {
  wait_started_kernel<<<1, 32, 0, st>>>(started, exited, target, err);
  return cudaGetLastError();
}

cudaError_t launch_gla_scan(const GlaParams& p, int B, cudaStream_t st) {
  size_t n = 0;
  for (int t = 0; t < p.n_tasks; ++t)
    n += static_cast<size_t>(B) * p.task[t].heads * p.task[t].v_tiles * p.task[t].dkp * kGlaTile;
  if (n == 0) return cudaSuccess;
  return launch_pdl(gla_scan_kernel, dim3(static_cast<unsigned>((n + 255) / 256)), dim3(256), 0, st, p, B);
}

cudaError_t launch_gla(const GlaParams& p, cudaStream_t st) {
  if (p.total_ctas <= 0) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(gla_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  return launch_pdl(gla_chunk_kernel, dim3(p.total_ctas), dim3(kThreads), kSmemBytes, st, p);
}

}  // namespace msgla
