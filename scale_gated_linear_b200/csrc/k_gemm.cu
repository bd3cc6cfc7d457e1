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
//               overlapping the next tile's main loop; 16-bit results are staged
//               per warp in shared memory (32 rows x 64 columns, 128-byte
//               swizzle) and written by TMA stores, so global writes are whole
//               lines instead of one 16-byte piece per row and instruction
// Epilogues (MS-GLA reading notes, Secs. 3.2-3.3):
//   kEpiProj      q | k | v columns to fp16, the low-rank gate columns to fp32
//   kEpiStoreF16  a coarse branch's Y^(s) = o W_o^T to fp16
//   kEpiFuse      the scale-1 branch's Y^(1) fused with the causal hold of the
//                 coarse branches and the fusion softmax weights (Eq. (11)):
//                 O_t = w_{t,1} Y^(1)_t + sum_s w_{t,s} Y^(s)_{floor((t+1)/s)-1}
//   kEpiProjGate  the forward's projection: q|k tiles pair W_q and W_k rows of the
//                 same 128 key channels and leave as the decay-scaled Qs = q 2^d,
//                 Ks = k 2^-d of the chunkwise GLA (d: the gate exponents of
//                 Sec. 2.1, launch_gate); v tiles leave as fp16
//   kEpiStoreF32  the low-rank gate inputs and fusion logits of the unpooled rows
//                 (fp32), optionally with the fusion weights of Eq. (10)
#include "msgla_internal.h"
#include "sm100_ptx.cuh"

namespace msgla {
namespace {

constexpr int kStages = 3;
constexpr int kThreads = 320;  // warp 0 TMA, warp 1 MMA, warps 2..9 epilogue
constexpr int kEpiThreads = 256;
constexpr int kStagerBytes = 32 * 128;              // one epilogue warp's staging buffer
constexpr int kGdBoxBytes = 32 * 32 * 4;            // gate exponents of 32 rows x 32 channels (fp32)
constexpr int kStagingBytes = 8 * 2 * kStagerBytes;  // eight epilogue warps, two buffers each

template <int BN>
struct GemmLayout {
  static constexpr int kABytes = kGemmBM * kGemmBK * 2;
  static constexpr int kBBytes = BN * kGemmBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStagingOffset = kStages * kStageBytes;
  static constexpr int kBarOffset = kStagingOffset + kStagingBytes;
  static constexpr int kSmemBytes = kBarOffset + 256 + 1024;  // barriers + 1024 B alignment slack
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

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

// n0: the tile's first output column (for a q|k tile of kEpiProjGate its first
// key channel, for its v tiles the first v column); brow0 / brow1: the first B
// row of the tile's column halves (CTA rank 0 / 1 of a pair, or the two
// 128-row B loads of a single-CTA 256-column tile).
struct TileCoord {
  int task, b, m0, n0, n_eff, kblocks, qk, brow0, brow1;
};

__device__ __forceinline__ TileCoord decode_tile(const GemmParams& p, int tile, int bn, int bm = kGemmBM) {
  TileCoord c;
  int ti = 0;
#pragma unroll 1
  for (int t = 1; t < p.n_tasks; ++t)
    if (tile >= p.task[t].tile_begin) ti = t;
  const GemmTask& T = p.task[ti];
  int local = tile - T.tile_begin;
  int half = -1;  // >= 0: which 128-column half of a full tile (GemmTask::half_from)
  if (T.half_from > 0 && local >= T.half_from) {
    const int hl = local - T.half_from;
    half = hl & 1;
    local = T.half_from + (hl >> 1);
  }
  const int n_tile = local % T.n_tiles;
  const int m_tile = (local / T.n_tiles) % T.m_tiles;
  c.task = ti;
  c.b = local / (T.n_tiles * T.m_tiles);
  c.m0 = m_tile * bm;
  c.kblocks = (T.K + kGemmBK - 1) / kGemmBK;
  c.qk = 0;
  if (T.epi == kEpiProjGate && n_tile < T.n_qk) {
    // 128 key channels of one head: W_q rows, then W_k rows of the same channels
    const int per_head = T.dkp / 128;
    c.qk = 1;
    c.n0 = (n_tile / per_head) * T.dkp + (n_tile % per_head) * 128;
    c.n_eff = 256;
    c.brow0 = c.n0;
    c.brow1 = T.nq + c.n0;
    return c;
  }
  int n_cols = T.N, b_first = 0;
  if (T.epi == kEpiProjGate) {  // v tiles
    c.n0 = (n_tile - T.n_qk) * bn;
    n_cols = T.nv;
    b_first = T.nq + T.nk;
  } else {
    c.n0 = n_tile * bn;
  }
  const int n_rem = n_cols - c.n0;
  c.n_eff = n_rem >= bn ? bn : ((n_rem + 15) / 16) * 16;
  if (half >= 0) {
    c.n0 += 128 * half;
    c.n_eff = 128;
  }
  c.brow0 = b_first + c.n0;
  c.brow1 = c.brow0 + (c.n_eff >> 1);
  return c;
}

// Whether this thread's accumulator row is a padded token of a masked scale-1
// projection. Read before the wait for the accumulator so that the load's latency
// hides behind the MMAs.
__device__ __forceinline__ bool row_is_padded(const GemmParams& p, const TileCoord& tc, int quad, int lane) {
  const GemmTask& T = p.task[tc.task];
  if ((T.epi != kEpiProj && T.epi != kEpiProjGate) || !T.mask) return false;
  const int row = tc.m0 + quad * 32 + lane;
  return row < T.rows && !__ldg(T.mask + static_cast<size_t>(tc.b) * T.rows + row);
}

// Per-warp staging of 16-bit output tiles: 32 accumulator rows x 64 columns in
// 32 rows of 128 bytes with the 128-byte swizzle (16-byte chunk j of row r at
// chunk j ^ (r & 7)), written by the warp and sent to global memory by one TMA
// store. Two buffers alternate, so a store's read of its buffer overlaps the
// filling of the other. Row r is the warp's lane r; every row's 64 columns
// arrive as two halves of 32 (one TMEM load each).
struct Stager {
  uint8_t* buf;  // 1 or 2 x 4 KB, 1024-byte aligned
  int lane;
  bool dbl;      // two buffers alternate (else one)
  // the buffer about to be filled is free: with two buffers at most the latest
  // store (which used the other one) may still be reading
  __device__ __forceinline__ void acquire() const {
    if (lane == 0) {
      if (dbl)
        bulk_wait_read1();
      else
        bulk_wait_read0();
    }
    __syncwarp();
  }
  __device__ __forceinline__ uint8_t* at(int sel) const { return buf + (dbl ? sel : 0) * kStagerBytes; }
  __device__ __forceinline__ void put(int sel, int half, const uint32_t (&pk)[16]) const {
    uint8_t* row = at(sel) + lane * 128;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      st_shared_v4(smem_u32(row + (((4 * half + j) ^ (lane & 7)) << 4)), pk[4 * j], pk[4 * j + 1], pk[4 * j + 2],
                   pk[4 * j + 3]);
  }
  // columns [col, col + 64) of rows [row0, row0 + 32) of batch element b
  __device__ __forceinline__ void store(int sel, const CUtensorMap* map, int col, int row0, int b) const {
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_3d(map, at(sel), col, row0, b);
      bulk_commit();
    }
  }
};

// Held coarse rows of one CTA tile in shared memory (kEpiFuse with one or two
// coarse branches): for coarse branch c, the rows i = floor((t+1)/s) - 1 of the
// tile's output rows t in [m0, m0 + 128) as four 64-column boxes of
// held_box_rows(s) rows of 128 bytes (128-byte swizzle), starting at row
// held_base(m0, s); rows before the first block and past the end are zero.
__device__ __forceinline__ int held_base(int m0, int s) { return (m0 + 1) / s - 1; }
struct Held {
  const uint8_t* smem[2];  // box 0 of each coarse branch
  int box_bytes[2];
  int lrow[2];             // this thread's held row within the boxes
  // box j (64 columns of every coarse branch) has its own barriers: full[j]
  // (the loader's TMA bytes landed, phase `parity` for this tile) and empty[j]
  // (one arrival per epilogue warp that has read it: four per box)
  uint64_t* full;
  uint64_t* empty;
  uint32_t parity;
  volatile int* abort_flag;
  // a 128-column half tile: the column group of epilogue warps g reads box 2 g
  // alone, and box 2 g + 1 carries nothing this tile (the loader completes its
  // round with a plain arrival, the group releases it unread)
  int half;
};

// Fusion weights w = softmax(z_t + b_fuse) of this thread's output row
// (Eq. (10), logits from the projection GEMM); the n0 == 0 tiles also store
// them. Computed before the accumulator is ready: the logit loads' latency
// hides behind the tile's MMAs.
struct FuseW {
  float wts[kMaxScales];
  float wmain;
};
__device__ __forceinline__ void fuse_weights(const GemmParams& p, const TileCoord& tc, int quad, int lane, int c_lo,
                                             FuseW& fw) {
  const GemmTask& T = p.task[tc.task];
  fw.wmain = 0.f;
  if (T.epi != kEpiFuse) return;
  const int row = tc.m0 + quad * 32 + lane;
  if (row >= T.rows) return;
  const size_t grow = static_cast<size_t>(tc.b) * T.rows + row;
  float zmax = -INFINITY;
  for (int j = 0; j < T.n_scales; ++j) {
    fw.wts[j] = __ldg(T.zf + grow * T.ldz + j) + __ldg(T.bfuse + j);
    zmax = fmaxf(zmax, fw.wts[j]);
  }
  float sum = 0.f;
  for (int j = 0; j < T.n_scales; ++j) {
    fw.wts[j] = __expf(fw.wts[j] - zmax);
    sum += fw.wts[j];
  }
  const float inv = 1.f / sum;
  for (int j = 0; j < T.n_scales; ++j) fw.wts[j] *= inv;
  if (tc.n0 == 0 && c_lo == 0)
    for (int j = 0; j < T.n_scales; ++j) T.w[grow * T.n_scales + j] = fw.wts[j];
  fw.wmain = fw.wts[T.main_index];
}

__device__ __forceinline__ void pack_f16x32(uint32_t (&pk)[16], const uint32_t (&v)[32]) {
#pragma unroll
  for (int e = 0; e < 16; ++e) pk[e] = pack_half2(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
}
__device__ __forceinline__ void pack_bf16x32(uint32_t (&pk)[16], const float (&a)[32]) {
#pragma unroll
  for (int e = 0; e < 16; ++e) pk[e] = pack_bf162(a[2 * e], a[2 * e + 1]);
}

// Columns [c_lo, c_hi) of the tile for the accumulator rows of TMEM lane
// quadrant `quad` (c_lo a multiple of 64). 16-bit destinations go through the
// warp's staging buffers in steps of 64 columns; the fp32 gate and fusion-logit
// columns of the projection are stored directly. For plain stores the TMEM load
// of the next 32 columns is in flight while the current ones are processed; the
// fused epilogue instead prefetches the held coarse rows one chunk ahead (both
// at once would not fit the register budget). `sel` is the warp's running
// staging-buffer index.
// Returns false if a bounded wait for held rows gave up (the error word is set).
__device__ __forceinline__ bool epilogue_tile(const GemmParams& p, const TileCoord& tc, uint32_t tacc, int quad,
                                              int lane, int c_lo, int c_hi, bool padded, const Stager& stg,
                                              int& sel, const FuseW& fw, const Held* held = nullptr) {
  const GemmTask& T = p.task[tc.task];
  const int row = tc.m0 + quad * 32 + lane;
  const int row0 = tc.m0 + quad * 32;
  const bool valid = row < T.rows;
  const size_t grow = static_cast<size_t>(tc.b) * T.rows + row;
  const float* wts = fw.wts;
  const float wmain = fw.wmain;
  const bool prefetch = T.epi == kEpiFuse && T.n_coarse <= 2 && !held;
  const uint4* base0 = nullptr;
  const uint4* base1 = nullptr;
  float wc0 = 0.f, wc1 = 0.f;
  if (T.epi == kEpiFuse) {
    if (prefetch && valid) {
      auto held = [&](int c, const uint4*& base, float& wc) {
        if (c >= T.n_coarse) return;
        const int i = (row + 1) / T.coarse_scale[c] - 1;
        if (i < 0) return;
        base = reinterpret_cast<const uint4*>(T.coarse_y[c] +
                                              (static_cast<size_t>(tc.b) * T.coarse_rows[c] + i) * T.N + tc.n0);
        wc = wts[T.coarse_index[c]];
      };
      held(0, base0, wc0);
      held(1, base1, wc1);
    }
  }
  uint4 cur0[4], cur1[4], nxt0[4], nxt1[4];
  auto load = [&](uint4 (&d0)[4], uint4 (&d1)[4], int c0) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      d0[j] = base0 ? __ldg(base0 + (c0 >> 3) + j) : make_uint4(0, 0, 0, 0);
      d1[j] = base1 ? __ldg(base1 + (c0 >> 3) + j) : make_uint4(0, 0, 0, 0);
    }
  };
  const int n_f16 = T.epi == kEpiProj ? T.nq + T.nk + T.nv : T.epi == kEpiProjGate ? T.nv : T.N;
  // one 32-column chunk (tile columns [c0, c0 + 32), values v); `half` places it
  // in the current staging buffer, `last` = no chunk of this tile follows
  auto chunk = [&](int c0, uint32_t (&v)[32], int half, bool last) __attribute__((always_inline)) {
    if (prefetch && !last) load(nxt0, nxt1, c0 + 32);
    const int col = tc.n0 + c0;
    if (col >= n_f16) {
      // fp32 gate / fusion-logit columns of the projection. Eq. (8) at scale 1
      // zeroes a padded row; the projections have no bias, so its q | k | v | g
      // columns are zero (the fusion logits read x_t and are kept)
      if (!valid) return;
      const int n_zeroed = T.nq + T.nk + T.nv + T.ng;
      if (padded)
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (col + j < n_zeroed) v[j] = 0u;
      // chunk column j is gate column gc + j (j < ng - gc), then logit column
      // gc + j - ng (< ldz when the branch carries logits); static indices keep
      // v in registers
      const int gc = col - n_f16;
      float* gp = T.g + grow * T.ng;
      float* zp = T.z ? T.z + grow * T.ldz : nullptr;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int c = gc + j;
        if (c < T.ng)
          gp[c] = __uint_as_float(v[j]);
        else if (T.nz > 0 && c - T.ng < T.ldz)
          zp[c - T.ng] = __uint_as_float(v[j]);
      }
      return;
    }
    const int col64 = col - 32 * half;
    const CUtensorMap* map = &T.tmOut[0];
    int dcol = col64;
    uint32_t pk[16];
    if (T.epi == kEpiProjGate) {  // a v tile
      map = &T.tmOut[2];
      if (padded)
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = 0u;
      pack_f16x32(pk, v);
    } else if (T.epi == kEpiProj) {
      if (col64 >= T.nq + T.nk) {
        map = &T.tmOut[2];
        dcol = col64 - T.nq - T.nk;
      } else if (col64 >= T.nq) {
        map = &T.tmOut[1];
        dcol = col64 - T.nq;
      }
      if (padded)
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = 0u;
      pack_f16x32(pk, v);
    } else if (T.epi == kEpiStoreF16) {
      pack_f16x32(pk, v);
    } else {
      float acc[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) acc[j] = wmain * __uint_as_float(v[j]);
      if (held) {
        // held coarse rows from shared memory: 16-byte pieces q of the chunk's
        // 64-column box, swizzled by the row
        const int box = held->half ? (c0 >> 6) * 2 : c0 >> 6, q0 = (c0 & 63) >> 3;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          if (c >= T.n_coarse) break;
          const float wgt = valid ? wts[T.coarse_index[c]] : 0.f;
          const int lr = held->lrow[c];
          const uint8_t* rowp = held->smem[c] + box * held->box_bytes[c] + lr * 128;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint4 u = *reinterpret_cast<const uint4*>(rowp + (((q0 + j) ^ (lr & 7)) << 4));
            const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float2 f = __half22float2(h[q]);
              acc[8 * j + 2 * q] = fmaf(wgt, f.x, acc[8 * j + 2 * q]);
              acc[8 * j + 2 * q + 1] = fmaf(wgt, f.y, acc[8 * j + 2 * q + 1]);
            }
          }
        }
      } else if (prefetch) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const __half2* h0 = reinterpret_cast<const __half2*>(&cur0[j]);
          const __half2* h1 = reinterpret_cast<const __half2*>(&cur1[j]);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 f0 = __half22float2(h0[q]), f1 = __half22float2(h1[q]);
            acc[8 * j + 2 * q] = fmaf(wc1, f1.x, fmaf(wc0, f0.x, acc[8 * j + 2 * q]));
            acc[8 * j + 2 * q + 1] = fmaf(wc1, f1.y, fmaf(wc0, f0.y, acc[8 * j + 2 * q + 1]));
          }
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          cur0[j] = nxt0[j];
          cur1[j] = nxt1[j];
        }
      } else if (valid) {
        for (int c = 0; c < T.n_coarse; ++c) {
          const int i = (row + 1) / T.coarse_scale[c] - 1;
          if (i < 0) continue;
          const __half* src = T.coarse_y[c] + (static_cast<size_t>(tc.b) * T.coarse_rows[c] + i) * T.N + col;
          add_scaled_f16x32(acc, src, wts[T.coarse_index[c]]);
        }
      }
      pack_bf16x32(pk, acc);
    }
    if (half == 0) stg.acquire();
    stg.put(sel, half, pk);
    if (half == 1) stg.store(sel, map, dcol, row0, tc.b);
  };
  if (c_lo >= c_hi) return true;
  uint32_t va[32], vb[32];
  if (prefetch) {
    load(cur0, cur1, c_lo);
    for (int c0 = c_lo; c0 < c_hi; c0 += 32) {
      const int half = ((c0 - c_lo) >> 5) & 1;
      tmem_ld32(tmem_addr(tacc, quad * 32, c0), va);
      tmem_wait_ld(va);
      chunk(c0, va, half, c0 + 32 >= c_hi);
      if (half) sel ^= 1;
    }
    return true;
  }
  tmem_ld32(tmem_addr(tacc, quad * 32, c_lo), va);
  tmem_wait_ld(va);
  for (int c0 = c_lo; c0 < c_hi; c0 += 64) {
    const bool has_b = c0 + 32 < c_hi, has_next = c0 + 64 < c_hi;
    const int hb = held && held->half ? (c0 >> 6) * 2 : c0 >> 6;  // held box of these columns
    // held rows: this 64-column box has landed
    if (held && !mbar_wait(&held->full[hb], held->parity, held->abort_flag, p.err)) return false;
    if (has_b) tmem_ld32(tmem_addr(tacc, quad * 32, c0 + 32), vb);
    chunk(c0, va, 0, !has_b);
    if (has_b) {
      tmem_wait_ld(vb);
      if (has_next) tmem_ld32(tmem_addr(tacc, quad * 32, c0 + 64), va);
      chunk(c0 + 32, vb, 1, !has_next);
      if (has_next) tmem_wait_ld(va);
    }
    if (held) {
      // this warp is done with the box: the loader may refill it for the next tile
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&held->empty[hb]);
      if (held->half) {
        // the sibling box of a half tile: complete its round unread
        if (!mbar_wait(&held->full[hb + 1], held->parity, held->abort_flag, p.err)) return false;
        if (lane == 0) mbar_arrive(&held->empty[hb + 1]);
      }
    }
    sel ^= 1;
  }
  return true;
}

// Columns [c_lo, c_hi) of a kEpiStoreF32 tile: fp32 rows stored directly (the
// gate inputs and fusion logits, 64 to 272 columns per row); the thread holding
// column 0 of a row also forms the fusion weights w = softmax(z + b_fuse) from
// the logits in columns 0..n_scales-1 when T.w is set (Eq. (10)).
__device__ __forceinline__ void epilogue_f32(const GemmParams& p, const TileCoord& tc, uint32_t tacc, int quad,
                                             int lane, int c_lo, int c_hi) {
  const GemmTask& T = p.task[tc.task];
  const int row = tc.m0 + quad * 32 + lane;
  const bool valid = row < T.rows;
  const size_t grow = static_cast<size_t>(tc.b) * T.rows + row;
#pragma unroll 1
  for (int c0 = c_lo; c0 < c_hi; c0 += 32) {
    uint32_t v[32];
    tmem_ld32(tmem_addr(tacc, quad * 32, c0), v);
    tmem_wait_ld(v);
    if (!valid) continue;
    const int col = tc.n0 + c0;
    if (col == 0 && T.w) {
      float zz[kMaxScales];
      float zmax = -INFINITY;
#pragma unroll
      for (int j = 0; j < kMaxScales; ++j) {
        zz[j] = j < T.n_scales ? __uint_as_float(v[j]) + __ldg(T.bfuse + j) : -INFINITY;
        zmax = fmaxf(zmax, zz[j]);
      }
      float sum = 0.f;
#pragma unroll
      for (int j = 0; j < kMaxScales; ++j) {
        zz[j] = j < T.n_scales ? __expf(zz[j] - zmax) : 0.f;
        sum += zz[j];
      }
      const float inv = 1.f / sum;
#pragma unroll
      for (int j = 0; j < kMaxScales; ++j)
        if (j < T.n_scales) T.w[grow * T.n_scales + j] = zz[j] * inv;
    }
    float* dst = T.f32 + grow * T.ldf + col;
    if (col + 32 <= T.N) {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        reinterpret_cast<float4*>(dst)[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                                        __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (col + j < T.N) dst[j] = __uint_as_float(v[j]);
    }
  }
}

// Two epilogue warps share each TMEM lane quadrant and split the tile's columns
// at a multiple of 64 (one staging step).
__device__ __forceinline__ void epi_columns(int warp, int n_eff, int& lo, int& hi) {
  const int mid = min(n_eff, ((n_eff / 2 + 63) / 64) * 64);
  const bool second = (warp - 2) >= 4;
  lo = second ? mid : 0;
  hi = second ? n_eff : mid;
}

// ---------------------------------------------------------------- gated projection
// Gate exponents of a q|k tile for one epilogue warp: 32 rows (its TMEM lane
// quadrant) x 32 key channels (group grp of its channel half) of d, fp32, loaded
// by TMA into the warp's 4 KB buffer (128-byte swizzle: 16-byte chunk j of row r
// at chunk j ^ (r & 7)); lane 0 issues it, gd_full completes when it lands.
struct GateExp {
  uint8_t* buf;
  uint64_t* full;
  uint32_t* phase;  // loads issued so far by this warp (parity of the next wait)
};
__device__ __forceinline__ void issue_gate_exponents(const GemmParams& p, const TileCoord& tc, int quad, int lane,
                                                     int ch, int grp, const GateExp& ge) {
  if (lane != 0) return;
  const GemmTask& T = p.task[tc.task];
  mbar_arrive_expect_tx(ge.full, kGdBoxBytes);
  tma_load_2d(&T.tmD, ge.full, ge.buf, tc.n0 + 64 * ch + 32 * grp, tc.b * T.rows + tc.m0 + quad * 32);
}

// Epilogue of a q|k tile of the gated projection (kEpiProjGate; MS-GLA reading
// notes, Sec. 2.1). The accumulator holds q (columns 0..127) and k (128..255) of
// the 128 key channels c0.. of one head for the CTA's 128 rows, which are one
// 128-row chunk of the GLA kernel. The thread of chunk row r and channel half ch
// takes channels c0 + 64 ch .., 32 at a time: with the gate exponents d = b - m
// of its row (b the cumulative sum of log2 alpha over the chunk's rows, m its
// value at row 63; launch_gate) it stores Qs = q 2^d and Ks = k 2^-d (fp16), the
// operands of the chunkwise GLA kernel, as two 32 x 32 boxes through the warp's
// staging buffer (Qs in its first 2 KB, Ks in the second; 64-byte swizzle, maps
// tmQK). The exponents of group 0 were requested before the accumulator wait
// (issue_gate_exponents); those of group 1 are requested as soon as group 0's
// are in registers. Only the side whose factor can exceed 1 is checked for the
// fp16 range (b does not increase along the chunk: Qs in rows 0..63, Ks in rows
// 64..127); an overflow latches kDevRange. Returns false if a bounded wait gave up.
__device__ __forceinline__ bool epilogue_qk(const GemmParams& p, const TileCoord& tc, uint32_t tacc, int quad,
                                            int lane, int ch, bool padded, const Stager& stg, const GateExp& ge,
                                            volatile int* abort_flag) {
  const GemmTask& T = p.task[tc.task];
  const int lrow = quad * 32 + lane;
  const int grow_side = lrow < 64 ? 0 : 1;
  uint8_t* buf = stg.at(0);
  uint32_t over = 0;
#pragma unroll
  for (int grp = 0; grp < 2; ++grp) {
    if (!mbar_wait(ge.full, *ge.phase & 1, abort_flag, p.err)) return false;
    ++*ge.phase;
    float d[32];
    {
      const uint8_t* row = ge.buf + lane * 128;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float4 x = *reinterpret_cast<const float4*>(row + ((j ^ (lane & 7)) << 4));
        d[4 * j] = x.x;
        d[4 * j + 1] = x.y;
        d[4 * j + 2] = x.z;
        d[4 * j + 3] = x.w;
      }
    }
    if (grp == 0) {
      // the buffer is read: the next 32 channels' exponents may land in it
      fence_proxy_async_smem();
      __syncwarp();
      issue_gate_exponents(p, tc, quad, lane, ch, 1, ge);
    }
    const int cb = tc.n0 + 64 * ch + 32 * grp;  // first key channel of this group
    stg.acquire();  // the previous group's stores have read the buffer
#pragma unroll
    for (int which = 0; which < 2; ++which) {
      uint32_t a[32];
      tmem_ld32(tmem_addr(tacc, quad * 32, which * 128 + 64 * ch + 32 * grp), a);
      tmem_wait_ld(a);
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float d0 = d[2 * e], d1 = d[2 * e + 1];
        const float s0 = ex2_approx(which ? -d0 : d0), s1 = ex2_approx(which ? -d1 : d1);
        const float v0 = padded ? 0.f : __uint_as_float(a[2 * e]) * s0;
        const float v1 = padded ? 0.f : __uint_as_float(a[2 * e + 1]) * s1;
        pk[e] = pack_half2(v0, v1);
        if (which == grow_side) half2_track_nonfinite(over, pk[e]);
      }
      // 64-byte rows, 16-byte chunk j of row r at chunk j ^ ((r >> 1) & 3)
      uint8_t* rowp = buf + which * 2048 + lane * 64;
#pragma unroll
      for (int j = 0; j < 4; ++j)
        st_shared_v4(smem_u32(rowp + ((j ^ ((lane >> 1) & 3)) << 4)), pk[4 * j], pk[4 * j + 1], pk[4 * j + 2],
                     pk[4 * j + 3]);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_3d(&T.tmQK[0], buf, cb, tc.m0 + quad * 32, tc.b);
      tma_store_3d(&T.tmQK[1], buf + 2048, cb, tc.m0 + quad * 32, tc.b);
      bulk_commit();
    }
  }
  if (over & 0x80008000u) atomicCAS(p.err, 0, kDevRange);
  return true;
}

// After a kEpiProjGate tile: once this warp's TMA stores have completed, count
// the warp's 32 rows in the 128-row block's counter (GemmParams::rows_done), with
// release order for the GLA kernel's acquire.
__device__ __forceinline__ void count_rows_done(const GemmParams& p, const TileCoord& tc, int lane) {
  const GemmTask& T = p.task[tc.task];
  if (!p.rows_done || T.epi != kEpiProjGate || lane != 0 || tc.m0 >= T.rows) return;
  bulk_wait0();
  fence_proxy_async_global();
  __threadfence();
  atomicAdd(p.rows_done + T.done_base + static_cast<size_t>(tc.b) * ((T.rows + 127) / 128) + tc.m0 / 128, 1ull);
}

// Prefetch the output tensor maps of every task (epilogue warps).
__device__ __forceinline__ void prefetch_out_maps(const GemmParams& p) {
  for (int t = 0; t < p.n_tasks; ++t) {
    for (int m = 0; m < 3; ++m) prefetch_tmap(&p.task[t].tmOut[m]);
    if (p.task[t].epi == kEpiProjGate) {
      for (int m = 0; m < 2; ++m) prefetch_tmap(&p.task[t].tmQK[m]);
      prefetch_tmap(&p.task[t].tmD);
    }
  }
}

// Producer side of a per-task input dependency (GemmTask::dep): before the first
// load of a task, wait for its producer running on another stream.
__device__ __forceinline__ bool task_ready(const GemmTask& T, int task, uint32_t& ready, volatile int* abort_flag,
                                           int* err) {
  if (!T.dep || ((ready >> task) & 1u)) return true;
  if (!wait_count(T.dep, T.dep_target, abort_flag, err)) return false;
  fence_proxy_async_global();
  ready |= 1u << task;
  return true;
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
  uint64_t* gd_full = acc_empty + 2;         // [8] per epilogue warp: its gate exponents landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gd_full + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  static_assert((2 * kStages + 12) * 8 + 8 <= 256, "barrier region");

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
    for (int w = 0; w < 8; ++w) mbar_init(&gd_full[w], 1);
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
  griddep_wait();
  griddep_launch();
  const uint32_t tmem = *tmem_slot;
  const int ntiles = p.total_tiles;

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer (runs ahead across tiles)
    for (int t = 0; t < p.n_tasks; ++t) {
      prefetch_tmap(&p.task[t].tmA);
      prefetch_tmap(&p.task[t].tmB);
    }
    uint32_t kbg = 0, ready = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < ntiles && ok; tile += gridDim.x) {
      const TileCoord tc = decode_tile(p, tile, BN);
      const GemmTask& T = p.task[tc.task];
      if (!task_ready(T, tc.task, ready, abort_flag, p.err)) break;
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
          tma_load_2d(&T.tmB, &full_bar[s], sb + h * 128 * kGemmBK * 2, kb * kGemmBK,
                      h == 0 ? tc.brow0 : (tc.qk ? tc.brow1 : tc.brow0 + h * 128));
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
    // one staging buffer per warp; the second 4 KB of its slot holds gate exponents
    const Stager stg{smem + Lay::kStagingOffset + (warp - 2) * 2 * kStagerBytes, lane};
    uint32_t gd_phase = 0;
    const GateExp ge{smem + Lay::kStagingOffset + (warp - 2) * 2 * kStagerBytes + kStagerBytes, &gd_full[warp - 2],
                     &gd_phase};
    int sel = 0;
    if (lane == 0) prefetch_out_maps(p);
    uint32_t it = 0;
    for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x, ++it) {
      const TileCoord tc = decode_tile(p, tile, BN);
      const uint32_t buf = it & 1;
      const bool padded = row_is_padded(p, tc, quad, lane);
      int lo, hi;
      epi_columns(warp, tc.n_eff, lo, hi);
      FuseW fw;
      fuse_weights(p, tc, quad, lane, lo, fw);
      if (tc.qk) issue_gate_exponents(p, tc, quad, lane, (warp - 2) >= 4 ? 1 : 0, 0, ge);
      if (!mbar_wait(&acc_full[buf], (it >> 1) & 1, abort_flag, p.err)) break;
      tc_fence_after();
      if (tc.qk) {
        if (!epilogue_qk(p, tc, tmem + buf * BN, quad, lane, (warp - 2) >= 4 ? 1 : 0, padded, stg, ge, abort_flag))
          break;
      } else if (p.task[tc.task].epi == kEpiStoreF32) {
        epilogue_f32(p, tc, tmem + buf * BN, quad, lane, lo, hi);
      } else {
        epilogue_tile(p, tc, tmem + buf * BN, quad, lane, lo, hi, padded, stg, sel, fw);
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);
      count_rows_done(p, tc, lane);
    }
    if (lane == 0) bulk_wait0();
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
//
// kHeld (the fused output launch with one or two coarse branches): warp 10 of
// each CTA TMA-loads the held coarse rows of the CTA's tile into shared memory
// during the tile's main loop, so the epilogue reads them there instead of
// gathering them from L2. This takes a 60 KB region: the ring has 4 stages and
// every epilogue warp one staging buffer.
constexpr int kPairStageBytes = 2 * kGemmBM * kGemmBK * 2;  // A half + B half = 32 KB
constexpr int kPairBN = 256, kPairBM = 256;
constexpr int kHeldBytes = 60 * 1024;

template <bool kHeld>
struct PairLayout {
  static constexpr int kStages = kHeld ? 4 : 5;
  static constexpr int kThreadsT = kHeld ? 352 : 320;  // + warp 10: held-row loader
  static constexpr int kStagingOffset = kStages * kPairStageBytes;
  static constexpr int kStagingBytesT = 8 * kStagerBytes;
  static constexpr int kHeldOffset = kStagingOffset + kStagingBytesT;
  // !kHeld: one 4 KB buffer per epilogue warp for the gate exponents of a q|k
  // tile (32 rows x 32 channels fp32, 128-byte swizzle), filled by TMA
  static constexpr int kGdOffset = kHeldOffset + (kHeld ? kHeldBytes : 0);
  static constexpr int kBarOffset = kGdOffset + (kHeld ? 0 : 8 * kGdBoxBytes);
  static constexpr int kSmemBytes = kBarOffset + 512 + 1024;  // barriers + 1024 B alignment slack
  static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
};

// Dynamic tile scheduling (GemmParams::tile_counter set): the leader's producer
// takes the next tile index from the counter and hands it to every role of both
// CTAs through a ring of kTileRing slots in shared memory (tile_full in each CTA,
// tile_empty in the leader, counting one arrival per consumer: the leader's MMA
// thread, the peer's producer and the eight epilogue warps of each CTA). -1 ends
// the sequence. A pair that starts late (its SMs still busy with another kernel)
// then takes only the tiles that are left.
constexpr int kTileRing = 4;
constexpr int kTileConsumers = 1 + 1 + 2 * 8;

template <bool kHeld>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairLayout<kHeld>::kThreadsT, 1)
    gemm_pair_kernel(const __grid_constant__ GemmParams p) {
  using Lay = PairLayout<kHeld>;
  constexpr int kStagesT = Lay::kStages;
  constexpr int kHeldBars = kHeld ? 4 : 1;
  static_assert((2 * kStagesT + 4 + 2 * kHeldBars + 2 * kTileRing + 8) * 8 + 4 * kTileRing + 8 <= 512, "barrier region");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full_bar = reinterpret_cast<uint64_t*>(smem + Lay::kBarOffset);
  uint64_t* empty_bar = full_bar + kStagesT;
  uint64_t* acc_full = empty_bar + kStagesT;  // [2]
  uint64_t* acc_empty = acc_full + 2;         // [2] (used in the leader)
  uint64_t* held_full = acc_empty + 2;        // kHeld [4]: box j of this CTA's held rows landed
  uint64_t* held_empty = held_full + kHeldBars;  // kHeld [4]: the epilogue warps are done with box j
  uint64_t* tile_full = held_empty + kHeldBars;  // [kTileRing] dynamic tiles
  uint64_t* tile_empty = tile_full + kTileRing;  // [kTileRing] (used in the leader)
  uint64_t* gd_full = tile_empty + kTileRing;    // [8] per epilogue warp: its gate exponents landed
  volatile int* tile_slot = reinterpret_cast<volatile int*>(gd_full + 8);  // [kTileRing]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(const_cast<int*>(tile_slot) + kTileRing);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint8_t* held_smem = smem + Lay::kHeldOffset;

  const int warp = warp_id(), lane = lane_id();
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const bool dyn = p.tile_counter != nullptr;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStagesT; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], 2 * kEpiThreads);
    }
    for (int j = 0; j < kHeldBars; ++j) {
      mbar_init(&held_full[j], 1);
      mbar_init(&held_empty[j], 4);  // the four epilogue warps of the box's column half
    }
    for (int r = 0; r < kTileRing; ++r) {
      mbar_init(&tile_full[r], 1);
      mbar_init(&tile_empty[r], kTileConsumers);
    }
    for (int w = 0; w < 8; ++w) mbar_init(&gd_full[w], 1);
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
  griddep_wait();
  griddep_launch();
  const uint32_t tmem = *tmem_slot;
  const int ntiles = p.total_tiles;
  // The it-th tile of this pair, or -1 when there are no more. Dynamic mode:
  // `fetch` (the leader's producer) takes it from the counter and publishes it;
  // every other caller reads it from the ring; `elected` callers (one lane per
  // warp, or the single-thread roles) arrive on the leader's tile_empty.
  auto next_tile = [&](int it, bool fetch, bool elected) -> int {
    if (!dyn) {
      const int t = pair + it * npairs;
      return t < ntiles ? t : -1;
    }
    const int slot = it % kTileRing;
    int t = -1;
    if (fetch) {
      if (it >= kTileRing && !mbar_wait(&tile_empty[slot], ((it / kTileRing) - 1) & 1, abort_flag, p.err)) return -1;
      t = static_cast<int>(atomicAdd(p.tile_counter, 1u));
      if (t >= ntiles) t = -1;
      tile_slot[slot] = t;
      st_cluster_u32(mapa_shared(smem_u32(const_cast<int*>(&tile_slot[slot])), 1), static_cast<uint32_t>(t));
      mbar_arrive(&tile_full[slot]);
      mbar_arrive_cluster(mapa_shared(smem_u32(&tile_full[slot]), 1));
      return t;
    }
    if (elected) {
      if (!mbar_wait_cluster(&tile_full[slot], (it / kTileRing) & 1, abort_flag, p.err)) return -1;
      t = tile_slot[slot];
      mbar_arrive_cluster(mapa_shared(smem_u32(&tile_empty[slot]), 0));
    }
    return t;
  };
  // held rows: coarse branch c occupies [held_off[c], +4 boxes)
  int held_off[2] = {0, 0}, held_box[2] = {0, 0};
  if (kHeld) {
    const GemmTask& T0 = p.task[0];
    for (int c = 0; c < 2 && c < T0.n_coarse; ++c) {
      held_box[c] = held_box_rows(T0.coarse_scale[c]) * 128;
      if (c == 1) held_off[1] = 4 * held_box[0];
    }
  }

  if (warp == 0 && lane == 0) {
    // ---------------- TMA producer of this CTA's halves
    for (int t = 0; t < p.n_tasks; ++t) {
      prefetch_tmap(&p.task[t].tmA);
      prefetch_tmap(&p.task[t].tmB);
    }
    uint32_t kbg = 0, ready = 0;
    bool ok = true;
    for (int it = 0; ok; ++it) {
      const int tile = next_tile(it, rank == 0, true);
      if (tile < 0) break;
      const TileCoord tc = decode_tile(p, tile, kPairBN, kPairBM);
      const GemmTask& T = p.task[tc.task];
      if (!task_ready(T, tc.task, ready, abort_flag, p.err)) break;
      const int arow = tc.m0 + 128 * static_cast<int>(rank);
      const int brow = rank ? tc.brow1 : tc.brow0;
      for (int kb = 0; kb < tc.kblocks; ++kb, ++kbg) {
        const uint32_t s = kbg % kStagesT;
        if (kbg >= kStagesT && !mbar_wait(&empty_bar[s], ((kbg / kStagesT) - 1) & 1, abort_flag, p.err)) {
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
    uint32_t kbg = 0;
    bool ok = true;
    for (uint32_t it = 0; ok; ++it) {
      const int tile = next_tile(static_cast<int>(it), false, true);
      if (tile < 0) break;
      const TileCoord tc = decode_tile(p, tile, kPairBN, kPairBM);
      const uint32_t buf = it & 1;
      if (it >= 2 && !mbar_wait(&acc_empty[buf], ((it >> 1) - 1) & 1, abort_flag, p.err)) break;
      tc_fence_after();
      const uint32_t idesc = idesc_f16(kPairBM, tc.n_eff, p.task[tc.task].ab_bf16, 0, 0);
      const uint32_t tacc = tmem + buf * kPairBN;
      for (int kb = 0; kb < tc.kblocks; ++kb, ++kbg) {
        const uint32_t s = kbg % kStagesT;
        if (!mbar_wait(&full_bar[s], (kbg / kStagesT) & 1, abort_flag, p.err)) {
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
  } else if (kHeld && warp == 10) {
    // ---------------- held coarse rows of this CTA's tiles (one tile ahead at most;
    // the fused launch schedules its tiles statically)
    if (lane == 0) {
      const GemmTask& T = p.task[0];
      for (int c = 0; c < 2 && c < T.n_coarse; ++c) prefetch_tmap(&T.tmOut[1 + c]);
      uint32_t it = 0;
      uint32_t bytes = 0;
      for (int c = 0; c < 2 && c < T.n_coarse; ++c) bytes += held_box[c];
      bool ok = true;
      for (int tile = pair; ok && tile < ntiles; tile += npairs, ++it) {
        const TileCoord tc = decode_tile(p, tile, kPairBN, kPairBM);
        const int m0 = tc.m0 + 128 * static_cast<int>(rank);
        // boxes in the order the epilogue releases them (the first 64 columns of
        // each column half first); each is refilled once its four warps are done
        const bool half = tc.n_eff == 128;  // a half tile: boxes 0 and 2 hold its two 64-column blocks
        for (int q = 0; q < 4; ++q) {
          const int j = (q >> 1) | ((q & 1) << 1);  // 0, 2, 1, 3
          if (it >= 1 && !mbar_wait(&held_empty[j], (it - 1) & 1, abort_flag, p.err)) {
            ok = false;
            break;
          }
          if (half && (j & 1)) {
            mbar_arrive(&held_full[j]);  // nothing to load: complete the box's round
            continue;
          }
          mbar_arrive_expect_tx(&held_full[j], bytes);
          const int col = tc.n0 + 64 * (half ? j >> 1 : j);
          for (int c = 0; c < 2 && c < T.n_coarse; ++c)
            tma_load_3d(&T.tmOut[1 + c], &held_full[j], held_smem + held_off[c] + j * held_box[c], col,
                        held_base(m0, T.coarse_scale[c]), tc.b);
        }
      }
    }
  } else if (warp >= 2 && warp < 10) {
    // ---------------- epilogue of this CTA's 128 accumulator rows
    const int quad = warp & 3;
    const uint32_t lead_empty0 = mapa_shared(smem_u32(&acc_empty[0]), 0);
    const uint32_t lead_empty1 = mapa_shared(smem_u32(&acc_empty[1]), 0);
    const Stager stg{smem + Lay::kStagingOffset + (warp - 2) * kStagerBytes, lane, false};
    uint32_t gd_phase = 0;
    const GateExp ge{smem + Lay::kGdOffset + (warp - 2) * kGdBoxBytes, &gd_full[warp - 2], &gd_phase};
    int sel = 0;
    if (lane == 0) prefetch_out_maps(p);
    for (uint32_t it = 0;; ++it) {
      int tile = next_tile(static_cast<int>(it), false, lane == 0);
      tile = __shfl_sync(0xffffffffu, tile, 0);
      if (tile < 0) break;
      TileCoord tc = decode_tile(p, tile, kPairBN, kPairBM);
      tc.m0 += 128 * static_cast<int>(rank);
      const uint32_t buf = it & 1;
      const bool padded = row_is_padded(p, tc, quad, lane);
      int lo, hi;
      epi_columns(warp, tc.n_eff, lo, hi);
      FuseW fw;
      fuse_weights(p, tc, quad, lane, lo, fw);
      if (!kHeld && tc.qk) issue_gate_exponents(p, tc, quad, lane, (warp - 2) >= 4 ? 1 : 0, 0, ge);
      if (!mbar_wait(&acc_full[buf], (it >> 1) & 1, abort_flag, p.err)) break;
      tc_fence_after();
      if (kHeld) {
        const GemmTask& T = p.task[tc.task];
        const int t = tc.m0 + quad * 32 + lane;
        Held h;
        for (int c = 0; c < 2; ++c) {
          h.smem[c] = held_smem + held_off[c];
          h.box_bytes[c] = held_box[c];
          h.lrow[c] = 0;
          if (c < T.n_coarse) {
            const int s = T.coarse_scale[c];
            h.lrow[c] = (t + 1) / s - 1 - held_base(tc.m0, s);
          }
        }
        h.full = held_full;
        h.empty = held_empty;
        h.parity = it & 1;
        h.abort_flag = abort_flag;
        h.half = tc.n_eff == 128;
        if (!epilogue_tile(p, tc, tmem + buf * kPairBN, quad, lane, lo, hi, padded, stg, sel, fw, &h)) break;
      } else if (!kHeld && tc.qk) {
        if (!epilogue_qk(p, tc, tmem + buf * kPairBN, quad, lane, (warp - 2) >= 4 ? 1 : 0, padded, stg, ge,
                         abort_flag))
          break;
      } else if (p.task[tc.task].epi == kEpiStoreF32) {
        epilogue_f32(p, tc, tmem + buf * kPairBN, quad, lane, lo, hi);
      } else {
        epilogue_tile(p, tc, tmem + buf * kPairBN, quad, lane, lo, hi, padded, stg, sel, fw);
      }
      tc_fence_before();
      mbar_arrive_cluster(buf ? lead_empty1 : lead_empty0);
      if (!kHeld) count_rows_done(p, tc, lane);
    }
    if (lane == 0) bulk_wait0();
  }
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 2 * kPairBN);
  }
  if (dyn && p.tile_exit && threadIdx.x == 0) {
    // this CTA takes no more tiles and waits for nothing more; the last CTA to
    // leave clears the counters for the next launch
    __threadfence();
    if (atomicAdd(p.tile_exit, 1u) + 1u == gridDim.x) {
      atomicExch(p.tile_counter, 0u);
      for (int i = 0; i < p.n_reset64; ++i) atomicExch(p.reset64 + i, 0ull);
      atomicExch(p.tile_exit, 0u);
    }
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
template <bool kHeld>
int max_active_pairs() {
  using Lay = PairLayout<kHeld>;
  static int n = -1;
  if (n < 0) {
    n = 0;
    if (cudaFuncSetAttribute(gemm_pair_kernel<kHeld>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Lay::kSmemBytes) == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2 * sm_count(), 1, 1);
      cfg.blockDim = dim3(Lay::kThreadsT, 1, 1);
      cfg.dynamicSmemBytes = Lay::kSmemBytes;
      cudaLaunchAttribute attr;
      attr.id = cudaLaunchAttributeClusterDimension;
      attr.val.clusterDim.x = 2;
      attr.val.clusterDim.y = 1;
      attr.val.clusterDim.z = 1;
      cfg.attrs = &attr;
      cfg.numAttrs = 1;
      int c = 0;
      if (cudaOccupancyMaxActiveClusters(&c, gemm_pair_kernel<kHeld>, &cfg) == cudaSuccess) n = c;
    }
    cudaGetLastError();  // clear a failed query
  }
  return n;
}

cudaError_t launch_gemm(const GemmParams& p, int bn, cudaStream_t st, int max_pairs) {
  if (p.total_tiles <= 0) return cudaSuccess;
  if (bn != 256) return cudaErrorInvalidValue;
  // the fused output launch with one or two coarse branches stages their held
  // rows in shared memory (the caller encodes tmOut[1 + c] for them)
  // (and only with full 256-column tiles: every 64-column box of held rows then
  // has the four epilogue warps that release it)
  const bool held = p.n_tasks == 1 && p.task[0].epi == kEpiFuse && p.task[0].n_coarse >= 1 &&
                    p.task[0].n_coarse <= 2 && p.task[0].N % kPairBN == 0 &&
                    held_rows_fit(p.task[0].coarse_scale, p.task[0].n_coarse);
  int pairs = held ? max_active_pairs<true>() : max_active_pairs<false>();
  if (max_pairs > 0 && pairs > max_pairs) pairs = max_pairs;
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
      T.n_tiles = T.epi == kEpiProjGate ? T.n_qk + (T.nv + kPairBN - 1) / kPairBN : (T.N + kPairBN - 1) / kPairBN;
      T.tile_begin = tiles;
      tiles += batches * T.m_tiles * T.n_tiles;
    }
    // the fused output launch: a last, partial wave of at most half the pairs runs
    // as twice as many 128-column half tiles
    if (held && tiles > pairs) {
      const int full = tiles / pairs * pairs, rest = tiles - full;
      if (rest > 0 && 2 * rest <= pairs) {
        q.task[0].half_from = full;
        tiles += rest;
      }
    }
    q.total_tiles = tiles;
    const int grid_pairs = tiles < pairs ? tiles : pairs;
    if (held)
      return launch_pdl(gemm_pair_kernel<true>, dim3(2 * grid_pairs), dim3(PairLayout<true>::kThreadsT),
                        PairLayout<true>::kSmemBytes, st, q);
    return launch_pdl(gemm_pair_kernel<false>, dim3(2 * grid_pairs), dim3(PairLayout<false>::kThreadsT),
                      PairLayout<false>::kSmemBytes, st, q);
  }
  int grid = p.total_tiles < sm_count() ? p.total_tiles : sm_count();
  if (max_pairs > 0 && grid > 2 * max_pairs) grid = 2 * max_pairs;
  const int smem = GemmLayout<256>::kSmemBytes;
  auto kern = gemm_kernel<256>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(grid), dim3(kThreads), smem, st, p);
}

}  // namespace msgla
