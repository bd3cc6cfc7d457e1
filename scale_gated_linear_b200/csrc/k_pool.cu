// k_pool.cu -- one pass over the layer input X per 128-row tile (sm_100a):
//   * U = X Wu^T on tcgen05 (M = 128 rows, N = ldu): the fusion logits
//     z_t = W_fuse x_t of Eq. (10) (MS-GLA reading notes, Sec. 3.3) and every
//     branch's low-rank gate input x_t W_g1^T (Sec. 2.1) of the unpooled rows;
//   * the mean pooling of Eq. (8) (Sec. 3.1) for every coarse scale, also on the
//     tensor cores and from the same shared-memory tiles of X, so X is read from
//     global memory once: with Pm the 0/1 matrix of pooled slots x tile rows
//     (slot m of scale s covers rows i s .. i s + s - 1; rows past the sequence
//     or padded by the mask are 0), the sums are Pm X (M = 128 slots, K = the
//     tile's 128 rows, N = the stage's 64 columns; X as an MN-major operand),
//     and each slot's sums are divided by its number of valid rows (at least 1);
//   * optionally the fusion weights w = softmax(z + b_fuse) (layers without a
//     scale-1 branch, whose fusion needs them as a separate array).
//
// One CTA per (sequence, 128-row tile), 192 threads:
//   warp 0     TMA producer: per 64-column K block, the tile's 128 x 64 slice of X
//              and the ldu x 64 slice of Wu (128-byte swizzle) into a ring stage
//   warp 1     TMEM allocation + tcgen05.mma issue: per stage the U products
//              (accumulated over the stages) and the stage's pooling product into
//              one of four pooled-sum buffers
//   warps 2-5  build Pm; per stage drain the pooled sums (one slot per TMEM lane:
//              scale, fp16, 128-byte row stores); at the end the U epilogue (one
//              accumulator row per thread, fp32 stores)
// Coarse scales must be powers of two up to 8 (slots: 64 + 32 + 16 <= 128), so
// pooled blocks never straddle a tile.
#include "msgla_internal.h"
#include "sm100_ptx.cuh"

namespace msgla {
namespace {

constexpr int kThreads = 192;
constexpr int kRows = 128;
constexpr int kABytes = kRows * 64 * 2;  // one 128 x 64 bf16 slice of X
constexpr int kPmBytes = 2 * kABytes;    // Pm: 128 slots x 128 rows bf16, two 64-column K blocks

enum {
  B_FULL = 0,
  B_EMPTY = kPoolUMaxStages,
  B_ACC = 2 * kPoolUMaxStages,
  B_PM,                                      // Pm is in shared memory (four warp arrivals)
  B_POOL_FULL,                               // [kPoolUBufs] pooled sums of a stage are in TMEM buffer j
  B_POOL_EMPTY = B_POOL_FULL + kPoolUBufs,   // [kPoolUBufs] buffer j drained (four warp arrivals)
  B_COUNT = B_POOL_EMPTY + kPoolUBufs
};

__global__ void __launch_bounds__(kThreads, 1) pool_u_kernel(const __grid_constant__ PoolUParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = p.stages;
  const int stage_bytes = kABytes + p.ldu * 128;
  uint8_t* pm = smem + S * stage_bytes;
  uint64_t* bar = reinterpret_cast<uint64_t*>(pm + kPmBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar + B_COUNT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = warp_id(), lane = lane_id();
  const int b = blockIdx.x / p.m_tiles;
  const int m0 = (blockIdx.x % p.m_tiles) * kRows;
  const int KB = p.d / 64;
  const bool pooling = p.n_coarse > 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&bar[B_FULL + s], 1);
      mbar_init(&bar[B_EMPTY + s], 1);
    }
    mbar_init(&bar[B_ACC], 1);
    mbar_init(&bar[B_PM], 4);
    for (int j = 0; j < kPoolUBufs; ++j) {
      mbar_init(&bar[B_POOL_FULL + j], 1);
      mbar_init(&bar[B_POOL_EMPTY + j], 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  griddep_wait();
  griddep_launch();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tpool = tmem + p.pool_col;  // pooled-sum buffers j: [pool_col + 64 j, +64)

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&p.tmX);
      prefetch_tmap(&p.tmW);
      for (int kb = 0; kb < KB; ++kb) {
        const int s = kb % S;
        if (kb >= S && !mbar_wait(&bar[B_EMPTY + s], ((kb / S) - 1) & 1, abort_flag, p.err)) break;
        uint8_t* sa = smem + s * stage_bytes;
        mbar_arrive_expect_tx(&bar[B_FULL + s], static_cast<uint32_t>(stage_bytes));
        tma_load_3d(&p.tmX, &bar[B_FULL + s], sa, kb * 64, m0, b);
        tma_load_2d(&p.tmW, &bar[B_FULL + s], sa + kABytes, kb * 64, 0);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id_u = idesc_f16(kRows, p.ldu, 1, 0, 0);
      const uint32_t id_pool = idesc_f16(kRows, 64, 1, 0, 1);  // Pm K-major, X MN-major
      const uint32_t spm = smem_u32(pm);
      bool ok = !pooling || mbar_wait(&bar[B_PM], 0, abort_flag, p.err);
      for (int kb = 0; kb < KB && ok; ++kb) {
        const int s = kb % S;
        if (!mbar_wait(&bar[B_FULL + s], (kb / S) & 1, abort_flag, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + s * stage_bytes), sb = sa + kABytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_f16(tmem, sdesc_sw128(sa + kk * 32, 16, 1024), sdesc_sw128(sb + kk * 32, 16, 1024), id_u,
                   (kb | kk) != 0);
        if (pooling) {
          // pooled sums of this stage's 64 columns: Pm [128 x 128] * X tile [128 rows x 64]
          const int j = kb % kPoolUBufs;
          if (kb >= kPoolUBufs && !mbar_wait(&bar[B_POOL_EMPTY + j], ((kb / kPoolUBufs) - 1) & 1, abort_flag, p.err)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_f16(tpool + 64 * j, sdesc_sw128(spm + (kk >> 2) * kABytes + (kk & 3) * 32, 16, 1024),
                     sdesc_sw128(sa + kk * 2048, kABytes, 1024), id_pool, kk != 0);
          umma_commit(&bar[B_POOL_FULL + j]);
        }
        umma_commit(&bar[B_EMPTY + s]);
      }
      if (ok) umma_commit(&bar[B_ACC]);
    }
  } else {
    // ---------------- warps 2-5: TMEM lane quadrant `quad`, lane = slot / row
    const int quad = warp & 3;
    const int m = quad * 32 + lane;  // pooling slot and U row of this thread
    // this slot's coarse branch, pooled row, first tile row and valid-row count
    int c = -1, prow = 0, r_lo = 0, width = 0;
    for (int l = 1; l <= 3; ++l) {
      const int cl = p.lvl_branch[l];
      if (cl < 0) continue;
      const int base = p.slot_base[l], n = kRows >> l;
      if (m >= base && m < base + n) {
        c = cl;
        width = 1 << l;
        r_lo = (m - base) << l;
        prow = (m0 >> l) + (m - base);
      }
    }
    float cnt = 0.f;
    uint32_t vbits = 0;  // valid rows of the slot's block
    for (int q = 0; q < width; ++q) {
      const int t = m0 + r_lo + q;
      if (t < p.L && (!p.M || p.M[static_cast<size_t>(b) * p.L + t])) {
        vbits |= 1u << q;
        cnt += 1.f;
      }
    }
    const bool store = c >= 0 && prow < p.rows[c];
    bool ok = true;
    if (pooling) {
      // row m of Pm: 1 (bf16 0x3F80) at the slot's valid rows, 0 elsewhere;
      // 16-byte chunk k of K block kb2 at chunk k ^ (m & 7) of the 128-byte row
#pragma unroll 1
      for (int ch = 0; ch < 16; ++ch) {
        const int r0 = ch * 8;
        uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int q = r0 + e - r_lo;
          if (c >= 0 && q >= 0 && q < width && ((vbits >> q) & 1u)) w[e >> 1] |= 0x3F80u << (16 * (e & 1));
        }
        st_shared_v4(smem_u32(pm + (ch >> 3) * kABytes + m * 128 + (((ch & 7) ^ (m & 7)) << 4)), w[0], w[1], w[2],
                     w[3]);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar[B_PM]);
      // per stage: the slot's 64 pooled sums -> means (fp16) -> 128 contiguous bytes
      const float inv = 1.f / fmaxf(cnt, 1.f);
      __half* dst = store ? p.Xp[c] + (static_cast<size_t>(b) * p.rows[c] + prow) * p.d : nullptr;
      uint32_t over = 0;
      for (int kb = 0; kb < KB; ++kb) {
        const int j = kb % kPoolUBufs;
        if (!mbar_wait(&bar[B_POOL_FULL + j], (kb / kPoolUBufs) & 1, abort_flag, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t va[32], vb[32];
        tmem_ld32(tmem_addr(tpool, quad * 32, 64 * j), va);
        tmem_ld32(tmem_addr(tpool, quad * 32, 64 * j + 32), vb);
        tmem_wait_ld(va);
        tmem_wait_ld(vb);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar[B_POOL_EMPTY + j]);
        if (store) {
          uint4* o = reinterpret_cast<uint4*>(dst + kb * 64);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const uint32_t* r = q < 4 ? va + 8 * q : vb + 8 * (q - 4);
            uint4 x;
            x.x = pack_half2(__uint_as_float(r[0]) * inv, __uint_as_float(r[1]) * inv);
            x.y = pack_half2(__uint_as_float(r[2]) * inv, __uint_as_float(r[3]) * inv);
            x.z = pack_half2(__uint_as_float(r[4]) * inv, __uint_as_float(r[5]) * inv);
            x.w = pack_half2(__uint_as_float(r[6]) * inv, __uint_as_float(r[7]) * inv);
            half2_track_nonfinite(over, x.x);
            half2_track_nonfinite(over, x.y);
            half2_track_nonfinite(over, x.z);
            half2_track_nonfinite(over, x.w);
            o[q] = x;
          }
        }
      }
      if (over & 0x80008000u) atomicCAS(p.err, 0, kDevRange);
    }
    // U rows: the fusion logits and gate inputs of the unpooled rows
    if (ok && mbar_wait(&bar[B_ACC], 0, abort_flag, p.err)) {
      tc_fence_after();
      const int t = m0 + m;
      const size_t grow = static_cast<size_t>(b) * p.L + t;
#pragma unroll 1
      for (int c0 = 0; c0 < p.ldu; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem_addr(tmem, quad * 32, c0), v);
        tmem_wait_ld(v);
        if (t >= p.L) continue;
        if (c0 == 0 && p.w) {
          // fusion weights w = softmax(z + b_fuse) from the logits in columns 0..n_scales-1
          float zz[kMaxScales];
          float zmax = -INFINITY;
#pragma unroll
          for (int jj = 0; jj < kMaxScales; ++jj) {
            zz[jj] = jj < p.n_scales ? __uint_as_float(v[jj]) + __ldg(p.bfuse + jj) : -INFINITY;
            zmax = fmaxf(zmax, zz[jj]);
          }
          float sum = 0.f;
#pragma unroll
          for (int jj = 0; jj < kMaxScales; ++jj) {
            zz[jj] = jj < p.n_scales ? __expf(zz[jj] - zmax) : 0.f;
            sum += zz[jj];
          }
          const float inv = 1.f / sum;
#pragma unroll
          for (int jj = 0; jj < kMaxScales; ++jj)
            if (jj < p.n_scales) p.w[grow * p.n_scales + jj] = zz[jj] * inv;
        }
        float* dst = p.U + grow * p.ldu + c0;
        if (c0 + 32 <= p.ldu) {
#pragma unroll
          for (int e = 0; e < 8; ++e)
            reinterpret_cast<float4*>(dst)[e] = make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                                                            __uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3]));
        } else {
#pragma unroll
          for (int e = 0; e < 16; ++e) dst[e] = __uint_as_float(v[e]);  // ldu is a multiple of 16
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, p.tmem_cols);
  }
}

}  // namespace

int pool_u_smem_bytes(int ldu, int stages) {
  return stages * (kABytes + ldu * 128) + kPmBytes + 1024 + 8 * B_COUNT + 16;
}

cudaError_t launch_pool_u(const PoolUParams& p, cudaStream_t st) {
  if (p.B * p.m_tiles == 0) return cudaSuccess;
  const int smem = pool_u_smem_bytes(p.ldu, p.stages);
  cudaError_t e = cudaFuncSetAttribute(pool_u_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(pool_u_kernel, dim3(p.B * p.m_tiles), dim3(kThreads), smem, st, p);
}

}  // namespace msgla
