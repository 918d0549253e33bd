// fp32-accurate rank-128 updates on the tcgen05 tensor cores:
//     C[m][c] -= sum_{t < 128} P[m][t] * Q[c][t]
// for one 128 x 128 tile of C per CTA.
//
// The pages' method needs full fp32 accuracy here (page "GPTQ, with the code
// open", section "Paper vs. code": TF32 is switched off because the Cholesky
// chain needs full 32-bit precision).  Each operand therefore arrives split
// in two fp32 arrays, hi = TF32(x) (round to nearest) and lo = x - hi (exact),
// and the product is taken as  P_hi Q_hi + P_hi Q_lo + P_lo Q_hi  with
// tcgen05.mma kind::tf32 (fp32 accumulation in TMEM).  The dropped P_lo Q_lo
// term and the TF32 truncation of lo are below 2^-21 relative per product.
//
// Structure: 128 threads.  Lane 0 of warp 0 streams the four 128 x 32 fp32
// tiles (P_hi, P_lo, Q_hi, Q_lo) of each of the 4 k-blocks through a 3-stage
// TMA ring (128-byte swizzle); lane 0 of warp 1 issues 3 x 4 MMAs
// (M = N = 128, K = 8) per k-block; then all four warps drain the 128 x 128
// fp32 accumulator (warp w reads TMEM lanes 32w..32w+31) and subtract it from
// C, masked to the tile's valid extent.  No multicast; every wait is bounded.
//
// `Decoder` maps blockIdx to a tile:  tile(bx, by) -> PgTile.  On a wait
// timeout the kernel writes `timeout_code` to `info` (if given) and exits.
#pragma once
#include <algorithm>
#include <cstdint>

#include "gptq_internal.cuh"
#include "sm100_ptx.cuh"

namespace gptq {

constexpr int kPgThreads = 128;
constexpr int kPgStages = 3;
constexpr int kPgKBlocks = kBlock / 32;                 // 4 k-blocks of 32 fp32
constexpr int kPgTileBytes = 128 * 32 * 4;              // one 128 x 32 fp32 tile
constexpr int kPgStageBytes = 4 * kPgTileBytes;         // P_hi, P_lo, Q_hi, Q_lo
constexpr size_t kPgSmemBytes = (size_t)kPgStages * kPgStageBytes + 1024 + 256;
constexpr uint32_t kPgTmemCols = 128;

struct PgTile {
  float* C;       // tile origin in C
  int64_t ldc;
  int prow, pkx;  // P tile: rows [prow, prow+128), columns [pkx, pkx+128)
  int qrow, qkx;  // Q tile: rows [qrow, qrow+128), columns [qkx, qkx+128)
  int mext, cext; // valid rows / columns of the C tile
  int valid;      // 0: nothing to do
};

__device__ __forceinline__ void pg_abort(volatile int* abort_flag, int32_t* info,
                                         int32_t code) {
  *abort_flag = 1;
  if (info) atomicExch(info, code);
}

template <class Decoder>
__global__ void __launch_bounds__(kPgThreads, 1)
    panel_gemm_kernel(const __grid_constant__ CUtensorMap mPh, const __grid_constant__ CUtensorMap mPl,
                      const __grid_constant__ CUtensorMap mQh, const __grid_constant__ CUtensorMap mQl,
                      const Decoder dec, int32_t* info, int32_t timeout_code,
                      const int32_t* skip_if_nonzero) {
  if (skip_if_nonzero && *(volatile const int32_t*)skip_if_nonzero != 0) return;
  const PgTile t = dec.tile(blockIdx.x, blockIdx.y);
  if (!t.valid) return;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kPgStages * kPgStageBytes);
  uint64_t* full = bars;                 // [kPgStages]
  uint64_t* empty = bars + kPgStages;    // [kPgStages]
  uint64_t* done = bars + 2 * kPgStages; // accumulator complete (also the abort drain)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  constexpr uint64_t kLimit = (uint64_t)kGridWaitLimitNs;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kPgStages; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    ptx::mbar_init(done, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, kPgTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------------------- TMA producer
    ptx::prefetch_tmap(&mPh);
    ptx::prefetch_tmap(&mPl);
    ptx::prefetch_tmap(&mQh);
    ptx::prefetch_tmap(&mQl);
    int issued_parity[kPgStages] = {-1, -1, -1};
    bool ok = true;
    for (int kb = 0; kb < kPgKBlocks; ++kb) {
      const int st = kb % kPgStages;
      if (kb >= kPgStages &&
          !ptx::mbar_wait_bounded(&empty[st], (uint32_t)((kb / kPgStages - 1) & 1), abort_flag,
                                  kLimit)) {
        ok = false;
        break;
      }
      uint8_t* sb = smem + st * kPgStageBytes;
      ptx::mbar_arrive_expect_tx(&full[st], kPgStageBytes);
      ptx::tma_load_2d(sb + 0 * kPgTileBytes, &mPh, &full[st], t.pkx + 32 * kb, t.prow);
      ptx::tma_load_2d(sb + 1 * kPgTileBytes, &mPl, &full[st], t.pkx + 32 * kb, t.prow);
      ptx::tma_load_2d(sb + 2 * kPgTileBytes, &mQh, &full[st], t.qkx + 32 * kb, t.qrow);
      ptx::tma_load_2d(sb + 3 * kPgTileBytes, &mQl, &full[st], t.qkx + 32 * kb, t.qrow);
      issued_parity[st] = (kb / kPgStages) & 1;
    }
    if (!ok) {
      pg_abort(abort_flag, info, timeout_code);
      volatile int never = 0;
      for (int s = 0; s < kPgStages; ++s)
        if (issued_parity[s] >= 0)
          ptx::mbar_wait_bounded(&full[s], (uint32_t)issued_parity[s], &never, kLimit);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc = ptx::idesc_tf32_f32(128, 128);
    bool ok = true;
    for (int kb = 0; kb < kPgKBlocks; ++kb) {
      const int st = kb % kPgStages;
      if (!ptx::mbar_wait_bounded(&full[st], (uint32_t)((kb / kPgStages) & 1), abort_flag,
                                  kLimit)) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      const uint32_t sb = ptx::smem_u32(smem + st * kPgStageBytes);
      const uint64_t ph = ptx::smem_desc_sw128(sb + 0 * kPgTileBytes);
      const uint64_t pl = ptx::smem_desc_sw128(sb + 1 * kPgTileBytes);
      const uint64_t qh = ptx::smem_desc_sw128(sb + 2 * kPgTileBytes);
      const uint64_t ql = ptx::smem_desc_sw128(sb + 3 * kPgTileBytes);
#pragma unroll
      for (int k = 0; k < 4; ++k) {  // K = 8 fp32 = 32 bytes per MMA
        ptx::mma_tf32(tmem_base, ph + 2 * k, qh + 2 * k, idesc, (kb > 0 || k > 0) ? 1u : 0u);
        ptx::mma_tf32(tmem_base, ph + 2 * k, ql + 2 * k, idesc, 1u);
        ptx::mma_tf32(tmem_base, pl + 2 * k, qh + 2 * k, idesc, 1u);
      }
      ptx::mma_commit(&empty[st]);
    }
    // `done` completes when every MMA issued above has finished (also on abort)
    ptx::mma_commit(done);
    if (!ok) pg_abort(abort_flag, info, timeout_code);
  }

  // ------------------------------------------------------------ epilogue
  const bool ready = ptx::mbar_wait_bounded(done, 0, abort_flag, kLimit);
  if (!ready) pg_abort(abort_flag, info, timeout_code);
  __syncwarp();
  // warp-uniform decision: tcgen05.ld below needs all 32 lanes
  const bool go = __all_sync(0xffffffffu, ready && !*abort_flag);
  ptx::tc_fence_after();
  if (go) {
    const int row = warp * 32 + lane;
    float* crow = t.C + (int64_t)row * t.ldc;
    const bool vec = t.cext == 128 && (t.ldc % 4) == 0 &&
                     (reinterpret_cast<uintptr_t>(t.C) % 16) == 0;
#pragma unroll 1
    for (int ch = 0; ch < 4; ++ch) {
      uint32_t v[32];
      ptx::tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(warp * 32) << 16) + (uint32_t)(ch * 32), v);
      ptx::tmem_ld_wait();
      if (row < t.mext) {
        if (vec) {
          float4* c4 = reinterpret_cast<float4*>(crow + ch * 32);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            float4 x = c4[j];
            x.x -= __uint_as_float(v[4 * j + 0]);
            x.y -= __uint_as_float(v[4 * j + 1]);
            x.z -= __uint_as_float(v[4 * j + 2]);
            x.w -= __uint_as_float(v[4 * j + 3]);
            c4[j] = x;
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int col = ch * 32 + j;
            if (col < t.cext) crow[col] -= __uint_as_float(v[j]);
          }
        }
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, kPgTmemCols);
  }
}

// hi / lo split of one value for the kernel above.
__device__ __forceinline__ void tf32_split(float x, float& hi, float& lo) {
  hi = ptx::tf32_hi(x);
  lo = x - hi;
}

// ===========================================================================
// Persistent form of the same update.  Work is a list of items; an item is a
// 128-row block of P (kept in shared memory, both halves, all of K = 128:
// 128 KB) and a run of `nq` consecutive 128-column tiles whose Q rows and C
// tiles follow one another:
//   tile t of item i:  Q rows [qrow0 + 128 t, +128),  C = C0 + 128 t (columns).
// Items are cut into units of at most `chunk` tiles; one CTA per SM walks the
// units.  Warp 0 (lane 0) loads P once per unit and streams the Q k-blocks
// through a 2-stage ring; warp 1 (lane 0) issues the 3 x 4 MMAs per k-block
// into one of two TMEM accumulators; warps 2..9 drain the other accumulator
// into C (two warps per TMEM lane quarter, 64 columns each), so the C
// read-modify-write of one tile overlaps the MMAs of the next.
//
// Decoder: __host__ __device__ int num_items() const;
//          __host__ __device__ int item_nq(int i) const;
//          __device__ PgItem item(int i) const;
// ===========================================================================
struct PgItem {
  float* C0;
  int64_t ldc;
  int prow, pkx;    // P block: rows [prow, prow+128), columns [pkx, pkx+128)
  int qrow0, qkx;   // Q rows of tile t start at qrow0 + 128 t; columns [qkx, qkx+128)
  int nq;           // tiles in the item
  int mext;         // valid rows of its C tiles
  int cext_last;    // valid columns of its last C tile (the others have 128)
};

constexpr int kPg2Threads = 320;
constexpr int kPg2QStages = 2;
constexpr int kPg2PBytes = kPgKBlocks * 2 * kPgTileBytes;   // 128 KB
constexpr int kPg2QStageBytes = 2 * kPgTileBytes;           // one k-block of Q_hi, Q_lo
constexpr size_t kPg2SmemBytes =
    (size_t)kPg2PBytes + kPg2QStages * kPg2QStageBytes + 1024 + 256;
constexpr uint32_t kPg2TmemCols = 256;

template <class Decoder>
__device__ __forceinline__ void pg2_unit(const Decoder& dec, int u, int chunk, int& item, int& qb,
                                         int& qe) {
  int i = 0;
  while (true) {
    const int nq = dec.item_nq(i);
    const int nu = (nq + chunk - 1) / chunk;
    if (u < nu) {
      item = i;
      qb = u * chunk;
      qe = min(nq, qb + chunk);
      return;
    }
    u -= nu;
    ++i;
  }
}

template <class Decoder>
__global__ void __launch_bounds__(kPg2Threads, 1)
    panel_gemm2_kernel(const __grid_constant__ CUtensorMap mPh,
                       const __grid_constant__ CUtensorMap mPl,
                       const __grid_constant__ CUtensorMap mQh,
                       const __grid_constant__ CUtensorMap mQl, const Decoder dec, int chunk,
                       int units, int32_t* info, int32_t timeout_code,
                       const int32_t* skip_if_nonzero) {
  if (skip_if_nonzero && *(volatile const int32_t*)skip_if_nonzero != 0) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sP = smem;
  uint8_t* sQ = smem + kPg2PBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sQ + kPg2QStages * kPg2QStageBytes);
  uint64_t* pfull = bars;
  uint64_t* pempty = bars + 1;
  uint64_t* qfull = bars + 2;                 // [kPg2QStages]
  uint64_t* qempty = qfull + kPg2QStages;     // [kPg2QStages]
  uint64_t* tfull = qempty + kPg2QStages;     // [2]
  uint64_t* tempty = tfull + 2;               // [2]
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  constexpr uint64_t kLimit = (uint64_t)kGridWaitLimitNs;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    ptx::mbar_init(pfull, 1);
    ptx::mbar_init(pempty, 1);
    for (int s = 0; s < kPg2QStages; ++s) {
      ptx::mbar_init(&qfull[s], 1);
      ptx::mbar_init(&qempty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(&tfull[a], 1);
      ptx::mbar_init(&tempty[a], 256);
    }
    ptx::mbar_init(drain, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, kPg2TmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ TMA producer
      ptx::prefetch_tmap(&mPh);
      ptx::prefetch_tmap(&mPl);
      ptx::prefetch_tmap(&mQh);
      ptx::prefetch_tmap(&mQl);
      int qst = 0;
      uint32_t qph = 0;
      int ku = 0;
      bool ok = true;
      int p_issued = 0;
      int q_last_parity[kPg2QStages] = {-1, -1};
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++ku) {
        int it, qb, qe;
        pg2_unit(dec, u, chunk, it, qb, qe);
        const PgItem I = dec.item(it);
        if (ku > 0 &&
            !ptx::mbar_wait_bounded(pempty, (uint32_t)((ku - 1) & 1), abort_flag, kLimit)) {
          ok = false;
          break;
        }
        ptx::mbar_arrive_expect_tx(pfull, kPg2PBytes);
        for (int kb = 0; kb < kPgKBlocks; ++kb) {
          ptx::tma_load_2d(sP + kb * 2 * kPgTileBytes, &mPh, pfull, I.pkx + 32 * kb, I.prow);
          ptx::tma_load_2d(sP + kb * 2 * kPgTileBytes + kPgTileBytes, &mPl, pfull,
                           I.pkx + 32 * kb, I.prow);
        }
        p_issued = ku + 1;
        for (int q = qb; q < qe && ok; ++q) {
          for (int kb = 0; kb < kPgKBlocks; ++kb) {
            if (!ptx::mbar_wait_bounded(&qempty[qst], qph ^ 1, abort_flag, kLimit)) {
              ok = false;
              break;
            }
            uint8_t* sb = sQ + qst * kPg2QStageBytes;
            ptx::mbar_arrive_expect_tx(&qfull[qst], kPg2QStageBytes);
            ptx::tma_load_2d(sb, &mQh, &qfull[qst], I.qkx + 32 * kb, I.qrow0 + 128 * q);
            ptx::tma_load_2d(sb + kPgTileBytes, &mQl, &qfull[qst], I.qkx + 32 * kb,
                             I.qrow0 + 128 * q);
            q_last_parity[qst] = (int)qph;
            if (++qst == kPg2QStages) {
              qst = 0;
              qph ^= 1;
            }
          }
        }
      }
      if (!ok || *abort_flag) {
        pg_abort(abort_flag, info, timeout_code);
        volatile int never = 0;  // wait (bounded) for this CTA's own copies in flight
        if (p_issued > 0)
          ptx::mbar_wait_bounded(pfull, (uint32_t)((p_issued - 1) & 1), &never, kLimit);
        for (int s = 0; s < kPg2QStages; ++s)
          if (q_last_parity[s] >= 0)
            ptx::mbar_wait_bounded(&qfull[s], (uint32_t)q_last_parity[s], &never, kLimit);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc = ptx::idesc_tf32_f32(128, 128);
      int qst = 0;
      uint32_t qph = 0;
      int acc = 0;
      uint32_t aph = 0;
      int ku = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++ku) {
        int it, qb, qe;
        pg2_unit(dec, u, chunk, it, qb, qe);
        if (!ptx::mbar_wait_bounded(pfull, (uint32_t)(ku & 1), abort_flag, kLimit)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        for (int q = qb; q < qe && ok; ++q) {
          if (!ptx::mbar_wait_bounded(&tempty[acc], aph ^ 1, abort_flag, kLimit)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t d = tmem_base + (uint32_t)(acc * 128);
          for (int kb = 0; kb < kPgKBlocks; ++kb) {
            if (!ptx::mbar_wait_bounded(&qfull[qst], qph, abort_flag, kLimit)) {
              ok = false;
              break;
            }
            ptx::tc_fence_after();
            const uint32_t pb = ptx::smem_u32(sP + kb * 2 * kPgTileBytes);
            const uint32_t qbase = ptx::smem_u32(sQ + qst * kPg2QStageBytes);
            const uint64_t ph = ptx::smem_desc_sw128(pb);
            const uint64_t pl = ptx::smem_desc_sw128(pb + kPgTileBytes);
            const uint64_t qh = ptx::smem_desc_sw128(qbase);
            const uint64_t ql = ptx::smem_desc_sw128(qbase + kPgTileBytes);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              ptx::mma_tf32(d, ph + 2 * k, qh + 2 * k, idesc, (kb > 0 || k > 0) ? 1u : 0u);
              ptx::mma_tf32(d, ph + 2 * k, ql + 2 * k, idesc, 1u);
              ptx::mma_tf32(d, pl + 2 * k, qh + 2 * k, idesc, 1u);
            }
            ptx::mma_commit(&qempty[qst]);
            if (++qst == kPg2QStages) {
              qst = 0;
              qph ^= 1;
            }
          }
          if (!ok) break;
          ptx::mma_commit(&tfull[acc]);
          acc ^= 1;
          if (acc == 0) aph ^= 1;
        }
        if (!ok) break;
        ptx::mma_commit(pempty);  // P may be reloaded once these MMAs are done
      }
      if (ok && ku > 0) {
        // the last commit's arrive must land before the CTA can exit
        volatile int never = 0;
        ptx::mbar_wait_bounded(pempty, (uint32_t)((ku - 1) & 1), &never, kLimit);
      }
      if (!ok || *abort_flag) {
        pg_abort(abort_flag, info, timeout_code);
        ptx::mma_commit(drain);
        volatile int never = 0;
        ptx::mbar_wait_bounded(drain, 0, &never, kLimit);
      }
    }
  } else {
    // -------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;  // columns [64 half, 64 half + 64)
    int acc = 0;
    uint32_t aph = 0;
    bool stop = false;
    for (int u = blockIdx.x; u < units && !stop; u += gridDim.x) {
      int it, qb, qe;
      pg2_unit(dec, u, chunk, it, qb, qe);
      const PgItem I = dec.item(it);
      for (int q = qb; q < qe; ++q) {
        const bool ready = ptx::mbar_wait_bounded(&tfull[acc], aph, abort_flag, kLimit);
        __syncwarp();
        if (!__all_sync(0xffffffffu, ready && !*abort_flag)) {
          if (!ready) pg_abort(abort_flag, info, timeout_code);
          stop = true;
          break;
        }
        ptx::tc_fence_after();
        const int row = quarter * 32 + lane;
        float* crow = I.C0 + (int64_t)row * I.ldc + (int64_t)q * 128;
        const int cext = (q == I.nq - 1) ? I.cext_last : 128;
        const bool vec = cext == 128 && (I.ldc % 4) == 0 &&
                         (reinterpret_cast<uintptr_t>(I.C0) % 16) == 0;
#pragma unroll 1
        for (int ch = 0; ch < 2; ++ch) {
          const int col0 = half * 64 + ch * 32;
          uint32_t v[32];
          ptx::tmem_ld_32x32b_x32(
              tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * 128 + col0), v);
          ptx::tmem_ld_wait();
          if (row < I.mext) {
            if (vec) {
              float4* c4 = reinterpret_cast<float4*>(crow + col0);
              float4 cv[8];
#pragma unroll
              for (int j = 0; j < 8; ++j) cv[j] = c4[j];
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                cv[j].x -= __uint_as_float(v[4 * j + 0]);
                cv[j].y -= __uint_as_float(v[4 * j + 1]);
                cv[j].z -= __uint_as_float(v[4 * j + 2]);
                cv[j].w -= __uint_as_float(v[4 * j + 3]);
                c4[j] = cv[j];
              }
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (col0 + j < cext) crow[col0 + j] -= __uint_as_float(v[j]);
            }
          }
        }
        ptx::tc_fence_before();
        ptx::mbar_arrive(&tempty[acc]);
        acc ^= 1;
        if (acc == 0) aph ^= 1;
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, kPg2TmemCols);
  }
}

// Host side: the chunk size (tiles per unit) that minimises the estimated
// time, counting one P load as one tile of work, and the resulting unit count.
template <class Decoder>
inline void pg2_plan(const Decoder& dec, int sms, int& chunk, int& units) {
  int total = 0, maxnq = 1;
  for (int i = 0; i < dec.num_items(); ++i) {
    total += dec.item_nq(i);
    maxnq = std::max(maxnq, dec.item_nq(i));
  }
  double best = 1e30;
  chunk = 1;
  units = 0;
  for (int c = 1; c <= maxnq; ++c) {
    int nu = 0;
    for (int i = 0; i < dec.num_items(); ++i) nu += (dec.item_nq(i) + c - 1) / c;
    const int waves = (nu + sms - 1) / sms;
    const double cost = (double)waves * (c + 1);
    if (cost < best - 1e-9) {
      best = cost;
      chunk = c;
      units = nu;
    }
  }
  (void)total;
}

}  // namespace gptq
