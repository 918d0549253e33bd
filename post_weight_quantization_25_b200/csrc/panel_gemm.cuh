// fp32-accurate rank-128 updates on the tcgen05 tensor cores:
//     C[m][c] -= sum_{t < 128} P[m][t] * Q[c][t]
// over a list of 128 x 128 tiles of C, by a persistent kernel.
//
// The pages' method needs full fp32 accuracy here (page "GPTQ, with the code
// open", section "Paper vs. code": TF32 is switched off because the Cholesky
// chain needs full 32-bit precision).  Each operand therefore arrives split
// in two fp32 arrays, hi = TF32(x) (round to nearest) and lo = x - hi (exact),
// and the product is taken as  P_hi Q_hi + P_hi Q_lo + P_lo Q_hi  with
// tcgen05.mma kind::tf32 (fp32 accumulation in TMEM).  The dropped P_lo Q_lo
// term and the TF32 truncation of lo are below 2^-21 relative per product.
//
// Work is a list of items.  An item is a 128-row block of P (kept in shared
// memory, both halves, all of K = 128: 128 KB) and a run of `nq` consecutive
// 128-column tiles whose Q rows and C tiles follow one another:
//   tile t of item i:  Q rows [qrow0 + 128 t, +128),  C columns + 128 t.
// Items are cut into units of at most `chunk` tiles; one CTA per SM walks the
// units.  Warp 0 (lane 0) loads P once per unit and streams the Q k-blocks
// through a 2-stage TMA ring; warp 1 (lane 0) issues the 3 x 4 MMAs per
// k-block into one of two TMEM accumulators; warps 2..9 drain the other
// accumulator (two warps per TMEM lane quarter, 64 columns each), so the C
// update of one tile overlaps the MMAs of the next.
//
// The C update (kReduce = true) is a TMA bulk reduce-add: each epilogue
// warp writes -acc for a 32 x 32 piece into its own shared-memory staging
// buffer (128-byte swizzle) and one lane issues cp.reduce.async.bulk.tensor
// .add into C, so C is never read into the SM and the adds happen in L2
// (fp32, round to nearest; each element gets exactly one add per launch).
// It needs C's row stride to be a multiple of 16 bytes; otherwise
// (kReduce = false) the epilogue reads, subtracts and writes C itself.
// No multicast anywhere.  Every wait is bounded (limit_ns): on a timeout the
// kernel writes `timeout_code` to `info` (if given), lets its own copies and
// MMAs finish, frees TMEM and exits.  `gate` (test hook, normally null): the
// producer first waits for *gate != 0, within the same limit.
//
// Decoder: __host__ __device__ int num_items() const;
//          __host__ __device__ int item_nq(int i) const;
//          __device__ PgItem item(int i) const;
#pragma once
#include <algorithm>
#include <cstdint>

#include "gptq_internal.cuh"
#include "sm100_ptx.cuh"

namespace gptq {

constexpr int kPgKBlocks = kBlock / 32;                 // 4 k-blocks of 32 fp32
constexpr int kPgTileBytes = 128 * 32 * 4;              // one 128 x 32 fp32 tile

struct PgItem {
  float* C0;        // (read-modify-write epilogue) C origin of tile 0
  int64_t ldc;
  int cmap;         // (reduce epilogue) which C tensor map: 0 or 1
  int cx0, cy0;     // (reduce epilogue) C origin of tile 0: column, row
  int prow, pkx;    // P block: rows [prow, prow+128), columns [pkx, pkx+128)
  int qrow0, qkx;   // Q rows of tile t start at qrow0 + 128 t; columns [qkx, qkx+128)
  int nq;           // tiles in the item
  int mext;         // valid rows of its C tiles
  int cext_last;    // valid columns of its last C tile (the others have 128)
  int nkb;          // (stream_gemm_kernel) k-blocks of 32: K = 32 nkb
};

constexpr int kPg2Threads = 320;
constexpr int kPg2QStages = 2;
constexpr int kPg2PBytes = kPgKBlocks * 2 * kPgTileBytes;   // 128 KB
constexpr int kPg2QStageBytes = 2 * kPgTileBytes;           // one k-block of Q_hi, Q_lo
constexpr int kPg2StageOut = 32 * 32 * 4;                   // one warp's 32 x 32 C piece
__host__ __device__ constexpr size_t pg2_smem_bytes(bool reduce) {
  return (size_t)kPg2PBytes + kPg2QStages * kPg2QStageBytes +
         (reduce ? 8 * kPg2StageOut : 0) + 1024 + 256;
}
constexpr uint32_t kPg2TmemCols = 256;

__device__ __forceinline__ void pg_abort(volatile int* abort_flag, int32_t* info,
                                         int32_t code) {
  *abort_flag = 1;
  if (info) atomicExch(info, code);
}

// One 32 x 32 piece of a tile's epilogue, by one of the eight epilogue warps:
// rows [32 quarter, +32) (this lane: row 32 quarter + lane) and columns
// [col0, +32) of C tile q of item I take -v (TMA reduce-add from the warp's
// staging buffer, or a read-modify-write of C).
template <bool kReduce>
__device__ __forceinline__ void pg_emit_piece(const PgItem& I, int q, int quarter, int col0,
                                              int lane, float* stage, const float (&v)[32],
                                              const CUtensorMap& mC0, const CUtensorMap& mC1) {
  const int row = quarter * 32 + lane;
  const int cext = (q == I.nq - 1) ? I.cext_last : 128;
  if (kReduce) {
    // pieces wholly past C's edge are skipped (no reduce starts outside C)
    if (quarter * 32 >= I.mext || col0 >= cext) return;
    // -v for rows [32 quarter, +32) x columns [col0, +32) of the tile,
    // 128-byte swizzle: 16-byte chunk c of row r sits at chunk c ^ (r & 7)
    if (lane == 0) ptx::bulk_wait_read0();  // the previous piece left the buffer
    __syncwarp();
    float4* srow = reinterpret_cast<float4*>(stage + lane * 32);
#pragma unroll
    for (int c4 = 0; c4 < 8; ++c4)
      srow[c4 ^ (lane & 7)] =
          make_float4(-v[4 * c4 + 0], -v[4 * c4 + 1], -v[4 * c4 + 2], -v[4 * c4 + 3]);
    ptx::fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      ptx::tma_reduce_add_2d(I.cmap ? &mC1 : &mC0, stage, I.cx0 + 128 * q + col0,
                             I.cy0 + quarter * 32);
      ptx::bulk_commit();
    }
  } else if (row < I.mext) {
    float* crow = I.C0 + (int64_t)row * I.ldc + (int64_t)q * 128;
    const bool vec =
        cext == 128 && (I.ldc % 4) == 0 && (reinterpret_cast<uintptr_t>(I.C0) % 16) == 0;
    if (vec) {
      float4* c4 = reinterpret_cast<float4*>(crow + col0);
      float4 cv[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) cv[j] = c4[j];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        cv[j].x -= v[4 * j + 0];
        cv[j].y -= v[4 * j + 1];
        cv[j].z -= v[4 * j + 2];
        cv[j].w -= v[4 * j + 3];
        c4[j] = cv[j];
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (col0 + j < cext) crow[col0 + j] -= v[j];
    }
  }
}

// 32 accumulator columns of this warp's TMEM lane quarter as floats.
__device__ __forceinline__ void pg_load_piece(uint32_t acc_tmem, int quarter, int col0,
                                              float (&v)[32]) {
  uint32_t u[32];
  ptx::tmem_ld_32x32b_x32(acc_tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)col0, u);
  ptx::tmem_ld_wait();
#pragma unroll
  for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(u[j]);
}

// One tile's epilogue straight from TMEM: accumulator columns [64 half, +64)
// of the tile at TMEM column acc_tmem.
template <bool kReduce>
__device__ __forceinline__ void pg_tile_epilogue(const PgItem& I, int q, uint32_t acc_tmem,
                                                 int quarter, int half, int lane, float* stage,
                                                 const CUtensorMap& mC0, const CUtensorMap& mC1) {
#pragma unroll 1
  for (int ch = 0; ch < 2; ++ch) {
    const int col0 = half * 64 + ch * 32;
    float v[32];
    pg_load_piece(acc_tmem, quarter, col0, v);
    pg_emit_piece<kReduce>(I, q, quarter, col0, lane, stage, v, mC0, mC1);
  }
}

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

template <class Decoder, bool kReduce>
__global__ void __launch_bounds__(kPg2Threads, 1)
    panel_gemm2_kernel(const __grid_constant__ CUtensorMap mPh,
                       const __grid_constant__ CUtensorMap mPl,
                       const __grid_constant__ CUtensorMap mQh,
                       const __grid_constant__ CUtensorMap mQl,
                       const __grid_constant__ CUtensorMap mC0,
                       const __grid_constant__ CUtensorMap mC1, const Decoder dec, int chunk,
                       int units, int32_t* info, int32_t timeout_code,
                       const int32_t* skip_if_nonzero, const int32_t* gate,
                       uint64_t limit_ns) {
  if (skip_if_nonzero && *(volatile const int32_t*)skip_if_nonzero != 0) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sP = smem;
  uint8_t* sQ = smem + kPg2PBytes;
  uint8_t* sOut = sQ + kPg2QStages * kPg2QStageBytes;         // [8][32 x 32 fp32] if kReduce
  uint64_t* bars = reinterpret_cast<uint64_t*>(sOut + (kReduce ? 8 * kPg2StageOut : 0));
  uint64_t* pfull = bars;
  uint64_t* pempty = bars + 1;
  uint64_t* qfull = bars + 2;                 // [kPg2QStages]
  uint64_t* qempty = qfull + kPg2QStages;     // [kPg2QStages]
  uint64_t* tfull = qempty + kPg2QStages;     // [2]
  uint64_t* tempty = tfull + 2;               // [2]
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  constexpr uint64_t kDrainLimit = (uint64_t)kGridWaitLimitNs;  // waits for own work in flight
  const uint64_t kLimit = limit_ns;                              // every pipeline wait

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
      ok = ptx::gate_wait_bounded(gate, kLimit);
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
          ptx::mbar_wait_bounded(pfull, (uint32_t)((p_issued - 1) & 1), &never, kDrainLimit);
        for (int s = 0; s < kPg2QStages; ++s)
          if (q_last_parity[s] >= 0)
            ptx::mbar_wait_bounded(&qfull[s], (uint32_t)q_last_parity[s], &never, kDrainLimit);
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
        ptx::mbar_wait_bounded(pempty, (uint32_t)((ku - 1) & 1), &never, kDrainLimit);
      }
      if (!ok || *abort_flag) {
        pg_abort(abort_flag, info, timeout_code);
        ptx::mma_commit(drain);
        volatile int never = 0;
        ptx::mbar_wait_bounded(drain, 0, &never, kDrainLimit);
      }
    }
  } else {
    // -------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;  // columns [64 half, 64 half + 64)
    float* stage = reinterpret_cast<float*>(sOut + (warp - 2) * kPg2StageOut);
    if (kReduce && lane == 0) {
      ptx::prefetch_tmap(&mC0);
      ptx::prefetch_tmap(&mC1);
    }
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
        pg_tile_epilogue<kReduce>(I, q, tmem_base + (uint32_t)(acc * 128), quarter, half, lane,
                                  stage, mC0, mC1);
        ptx::tc_fence_before();
        ptx::mbar_arrive(&tempty[acc]);
        acc ^= 1;
        if (acc == 0) aph ^= 1;
      }
    }
    // every reduce this warp issued has completed before the CTA exits
    if (kReduce && lane == 0) ptx::bulk_wait_all0();
    __syncwarp();
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, kPg2TmemCols);
  }
}

// ===========================================================================
// The same fp32-accurate update for long K:  C -= P Q^T  with K = 32 nkb per
// item (nkb a multiple of 4), both operands streamed.  A unit is one
// 128 x 128 C tile; for each of its k-blocks of 32 the producer loads the P
// and Q k-blocks (hi and lo, 64 KB) into a 3-stage TMA ring and the MMA warp
// issues the three TF32 products (12 MMAs).  The tensor cores' fp32 sum in
// TMEM loses accuracy with the length of the chain of MMAs it accumulates,
// so every 128 of K (48 MMAs, as in panel_gemm2_kernel) starts a fresh sum in
// the other of two TMEM accumulators; the epilogue warps add the pieces in
// registers with IEEE adds and subtract the tile from C once at the end (as
// panel_gemm2_kernel does), while the MMAs of the next piece run.  C is read
// and written once per launch whatever K is, which is what deferring many
// rank-128 updates into one buys.
// ===========================================================================
constexpr int kSgStages = 3;
constexpr int kSgStageBytes = 4 * kPgTileBytes;            // P hi, P lo, Q hi, Q lo
constexpr int kSgPieceKb = kBlock / 32;                    // k-blocks per fresh TMEM sum
__host__ __device__ constexpr size_t sg_smem_bytes(bool reduce) {
  return (size_t)kSgStages * kSgStageBytes + (reduce ? 8 * kPg2StageOut : 0) + 1024 + 256;
}

template <class Decoder, bool kReduce>
__global__ void __launch_bounds__(kPg2Threads, 1)
    stream_gemm_kernel(const __grid_constant__ CUtensorMap mPh,
                       const __grid_constant__ CUtensorMap mPl,
                       const __grid_constant__ CUtensorMap mQh,
                       const __grid_constant__ CUtensorMap mQl,
                       const __grid_constant__ CUtensorMap mC0,
                       const __grid_constant__ CUtensorMap mC1, const Decoder dec, int units,
                       int32_t* info, int32_t timeout_code, const int32_t* skip_if_nonzero,
                       const int32_t* gate, uint64_t limit_ns) {
  if (skip_if_nonzero && *(volatile const int32_t*)skip_if_nonzero != 0) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sS = smem;                                            // [kSgStages] stages
  uint8_t* sOut = sS + kSgStages * kSgStageBytes;                // [8][32 x 32 fp32] if kReduce
  uint64_t* bars = reinterpret_cast<uint64_t*>(sOut + (kReduce ? 8 * kPg2StageOut : 0));
  uint64_t* full = bars;                       // [kSgStages]
  uint64_t* empty = full + kSgStages;          // [kSgStages]
  uint64_t* tfull = empty + kSgStages;         // [2]
  uint64_t* tempty = tfull + 2;                // [2]
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  constexpr uint64_t kDrainLimit = (uint64_t)kGridWaitLimitNs;
  const uint64_t kLimit = limit_ns;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int st = 0; st < kSgStages; ++st) {
      ptx::mbar_init(&full[st], 1);
      ptx::mbar_init(&empty[st], 1);
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
      int st = 0;
      uint32_t ph = 0;
      int last_parity[kSgStages];
      for (int i = 0; i < kSgStages; ++i) last_parity[i] = -1;
      bool ok = ptx::gate_wait_bounded(gate, kLimit);
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        int it, q, qe;
        pg2_unit(dec, u, 1, it, q, qe);
        const PgItem I = dec.item(it);
        for (int kb = 0; kb < I.nkb; ++kb) {
          if (!ptx::mbar_wait_bounded(&empty[st], ph ^ 1, abort_flag, kLimit)) {
            ok = false;
            break;
          }
          uint8_t* sb = sS + st * kSgStageBytes;
          ptx::mbar_arrive_expect_tx(&full[st], kSgStageBytes);
          ptx::tma_load_2d(sb, &mPh, &full[st], I.pkx + 32 * kb, I.prow);
          ptx::tma_load_2d(sb + kPgTileBytes, &mPl, &full[st], I.pkx + 32 * kb, I.prow);
          ptx::tma_load_2d(sb + 2 * kPgTileBytes, &mQh, &full[st], I.qkx + 32 * kb,
                           I.qrow0 + 128 * q);
          ptx::tma_load_2d(sb + 3 * kPgTileBytes, &mQl, &full[st], I.qkx + 32 * kb,
                           I.qrow0 + 128 * q);
          last_parity[st] = (int)ph;
          if (++st == kSgStages) {
            st = 0;
            ph ^= 1;
          }
        }
      }
      if (!ok || *abort_flag) {
        pg_abort(abort_flag, info, timeout_code);
        volatile int never = 0;  // wait (bounded) for this CTA's own copies in flight
        for (int i = 0; i < kSgStages; ++i)
          if (last_parity[i] >= 0)
            ptx::mbar_wait_bounded(&full[i], (uint32_t)last_parity[i], &never, kDrainLimit);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc = ptx::idesc_tf32_f32(128, 128);
      int st = 0;
      uint32_t ph = 0;
      int acc = 0;
      uint32_t aph = 0;
      bool ok = true;
      int issued = 0;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        int it, q, qe;
        pg2_unit(dec, u, 1, it, q, qe);
        const int nkb = dec.item(it).nkb;
        for (int kb0 = 0; kb0 < nkb && ok; kb0 += kSgPieceKb) {
          // a fresh TMEM sum for the piece of k-blocks [kb0, kb0 + kSgPieceKb)
          if (!ptx::mbar_wait_bounded(&tempty[acc], aph ^ 1, abort_flag, kLimit)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t d = tmem_base + (uint32_t)(acc * 128);
          for (int kb = kb0; kb < kb0 + kSgPieceKb; ++kb) {
            if (!ptx::mbar_wait_bounded(&full[st], ph, abort_flag, kLimit)) {
              ok = false;
              break;
            }
            ptx::tc_fence_after();
            const uint32_t base = ptx::smem_u32(sS + st * kSgStageBytes);
            const uint64_t phd = ptx::smem_desc_sw128(base);
            const uint64_t pld = ptx::smem_desc_sw128(base + kPgTileBytes);
            const uint64_t qhd = ptx::smem_desc_sw128(base + 2 * kPgTileBytes);
            const uint64_t qld = ptx::smem_desc_sw128(base + 3 * kPgTileBytes);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              ptx::mma_tf32(d, phd + 2 * k, qhd + 2 * k, idesc,
                            (kb > kb0 || k > 0) ? 1u : 0u);
              ptx::mma_tf32(d, phd + 2 * k, qld + 2 * k, idesc, 1u);
              ptx::mma_tf32(d, pld + 2 * k, qhd + 2 * k, idesc, 1u);
            }
            ptx::mma_commit(&empty[st]);
            ++issued;
            if (++st == kSgStages) {
              st = 0;
              ph ^= 1;
            }
          }
          if (!ok) break;
          ptx::mma_commit(&tfull[acc]);
          acc ^= 1;
          if (acc == 0) aph ^= 1;
        }
      }
      if (!ok || *abort_flag) pg_abort(abort_flag, info, timeout_code);
      // every MMA issued above is complete before the CTA tears down (bounded)
      if (issued > 0 || !ok) {
        ptx::mma_commit(drain);
        volatile int never = 0;
        ptx::mbar_wait_bounded(drain, 0, &never, kDrainLimit);
      }
    }
  } else {
    // -------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;  // columns [64 half, 64 half + 64)
    float* stage = reinterpret_cast<float*>(sOut + (warp - 2) * kPg2StageOut);
    if (kReduce && lane == 0) {
      ptx::prefetch_tmap(&mC0);
      ptx::prefetch_tmap(&mC1);
    }
    int acc = 0;
    uint32_t aph = 0;
    bool stop = false;
    for (int u = blockIdx.x; u < units && !stop; u += gridDim.x) {
      int it, q, qe;
      pg2_unit(dec, u, 1, it, q, qe);
      const PgItem I = dec.item(it);
      float sum[2][32];
#pragma unroll
      for (int ch = 0; ch < 2; ++ch)
#pragma unroll
        for (int j = 0; j < 32; ++j) sum[ch][j] = 0.f;
      for (int kb0 = 0; kb0 < I.nkb; kb0 += kSgPieceKb) {
        const bool ready = ptx::mbar_wait_bounded(&tfull[acc], aph, abort_flag, kLimit);
        __syncwarp();
        if (!__all_sync(0xffffffffu, ready && !*abort_flag)) {
          if (!ready) pg_abort(abort_flag, info, timeout_code);
          stop = true;
          break;
        }
        ptx::tc_fence_after();
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          float v[32];
          pg_load_piece(tmem_base + (uint32_t)(acc * 128), quarter, half * 64 + ch * 32, v);
#pragma unroll
          for (int j = 0; j < 32; ++j) sum[ch][j] += v[j];
        }
        ptx::tc_fence_before();
        ptx::mbar_arrive(&tempty[acc]);
        acc ^= 1;
        if (acc == 0) aph ^= 1;
      }
      if (stop) break;
#pragma unroll
      for (int ch = 0; ch < 2; ++ch)
        pg_emit_piece<kReduce>(I, q, quarter, half * 64 + ch * 32, lane, stage, sum[ch], mC0,
                               mC1);
    }
    // every reduce this warp issued has completed before the CTA exits
    if (kReduce && lane == 0) ptx::bulk_wait_all0();
    __syncwarp();
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, kPg2TmemCols);
  }
}

// Units (tiles) of a stream_gemm_kernel launch.
template <class Decoder>
inline int sg_units(const Decoder& dec) {
  int nu = 0;
  for (int i = 0; i < dec.num_items(); ++i) nu += dec.item_nq(i);
  return nu;
}

// hi / lo split of one value for the kernel above.
__device__ __forceinline__ void tf32_split(float x, float& hi, float& lo) {
  hi = ptx::tf32_hi(x);
  lo = x - hi;
}

// Host side: the chunk size (tiles per unit) that minimises the estimated
// time, counting one P load as one tile of work, and the resulting unit count.
template <class Decoder>
inline void pg2_plan(const Decoder& dec, int sms, int& chunk, int& units) {
  int maxnq = 1;
  for (int i = 0; i < dec.num_items(); ++i) maxnq = std::max(maxnq, dec.item_nq(i));
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
}

}  // namespace gptq
