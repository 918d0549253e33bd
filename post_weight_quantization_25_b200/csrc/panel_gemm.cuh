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

}  // namespace gptq
