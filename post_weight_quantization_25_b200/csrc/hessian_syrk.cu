// Calibration Hessian  H += alpha * X X^T  on the tcgen05 tensor cores.
//
// Page "GPTQ, with the code open", section "Measuring damage where it
// matters": H = 2 X X^T prices the layer-output damage exactly; section
// "Paper vs. code": H is accumulated over calibration batches.
//
// Design (sm_100a):
//  * X is n features x N tokens, token-contiguous, so both GEMM operands are
//    K-major rows of X.  Only tiles that touch the upper triangle are computed
//    (128 x 256 output tiles, I <= 2J + 1); the lower triangle is mirrored
//    afterwards.
//  * Work unit = (tile, chunk of tokens).  The number of token chunks is
//    picked so that the units fill whole waves of the SMs; a persistent grid
//    of one CTA per SM walks the units in token-chunk-major order, so the
//    CTAs that run together read the same slab of X and it is served from L2.
//  * Per CTA: warp 0 issues TMA loads (128-byte swizzle, 4-stage ring of
//    128x64 + 256x64 bf16 tiles), warp 1 issues tcgen05.mma kind::f16
//    (M=128, N=256, K=16; fp32 accumulators in TMEM, two 256-column buffers
//    so the epilogue of one piece overlaps the MMAs of the next), warps 2-9
//    drain TMEM with tcgen05.ld.
//  * Accuracy: the fp32 sum the tensor cores keep in TMEM loses more than
//    IEEE round-to-nearest would over a long chain of MMAs; measured on this
//    kernel, the relative error of H grew in proportion to the number of
//    MMAs accumulated into one TMEM tile (about 1.2e-7 per K = 16 MMA).  So
//    a unit's token range is cut into pieces of kSubKb k-blocks (1024
//    tokens, 64 MMAs); each piece starts a fresh TMEM sum, and the epilogue
//    adds the pieces into an fp32 register copy of the tile with ordinary
//    IEEE adds.  At the end of the unit it adds alpha * tile into H, masked
//    to the upper triangle (the split-K reduction).
//  * Ordered split-K reduction: the token chunks of a tile are added into H
//    in chunk order.  A per-tile counter in global memory (a turnstile) holds
//    how many chunks have been added; the unit of chunk c waits (acquire)
//    until it reads c, adds its tile by reductions in L2 (red.add, which
//    return nothing, so the epilogue does not wait on L2 round trips), makes
//    them visible (fence) and publishes c + 1 (release).  Only one chunk adds
//    into a tile at a time, so every element takes its adds in chunk order
//    and H is the same bit for bit from run to run.  Units are walked in chunk-major order by a
//    persistent grid whose CTAs are all resident, so chunk c - 1 of a tile is
//    always taken before chunk c and the wait ends.
//  * No multicast loads.  Every wait is bounded: on timeout the CTA stops,
//    writes GPTQ_ERR_TIMEOUT to `info`, waits for its own copies and MMAs,
//    frees TMEM and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <mutex>

#include "gptq_internal.cuh"
#include "sm100_ptx.cuh"

namespace gptq {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int NUM_THREADS = 320;          // TMA warp, MMA warp, 8 epilogue warps
constexpr int kSubKb = 16;                // k-blocks per fresh TMEM sum (1024 tokens)
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr size_t SMEM_BYTES = (size_t)STAGES * STAGE_BYTES + 1024 + 256;
constexpr uint64_t WAIT_LIMIT_NS = (uint64_t)kGridWaitLimitNs;

struct SyrkArgs {
  float* H;
  int n;
  float alpha;
  int nkb;          // k-blocks of BK tokens
  int kb_per_unit;  // k-blocks per unit (last chunk may be shorter)
  int ntiles;       // tiles touching the upper triangle
  int nI;           // row blocks of BM
  int units;        // ntiles * token chunks
  int vec4;         // H row starts are 16-byte aligned
  int32_t* info;
  uint32_t* flags;  // [ntiles] chunks of each tile added so far
  const int32_t* gate;  // test gate of the bounded waits (null: none)
  uint64_t limit_ns;    // limit of every pipeline wait
};

// Tile t of the J-major enumeration: column block J holds row blocks 0..min(nI, 2J+2)-1.
__device__ __forceinline__ void decode_tile(int t, int nI, int& I, int& J) {
  J = 0;
  while (true) {
    const int c = min(nI, 2 * J + 2);
    if (t < c) {
      I = t;
      return;
    }
    t -= c;
    ++J;
  }
}

__device__ __forceinline__ void raise_abort(volatile int* abort_flag, int32_t* info) {
  *abort_flag = 1;
  if (info) atomicExch(info, (int32_t)GPTQ_ERR_TIMEOUT);
}

constexpr int kEpiBar = 1;                 // named barrier of the 8 epilogue warps
constexpr int kEpiThreads = NUM_THREADS - 64;

// The ordered add of one unit's tile (this thread's row, 128 columns from
// cbase) into H: wait for the turnstile to show `chunk`, add, publish
// chunk + 1.  Called by all epilogue threads together; returns false (for
// all of them) if the wait gave up.
__device__ __forceinline__ bool ordered_add(float* H, int n, int row, int cbase, float alpha,
                                            int vec4, const float (&tile)[128], uint32_t* flag,
                                            uint32_t chunk, volatile int* abort_flag,
                                            int32_t* info, uint64_t limit_ns, bool waiter) {
  bool ok = true;
  if (waiter) {
    ok = ptx::flag_wait_bounded(flag, chunk, abort_flag, limit_ns);
    if (!ok) raise_abort(abort_flag, info);
  }
  ok = ptx::named_bar_and(kEpiBar, kEpiThreads, ok);
  if (!ok) return false;
  if (row < n) {
    // reductions in L2 (no value comes back, so nothing waits on a round
    // trip); the turnstile lets one unit at a time add into the tile, so each
    // element still takes its chunks' adds one after another in chunk order,
    // each an IEEE round-to-nearest fp32 add
    float* hrow = H + (int64_t)row * n;
#pragma unroll
    for (int j4 = 0; j4 < 32; ++j4) {
      const int c = cbase + 4 * j4;
      if (c + 3 < row || c >= n) continue;
      const float f0 = alpha * tile[4 * j4 + 0];
      const float f1 = alpha * tile[4 * j4 + 1];
      const float f2 = alpha * tile[4 * j4 + 2];
      const float f3 = alpha * tile[4 * j4 + 3];
      if (vec4 && c >= row && c + 3 < n) {
        atomicAdd(reinterpret_cast<float4*>(hrow + c), make_float4(f0, f1, f2, f3));
      } else {
        const float fv[4] = {f0, f1, f2, f3};
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (c + i >= row && c + i < n) atomicAdd(hrow + c + i, fv[i]);
      }
    }
    __threadfence();   // this thread's reductions are performed before the release below
  }
  // every thread's stores are done before the next chunk may start
  ptx::named_bar_sync(kEpiBar, kEpiThreads);
  if (waiter) {
    __threadfence();
    ptx::st_release_gpu(flag, chunk + 1);
  }
  return true;
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    syrk_bf16_kernel(const __grid_constant__ CUtensorMap mapA,
                     const __grid_constant__ CUtensorMap mapB, const SyrkArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
  uint64_t* full = bars;                 // [STAGES] TMA landed
  uint64_t* empty = bars + STAGES;       // [STAGES] MMAs done reading
  uint64_t* tfull = bars + 2 * STAGES;   // [2] accumulator ready
  uint64_t* tempty = tfull + 2;          // [2] accumulator drained
  uint64_t* drain = tempty + 2;          // [1] MMA drain on abort
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
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
    ptx::tmem_alloc(tmem_slot, TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      ptx::prefetch_tmap(&mapA);
      ptx::prefetch_tmap(&mapB);
      int stage = 0;
      uint32_t phase = 0;
      int last_parity[STAGES];
      for (int s = 0; s < STAGES; ++s) last_parity[s] = -1;
      bool ok = ptx::gate_wait_bounded(args.gate, args.limit_ns);
      for (int u = blockIdx.x; u < args.units && ok; u += gridDim.x) {
        int I, J;
        decode_tile(u % args.ntiles, args.nI, I, J);
        const int kb0 = (u / args.ntiles) * args.kb_per_unit;
        const int kb1 = min(kb0 + args.kb_per_unit, args.nkb);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!ptx::mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, args.limit_ns)) {
            ok = false;
            break;
          }
          ptx::mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
          ptx::tma_load_2d(sA + stage * A_BYTES, &mapA, &full[stage], kb * BK, I * BM);
          ptx::tma_load_2d(sB + stage * B_BYTES, &mapB, &full[stage], kb * BK, J * BN);
          last_parity[stage] = (int)phase;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok || *abort_flag) {
        raise_abort(abort_flag, args.info);
        // wait (bounded) for this CTA's own copies still in flight
        volatile int never = 0;
        for (int s = 0; s < STAGES; ++s)
          if (last_parity[s] >= 0)
            ptx::mbar_wait_bounded(&full[s], (uint32_t)last_parity[s], &never, WAIT_LIMIT_NS);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      constexpr uint32_t idesc = ptx::idesc_bf16_f32(BM, BN);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t aphase = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < args.units && ok; u += gridDim.x) {
        const int kb0 = (u / args.ntiles) * args.kb_per_unit;
        const int kb1 = min(kb0 + args.kb_per_unit, args.nkb);
        for (int p0 = kb0; p0 < kb1 && ok; p0 += kSubKb) {
          const int p1 = min(p0 + kSubKb, kb1);
          if (!ptx::mbar_wait_bounded(&tempty[acc], aphase ^ 1, abort_flag, args.limit_ns)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
          for (int kb = p0; kb < p1; ++kb) {
            if (!ptx::mbar_wait_bounded(&full[stage], phase, abort_flag, args.limit_ns)) {
              ok = false;
              break;
            }
            ptx::tc_fence_after();
            const uint64_t adesc = ptx::smem_desc_sw128(ptx::smem_u32(sA + stage * A_BYTES));
            const uint64_t bdesc = ptx::smem_desc_sw128(ptx::smem_u32(sB + stage * B_BYTES));
#pragma unroll
            for (int k = 0; k < BK / 16; ++k)
              ptx::mma_bf16(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc,
                            (kb > p0 || k > 0) ? 1u : 0u);
            ptx::mma_commit(&empty[stage]);
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1;
            }
          }
          if (!ok) break;
          ptx::mma_commit(&tfull[acc]);
          acc ^= 1;
          if (acc == 0) aphase ^= 1;
        }
      }
      if (!ok || *abort_flag) {
        raise_abort(abort_flag, args.info);
        ptx::mma_commit(drain);  // completes when every MMA issued above is done
        volatile int never = 0;
        ptx::mbar_wait_bounded(drain, 0, &never, WAIT_LIMIT_NS);
      }
    }
  } else {
    // -------------------------------------------------- epilogue (warps 2..9)
    // warp w reads TMEM lanes [32 (w % 4), +32) (rows of the tile) and
    // columns [128 half, +128) of the accumulator.  Every decision to stop is
    // taken by all 256 epilogue threads together (named barrier with AND).
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    int acc = 0;
    uint32_t aphase = 0;
    const int n = args.n;
    for (int u = blockIdx.x; u < args.units; u += gridDim.x) {
      int I, J;
      decode_tile(u % args.ntiles, args.nI, I, J);
      const int kb0 = (u / args.ntiles) * args.kb_per_unit;
      const int kb1 = min(kb0 + args.kb_per_unit, args.nkb);
      const int row_lo = I * BM + q * 32;
      const int row = row_lo + lane;
      const int cbase = J * BN + half * 128;
      float tile[128];
#pragma unroll
      for (int j = 0; j < 128; ++j) tile[j] = 0.f;
      bool ok = true;
      for (int p0 = kb0; p0 < kb1; p0 += kSubKb) {
        bool ready = ptx::mbar_wait_bounded(&tfull[acc], aphase, abort_flag, args.limit_ns);
        if (!ready) raise_abort(abort_flag, args.info);
        if (!ptx::named_bar_and(kEpiBar, kEpiThreads, ready)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          const int col0 = cbase + ch * 32;
          // warp-uniform: pieces past n or wholly below the diagonal are not needed
          if (col0 < n && col0 + 31 >= row_lo) {
            uint32_t v[32];
            ptx::tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) +
                                        (uint32_t)(acc * BN + half * 128 + ch * 32),
                                    v);
            ptx::tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) tile[ch * 32 + j] += __uint_as_float(v[j]);
          }
        }
        ptx::tc_fence_before();
        ptx::mbar_arrive(&tempty[acc]);
        acc ^= 1;
        if (acc == 0) aphase ^= 1;
      }
      if (!ok) break;
      const int t = u % args.ntiles;
      if (!ordered_add(args.H, n, row, cbase, args.alpha, args.vec4, tile, args.flags + t,
                       (uint32_t)(u / args.ntiles), abort_flag, args.info, args.limit_ns,
                       warp == 2 && lane == 0))
        break;
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ===========================================================================
// The same SYRK on CTA pairs (clusters of 2): one tcgen05.mma.cta_group::2
// (M = 256, N = 256, K = 16) covers a 256 x 256 tile of H.  CTA r of the
// pair loads its own 128 rows of A (tile rows 128 r..) and its own half of
// B (tile columns 128 r..), 32 KB per 64-token k-block instead of 48 KB per
// SM, so the operand feed from L2 per unit of MMA work drops by a third.
//  * Both CTAs' TMA loads count on the leader's (rank 0) `full` barrier; only
//    the leader's producer posts the expected bytes (both CTAs' share).
//  * Only the leader issues MMAs; each commit arrives on the `empty` /
//    `tfull` barrier at the same offset in both CTAs.
//  * Each CTA drains its own TMEM (its 128 rows x 256 columns); one lane per
//    epilogue warp arrives on the leader's `tempty` (16 arrivals per piece).
//  * TMEM is allocated and freed by one warp in each CTA (cta_group::2);
//    cluster barriers order set-up and tear-down.
// Tiles (I2, J) with I2 <= J cover the upper triangle in 256 x 256 blocks.
// Accuracy handling is the single-CTA kernel's: fresh TMEM sums every
// kSubKb k-blocks, added in an fp32 register tile, the ordered split-K add per unit.
// ===========================================================================
constexpr int P_STAGES = 6;
constexpr int P_A_BYTES = 128 * BK * 2;   // this CTA's A rows
constexpr int P_B_BYTES = 128 * BK * 2;   // this CTA's half of B
constexpr int P_STAGE_BYTES = P_A_BYTES + P_B_BYTES;
constexpr size_t P_SMEM_BYTES = (size_t)P_STAGES * P_STAGE_BYTES + 1024 + 256;

struct SyrkPairArgs {
  float* H;
  int n;
  float alpha;
  int nkb;          // k-blocks of BK tokens
  int kb_per_unit;
  int ntiles;       // 256 x 256 tiles touching the upper triangle
  int units;        // ntiles * token chunks
  int vec4;
  int32_t* info;
  uint32_t* flags;  // [2][ntiles] chunks of each tile half (CTA rank) added so far
  const int32_t* gate;
  uint64_t limit_ns;
};

// Tile t of the J-major enumeration: column block J holds row blocks 0..J.
__device__ __forceinline__ void decode_tile_pair(int t, int& I2, int& J) {
  J = 0;
  while ((J + 1) * (J + 2) / 2 <= t) ++J;
  I2 = t - J * (J + 1) / 2;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    syrk_bf16_pair_kernel(const __grid_constant__ CUtensorMap mapA,
                          const __grid_constant__ CUtensorMap mapB, const SyrkPairArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + P_STAGES * P_A_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + P_STAGES * P_STAGE_BYTES);
  uint64_t* full = bars;                   // [P_STAGES] (the leader's counts both CTAs' loads)
  uint64_t* empty = bars + P_STAGES;       // [P_STAGES]
  uint64_t* tfull = bars + 2 * P_STAGES;   // [2]
  uint64_t* tempty = tfull + 2;            // [2] (the leader's: 16 warp arrivals)
  uint64_t* drain = tempty + 2;            // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  if (threadIdx.x == 0) {
    for (int s = 0; s < P_STAGES; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(&tfull[a], 1);
      ptx::mbar_init(&tempty[a], 16);
    }
    ptx::mbar_init(drain, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(tmem_slot, TMEM_COLS);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  ptx::cluster_sync();  // barriers and TMEM of both CTAs exist before any cross-CTA use
  ptx::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer (both CTAs)
      ptx::prefetch_tmap(&mapA);
      ptx::prefetch_tmap(&mapB);
      int stage = 0;
      uint32_t phase = 0;
      int last_parity[P_STAGES];  // leader: last phase of full[s] it armed
      for (int s = 0; s < P_STAGES; ++s) last_parity[s] = -1;
      bool ok = ptx::gate_wait_bounded(args.gate, args.limit_ns);
      for (int u = pair; u < args.units && ok; u += npairs) {
        int I2, J;
        decode_tile_pair(u % args.ntiles, I2, J);
        const int kb0 = (u / args.ntiles) * args.kb_per_unit;
        const int kb1 = min(kb0 + args.kb_per_unit, args.nkb);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!ptx::mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, args.limit_ns)) {
            ok = false;
            break;
          }
          if (leader) {
            ptx::mbar_arrive_expect_tx(&full[stage], 2 * P_STAGE_BYTES);
            last_parity[stage] = (int)phase;
          }
          const uint32_t fb = ptx::mapa_shared(&full[stage], 0);
          ptx::tma_load_2d_pair(sA + stage * P_A_BYTES, &mapA, fb, kb * BK,
                                I2 * 256 + (int)rank * 128);
          ptx::tma_load_2d_pair(sB + stage * P_B_BYTES, &mapB, fb, kb * BK,
                                J * 256 + (int)rank * 128);
          if (++stage == P_STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok || *abort_flag) {
        raise_abort(abort_flag, args.info);
        // Loads still in flight must land before the pair tears down.  Both
        // CTAs' loads of a stage complete on the leader's full[] barrier, so
        // the leader waits (bounded) for the last phase it armed on each
        // stage; the other CTA is held by the final cluster barrier until
        // the leader gets there.
        if (leader) {
          volatile int never = 0;
          for (int s = 0; s < P_STAGES; ++s)
            if (last_parity[s] >= 0)
              ptx::mbar_wait_bounded(&full[s], (uint32_t)last_parity[s], &never, WAIT_LIMIT_NS);
        }
      } else {
        // tail: every stage is released once more, so the MMA commits'
        // arrivals on this CTA's `empty` barriers have all landed
        for (int i = 0; i < P_STAGES; ++i) {
          if (!ptx::mbar_wait_bounded(&empty[stage], phase ^ 1, abort_flag, args.limit_ns)) break;
          if (++stage == P_STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------ MMA issuer (leader only)
      constexpr uint32_t idesc = ptx::idesc_bf16_f32(256, 256);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t aphase = 0;
      bool ok = true;
      for (int u = pair; u < args.units && ok; u += npairs) {
        const int kb0 = (u / args.ntiles) * args.kb_per_unit;
        const int kb1 = min(kb0 + args.kb_per_unit, args.nkb);
        for (int p0 = kb0; p0 < kb1 && ok; p0 += kSubKb) {
          const int p1 = min(p0 + kSubKb, kb1);
          if (!ptx::mbar_wait_bounded(&tempty[acc], aphase ^ 1, abort_flag, args.limit_ns)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
          for (int kb = p0; kb < p1; ++kb) {
            if (!ptx::mbar_wait_bounded(&full[stage], phase, abort_flag, args.limit_ns)) {
              ok = false;
              break;
            }
            ptx::tc_fence_after();
            const uint64_t adesc = ptx::smem_desc_sw128(ptx::smem_u32(sA + stage * P_A_BYTES));
            const uint64_t bdesc = ptx::smem_desc_sw128(ptx::smem_u32(sB + stage * P_B_BYTES));
#pragma unroll
            for (int k = 0; k < BK / 16; ++k)
              ptx::mma_bf16_pair(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc,
                                 (kb > p0 || k > 0) ? 1u : 0u);
            ptx::mma_commit_pair(&empty[stage], 0x3);
            if (++stage == P_STAGES) {
              stage = 0;
              phase ^= 1;
            }
          }
          if (!ok) break;
          ptx::mma_commit_pair(&tfull[acc], 0x3);
          acc ^= 1;
          if (acc == 0) aphase ^= 1;
        }
      }
      if (!ok || *abort_flag) raise_abort(abort_flag, args.info);
      // every MMA issued above is complete before tear-down (bounded)
      ptx::mma_commit_pair(drain, 0x1);
      volatile int never = 0;
      ptx::mbar_wait_bounded(drain, 0, &never, WAIT_LIMIT_NS);
    }
  } else {
    // -------------------------------------------------- epilogue (warps 2..9, both CTAs)
    const int q = warp & 3;              // TMEM lanes [32q, 32q + 32): rows of this CTA's half
    const int half = (warp - 2) >> 2;    // accumulator columns [128 half, +128)
    const uint32_t tempty_leader0 = ptx::mapa_shared(&tempty[0], 0);
    const uint32_t tempty_leader1 = ptx::mapa_shared(&tempty[1], 0);
    int acc = 0;
    uint32_t aphase = 0;
    const int n = args.n;
    for (int u = pair; u < args.units; u += npairs) {
      int I2, J;
      decode_tile_pair(u % args.ntiles, I2, J);
      const int kb0 = (u / args.ntiles) * args.kb_per_unit;
      const int kb1 = min(kb0 + args.kb_per_unit, args.nkb);
      const int row_lo = I2 * 256 + (int)rank * 128 + q * 32;
      const int row = row_lo + lane;
      const int cbase = J * 256 + half * 128;
      float tile[128];
#pragma unroll
      for (int j = 0; j < 128; ++j) tile[j] = 0.f;
      bool ok = true;
      for (int p0 = kb0; p0 < kb1; p0 += kSubKb) {
        bool ready = ptx::mbar_wait_bounded(&tfull[acc], aphase, abort_flag, args.limit_ns);
        if (!ready) raise_abort(abort_flag, args.info);
        if (!ptx::named_bar_and(kEpiBar, kEpiThreads, ready)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          const int col0 = cbase + ch * 32;
          // warp-uniform: pieces past n or wholly below the diagonal are not needed
          if (col0 < n && col0 + 31 >= row_lo) {
            uint32_t v[32];
            ptx::tmem_ld_32x32b_x32(tmem_base + ((uint32_t)(q * 32) << 16) +
                                        (uint32_t)(acc * BN + half * 128 + ch * 32),
                                    v);
            ptx::tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) tile[ch * 32 + j] += __uint_as_float(v[j]);
          }
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
        acc ^= 1;
        if (acc == 0) aphase ^= 1;
      }
      if (!ok) break;
      const int t = u % args.ntiles;
      if (!ordered_add(args.H, n, row, cbase, args.alpha, args.vec4, tile,
                       args.flags + (int)rank * args.ntiles + t, (uint32_t)(u / args.ntiles),
                       abort_flag, args.info, args.limit_ns, warp == 2 && lane == 0))
        break;
    }
  }

  ptx::tc_fence_before();
  ptx::cluster_sync();  // both CTAs done with every load, MMA and TMEM read
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

// hi = bf16(x) (round to nearest even), lo = bf16(x - hi)
__global__ void split_bf16_kernel(const float* __restrict__ X, int64_t n, int64_t ntok,
                                  int64_t ldx, __nv_bfloat16* __restrict__ hi,
                                  __nv_bfloat16* __restrict__ lo, int64_t ldo) {
  const int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int64_t r = blockIdx.y;
  if (t >= ntok) return;
  const float x = X[r * ldx + t];
  const __nv_bfloat16 h = __float2bfloat16_rn(x);
  hi[r * ldo + t] = h;
  lo[r * ldo + t] = __float2bfloat16_rn(x - __bfloat162float(h));
}

// H[c][r] = H[r][c] for c > r, 32 x 32 tiles through shared memory.
__global__ void __launch_bounds__(256) mirror_upper_kernel(float* __restrict__ H, int n) {
  __shared__ float T[32][33];
  const int I = blockIdx.y, J = blockIdx.x;
  if (I > J) return;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int a = ty; a < 32; a += 8) {
    const int r = 32 * I + a, c = 32 * J + tx;
    T[a][tx] = (r < n && c < n) ? H[(int64_t)r * n + c] : 0.f;
  }
  __syncthreads();
  for (int a = ty; a < 32; a += 8) {
    const int r = 32 * J + a, c = 32 * I + tx;  // destination (lower): row r, col c
    if (r < n && c < n && c < r) H[(int64_t)r * n + c] = T[tx][a];
  }
}

bool make_map(CUtensorMap* map, const void* base, int64_t rows, int64_t ntok, int64_t ld,
              uint32_t box_rows) {
  return make_tma_2d(map, base, /*bf16=*/true, rows, ntok, ld, BK, box_rows);
}

}  // namespace

namespace {

// Fewest token chunks that fill `slots` parallel workers' waves to >= 97 %
// (at least 8 k-blocks per unit), else the best fill found.
int choose_chunks(int ntiles, int nkb, int slots) {
  int best_kc = 1;
  double best_eff = -1.0;
  const int max_kc = std::max(1, std::min(nkb / 8, 512));
  for (int kc = 1; kc <= max_kc; ++kc) {
    const long units = (long)ntiles * kc;
    const long waves = (units + slots - 1) / slots;
    const double eff = (double)units / (double)(waves * slots);
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best_kc = kc;
    }
    if (eff >= 0.97) break;
  }
  return best_kc;
}

// Concurrent CTA pairs the pair kernel can have on the current device (0 if
// it cannot launch there).  A property of the device and the kernel, so it is
// looked up once per device and kept (under a lock).
int pair_slots() {
  constexpr int kMaxDev = 64;
  static std::mutex mu;
  static int cached[kMaxDev];
  static bool have[kMaxDev] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (have[dev]) return cached[dev];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * 74, 1, 1);
  cfg.blockDim = dim3(NUM_THREADS, 1, 1);
  cfg.dynamicSmemBytes = P_SMEM_BYTES;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = 2;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int clusters = 0;
  if (cudaFuncSetAttribute(syrk_bf16_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)P_SMEM_BYTES) != cudaSuccess ||
      cudaOccupancyMaxActiveClusters(&clusters, syrk_bf16_pair_kernel, &cfg) != cudaSuccess) {
    cudaGetLastError();
    clusters = 0;
  }
  cached[dev] = clusters;
  have[dev] = true;
  return clusters;
}

int pair_tiles(int64_t n) {
  const int nJ = (int)((n + 255) / 256);
  return nJ * (nJ + 1) / 2;
}

int single_tiles(int64_t n) {
  const int nI = (int)((n + BM - 1) / BM), nJ = (int)((n + BN - 1) / BN);
  int t = 0;
  for (int J = 0; J < nJ; ++J) t += std::min(nI, 2 * J + 2);
  return t;
}

}  // namespace

size_t syrk_flag_bytes(int64_t n) {
  return sizeof(uint32_t) * (size_t)std::max(2 * pair_tiles(n), single_tiles(n));
}

cudaError_t launch_syrk_bf16(float* H, int64_t n, const void* A, const void* B, int64_t ntok,
                             int64_t ld, float alpha, int32_t* info, void* flags,
                             cudaStream_t s) {
  if (n <= 0 || ntok <= 0) return cudaSuccess;
  const int sms = num_sms();
  const int nkb = (int)((ntok + BK - 1) / BK);
  const int vec4 = ((n % 4) == 0 && (reinterpret_cast<uintptr_t>(H) % 16) == 0) ? 1 : 0;
  const WaitGate wg = current_wait_gate();
  cudaError_t e;
  // the turnstile counts start at zero for every launch
  if ((e = cudaMemsetAsync(flags, 0, syrk_flag_bytes(n), s)) != cudaSuccess) return e;
  // CTA pairs for layers of at least 256 inputs, when the device can co-schedule them
  const int slots = n >= 256 ? pair_slots() : 0;
  if (slots > 0) {
    CUtensorMap mapA, mapB;
    if (!make_map(&mapA, A, n, ntok, ld, 128) || !make_map(&mapB, B, n, ntok, ld, 128))
      return cudaErrorInvalidValue;
    SyrkPairArgs a;
    a.H = H;
    a.n = (int)n;
    a.alpha = alpha;
    a.nkb = nkb;
    a.ntiles = pair_tiles(n);
    const int kc = choose_chunks(a.ntiles, nkb, slots);
    a.kb_per_unit = (nkb + kc - 1) / kc;
    a.units = a.ntiles * ((nkb + a.kb_per_unit - 1) / a.kb_per_unit);
    a.vec4 = vec4;
    a.info = info;
    a.flags = static_cast<uint32_t*>(flags);
    a.gate = wg.gate;
    a.limit_ns = wg.limit_ns;
    // every pair of the persistent grid must be resident at once (the
    // turnstile waits on units of other pairs): no more pairs than slots
    const int pairs = std::min(slots, a.units);
    if ((e = cudaFuncSetAttribute(syrk_bf16_pair_kernel,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)P_SMEM_BYTES)) != cudaSuccess)
      return e;
    syrk_bf16_pair_kernel<<<2 * pairs, NUM_THREADS, P_SMEM_BYTES, s>>>(mapA, mapB, a);
    note_launch();
    return cudaGetLastError();
  }
  CUtensorMap mapA, mapB;
  if (!make_map(&mapA, A, n, ntok, ld, BM) || !make_map(&mapB, B, n, ntok, ld, BN))
    return cudaErrorInvalidValue;
  SyrkArgs a;
  a.H = H;
  a.n = (int)n;
  a.alpha = alpha;
  a.nkb = nkb;
  a.nI = (int)((n + BM - 1) / BM);
  a.ntiles = single_tiles(n);
  const int best_kc = choose_chunks(a.ntiles, nkb, sms);
  a.kb_per_unit = (a.nkb + best_kc - 1) / best_kc;
  const int kchunks = (a.nkb + a.kb_per_unit - 1) / a.kb_per_unit;
  a.units = a.ntiles * kchunks;
  a.vec4 = vec4;
  a.info = info;
  a.flags = static_cast<uint32_t*>(flags);
  a.gate = wg.gate;
  a.limit_ns = wg.limit_ns;
  if ((e = cudaFuncSetAttribute(syrk_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)SMEM_BYTES)) != cudaSuccess)
    return e;
  const int grid = std::min(sms, a.units);
  syrk_bf16_kernel<<<grid, NUM_THREADS, SMEM_BYTES, s>>>(mapA, mapB, a);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_split_bf16(const float* X, int64_t n, int64_t ntok, int64_t ldx, void* hi,
                              void* lo, int64_t ldo, cudaStream_t s) {
  if (n <= 0 || ntok <= 0) return cudaSuccess;
  dim3 grid((unsigned)((ntok + 255) / 256), (unsigned)n);
  split_bf16_kernel<<<grid, 256, 0, s>>>(X, n, ntok, ldx, static_cast<__nv_bfloat16*>(hi),
                                         static_cast<__nv_bfloat16*>(lo), ldo);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_mirror_upper(float* H, int64_t n, cudaStream_t s) {
  const unsigned nt = (unsigned)((n + 31) / 32);
  mirror_upper_kernel<<<dim3(nt, nt), 256, 0, s>>>(H, (int)n);
  note_launch();
  return cudaGetLastError();
}

}  // namespace gptq
