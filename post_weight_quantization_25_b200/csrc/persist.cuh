// The machinery shared by the persistent task-queue kernels (the sweep and
// the factorisation): one CTA per SM, kPg2Threads threads, the shared memory
// and TMEM of one panel_gemm2 CTA, and the fp32-accurate rank-128 update
//     C[rows of the item][its tiles] -= P Q^T      (K = 128)
// run as one task by the CTA's producer (warp 0), MMA issuer (warp 1) and
// epilogue warps (2 .. 9), exactly as in panel_gemm2_kernel: P (128 rows x
// 128, TF32 part and remainder) is loaded once per task, Q streams through a
// two-stage TMA ring, three TF32 MMAs per k-step accumulate in one of two
// TMEM buffers, and the epilogue lands each tile in C by TMA reduce-add.
// The pipeline state (ring stages, barrier phases) carries over from task to
// task.  Every wait is bounded; a failed wait raises the CTA's abort flag,
// records the timeout code in `info` (if no error was recorded before) and
// waits (bounded) for the CTA's own copies and MMAs.
#pragma once
#include <cstdint>

#include "panel_gemm.cuh"
#include "sm100_ptx.cuh"

namespace gptq {

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// first error wins
__device__ __forceinline__ void persist_abort(volatile int* abort_flag, int32_t* info,
                                              int32_t code) {
  *abort_flag = 1;
  if (info) atomicCAS(info, 0, code);
}

static_assert(kPg2QStages == 2, "the Q ring's last-load parities are two scalars");

// The update pipeline's state, kept in shared memory between tasks so that it
// holds no registers while a CTA runs other kinds of task.
struct PgPipeState {
  int p_loads;        // P blocks loaded (= consumed: the producer and the MMA agree after a task)
  int qst;            // Q ring stage
  uint32_t qph;
  int acc;            // TMEM accumulator
  uint32_t aph;
  int q_last0, q_last1;  // parity of the last load into Q stage 0 / 1 (-1: none yet)
  int last_pempty;    // parity of the last commit on pempty (-1: none yet)
};

struct PersistCta {
  uint8_t* smem;  // 1024-aligned; the update's buffers, free between tasks
  uint32_t tmem_base;
  uint64_t limit;

  // the regions and barriers (fixed offsets from smem)
  __device__ __forceinline__ uint8_t* sP() const { return smem; }
  __device__ __forceinline__ uint8_t* sQ() const { return smem + kPg2PBytes; }
  __device__ __forceinline__ uint8_t* sOut() const {
    return smem + kPg2PBytes + kPg2QStages * kPg2QStageBytes;
  }
  __device__ __forceinline__ uint64_t* bars() const {
    return reinterpret_cast<uint64_t*>(sOut() + 8 * kPg2StageOut);
  }
  __device__ __forceinline__ uint64_t* pfull() const { return bars(); }
  __device__ __forceinline__ uint64_t* pempty() const { return bars() + 1; }
  __device__ __forceinline__ uint64_t* qfull(int q) const { return bars() + 2 + q; }
  __device__ __forceinline__ uint64_t* qempty(int q) const { return bars() + 2 + kPg2QStages + q; }
  __device__ __forceinline__ uint64_t* tfull(int c) const { return bars() + 2 + 2 * kPg2QStages + c; }
  __device__ __forceinline__ uint64_t* tempty(int c) const {
    return bars() + 4 + 2 * kPg2QStages + c;
  }
  __device__ __forceinline__ uint64_t* drain() const { return bars() + 6 + 2 * kPg2QStages; }
  __device__ __forceinline__ uint32_t* tmem_slot() const {
    return reinterpret_cast<uint32_t*>(bars() + 7 + 2 * kPg2QStages);
  }
  __device__ __forceinline__ volatile int* abort_flag() const {
    return reinterpret_cast<volatile int*>(tmem_slot() + 1);
  }
  // two words the kernels use to broadcast thread 0's decisions
  __device__ __forceinline__ volatile int* task_slot() const { return abort_flag() + 1; }
  __device__ __forceinline__ volatile int* skip_slot() const { return abort_flag() + 2; }
  __device__ __forceinline__ PgPipeState* state() const {
    return reinterpret_cast<PgPipeState*>(sOut() + 8 * kPg2StageOut + 128);
  }

  // Every thread: carve shared memory, initialise the barriers, allocate TMEM.
  __device__ __forceinline__ void init(uint8_t* smem_raw, uint64_t limit_ns) {
    static_assert(sizeof(PgPipeState) <= 128, "the pipeline state fits its slot");
    smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                      ~static_cast<uintptr_t>(1023));
    limit = limit_ns;
    const int tid = threadIdx.x, warp = tid >> 5;
    if (tid == 0) {
      ptx::mbar_init(pfull(), 1);
      ptx::mbar_init(pempty(), 1);
      for (int q = 0; q < kPg2QStages; ++q) {
        ptx::mbar_init(qfull(q), 1);
        ptx::mbar_init(qempty(q), 1);
      }
      for (int c = 0; c < 2; ++c) {
        ptx::mbar_init(tfull(c), 1);
        ptx::mbar_init(tempty(c), 256);
      }
      ptx::mbar_init(drain(), 1);
      *abort_flag() = 0;
      PgPipeState* st = state();
      st->p_loads = 0;
      st->qst = 0;
      st->qph = 0;
      st->acc = 0;
      st->aph = 0;
      st->q_last0 = st->q_last1 = -1;
      st->last_pempty = -1;
      ptx::fence_mbar_init();
    }
    if (warp == 1) {
      ptx::tmem_alloc(tmem_slot(), kPg2TmemCols);
      ptx::tmem_relinquish();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    tmem_base = *tmem_slot();
  }

  // Every thread: the next task index (taken by thread 0), or -1 once the
  // CTA should stop (no task left, or an abort).
  __device__ __forceinline__ int next_task(uint32_t* counter, int total) {
    if (threadIdx.x == 0) *task_slot() = (int)atomicAdd(counter, 1u);
    __syncthreads();
    const int t = *task_slot();
    const bool stop = *abort_flag() != 0;
    __syncthreads();
    return (t >= total || stop) ? -1 : t;
  }

  // Every thread, after the task's waits and a CTA barrier: one update task.
  // On return the epilogue warps' reduce-adds have landed and are ordered
  // before the generic proxy; the caller synchronises the CTA and publishes.
  __device__ __forceinline__ void update(const PgItem& I, const CUtensorMap& mPh,
                                         const CUtensorMap& mPl, const CUtensorMap& mQh,
                                         const CUtensorMap& mQl, const CUtensorMap& mC0,
                                         const CUtensorMap& mC1, int32_t* info,
                                         int32_t timeout_code) {
    constexpr uint64_t kDrainLimit = (uint64_t)kGridWaitLimitNs;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    volatile int* abort_flag = this->abort_flag();
    uint8_t* sP = this->sP();
    uint8_t* sQ = this->sQ();
    uint8_t* sOut = this->sOut();
    uint64_t* pfull = this->pfull();
    uint64_t* pempty = this->pempty();
    uint64_t* qfull = this->qfull(0);
    uint64_t* qempty = this->qempty(0);
    uint64_t* tfull = this->tfull(0);
    uint64_t* tempty = this->tempty(0);
    uint64_t* drain = this->drain();
    PgPipeState* stp = state();
    int p_loads = stp->p_loads, qst = stp->qst, acc = stp->acc;
    uint32_t qph = stp->qph, aph = stp->aph;
    int q_last0 = stp->q_last0, q_last1 = stp->q_last1, last_pempty = stp->last_pempty;
    if (warp == 0) {
      if (lane == 0) {
        // producer: P (all of K = 128), then Q per tile
        bool ok = p_loads == 0 ||
                  ptx::mbar_wait_bounded(pempty, (uint32_t)((p_loads - 1) & 1), abort_flag, limit);
        if (ok) {
          ptx::mbar_arrive_expect_tx(pfull, kPg2PBytes);
          for (int kb = 0; kb < kPgKBlocks; ++kb) {
            ptx::tma_load_2d(sP + kb * 2 * kPgTileBytes, &mPh, pfull, I.pkx + 32 * kb, I.prow);
            ptx::tma_load_2d(sP + kb * 2 * kPgTileBytes + kPgTileBytes, &mPl, pfull,
                             I.pkx + 32 * kb, I.prow);
          }
          ++p_loads;
          for (int q = 0; q < I.nq && ok; ++q)
            for (int kb = 0; kb < kPgKBlocks; ++kb) {
              if (!ptx::mbar_wait_bounded(&qempty[qst], qph ^ 1, abort_flag, limit)) {
                ok = false;
                break;
              }
              uint8_t* sb = sQ + qst * kPg2QStageBytes;
              ptx::mbar_arrive_expect_tx(&qfull[qst], kPg2QStageBytes);
              ptx::tma_load_2d(sb, &mQh, &qfull[qst], I.qkx + 32 * kb, I.qrow0 + 128 * q);
              ptx::tma_load_2d(sb + kPgTileBytes, &mQl, &qfull[qst], I.qkx + 32 * kb,
                               I.qrow0 + 128 * q);
              if (qst == 0)
                q_last0 = (int)qph;
              else
                q_last1 = (int)qph;
              if (++qst == kPg2QStages) {
                qst = 0;
                qph ^= 1;
              }
            }
        }
        if (!ok) {
          persist_abort(abort_flag, info, timeout_code);
          volatile int never = 0;  // this CTA's own copies in flight
          ptx::mbar_wait_bounded(pfull, (uint32_t)((p_loads - 1) & 1), &never, kDrainLimit);
          if (q_last0 >= 0) ptx::mbar_wait_bounded(&qfull[0], (uint32_t)q_last0, &never, kDrainLimit);
          if (q_last1 >= 0) ptx::mbar_wait_bounded(&qfull[1], (uint32_t)q_last1, &never, kDrainLimit);
        }
        stp->q_last0 = q_last0;
        stp->q_last1 = q_last1;
      }
    } else if (warp == 1) {
      if (lane == 0) {
        // MMA issuer
        constexpr uint32_t idesc = ptx::idesc_tf32_f32(128, 128);
        bool ok = ptx::mbar_wait_bounded(pfull, (uint32_t)(p_loads & 1), abort_flag, limit);
        if (ok) {
          ptx::tc_fence_after();
          for (int q = 0; q < I.nq && ok; ++q) {
            if (!ptx::mbar_wait_bounded(&tempty[acc], aph ^ 1, abort_flag, limit)) {
              ok = false;
              break;
            }
            ptx::tc_fence_after();
            const uint32_t d = tmem_base + (uint32_t)(acc * 128);
            for (int kb = 0; kb < kPgKBlocks; ++kb) {
              if (!ptx::mbar_wait_bounded(&qfull[qst], qph, abort_flag, limit)) {
                ok = false;
                break;
              }
              ptx::tc_fence_after();
              const uint32_t pb = ptx::smem_u32(sP + kb * 2 * kPgTileBytes);
              const uint32_t qb = ptx::smem_u32(sQ + qst * kPg2QStageBytes);
              const uint64_t ph = ptx::smem_desc_sw128(pb);
              const uint64_t pl = ptx::smem_desc_sw128(pb + kPgTileBytes);
              const uint64_t qh = ptx::smem_desc_sw128(qb);
              const uint64_t ql = ptx::smem_desc_sw128(qb + kPgTileBytes);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                ptx::mma_tf32(d, ph + 2 * kk, qh + 2 * kk, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
                ptx::mma_tf32(d, ph + 2 * kk, ql + 2 * kk, idesc, 1u);
                ptx::mma_tf32(d, pl + 2 * kk, qh + 2 * kk, idesc, 1u);
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
          if (ok) {
            ptx::mma_commit(pempty);
            last_pempty = p_loads & 1;
          }
        }
        ++p_loads;  // the MMA thread counts the P blocks it consumed
        if (!ok) {
          persist_abort(abort_flag, info, timeout_code);
          ptx::mma_commit(drain);
          volatile int never = 0;
          ptx::mbar_wait_bounded(drain, 0, &never, kDrainLimit);
        }
        // the state after the task (the producer's ring and P counts agree)
        stp->p_loads = p_loads;
        stp->qst = qst;
        stp->qph = qph;
        stp->acc = acc;
        stp->aph = aph;
        stp->last_pempty = last_pempty;
      }
    } else {
      // epilogue: warps 2 .. 9
      const int quarter = warp & 3;
      const int half = (warp - 2) >> 2;
      float* stage = reinterpret_cast<float*>(sOut + (warp - 2) * kPg2StageOut);
      for (int q = 0; q < I.nq; ++q) {
        const bool ready = ptx::mbar_wait_bounded(&tfull[acc], aph, abort_flag, limit);
        __syncwarp();
        if (!__all_sync(0xffffffffu, ready && !*abort_flag)) {
          if (!ready) persist_abort(abort_flag, info, timeout_code);
          break;
        }
        ptx::tc_fence_after();
        pg_tile_epilogue<true>(I, q, tmem_base + (uint32_t)(acc * 128), quarter, half, lane,
                               stage, mC0, mC1);
        ptx::tc_fence_before();
        ptx::mbar_arrive(&tempty[acc]);
        acc ^= 1;
        if (acc == 0) aph ^= 1;
      }
      // every reduce this warp issued has landed (and is ordered before the
      // generic proxy's accesses) before the caller publishes the tiles
      if (lane == 0) {
        ptx::bulk_wait_all0();
        fence_proxy_async_global();
      }
      __syncwarp();
    }
  }

  // Every thread, once the task loop is over: wait (bounded) for the last
  // commit on pempty, then free TMEM.
  __device__ __forceinline__ void teardown() {
    constexpr uint64_t kDrainLimit = (uint64_t)kGridWaitLimitNs;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int last_pempty = state()->last_pempty;
    if (warp == 1 && lane == 0 && last_pempty >= 0) {
      volatile int never = 0;
      ptx::mbar_wait_bounded(pempty(), (uint32_t)last_pempty, &never, kDrainLimit);
    }
    ptx::tc_fence_before();
    __syncthreads();
    if (warp == 1) {
      ptx::tc_fence_after();
      ptx::tmem_dealloc(tmem_base, kPg2TmemCols);
    }
  }
};

}  // namespace gptq
