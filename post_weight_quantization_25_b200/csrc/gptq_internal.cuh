// Internal launch interface between the C-ABI layer (gptq_api.cu) and the
// kernel files.  Every launcher enqueues on `s` and returns the CUDA error of
// the launch (cudaSuccess when nothing had to run).
#pragma once
#include <cstdint>
#include <mutex>
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include "../../include/gptq.h"

namespace gptq {

constexpr int kBlock = 128;            // lazy-update block of the sweep / Cholesky panel
constexpr int kGridWaitLimitNs = 1000000000;  // 1 s: upper bound of any in-kernel wait

// NVTX range around one C-ABI call (host side: the call's argument checks
// and enqueue; the kernels it enqueues show up under it in a profiler's
// timeline).  NVTX is header-only; without a tool attached a push or pop is a
// check of a null hook and costs a few nanoseconds.
struct NvtxScope {
  explicit NvtxScope(const char* name) { nvtxRangePushA(name); }
  ~NvtxScope() { nvtxRangePop(); }
  NvtxScope(const NvtxScope&) = delete;
  NvtxScope& operator=(const NvtxScope&) = delete;
};

// ---- device-side index checks (debug builds)
// Built with -DGPTQ_DEVICE_CHECKS (libgptq_b200_debug.so), the kernels that
// index with caller-supplied arrays (a group index g_idx, a permutation)
// test every such index before they use it; an index out of range is not
// used (the value it would have produced is left 0) and its kind is OR-ed
// into a per-translation-unit device word that gptq_device_checks reads.
// In release builds index_ok is a constant true and costs nothing.
enum : uint32_t { kCheckGroupIndex = 1u, kCheckPermutation = 2u };
namespace {
#ifdef GPTQ_DEVICE_CHECKS
__device__ uint32_t g_dev_checks;
#endif
__device__ __forceinline__ bool index_ok(int64_t i, int64_t lim, uint32_t what) {
#ifdef GPTQ_DEVICE_CHECKS
  if (i >= 0 && i < lim) return true;
  atomicOr(&g_dev_checks, what);
  return false;
#else
  (void)i;
  (void)lim;
  (void)what;
  return true;
#endif
}
// Host: this translation unit's recorded checks, then cleared (0 in release
// builds).  Synchronous.
inline uint32_t take_unit_device_checks() {
#ifdef GPTQ_DEVICE_CHECKS
  uint32_t v = 0, z = 0;
  if (cudaMemcpyFromSymbol(&v, g_dev_checks, sizeof(v)) != cudaSuccess) return ~0u;
  if (cudaMemcpyToSymbol(g_dev_checks, &z, sizeof(z)) != cudaSuccess) return ~0u;
  return v;
#else
  return 0u;
#endif
}
}  // namespace
uint32_t take_device_checks_pack();
uint32_t take_device_checks_sweep();

int num_sms();
// 2-D TMA descriptor (128-byte swizzle, zero fill out of bounds) for a
// row-major rows x cols matrix of bf16 (bf16 = true) or fp32 elements with a
// row stride of ld elements; boxes of box_cols x box_rows.  Host only.
bool make_tma_2d(CUtensorMap* map, const void* base, bool bf16, int64_t rows, int64_t cols,
                 int64_t ld, uint32_t box_cols, uint32_t box_rows);
// Counts one kernel enqueued by this library (read by gptq_launch_count).
void note_launch();

// Events that order a caller-given side stream against the caller's stream
// for the duration of one call's enqueue: created by create(), destroyed by
// the destructor (CUDA frees an event whose recorded work is still pending
// once that work completes, so destroying right after the enqueue is safe).
// The library keeps no stream or event between calls.
struct SideEvents {
  cudaEvent_t ev[4] = {nullptr, nullptr, nullptr, nullptr};
  bool create();
  ~SideEvents();
};

// Test hook for the bounded waits (see gptq_set_wait_gate in gptq.h): the
// producer of every tensor-core kernel enqueued afterwards by the calling
// host thread first waits for *gate != 0, giving up after limit_ns.  With no
// gate set (the default) gate is null and limit_ns = kGridWaitLimitNs.
struct WaitGate {
  const int32_t* gate;
  uint64_t limit_ns;
};
WaitGate current_wait_gate();

// ---- Hessian (hessian_syrk.cu)
// H(upper incl. diagonal) += alpha * A_rows * B_rows^T over tokens [0, ntok),
// A and B are n x ntok bf16 with row stride ld (elements).  `flags`: device
// scratch of syrk_flag_bytes(n) bytes (256-byte aligned) for the ordered
// split-K reduction; zeroed by the launcher.
cudaError_t launch_syrk_bf16(float* H, int64_t n, const void* A, const void* B, int64_t ntok,
                             int64_t ld, float alpha, int32_t* info, void* flags,
                             cudaStream_t s);
size_t syrk_flag_bytes(int64_t n);
// fp32 X -> bf16 hi / lo parts (n x ntok, row stride ldo).
cudaError_t launch_split_bf16(const float* X, int64_t n, int64_t ntok, int64_t ldx, void* hi,
                              void* lo, int64_t ldo, cudaStream_t s);
// H[c][r] = H[r][c] for c > r.
cudaError_t launch_mirror_upper(float* H, int64_t n, cudaStream_t s);

// ---- Cholesky / inverse (cholesky.cu)
// side: a second stream for the look-ahead, or null (everything on s).
cudaError_t launch_cholesky_inverse(const float* H, int64_t n, float percdamp, int actorder,
                                    float* U, int32_t* perm, uint8_t* dead, int32_t* info,
                                    void* ws, cudaStream_t s, cudaStream_t side);
size_t cholesky_workspace_bytes(int64_t n);

// ---- sweep (sweep.cu)
cudaError_t launch_quantize_layer(const void* W, int wt, int64_t rows, int64_t n, const float* U,
                                  const int32_t* perm, const uint8_t* dead, int bits,
                                  int group_size, int sym, uint8_t* codes, float* scales,
                                  uint8_t* zeros, int32_t* g_idx, float* Wq, float* row_loss,
                                  void* ws, int32_t* info, cudaStream_t s, cudaStream_t side);
size_t quantize_workspace_bytes(int64_t rows, int64_t n);
// out[i] = a[i] / b[i] by the sweep's division routine (fdiv.cuh)
cudaError_t launch_selftest_division(const float* a, const float* b, int64_t count, float* out,
                                     cudaStream_t s);

// ---- storage (pack.cu)
cudaError_t launch_pack_int4(const uint8_t* codes, int64_t rows, int64_t n, uint32_t* out,
                             cudaStream_t s);
cudaError_t launch_pack_int3(const uint8_t* codes, int64_t rows, int64_t n, uint32_t* out,
                             cudaStream_t s);
// y (batch x rows fp32) = x (batch x n, bf16 or fp32) w_hat^T, w_hat dequantized on the fly;
// with perm, column k of the packed rows multiplies x[perm[k]].
cudaError_t launch_dequant_matvec(const uint32_t* packed, int bits, int64_t rows, int64_t n,
                                  const float* scales, const uint8_t* zeros, int group_size,
                                  int64_t n_groups, const int32_t* g_idx, const int32_t* perm,
                                  const void* x, int x_bf16, int64_t batch, float* y,
                                  void* ws, cudaStream_t s);
// scratch of launch_dequant_matvec: x re-laid out as batch x n bf16
size_t dequant_matvec_workspace_bytes(int64_t batch, int64_t n);
// dst[r][k] = src[r][perm[k]] (rows x n bytes)
cudaError_t launch_gather_columns_u8(const uint8_t* src, int64_t rows, int64_t n,
                                     const int32_t* perm, uint8_t* dst, cudaStream_t s);

// ---- Hadamard rotation (hadamard.cu)
// cols = false: out[r][c0 + j] = (1/sqrt(b)) sum_i H_b[j][i] s[c0 + i] in[r][c0 + i]
//               for a = rows, b_ = n (row stride ld_in / ld_out elements);
// cols = true:  the same along the first axis of an n x ntok matrix (a = n,
//               b_ = ntok).  block in {32, ..., 1024}, n % block == 0.
cudaError_t launch_hadamard(bool cols, int block, int in_bf16, int out_bf16, const void* in,
                            int64_t ld_in, void* out, int64_t ld_out, int64_t a, int64_t b_,
                            const float* signs, cudaStream_t s);
cudaError_t launch_dequant(const uint32_t* packed, int bits, int64_t rows, int64_t n,
                           const float* scales, const uint8_t* zeros, int group_size,
                           int64_t n_groups, const int32_t* g_idx, void* out, int out_bf16,
                           cudaStream_t s);

}  // namespace gptq
