// The GPTQ column sweep with lazy block updates.
//
// Page "GPTQ, with the code open":
//  * section "What quantization is, and why anyone bothers": the ruler
//    scale = (max - min) / (2^b - 1), zero point rounded to a whole tick,
//    w_hat = scale (q - zero);
//  * section "The repair rule" + "From one repair to a whole model": after
//    column j is rounded, the still-free columns move by
//    -(w - w_hat) / U[j][j] * U[j, j+1:] (the OBS update read off the rows of
//    the Cholesky factor); per-weight loss (w - w_hat)^2 / (2 U_jj^2); repairs
//    inside the current block of 128 columns at once, the rest deferred to
//    one product per block; per-row rulers fitted before any repair, drifted
//    weights clamped to the end ticks;
//  * section "Paper vs. code": a new ruler every group of columns, fitted
//    when the sweep reaches it; act-order; dead inputs zeroed.
//
// Data flow per layer (all fp32, IEEE division, round-half-to-even):
//   gather:    Wf = W[:, perm] with dead columns zeroed (sweep order);
//              per-row rulers when there are no groups
//   per block [i1, i2):  sweep_block (one warp per row, U's diagonal block in
//              shared memory) -> codes, rulers, Err = err terms of the block;
//              trailing: Wf[:, i2:] -= Err U[i1:i2, i2:]
//   unpermute: codes / Wq back to the original column order, g_idx.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>

#include "gptq_internal.cuh"
#include "panel_gemm.cuh"
#include "persist.cuh"
#include "fdiv.cuh"
#include "stage.cuh"

namespace gptq {
namespace {

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

constexpr int32_t kSweepInfoTimeout = -2;  // `info` value when a device wait gave up

// Two-level blocking for wide layers: the lazy update inside a super-block of
// kSuperCols columns is applied per 128-column block (K = 128), the update of
// the columns past the super-block once per super-block (K = kSuperCols), so
// those columns are read and written once per super-block instead of once
// per block.  Narrower layers use one level (the super-block is the block).
constexpr int kSuperCols = 1024;
constexpr int64_t kTwoLevelMinN = 8192;
int64_t super_cols(int64_t n) { return n >= kTwoLevelMinN ? kSuperCols : kBlock; }

struct SweepWs {
  float* Wf;          // rows x n, sweep order; after the sweep holds w_hat
  float* Err_hi[2];   // rows x S: a super-block's err terms, TF32 part (super-blocks alternate)
  float* Err_lo[2];   // rows x S: remainder (err - Err_hi)
  int64_t lde;        // S = super_cols(n)
  uint8_t* codes_sw;  // rows x n, sweep order
  int32_t* pos;       // n: sweep position of each original column
  float* UT_hi;       // n x ldut: U^T, TF32 part (the lazy update's K-major operand)
  float* UT_lo;       // n x ldut: remainder
  int64_t ldut;
};

int64_t ut_ld(int64_t n) { return (n + 3) / 4 * 4; }

// Layers narrower than the two-level width, with rows 16-byte aligned, are
// swept by the persistent kernel, which keeps every block's err terms.
bool use_persistent(int64_t n) { return n > kBlock && n < kTwoLevelMinN && n % 4 == 0; }
int64_t persist_lde(int64_t n) { return (n + kBlock - 1) / kBlock * kBlock; }
size_t persist_ctr_bytes(int64_t rows, int64_t n) {
  const int64_t RB = (rows + kBlock - 1) / kBlock, nb = persist_lde(n) / kBlock;
  return align_up(sizeof(uint32_t) * (size_t)(1 + RB + RB * nb), 256);
}
// bytes of the err-term region: two super-blocks (hi and lo) or, for the
// persistent sweep, every block (hi and lo)
size_t err_region_bytes(int64_t rows, int64_t n) {
  const size_t two = 4 * align_up(sizeof(float) * rows * super_cols(n), 256);
  const size_t all = use_persistent(n) ? 2 * align_up(sizeof(float) * rows * persist_lde(n), 256)
                                       : 0;
  return std::max(two, all);
}

struct SweepWsExtra {
  uint32_t* ctr;  // counters of the persistent sweep
};

// S: the super-block width in use (at most super_cols(n), which sizes the
// workspace); persist: the err terms of every block instead of two super-blocks
SweepWs carve(void* ws, int64_t rows, int64_t n, int64_t S, bool persist = false,
              SweepWsExtra* extra = nullptr) {
  char* p = static_cast<char*>(ws);
  SweepWs w;
  w.Wf = reinterpret_cast<float*>(p);
  p += align_up(sizeof(float) * rows * n, 256);
  char* err = p;
  if (persist) {
    w.lde = persist_lde(n);
    w.Err_hi[0] = w.Err_hi[1] = reinterpret_cast<float*>(err);
    w.Err_lo[0] = w.Err_lo[1] =
        reinterpret_cast<float*>(err + align_up(sizeof(float) * rows * w.lde, 256));
  } else {
    w.lde = S;
    for (int b = 0; b < 2; ++b) {
      w.Err_hi[b] = reinterpret_cast<float*>(p);
      p += align_up(sizeof(float) * rows * w.lde, 256);
      w.Err_lo[b] = reinterpret_cast<float*>(p);
      p += align_up(sizeof(float) * rows * w.lde, 256);
    }
  }
  p = err + err_region_bytes(rows, n);
  if (extra) extra->ctr = reinterpret_cast<uint32_t*>(p);
  p += use_persistent(n) ? persist_ctr_bytes(rows, n) : 0;
  w.codes_sw = reinterpret_cast<uint8_t*>(p);
  p += align_up((size_t)rows * n, 256);
  w.pos = reinterpret_cast<int32_t*>(p);
  p += align_up(sizeof(int32_t) * n, 256);
  w.ldut = ut_ld(n);
  w.UT_hi = reinterpret_cast<float*>(p);
  p += align_up(sizeof(float) * n * w.ldut, 256);
  w.UT_lo = reinterpret_cast<float*>(p);
  return w;
}

// UT[a][b] = U[b][a], split into TF32 part and remainder; columns past n are 0.
__global__ void __launch_bounds__(256) ut_split_kernel(const float* __restrict__ U, int n,
                                                       int64_t ldut, float* __restrict__ hi,
                                                       float* __restrict__ lo) {
  __shared__ float T[32][33];
  const int bx = blockIdx.x, by = blockIdx.y;  // output tile: rows 32 by, cols 32 bx
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  for (int i = ty; i < 32; i += 8) {
    const int r = 32 * bx + i, c = 32 * by + tx;  // source U[r][c]
    T[i][tx] = (r < n && c < n) ? U[(int64_t)r * n + c] : 0.f;
  }
  __syncthreads();
  for (int i = ty; i < 32; i += 8) {
    const int a = 32 * by + i, b = 32 * bx + tx;  // destination UT[a][b] = U[b][a]
    if (a < n && b < ldut) {
      float h, l;
      tf32_split(T[tx][i], h, l);
      hi[(int64_t)a * ldut + b] = h;
      lo[(int64_t)a * ldut + b] = l;
    }
  }
}

// The lazy update  Wf[:, c0:c1] -= Err U[i1:i1+128, c0:c1]  as items for the
// tensor-core panel GEMM: P = Err (rows x 128), Q = U^T rows c0.. (columns
// i1..i1+128), C = Wf.  Item i = rows [128 i, 128 i + 128) of Wf, with its P
// block (the err terms) kept resident while the tiles of columns c0,
// c0 + 128, ... stream by.
struct SweepTrailItems {
  float* Wf;
  int rows, n, i1, c0, c1;
  int pk;  // column of the block's err terms in the super-block buffer
  __host__ __device__ int num_items() const { return (rows + 127) / 128; }
  __host__ __device__ int item_nq(int) const { return (c1 - c0 + 127) / 128; }
  __device__ PgItem item(int i) const {
    PgItem I;
    I.C0 = Wf + (int64_t)i * 128 * n + c0;
    I.ldc = n;
    I.cmap = 0;
    I.cx0 = c0;
    I.cy0 = 128 * i;
    I.prow = 128 * i;
    I.pkx = pk;
    I.qrow0 = c0;
    I.qkx = i1;
    I.nq = item_nq(i);
    I.mext = min(128, rows - 128 * i);
    I.cext_last = c1 - c0 - 128 * (I.nq - 1);
    I.nkb = kBlock / 32;
    return I;
  }
};

// The update past a finished super-block [s1, s1 + S):
//   Wf[:, c0:c1] -= Err_S U[s1:s1+S, c0:c1]   (K = S, stream_gemm_kernel)
// Item i = rows [128 i, 128 i + 128) of Wf; its tiles run over the columns.
struct SweepSuperItems {
  float* Wf;
  int rows, n, s1, S, c0, c1;
  __host__ __device__ int num_items() const { return (rows + 127) / 128; }
  __host__ __device__ int item_nq(int) const { return (c1 - c0 + 127) / 128; }
  __device__ PgItem item(int i) const {
    PgItem I;
    I.C0 = Wf + (int64_t)i * 128 * n + c0;
    I.ldc = n;
    I.cmap = 0;
    I.cx0 = c0;
    I.cy0 = 128 * i;
    I.prow = 128 * i;
    I.pkx = 0;
    I.qrow0 = c0;
    I.qkx = s1;
    I.nq = item_nq(i);
    I.mext = min(128, rows - 128 * i);
    I.cext_last = c1 - c0 - 128 * (I.nq - 1);
    I.nkb = S / 32;
    return I;
  }
};

// The ruler for values spanning [mn, mx]: range stretched to include 0
// ([-1, 1] when flat), scale = (xmax - xmin) / maxq, zero = rint(-xmin / scale).
// Symmetric ruler (opt-in): the range becomes [-m, m], m = max(-xmin, xmax),
// with the same scale formula and the zero point on the middle tick.
__device__ __forceinline__ void fit_ruler(float mn, float mx, float maxq, int sym, float& scale,
                                          float& zf) {
  float xmin = fminf(mn, 0.f), xmax = fmaxf(mx, 0.f);
  if (sym) {
    const float m = fmaxf(-xmin, xmax);
    xmin = -m;
    xmax = m;
  }
  if (xmin == 0.f && xmax == 0.f) {
    xmin = -1.f;
    xmax = 1.f;
  }
  scale = __fdiv_rn(xmax - xmin, maxq);
  zf = sym ? 0.5f * (maxq + 1.f) : rintf(__fdiv_rn(-xmin, scale));
}

__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__global__ void pos_kernel(const int32_t* __restrict__ perm, int n, int32_t* __restrict__ pos) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= n) return;
  const int pk = perm ? perm[k] : k;
  if (index_ok(pk, n, kCheckPermutation)) pos[pk] = k;
}

// One CTA per row: Wf[r][k] = dead[perm[k]] ? 0 : W[r][perm[k]]; per-row ruler
// (group_size <= 0) from the min / max of that row; row_loss[r] = 0.
template <typename T>
__global__ void __launch_bounds__(256) gather_w_kernel(
    const T* __restrict__ W, int n, const int32_t* __restrict__ perm,
    const uint8_t* __restrict__ dead, float* __restrict__ Wf, int per_row, float maxq, int sym,
    float* __restrict__ scales, uint8_t* __restrict__ zeros, float* __restrict__ row_loss) {
  extern __shared__ float wrow[];
  __shared__ float red[2][8];
  const int r = blockIdx.x;
  const T* src = W + (int64_t)r * n;
  // 16-byte loads of W (with the matching dead flags) and 4-column outputs
  // when the rows allow it (the same values either way)
  constexpr int VI = 16 / (int)sizeof(T);
  const bool vin = n % VI == 0 && reinterpret_cast<uintptr_t>(src) % 16 == 0 &&
                   reinterpret_cast<uintptr_t>(dead) % VI == 0;
  if (vin) {
    for (int j = threadIdx.x; j < n / VI; j += blockDim.x) {
      const uint4 raw = reinterpret_cast<const uint4*>(src)[j];
      const T* e = reinterpret_cast<const T*>(&raw);
#pragma unroll
      for (int i = 0; i < VI; ++i) wrow[VI * j + i] = dead[VI * j + i] ? 0.f : (float)e[i];
    }
  } else {
    for (int j = threadIdx.x; j < n; j += blockDim.x) wrow[j] = dead[j] ? 0.f : (float)src[j];
  }
  __syncthreads();
  float mn = INFINITY, mx = -INFINITY;
  float* dst = Wf + (int64_t)r * n;
  const bool vout = n % 4 == 0 && reinterpret_cast<uintptr_t>(dst) % 16 == 0 &&
                    (!perm || reinterpret_cast<uintptr_t>(perm) % 16 == 0);
  if (vout) {
    for (int k4 = threadIdx.x; k4 < n / 4; k4 += blockDim.x) {
      const int4 k = perm ? reinterpret_cast<const int4*>(perm)[k4]
                          : make_int4(4 * k4, 4 * k4 + 1, 4 * k4 + 2, 4 * k4 + 3);
      const float4 v = make_float4(index_ok(k.x, n, kCheckPermutation) ? wrow[k.x] : 0.f,
                                   index_ok(k.y, n, kCheckPermutation) ? wrow[k.y] : 0.f,
                                   index_ok(k.z, n, kCheckPermutation) ? wrow[k.z] : 0.f,
                                   index_ok(k.w, n, kCheckPermutation) ? wrow[k.w] : 0.f);
      reinterpret_cast<float4*>(dst)[k4] = v;
      mn = fminf(fminf(mn, fminf(v.x, v.y)), fminf(v.z, v.w));
      mx = fmaxf(fmaxf(mx, fmaxf(v.x, v.y)), fmaxf(v.z, v.w));
    }
  } else {
    for (int k = threadIdx.x; k < n; k += blockDim.x) {
      const int pk = perm ? perm[k] : k;
      const float v = index_ok(pk, n, kCheckPermutation) ? wrow[pk] : 0.f;
      dst[k] = v;
      mn = fminf(mn, v);
      mx = fmaxf(mx, v);
    }
  }
  if (per_row) {
    mn = warp_min(mn);
    mx = warp_max(mx);
    if ((threadIdx.x & 31) == 0) {
      red[0][threadIdx.x >> 5] = mn;
      red[1][threadIdx.x >> 5] = mx;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      for (int i = 1; i < 8; ++i) {
        mn = fminf(mn, red[0][i]);
        mx = fmaxf(mx, red[1][i]);
      }
      float scale, zf;
      fit_ruler(mn, mx, maxq, sym, scale, zf);
      scales[r] = scale;
      zeros[r] = (uint8_t)zf;
    }
  }
  if (row_loss && threadIdx.x == 0) row_loss[r] = 0.f;
}

// One block [i1, i1 + bsz) of the sweep.  A team of kSweepLanes = 4 lanes
// works one row; a CTA of 128 threads holds 32 rows.
//
// The CTA stages U's 128 x 128 diagonal block and its rows' 128 columns of
// Wf in shared memory.  The block is swept in sub-blocks of kSub = 16
// columns: lane q of a team loads columns q, q + 4, q + 8, q + 12 of the
// sub-block into registers, and the 16 column steps run fully unrolled:
// every lane of the team rounds the step's column itself (its value is
// carried from step to step; the owner of the column after next sends it
// one step ahead), and each lane repairs its later columns of the
// sub-block.  Then the sub-block's 16 error terms
// (all lanes hold them) update the rest of the block in shared memory, lane
// q taking the 4-column chunks q, q + 4, ... (a rolled rank-16 update).
// Every column receives fmaf(-err_j, U[j][c], w) for j = 0, 1, ... in column
// order, the same operations in the same order as one repair per column
// step.  The sub-block loop is rolled, so the code stays small enough for
// the instruction caches (a fully unrolled 128-step sweep does not fit them).
//   GS = 0:   per-row ruler (already in scales / zeros)
//   GS = 128: groups of a multiple of 128 columns, fitted at a block start that
//             is a group start, from the current Wf
//   GS = 32, 64: groups inside the block, fitted on the current values
// Columns past bsz (a short last block) hold 0 and their U rows are 0 with
// 1/U_jj = 1: they round to the zero point with no error and change nothing.
constexpr int kSweepLanes = 4;                          // lanes per row (a team)
constexpr int kSweepThreads = 128;
constexpr int kSweepRows = kSweepThreads / kSweepLanes; // rows per CTA
constexpr int kSub = 16;                                // columns per unrolled sub-block
constexpr int kSubSlots = kSub / kSweepLanes;           // columns per lane in a sub-block
constexpr int kWbPitch = 132;                           // floats per row of the staged W block
constexpr int kCbPitch = kBlock + 16;                   // bytes per row of the staged codes
// Ud [128][128] | Wb, Eb [32][kWbPitch] | rd, hrd2 [128] | Cb [32][kCbPitch] (bytes)
constexpr size_t kSweepSmemBytes =
    sizeof(float) * (kBlock * kBlock + 2 * kSweepRows * kWbPitch + 2 * kBlock) +
    kSweepRows * kCbPitch;

__device__ __forceinline__ float team_min(float v) {
#pragma unroll
  for (int o = 1; o < kSweepLanes; o <<= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float team_max(float v) {
#pragma unroll
  for (int o = 1; o < kSweepLanes; o <<= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Issues (does not wait for) the 16-byte async copies of U's diagonal block
// [i1, i1 + 128)^2 into the body's Ud (n a multiple of 4; 0 past bsz).
__device__ __forceinline__ void sweep_stage_u(float* smem, int tid, const float* __restrict__ U,
                                              int n, int i1, int bsz) {
  const float* us = U + (int64_t)i1 * n + i1;
  for (int f = tid; f < kBlock * kBlock / 4; f += kSweepThreads) {
    const int a = f >> 5, c = (f & 31) * 4;
    const bool ok = a < bsz && c < bsz;
    ptx::cp_async_16z(smem + a * kBlock + c, ok ? us + (int64_t)a * n + c : us, ok ? 16 : 0);
  }
}

// The sweep of one block by threads 0 .. kSweepThreads - 1 of a CTA, for
// rows [r0, r0 + kSweepRows): `smem` holds kSweepSmemBytes, `bar` is the
// barrier they synchronise on (0: __syncthreads, else a named barrier of
// kSweepThreads threads).  Shared by the one-block kernel and the persistent
// sweep; the latter issues the copies of U's block itself (u_issued, n a
// multiple of 4) before it waits for the block's columns to be up to date.
template <int GS>
__device__ __forceinline__ void sweep_block_body(
    float* smem, int tid, int r0, int bar, float* __restrict__ Wf, int rows, int n,
    const float* __restrict__ U, int i1, int bsz, float maxq, int sym, int gsize, int G,
    float* __restrict__ Err_hi, float* __restrict__ Err_lo, int lde,
    uint8_t* __restrict__ codes_sw, float* __restrict__ scales, uint8_t* __restrict__ zeros,
    float* __restrict__ row_loss, bool u_issued = false) {
  constexpr int L = kSweepLanes, NS = kSubSlots;
  auto sync = [bar]() {
    if (bar == 0)
      __syncthreads();
    else
      ptx::named_bar_sync(bar, kSweepThreads);
  };
  float* Ud = smem;                       // [128][128]  U[i1 + a][i1 + b], 0 past bsz
  float* Wb = Ud + kBlock * kBlock;       // [32][kWbPitch]  this CTA's rows of the block; w_hat
  float* Eb = Wb + kSweepRows * kWbPitch; // [32][kWbPitch]  their error terms
  float* rd = Eb + kSweepRows * kWbPitch; // [128]  1 / U_jj
  float* hrd2 = rd + kBlock;              // [128]  1 / (2 U_jj^2)
  uint8_t* Cb = reinterpret_cast<uint8_t*>(hrd2 + kBlock);  // [32][kCbPitch]  their codes
  const int vr = min(kSweepRows, rows - r0);
  if ((n % 4) == 0) {
    // 16-byte async copies, all in flight at once; bsz is a multiple of 4 here
    const float* ws = Wf + (int64_t)r0 * n + i1;
    if (!u_issued) sweep_stage_u(smem, tid, U, n, i1, bsz);
    for (int f = tid; f < kSweepRows * kBlock / 4; f += kSweepThreads) {
      const int a = f >> 5, c = (f & 31) * 4;
      const bool ok = a < vr && c < bsz;
      ptx::cp_async_16z(Wb + a * kWbPitch + c, ok ? ws + (int64_t)a * n + c : ws, ok ? 16 : 0);
    }
    ptx::cp_async_wait_all();
  } else {
    stage_block_128<kSweepThreads>(
        U + (int64_t)i1 * n + i1, n, bsz, bsz, /*lower=*/false, false,
        [&](int a, int b, float v) { Ud[a * kBlock + b] = v; }, [](int, int) { return 0.f; });
    for (int f = tid; f < kSweepRows * kBlock; f += kSweepThreads) {
      const int a = f >> 7, c = f & 127;
      Wb[a * kWbPitch + c] = (a < vr && c < bsz) ? Wf[(int64_t)(r0 + a) * n + i1 + c] : 0.f;
    }
  }
  sync();
  for (int i = tid; i < kBlock; i += kSweepThreads) {
    const float d = (i < bsz) ? Ud[i * kBlock + i] : 1.f;
    rd[i] = 1.f / d;
    hrd2[i] = 0.5f / (d * d);
  }
  sync();

  const int lane = tid & 31;
  const int q = lane % L;                 // lane within the team
  const int rl = tid / L;                 // row within the CTA
  const int r = r0 + rl;
  const bool active = rl < vr;
  float* wrow = Wb + rl * kWbPitch;
  float scale = 1.f, zf = 0.f;
  if (GS == 0) {
    if (active) {
      scale = scales[r];
      zf = (float)zeros[r];
    }
  } else if (GS == 128) {
    const int g = i1 / gsize;
    if (i1 % gsize == 0) {
      float mn = INFINITY, mx = -INFINITY;
      for (int c = q; c < kBlock; c += L) {
        mn = fminf(mn, wrow[c]);
        mx = fmaxf(mx, wrow[c]);
      }
      const int end = min(i1 + gsize, n);
      if (active)
        for (int c = i1 + kBlock + q; c < end; c += L) {
          const float v = Wf[(int64_t)r * n + c];
          mn = fminf(mn, v);
          mx = fmaxf(mx, v);
        }
      fit_ruler(team_min(mn), team_max(mx), maxq, sym, scale, zf);
      if (active && q == 0) {
        scales[(int64_t)r * G + g] = scale;
        zeros[(int64_t)r * G + g] = (uint8_t)zf;
      }
    } else if (active) {
      scale = scales[(int64_t)r * G + g];
      zf = (float)zeros[(int64_t)r * G + g];
    }
  }
  // w / scale, correctly rounded, with the reciprocal of the scale computed
  // once per ruler (Markstein's method, fdiv.cuh)
  MDiv md = md_prepare(scale);
  float loss = 0.f;
  float* erow = Eb + rl * kWbPitch;
  uint8_t* crow = Cb + rl * kCbPitch;

#pragma unroll 1
  for (int c0 = 0; c0 < kBlock; c0 += kSub) {
    // this lane's columns c0 + L s + q of the sub-block
    float cur[NS];
#pragma unroll
    for (int s = 0; s < NS; ++s) cur[s] = wrow[c0 + L * s + q];
    constexpr int kGS = (GS == 32 || GS == 64) ? GS : kBlock;  // in-block group size
    if ((GS == 32 || GS == 64) && (c0 % kGS) == 0) {
      // the group [c0, c0 + GS) of the block, current (repaired) values
      float mn = INFINITY, mx = -INFINITY;
#pragma unroll
      for (int s = 0; s < NS; ++s) {
        mn = fminf(mn, cur[s]);
        mx = fmaxf(mx, cur[s]);
      }
      for (int c = c0 + kSub + q; c < c0 + kGS; c += L) {
        mn = fminf(mn, wrow[c]);
        mx = fmaxf(mx, wrow[c]);
      }
      fit_ruler(team_min(mn), team_max(mx), maxq, sym, scale, zf);
      md = md_prepare(scale);
      if (active && q == 0 && c0 < bsz) {  // groups past the last column do not exist
        const int g = (i1 + c0) / kGS;
        scales[(int64_t)r * G + g] = scale;
        zeros[(int64_t)r * G + g] = (uint8_t)zf;
      }
    }
    float ev_sub[kSub];   // the sub-block's error terms (every lane of the team)
    float e_own[NS];      // this lane's own columns' error terms
    uint32_t cw = 0u;     // this lane's own columns' codes, one byte each
    // Every lane of the team rounds the step's column itself, so the error
    // term needs no exchange: xk is column jj's current value, and xn is
    // column jj + 1's value before step jj's repair, which its owner sends
    // one step ahead (the send is off the chain of dependent steps).  Both
    // are the owner's register values bit for bit.
    float xk = wrow[c0];
    float xn = wrow[c0 + 1];
#pragma unroll
    for (int k = 0; k < kSub; ++k) {
      const int jj = c0 + k;
      const int s = k / L, ko = k % L;   // the step's slot, and its owner lane
      const float x = xk;
      float qv = rintf(md_div(x, md)) + zf;
      qv = fminf(fmaxf(qv, 0.f), maxq);
      const float wh = __fmul_rn(scale, qv - zf);
      const float e = x - wh;
      const float ev = e * rd[jj];
      ev_sub[k] = ev;
      const bool own = (q == ko);
      loss = own ? fmaf(e * e, hrd2[jj], loss) : loss;
      cur[s] = own ? wh : cur[s];
      e_own[s] = own ? ev : e_own[s];
      cw |= own ? (((uint32_t)qv) << (8 * s)) : 0u;
      const float* urow = Ud + jj * kBlock + c0;
      // the next column, repaired by this step: the chain to the next step
      if (k + 1 < kSub) xk = fmaf(-ev, urow[k + 1], xn);
      // repair this lane's later columns of the sub-block
#pragma unroll
      for (int s2 = s; s2 < NS; ++s2)
        if (s2 > s || q > ko) cur[s2] = fmaf(-ev, urow[L * s2 + q], cur[s2]);
      // column jj + 2 after this step's repair, from its owner
      if (k + 2 < kSub) xn = __shfl_sync(0xffffffffu, cur[(k + 2) / L], (k + 2) % L, L);
    }
    // the sub-block's results, staged for the block's coalesced write-out:
    // w_hat in place of the columns just swept (no later step reads them),
    // the error terms and the codes
#pragma unroll
    for (int s = 0; s < NS; ++s) {
      const int c = c0 + L * s + q;
      wrow[c] = cur[s];
      erow[c] = e_own[s];
      crow[c] = (uint8_t)((cw >> (8 * s)) & 0xFFu);
    }
    // rank-16 update of the block's later columns (shared memory), lane q
    // taking the 4-column chunks q, q + L, ...; all of a lane's chunks are
    // held in registers and updated together, step j by step j, so their
    // FMA chains run side by side
    constexpr int kMaxChunks = (kBlock - kSub) / (4 * L);
    const int nch = (kBlock - c0 - kSub) / (4 * L);   // the same for every lane
    float* wch = wrow + c0 + kSub + 4 * q;
    float4 w4[kMaxChunks];
#pragma unroll
    for (int i = 0; i < kMaxChunks; ++i)
      if (i < nch) w4[i] = *reinterpret_cast<const float4*>(wch + 4 * L * i);
#pragma unroll
    for (int j = 0; j < kSub; ++j) {
      const float ne = -ev_sub[j];
      const float* urow = Ud + (c0 + j) * kBlock + c0 + kSub + 4 * q;
#pragma unroll
      for (int i = 0; i < kMaxChunks; ++i) {
        if (i < nch) {
          const float4 u = *reinterpret_cast<const float4*>(urow + 4 * L * i);
          w4[i].x = fmaf(ne, u.x, w4[i].x);
          w4[i].y = fmaf(ne, u.y, w4[i].y);
          w4[i].z = fmaf(ne, u.z, w4[i].z);
          w4[i].w = fmaf(ne, u.w, w4[i].w);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < kMaxChunks; ++i)
      if (i < nch) *reinterpret_cast<float4*>(wch + 4 * L * i) = w4[i];
    __syncwarp();  // the team's chunk writes land before the next sub-block's loads
  }
  if (row_loss) {
#pragma unroll
    for (int o = 1; o < L; o <<= 1) loss += __shfl_xor_sync(0xffffffffu, loss, o);
    if (active && q == 0) row_loss[r] += loss;
  }
  // write-out, whole row segments at a time: w_hat into Wf and the codes
  // (columns < bsz), the error terms split into TF32 part and remainder
  // (all 128 columns; those past bsz are 0)
  sync();
  for (int f = tid; f < kSweepRows * (kBlock / 4); f += kSweepThreads) {
    const int a = f / (kBlock / 4), c = (f % (kBlock / 4)) * 4;
    if (a >= vr) continue;
    const float4 e4 = *reinterpret_cast<const float4*>(Eb + a * kWbPitch + c);
    float4 h4, l4;
    tf32_split(e4.x, h4.x, l4.x);
    tf32_split(e4.y, h4.y, l4.y);
    tf32_split(e4.z, h4.z, l4.z);
    tf32_split(e4.w, h4.w, l4.w);
    *reinterpret_cast<float4*>(Err_hi + (int64_t)(r0 + a) * lde + c) = h4;
    *reinterpret_cast<float4*>(Err_lo + (int64_t)(r0 + a) * lde + c) = l4;
    const float* wsrc = Wb + a * kWbPitch + c;
    float* wdst = Wf + (int64_t)(r0 + a) * n + i1 + c;
    if ((n % 4) == 0 && c + 4 <= bsz) {
      *reinterpret_cast<float4*>(wdst) = *reinterpret_cast<const float4*>(wsrc);
    } else {
      for (int i = 0; i < 4 && c + i < bsz; ++i) wdst[i] = wsrc[i];
    }
  }
  for (int f = tid; f < kSweepRows * (kBlock / 16); f += kSweepThreads) {
    const int a = f / (kBlock / 16), c = (f % (kBlock / 16)) * 16;
    if (a >= vr) continue;
    const uint8_t* csrc = Cb + a * kCbPitch + c;
    uint8_t* cdst = codes_sw + (int64_t)(r0 + a) * n + i1 + c;
    if ((n % 16) == 0 && c + 16 <= bsz) {
      *reinterpret_cast<uint4*>(cdst) = *reinterpret_cast<const uint4*>(csrc);
    } else {
      for (int i = 0; i < 16 && c + i < bsz; ++i) cdst[i] = csrc[i];
    }
  }
}

template <int GS>
__global__ void __launch_bounds__(kSweepThreads) sweep_block_kernel(
    float* __restrict__ Wf, int rows, int n, const float* __restrict__ U, int i1, int bsz,
    float maxq, int sym, int gsize, int G, float* __restrict__ Err_hi, float* __restrict__ Err_lo,
    int lde, uint8_t* __restrict__ codes_sw, float* __restrict__ scales,
    uint8_t* __restrict__ zeros, float* __restrict__ row_loss) {
  extern __shared__ __align__(16) float smem[];
  sweep_block_body<GS>(smem, threadIdx.x, blockIdx.x * kSweepRows, 0, Wf, rows, n, U, i1, bsz,
                       maxq, sym, gsize, G, Err_hi, Err_lo, lde, codes_sw, scales, zeros,
                       row_loss);
}

// ===========================================================================
// The persistent sweep (layers narrower than the two-level width): one
// launch runs every block's sweep and every lazy update of a layer.
//
// The columns of block b's err terms go to the later 128-column tiles in two
// parts: the "near" tiles [b + 1, b + 1 + nw(b)) -- the next block, or the
// whole next group when a group ruler wider than a block starts there -- and
// the "far" tiles past them.  One CTA per SM takes tasks from a global
// counter in a fixed order in which every task comes after the tasks it
// depends on (so a CTA that waits, waits for a task some running CTA has
// already taken, and the waits end).  For each block s:
//   S(R, h, s)   the sweep of block s for 64 rows (half h of 128-row block R),
//                two 32-row slices at once on the CTA's first 256 threads
//   F(s - 1)     the far update by block s - 1 (chunks of up to kSpChunk
//                tiles), which runs on the SMs the sweep leaves free
//   N(s)         the near update by block s
// A 128-row block R keeps two kinds of counters in global memory: sweep
// tasks done (kSpSlices per block) and, per tile, blocks applied.  S(R, ., s)
// waits until tile s (and, at the start of a group wider than a block, every
// tile of the group) has received blocks 0 .. s - 1; an update by block b of
// tile c waits until block b is swept for all of R's rows and tile c has
// received blocks 0 .. b - 1.  So every tile gets its updates in block order
// and the result is the same bit for bit as the launch-by-launch form.
// Updates are the panel GEMM's rank-128 step on the tensor cores (P = the
// block's err terms, Q = U^T, C = Wf by TMA reduce-add).  All waits are
// bounded; writes are published with release stores after the proxy and
// memory fences, and read after acquire loads and a proxy fence.
// ===========================================================================
constexpr int kSpGroups = 2;                    // 32-row slices a sweep task runs at once
constexpr int kSpSlices = kBlock / (kSweepRows * kSpGroups);  // sweep tasks per row block, block
constexpr int kSpChunk = 4;                     // tiles per update task at most
static_assert(kSweepSmemBytes % 16 == 0 &&
                  kSpGroups * kSweepSmemBytes <= pg2_smem_bytes(true) - 1024 - 256,
              "a sweep task's slices reuse the update's shared memory");
static_assert(kSpGroups * kSweepThreads <= kPg2Threads, "one 128-thread group per slice");

struct SweepPersistArgs {
  float* Wf;
  int rows, n;
  const float* U;
  float maxq;
  int sym, gsize, G;
  int gw;     // tiles of a group ruler wider than a block (else 1)
  float* Eh;  // rows x lde: every block's err terms, TF32 part
  float* El;  // remainder
  int lde;
  uint8_t* codes_sw;
  float* scales;
  uint8_t* zeros;
  float* row_loss;
  uint32_t* ctr;  // [0] next task, [1 + R] sweep tasks done, [1 + RB + R nb + c] blocks applied
  int RB, nb;
  int32_t* info;
  const int32_t* gate;
  uint64_t limit_ns;
};

struct SpTask {
  int kind;  // 0 sweep, 1 update
  int R, s;  // row block; block (sweep) or the err terms' block (update)
  int slice;
  int c0, c1;  // update: tiles [c0, c1)
};

// near tiles of block b: [b + 1, b + 1 + sp_near(a, b))
__host__ __device__ inline int sp_near(const SweepPersistArgs& a, int b) {
  const int w = (a.gw > 1 && (b + 1) % a.gw == 0) ? a.gw : 1;
  return max(0, min(w, a.nb - b - 1));
}

struct SpStep {
  int nS, nF, nN;  // tasks per 128-row block of each kind
  int fs;          // first far tile of block s - 1
  int nwt;         // near tiles of block s
};

__host__ __device__ inline SpStep sp_step(const SweepPersistArgs& a, int s) {
  SpStep st;
  st.nS = kSpSlices;
  st.nwt = sp_near(a, s);
  st.nN = (st.nwt + kSpChunk - 1) / kSpChunk;
  st.fs = a.nb;
  st.nF = 0;
  if (s >= 1) {
    st.fs = s + sp_near(a, s - 1);
    st.nF = (max(0, a.nb - st.fs) + kSpChunk - 1) / kSpChunk;
  }
  return st;
}

__host__ __device__ inline int sp_total(const SweepPersistArgs& a) {
  int t = 0;
  for (int s = 0; s < a.nb; ++s) {
    const SpStep st = sp_step(a, s);
    t += a.RB * (st.nS + st.nF + st.nN);
  }
  return t;
}

__host__ __device__ inline SpTask sp_decode(const SweepPersistArgs& a, int t) {
  SpTask k;
  k.slice = 0;
  k.c0 = k.c1 = 0;
  for (int s = 0;; ++s) {
    const SpStep st = sp_step(a, s);
    const int nS = a.RB * st.nS, nF = a.RB * st.nF, nN = a.RB * st.nN;
    if (t < nS) {
      k.kind = 0;
      k.s = s;
      k.R = t / kSpSlices;
      k.slice = t % kSpSlices;
      return k;
    }
    t -= nS;
    if (t < nF + nN) {
      int chunk, base, end;
      k.kind = 1;
      if (t < nF) {   // the far chunks nearest to the sweep first
        k.R = t % a.RB;
        chunk = t / a.RB;
        k.s = s - 1;
        base = st.fs;
        end = a.nb;
      } else {
        t -= nF;
        k.R = t % a.RB;
        chunk = t / a.RB;
        k.s = s;
        base = s + 1;
        end = s + 1 + st.nwt;
      }
      k.c0 = base + chunk * kSpChunk;
      k.c1 = min(k.c0 + kSpChunk, end);
      return k;
    }
    t -= nF + nN;
  }
}

template <int GS>
__global__ void __launch_bounds__(kPg2Threads, 1)
    sweep_persist_kernel(const __grid_constant__ CUtensorMap mEh,
                         const __grid_constant__ CUtensorMap mEl,
                         const __grid_constant__ CUtensorMap mUh,
                         const __grid_constant__ CUtensorMap mUl,
                         const __grid_constant__ CUtensorMap mW, const SweepPersistArgs a) {
  extern __shared__ uint8_t smem_raw[];
  constexpr int32_t kTimeout = -2;
  PersistCta cta;
  cta.init(smem_raw, a.limit_ns);
  uint8_t* smem = cta.smem;
  volatile int* abort_flag = cta.abort_flag();
  const uint64_t kLimit = a.limit_ns;
  uint32_t* swept = a.ctr + 1;
  uint32_t* applied = a.ctr + 1 + a.RB;
  const int tid = threadIdx.x;
  if (tid == 0 && !ptx::gate_wait_bounded(a.gate, kLimit)) persist_abort(abort_flag, a.info, kTimeout);
  const int total = sp_total(a);

  while (true) {
    const int t = cta.next_task(a.ctr, total);
    if (t < 0) break;
    const SpTask k = sp_decode(a, t);
    if (k.kind == 0) {
      // ---------------------------------------------------------------- sweep task
      const int i1 = k.s * kBlock;
      const int bsz = min(kBlock, a.n - i1);
      const int grp = tid / kSweepThreads;   // slice of the task this thread sweeps
      const int r0 = k.R * kBlock + (k.slice * kSpGroups + grp) * kSweepRows;
      const bool mine = grp < kSpGroups && r0 < a.rows;
      float* gsm = reinterpret_cast<float*>(smem + grp * kSweepSmemBytes);
      // U's block does not depend on the wait: its copies go out first
      if (mine) sweep_stage_u(gsm, tid % kSweepThreads, a.U, a.n, i1, bsz);
      if (tid == 0) {
        // tile s has every earlier block's update; a group wider than a
        // block needs its other tiles as well
        int c_hi = k.s + 1;
        if (GS == 128 && a.gw > 1 && k.s % a.gw == 0) c_hi = min(a.nb, k.s + a.gw);
        bool ok = true;
        for (int c = k.s; c < c_hi && ok; ++c)
          ok = ptx::flag_wait_bounded(&applied[k.R * a.nb + c], (uint32_t)k.s, abort_flag, kLimit);
        if (!ok) persist_abort(abort_flag, a.info, kTimeout);
        fence_proxy_async_global();
      }
      __syncthreads();
      if (*abort_flag) {
        ptx::cp_async_wait_all();   // this thread's copies land before the CTA leaves
        continue;
      }
      if (mine) {
        sweep_block_body<GS>(gsm, tid % kSweepThreads, r0, 1 + grp, a.Wf, a.rows, a.n, a.U, i1,
                             bsz, a.maxq, a.sym, a.gsize, a.G, a.Eh + i1, a.El + i1, a.lde,
                             a.codes_sw, a.scales, a.zeros, a.row_loss, /*u_issued=*/true);
        // this thread's writes (shared memory the next task's TMA loads
        // overwrite; Wf and the err terms other CTAs read by TMA) are ordered
        // before the async proxy's accesses
        asm volatile("fence.proxy.async;" ::: "memory");
      }
      __syncthreads();
      if (tid == 0) {
        __threadfence();
        atomicAdd(&swept[k.R], 1u);
      }
      continue;
    }
    // ------------------------------------------------------------------ update task
    PgItem I;
    I.C0 = a.Wf + (int64_t)k.R * kBlock * a.n + (int64_t)k.c0 * kBlock;
    I.ldc = a.n;
    I.cmap = 0;
    I.cx0 = k.c0 * kBlock;
    I.cy0 = k.R * kBlock;
    I.prow = k.R * kBlock;
    I.pkx = k.s * kBlock;
    I.qrow0 = k.c0 * kBlock;
    I.qkx = k.s * kBlock;
    I.nq = k.c1 - k.c0;
    I.mext = min(kBlock, a.rows - k.R * kBlock);
    I.cext_last = min(kBlock, a.n - (k.c1 - 1) * kBlock);
    I.nkb = kPgKBlocks;
    if (tid == 0) {
      // block s is swept for all of R's rows, and each tile has blocks 0 .. s - 1
      bool ok = ptx::flag_wait_bounded(&swept[k.R], (uint32_t)(kSpSlices * (k.s + 1)),
                                       abort_flag, kLimit);
      for (int c = k.c0; c < k.c1 && ok; ++c)
        ok = ptx::flag_wait_bounded(&applied[k.R * a.nb + c], (uint32_t)k.s, abort_flag, kLimit);
      if (!ok) persist_abort(abort_flag, a.info, kTimeout);
      fence_proxy_async_global();
    }
    __syncthreads();
    if (*abort_flag) continue;
    cta.update(I, mEh, mEl, mUh, mUl, mW, mW, a.info, kTimeout);
    __syncthreads();
    if (tid == 0 && !*abort_flag) {
      __threadfence();
      for (int c = k.c0; c < k.c1; ++c)
        ptx::st_release_gpu(&applied[k.R * a.nb + c], (uint32_t)(k.s + 1));
    }
  }
  cta.teardown();
}

// One CTA per row: codes[r][c] = codes_sw[r][pos[c]], Wq[r][c] = Wf[r][pos[c]].
__global__ void __launch_bounds__(256) unpermute_kernel(const uint8_t* __restrict__ codes_sw,
                                                        const float* __restrict__ Wf, int n,
                                                        const int32_t* __restrict__ pos,
                                                        uint8_t* __restrict__ codes,
                                                        float* __restrict__ Wq) {
  extern __shared__ float srow[];
  uint8_t* crow = reinterpret_cast<uint8_t*>(srow + (Wq ? n : 0));
  const int r = blockIdx.x;
  const uint8_t* csrc = codes_sw + (int64_t)r * n;
  uint8_t* cdst = codes + (int64_t)r * n;
  float* wdst = Wq ? Wq + (int64_t)r * n : nullptr;
  // 16-byte staging and 4-column outputs when the rows allow it (same bytes)
  const bool vin = n % 16 == 0 && reinterpret_cast<uintptr_t>(csrc) % 16 == 0 &&
                   (!Wq || reinterpret_cast<uintptr_t>(Wf) % 16 == 0);
  const bool vout = n % 4 == 0 && reinterpret_cast<uintptr_t>(cdst) % 4 == 0 &&
                    reinterpret_cast<uintptr_t>(pos) % 16 == 0 &&
                    (!Wq || reinterpret_cast<uintptr_t>(wdst) % 16 == 0);
  if (vin) {
    for (int j = threadIdx.x; j < n / 16; j += blockDim.x) {
      reinterpret_cast<uint4*>(crow)[j] = reinterpret_cast<const uint4*>(csrc)[j];
      if (Wq)
        for (int q = 0; q < 4; ++q)
          reinterpret_cast<float4*>(srow)[4 * j + q] =
              reinterpret_cast<const float4*>(Wf + (int64_t)r * n)[4 * j + q];
    }
  } else {
    for (int j = threadIdx.x; j < n; j += blockDim.x) {
      crow[j] = csrc[j];
      if (Wq) srow[j] = Wf[(int64_t)r * n + j];
    }
  }
  __syncthreads();
  if (vout) {
    for (int c4 = threadIdx.x; c4 < n / 4; c4 += blockDim.x) {
      int4 k = reinterpret_cast<const int4*>(pos)[c4];
      // positions come from the caller's permutation (checked in debug builds)
      if (!index_ok(k.x, n, kCheckPermutation)) k.x = 0;
      if (!index_ok(k.y, n, kCheckPermutation)) k.y = 0;
      if (!index_ok(k.z, n, kCheckPermutation)) k.z = 0;
      if (!index_ok(k.w, n, kCheckPermutation)) k.w = 0;
      reinterpret_cast<uint32_t*>(cdst)[c4] = (uint32_t)crow[k.x] | ((uint32_t)crow[k.y] << 8) |
                                              ((uint32_t)crow[k.z] << 16) |
                                              ((uint32_t)crow[k.w] << 24);
      if (Wq)
        reinterpret_cast<float4*>(wdst)[c4] = make_float4(srow[k.x], srow[k.y], srow[k.z], srow[k.w]);
    }
  } else {
    for (int c = threadIdx.x; c < n; c += blockDim.x) {
      int k = pos[c];
      if (!index_ok(k, n, kCheckPermutation)) k = 0;
      cdst[c] = crow[k];
      if (Wq) wdst[c] = srow[k];
    }
  }
}

__global__ void gidx_kernel(const int32_t* __restrict__ pos, int n, int gsize,
                            int32_t* __restrict__ g_idx) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c < n) g_idx[c] = gsize > 0 ? pos[c] / gsize : 0;
}

template <typename F>
cudaError_t set_smem(F* f, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

}  // namespace

namespace {
__global__ void selftest_division_kernel(const float* __restrict__ a, const float* __restrict__ b,
                                         int64_t count, float* __restrict__ out) {
  const int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (i < count) out[i] = md_div(a[i], md_prepare(b[i]));
}
}  // namespace

cudaError_t launch_selftest_division(const float* a, const float* b, int64_t count, float* out,
                                     cudaStream_t s) {
  if (count <= 0) return cudaSuccess;
  selftest_division_kernel<<<(unsigned)((count + 255) / 256), 256, 0, s>>>(a, b, count, out);
  note_launch();
  return cudaGetLastError();
}

size_t quantize_workspace_bytes(int64_t rows, int64_t n) {
  return align_up(sizeof(float) * rows * n, 256) + err_region_bytes(rows, n) +
         (use_persistent(n) ? persist_ctr_bytes(rows, n) : 0) + align_up((size_t)rows * n, 256) +
         align_up(sizeof(int32_t) * n, 256) + 2 * align_up(sizeof(float) * n * ut_ld(n), 256);
}

cudaError_t launch_quantize_layer(const void* W, int wt, int64_t rows64, int64_t n64,
                                  const float* U, const int32_t* perm, const uint8_t* dead,
                                  int bits, int group_size, int sym, uint8_t* codes,
                                  float* scales, uint8_t* zeros, int32_t* g_idx, float* Wq,
                                  float* row_loss, void* ws, int32_t* info, cudaStream_t s,
                                  cudaStream_t side_s) {
  const int rows = (int)rows64, n = (int)n64;
  // A group ruler wider than a block is fitted on all of the group's current
  // columns, so a group must not cross a super-block's end (the columns past
  // it get the super-block's updates only at its end): other group sizes use
  // one level.
  int64_t S64 = super_cols(n64);
  if (S64 > kBlock && group_size > kBlock && S64 % group_size != 0 && group_size % S64 != 0)
    S64 = kBlock;
  const bool persist = use_persistent(n64);
  SweepWsExtra extra{};
  SweepWs w = carve(ws, rows64, n64, S64, persist, &extra);
  const float maxq = (float)((1 << bits) - 1);
  const int per_row = group_size <= 0;
  const int G = per_row ? 1 : (n + group_size - 1) / group_size;
  const int gmode = per_row ? 0 : (group_size >= kBlock ? 1 : 2);
  cudaError_t e;

  if (info && (e = cudaMemsetAsync(info, 0, sizeof(int32_t), s)) != cudaSuccess) return e;
  pos_kernel<<<(n + 255) / 256, 256, 0, s>>>(perm, n, w.pos);
  note_launch();
  const size_t row_smem = sizeof(float) * (size_t)n;
  if (wt == GPTQ_BF16) {
    if ((e = set_smem(gather_w_kernel<__nv_bfloat16>, row_smem)) != cudaSuccess) return e;
    gather_w_kernel<__nv_bfloat16><<<rows, 256, row_smem, s>>>(
        static_cast<const __nv_bfloat16*>(W), n, perm, dead, w.Wf, per_row, maxq, sym, scales,
        zeros, row_loss);
    note_launch();
  } else {
    if ((e = set_smem(gather_w_kernel<float>, row_smem)) != cudaSuccess) return e;
    gather_w_kernel<float><<<rows, 256, row_smem, s>>>(static_cast<const float*>(W), n, perm,
                                                       dead, w.Wf, per_row, maxq, sym, scales,
                                                       zeros, row_loss);
    note_launch();
  }

  const size_t us_smem = kSweepSmemBytes;
  if ((e = set_smem(sweep_block_kernel<0>, us_smem)) != cudaSuccess) return e;
  if ((e = set_smem(sweep_block_kernel<128>, us_smem)) != cudaSuccess) return e;
  if ((e = set_smem(sweep_block_kernel<32>, us_smem)) != cudaSuccess) return e;
  if ((e = set_smem(sweep_block_kernel<64>, us_smem)) != cudaSuccess) return e;
  const int sweep_ctas = (rows + kSweepRows - 1) / kSweepRows;
  const int sms = num_sms();

  if (persist) {
    // one launch for every block's sweep and every lazy update (the side
    // stream is not needed)
    ut_split_kernel<<<dim3((unsigned)((w.ldut + 31) / 32), (unsigned)((n + 31) / 32)), 256, 0, s>>>(
        U, n, w.ldut, w.UT_hi, w.UT_lo);
    note_launch();
    CUtensorMap pEh, pEl, pUh, pUl, pW;
    if (!make_tma_2d(&pEh, w.Err_hi[0], false, rows, w.lde, w.lde, 32, 128) ||
        !make_tma_2d(&pEl, w.Err_lo[0], false, rows, w.lde, w.lde, 32, 128) ||
        !make_tma_2d(&pUh, w.UT_hi, false, n, n, w.ldut, 32, 128) ||
        !make_tma_2d(&pUl, w.UT_lo, false, n, n, w.ldut, 32, 128) ||
        !make_tma_2d(&pW, w.Wf, false, rows, n, n, 32, 32))
      return cudaErrorInvalidValue;
    if ((e = cudaMemsetAsync(extra.ctr, 0, persist_ctr_bytes(rows64, n64), s)) != cudaSuccess)
      return e;
    const WaitGate pg = current_wait_gate();
    SweepPersistArgs a;
    a.Wf = w.Wf;
    a.rows = rows;
    a.n = n;
    a.U = U;
    a.maxq = maxq;
    a.sym = sym;
    a.gsize = group_size;
    a.G = G;
    a.gw = gmode == 1 ? group_size / kBlock : 1;
    a.Eh = w.Err_hi[0];
    a.El = w.Err_lo[0];
    a.lde = (int)w.lde;
    a.codes_sw = w.codes_sw;
    a.scales = scales;
    a.zeros = zeros;
    a.row_loss = row_loss;
    a.ctr = extra.ctr;
    a.RB = (rows + kBlock - 1) / kBlock;
    a.nb = (int)(w.lde / kBlock);
    a.info = info;
    a.gate = pg.gate;
    a.limit_ns = pg.limit_ns;
    const int grid = std::min(sms, sp_total(a));
    const size_t smem = pg2_smem_bytes(true);
#define GPTQ_PERSIST_LAUNCH(GSV)                                                             \
  if ((e = cudaFuncSetAttribute(sweep_persist_kernel<GSV>,                                  \
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != \
      cudaSuccess)                                                                          \
    return e;                                                                               \
  sweep_persist_kernel<GSV><<<grid, kPg2Threads, smem, s>>>(pEh, pEl, pUh, pUl, pW, a)
    if (gmode == 0) {
      GPTQ_PERSIST_LAUNCH(0);
    } else if (gmode == 1) {
      GPTQ_PERSIST_LAUNCH(128);
    } else if (group_size == 32) {
      GPTQ_PERSIST_LAUNCH(32);
    } else {
      GPTQ_PERSIST_LAUNCH(64);
    }
#undef GPTQ_PERSIST_LAUNCH
    note_launch();
  } else {
  // operands of the lazy update on the tensor cores; with a row stride that
  // is a multiple of 16 bytes the update lands in Wf by TMA reduce-add
  const int S = (int)w.lde;  // super-block columns (kBlock: one level)
  CUtensorMap mEh[2], mEl[2], mUh, mUl, mW;
  const bool reduce = (n % 4) == 0;
  if (n > kBlock) {
    ut_split_kernel<<<dim3((unsigned)((w.ldut + 31) / 32), (unsigned)((n + 31) / 32)), 256, 0, s>>>(
        U, n, w.ldut, w.UT_hi, w.UT_lo);
    note_launch();
    for (int b = 0; b < 2; ++b)
      if (!make_tma_2d(&mEh[b], w.Err_hi[b], false, rows, S, S, 32, 128) ||
          !make_tma_2d(&mEl[b], w.Err_lo[b], false, rows, S, S, 32, 128))
        return cudaErrorInvalidValue;
    if (!make_tma_2d(&mUh, w.UT_hi, false, n, n, w.ldut, 32, 128) ||
        !make_tma_2d(&mUl, w.UT_lo, false, n, n, w.ldut, 32, 128))
      return cudaErrorInvalidValue;
    if (reduce) {
      if (!make_tma_2d(&mW, w.Wf, false, rows, n, n, 32, 32)) return cudaErrorInvalidValue;
    } else {
      mW = mUh;  // not read by the read-modify-write epilogue
    }
    if ((e = cudaFuncSetAttribute(reduce ? (const void*)panel_gemm2_kernel<SweepTrailItems, true>
                                         : (const void*)panel_gemm2_kernel<SweepTrailItems, false>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)pg2_smem_bytes(reduce))) != cudaSuccess)
      return e;
    if (S > kBlock &&
        (e = cudaFuncSetAttribute(reduce ? (const void*)stream_gemm_kernel<SweepSuperItems, true>
                                         : (const void*)stream_gemm_kernel<SweepSuperItems, false>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)sg_smem_bytes(reduce))) != cudaSuccess)
      return e;
  }
  const WaitGate wg = current_wait_gate();
  // rank-128 update by block i1's err terms (column pk of buffer eb): columns [c0, c1)
  auto trail = [&](int eb, int i1, int pk, int c0, int c1, int max_grid, cudaStream_t st) {
    const SweepTrailItems dec{w.Wf, rows, n, i1, c0, c1, pk};
    int chunk = 1, units = 0;
    pg2_plan(dec, max_grid, chunk, units);
    const int grid = std::min(units, max_grid);
    if (reduce)
      panel_gemm2_kernel<SweepTrailItems, true><<<grid, kPg2Threads, pg2_smem_bytes(true), st>>>(
          mEh[eb], mEl[eb], mUh, mUl, mW, mW, dec, chunk, units, info, kSweepInfoTimeout,
          nullptr, wg.gate, wg.limit_ns);
    else
      panel_gemm2_kernel<SweepTrailItems, false><<<grid, kPg2Threads, pg2_smem_bytes(false), st>>>(
          mEh[eb], mEl[eb], mUh, mUl, mW, mW, dec, chunk, units, info, kSweepInfoTimeout,
          nullptr, wg.gate, wg.limit_ns);
    note_launch();
  };
  // the update past the super-block [s1, s1 + S) (all its err terms): columns [c0, c1)
  auto past = [&](int eb, int s1, int c0, int c1, int max_grid, cudaStream_t st) {
    if (S == kBlock) {
      trail(eb, s1, 0, c0, c1, max_grid, st);
      return;
    }
    const SweepSuperItems dec{w.Wf, rows, n, s1, S, c0, c1};
    const int units = sg_units(dec);
    const int grid = std::min(units, max_grid);
    if (reduce)
      stream_gemm_kernel<SweepSuperItems, true><<<grid, kPg2Threads, sg_smem_bytes(true), st>>>(
          mEh[eb], mEl[eb], mUh, mUl, mW, mW, dec, units, info, kSweepInfoTimeout, nullptr,
          wg.gate, wg.limit_ns);
    else
      stream_gemm_kernel<SweepSuperItems, false><<<grid, kPg2Threads, sg_smem_bytes(false), st>>>(
          mEh[eb], mEl[eb], mUh, mUl, mW, mW, dec, units, info, kSweepInfoTimeout, nullptr,
          wg.gate, wg.limit_ns);
    note_launch();
  };

  // Look-ahead (with a side stream).  After block b is swept, only the next
  // block's columns are updated on the caller's stream (the "near" update,
  // which the next sweep waits for); the update of every later column
  // ("far") runs on the side stream, on part of the SMs, while the next
  // block is swept.  Inside a super-block the updates are rank-128 and stop
  // at the super-block's end; after its last block, the update past it (all
  // its err terms at once) is split the same way.  Every column still
  // receives its updates in a fixed order -- each near update waits for the
  // far update issued before it -- so the result does not depend on how the
  // streams interleave.  The err terms of consecutive super-blocks go to two
  // buffers; the next writer of a buffer (the first sweep two super-blocks
  // on) runs after the caller's stream has waited for the last far update
  // that reads it.
  SideEvents side;
  const bool lookahead = n > 2 * kBlock && side_s != nullptr && side_s != s;
  if (lookahead && !side.create()) return cudaErrorMemoryAllocation;
  // SMs for the far updates, which run beside the next blocks' sweeps: what
  // one wave of the sweep's CTAs (two per SM) leaves, but at least half of
  // them -- on tall layers the far updates past a super-block are most of
  // the work, and a sweep that takes two waves costs less than starving them
  const int far_grid = std::max(sms / 2, sms - (sweep_ctas + 1) / 2);
  auto fork = [&]() -> cudaError_t {
    cudaError_t r = cudaEventRecord(side.ev[0], s);
    return r != cudaSuccess ? r : cudaStreamWaitEvent(side_s, side.ev[0], 0);
  };
  if (lookahead && (e = fork()) != cudaSuccess) return e;
  bool far_pending = false;   // a far update inside the super-block (ev[1]) is unwaited
  bool past_pending = false;  // a far update past a super-block (ev[2]) is unwaited
  bool last = false;
  for (int s1 = 0, sb = 0; s1 < n && !last; s1 += S, ++sb) {
    const int s2 = std::min(s1 + S, n);
    const int eb = sb & 1;
    for (int i1 = s1; i1 < s2; i1 += kBlock) {
      const int bsz = std::min(kBlock, n - i1);
      const int i2 = i1 + bsz;
      const int pk = i1 - s1;
#define GPTQ_SWEEP_LAUNCH(GSV)                                                                 \
  sweep_block_kernel<GSV><<<sweep_ctas, kSweepThreads, us_smem, s>>>(                          \
      w.Wf, rows, n, U, i1, bsz, maxq, sym, group_size, G, w.Err_hi[eb] + pk,                  \
      w.Err_lo[eb] + pk, S, w.codes_sw, scales, zeros, row_loss)
      if (gmode == 0)
        GPTQ_SWEEP_LAUNCH(0);
      else if (gmode == 1)
        GPTQ_SWEEP_LAUNCH(128);
      else if (group_size == 32)
        GPTQ_SWEEP_LAUNCH(32);
      else
        GPTQ_SWEEP_LAUNCH(64);
#undef GPTQ_SWEEP_LAUNCH
      note_launch();
      if (i2 >= n) {  // bsz == 128 below: only the last block is short
        last = true;
        break;
      }
      const bool inside = i2 < s2;        // more blocks of this super-block follow
      const int end = inside ? s2 : n;    // the columns this block's update reaches
      if (!lookahead) {
        if (inside)
          trail(eb, i1, pk, i2, end, sms, s);
        else
          past(eb, s1, i2, end, sms, s);
        continue;
      }
      // the near part is what the next sweep reads: the next block, or, when
      // the next block starts a group wider than a block, the whole group
      // (its ruler is fitted on all of the group's current columns)
      const int near_w = (gmode == 1 && i2 % group_size == 0) ? group_size : kBlock;
      const int near_end = std::min(i2 + near_w, end);
      if (near_end < end && (e = fork()) != cudaSuccess) return e;
      if (far_pending) {
        if ((e = cudaStreamWaitEvent(s, side.ev[1], 0)) != cudaSuccess) return e;
        far_pending = false;
      }
      if (past_pending) {
        if ((e = cudaStreamWaitEvent(s, side.ev[2], 0)) != cudaSuccess) return e;
        past_pending = false;
      }
      if (inside)
        trail(eb, i1, pk, i2, near_end, sms, s);
      else
        past(eb, s1, i2, near_end, sms, s);
      if (near_end < end) {
        if (inside) {
          trail(eb, i1, pk, near_end, end, far_grid, side_s);
          if ((e = cudaEventRecord(side.ev[1], side_s)) != cudaSuccess) return e;
          far_pending = true;
        } else {
          past(eb, s1, near_end, end, far_grid, side_s);
          if ((e = cudaEventRecord(side.ev[2], side_s)) != cudaSuccess) return e;
          past_pending = true;
        }
      }
    }
  }
  if (lookahead) {  // join: everything on the side stream precedes what follows on s
    if ((e = cudaEventRecord(side.ev[1], side_s)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(s, side.ev[1], 0)) != cudaSuccess)
      return e;
  }
  }  // one-block launches
  const size_t un_smem = (Wq ? sizeof(float) * (size_t)n : 0) + (size_t)n;
  if ((e = set_smem(unpermute_kernel, un_smem)) != cudaSuccess) return e;
  unpermute_kernel<<<rows, 256, un_smem, s>>>(w.codes_sw, w.Wf, n, w.pos, codes, Wq);
  note_launch();
  if (g_idx) {
    gidx_kernel<<<(n + 255) / 256, 256, 0, s>>>(w.pos, n, group_size, g_idx);
    note_launch();
  }
  return cudaGetLastError();
}

uint32_t take_device_checks_sweep() { return take_unit_device_checks(); }

}  // namespace gptq
