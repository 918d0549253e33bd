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
#include "fdiv.cuh"
#include "stage.cuh"

namespace gptq {
namespace {

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct SweepWs {
  float* Wf;          // rows x n, sweep order; after the sweep holds w_hat
  float* Err_hi[2];   // rows x 128: a block's err terms, TF32 part (blocks alternate)
  float* Err_lo[2];   // rows x 128: remainder (err - Err_hi)
  uint8_t* codes_sw;  // rows x n, sweep order
  int32_t* pos;       // n: sweep position of each original column
  float* UT_hi;       // n x ldut: U^T, TF32 part (the lazy update's K-major operand)
  float* UT_lo;       // n x ldut: remainder
  int64_t ldut;
};

int64_t ut_ld(int64_t n) { return (n + 3) / 4 * 4; }

SweepWs carve(void* ws, int64_t rows, int64_t n) {
  char* p = static_cast<char*>(ws);
  SweepWs w;
  w.Wf = reinterpret_cast<float*>(p);
  p += align_up(sizeof(float) * rows * n, 256);
  for (int b = 0; b < 2; ++b) {
    w.Err_hi[b] = reinterpret_cast<float*>(p);
    p += align_up(sizeof(float) * rows * kBlock, 256);
    w.Err_lo[b] = reinterpret_cast<float*>(p);
    p += align_up(sizeof(float) * rows * kBlock, 256);
  }
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
    I.qkx = i1;
    I.nq = item_nq(i);
    I.mext = min(128, rows - 128 * i);
    I.cext_last = c1 - c0 - 128 * (I.nq - 1);
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
  if (k < n) pos[perm ? perm[k] : k] = k;
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
  for (int j = threadIdx.x; j < n; j += blockDim.x) wrow[j] = dead[j] ? 0.f : (float)src[j];
  __syncthreads();
  float mn = INFINITY, mx = -INFINITY;
  float* dst = Wf + (int64_t)r * n;
  for (int k = threadIdx.x; k < n; k += blockDim.x) {
    const float v = wrow[perm ? perm[k] : k];
    dst[k] = v;
    mn = fminf(mn, v);
    mx = fmaxf(mx, v);
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

// One block [i1, i1 + bsz) of the sweep.  kSweepLanes lanes per row (a
// "team"); lane q of a team holds block columns q, q + L, ..., q + 128 - L
// (slot s = column / L, L = kSweepLanes).  Column jj is rounded in every lane
// of the team, the owner lane's (jj % L) error term is broadcast inside the
// team, and each lane repairs its columns past jj with row jj of U's diagonal
// block.  The loop over jj is unrolled, so slots left of jj are skipped at
// compile time.  4 lanes per row is the measured choice at 4096 rows; 16
// lanes (8 slots each, 80 registers, twice the CTAs) computes the same
// results but was slower there (2.15 ms against 1.52 ms per layer at 4096 x
// 4096), its CTAs crowding out the concurrent far update.
// Shared memory holds the block of U as  Uq[jj][q][slot] = U[i1+jj][i1+L slot+q]
// (team-lane-major; row pitch kUqPitch floats per lane, chosen so the 16-byte
// float4 reads of the 8 lanes of a phase hit distinct banks), plus 1/U_jj and
// 1/(2 U_jj^2).
//   GS = 0:   per-row ruler (already in scales / zeros)
//   GS = 128: groups of a multiple of 128 columns, fitted at a block start that
//             is a group start, from the current Wf
//   GS = 32, 64: groups inside the block, fitted on the current registers
constexpr int kSweepLanes = 4;                           // lanes per row (4 or 16)
constexpr int kSweepSlots = kBlock / kSweepLanes;        // columns per lane
constexpr int kSweepThreads = kSweepLanes == 4 ? 128 : 256;
constexpr int kUqPitch = kSweepLanes == 4 ? 36 : 12;     // floats per (jj, q)
constexpr int kUqRow = kSweepLanes * kUqPitch;           // floats per jj
constexpr size_t kSweepSmemBytes = sizeof(float) * (kBlock * kUqRow + 2 * kBlock);
static_assert(kSweepSlots % 4 == 0 && kUqPitch >= kSweepSlots, "sweep team layout");

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

template <int GS>
__global__ void __launch_bounds__(kSweepThreads) sweep_block_kernel(
    float* __restrict__ Wf, int rows, int n, const float* __restrict__ U, int i1, int bsz,
    float maxq, int sym, int gsize, int G, float* __restrict__ Err_hi, float* __restrict__ Err_lo,
    uint8_t* __restrict__ codes_sw, float* __restrict__ scales, uint8_t* __restrict__ zeros,
    float* __restrict__ row_loss) {
  constexpr int L = kSweepLanes, NS = kSweepSlots;
  extern __shared__ __align__(16) float smem[];
  float* Uq = smem;
  float* rd = smem + kBlock * kUqRow;
  float* hrd2 = rd + kBlock;
  stage_block_128<kSweepThreads>(
      U + (int64_t)i1 * n + i1, n, bsz, bsz, /*lower=*/false, (n % 4) == 0,
      [&](int a, int b, float v) { Uq[a * kUqRow + (b % L) * kUqPitch + (b / L)] = v; },
      [](int, int) { return 0.f; });
  __syncthreads();
  for (int i = threadIdx.x; i < kBlock; i += blockDim.x) {
    const float d = (i < bsz) ? Uq[i * kUqRow + (i % L) * kUqPitch + (i / L)] : 1.f;
    rd[i] = 1.f / d;
    hrd2[i] = 0.5f / (d * d);
  }
  __syncthreads();

  const int lane = threadIdx.x & 31;
  const int q = lane % L;
  const int r = (blockIdx.x * blockDim.x + threadIdx.x) / L;
  const bool active = r < rows;
  float* wrow = Wf + (int64_t)(active ? r : 0) * n + i1;
  float w[NS];
#pragma unroll
  for (int s = 0; s < NS; ++s) {
    const int c = L * s + q;
    w[s] = (active && c < bsz) ? wrow[c] : 0.f;
  }

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
#pragma unroll
      for (int s = 0; s < NS; ++s)
        if (L * s + q < bsz) {
          mn = fminf(mn, w[s]);
          mx = fmaxf(mx, w[s]);
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
  float e_out[NS];
  uint32_t cw[NS / 4];
#pragma unroll
  for (int s = 0; s < NS; ++s) e_out[s] = 0.f;
#pragma unroll
  for (int k = 0; k < NS / 4; ++k) cw[k] = 0u;
  float loss = 0.f;
  const float* uq_lane = Uq + q * kUqPitch;

#pragma unroll
  for (int s = 0; s < NS; ++s) {
#pragma unroll
  for (int k = 0; k < L; ++k) {
    // No early exit for a short last block: its columns past bsz hold 0 and
    // its U rows past bsz are 0 (with 1/U_jj = 1), so they round to the zero
    // point with no error and change nothing; keeping the 128 steps free of
    // branches lets the compiler overlap consecutive steps.
    const int jj = L * s + k;
    constexpr int kGS = (GS == 32 || GS == 64) ? GS : L;  // in-block group size
    if ((GS == 32 || GS == 64) && (jj % kGS) == 0) {
      // group [jj, jj + GS) of the block, current (repaired) values
      float mn = INFINITY, mx = -INFINITY;
#pragma unroll
      for (int s2 = s; s2 < s + kGS / L; ++s2)
        if (L * s2 + q < bsz) {
          mn = fminf(mn, w[s2]);
          mx = fmaxf(mx, w[s2]);
        }
      fit_ruler(team_min(mn), team_max(mx), maxq, sym, scale, zf);
      md = md_prepare(scale);
      if (active && q == 0 && jj < bsz) {  // groups past the last column do not exist
        const int g = (i1 + jj) / kGS;
        scales[(int64_t)r * G + g] = scale;
        zeros[(int64_t)r * G + g] = (uint8_t)zf;
      }
    }
    // every lane rounds its slot s; the owner's (q == jj % L) result is used
    const float x = w[s];
    float qv = rintf(md_div(x, md)) + zf;
    qv = fminf(fmaxf(qv, 0.f), maxq);
    const float wh = __fmul_rn(scale, qv - zf);
    const float e = x - wh;
    const float ev = e * rd[jj];
    const float err = __shfl_sync(0xffffffffu, ev, k, L);
    const float* urow = uq_lane + jj * kUqRow;
#pragma unroll
    for (int s4 = s >> 2; s4 < NS / 4; ++s4) {
      const float4 u = *reinterpret_cast<const float4*>(urow + 4 * s4);
      if (4 * s4 + 0 >= s) w[4 * s4 + 0] = fmaf(-err, u.x, w[4 * s4 + 0]);
      if (4 * s4 + 1 >= s) w[4 * s4 + 1] = fmaf(-err, u.y, w[4 * s4 + 1]);
      if (4 * s4 + 2 >= s) w[4 * s4 + 2] = fmaf(-err, u.z, w[4 * s4 + 2]);
      if (4 * s4 + 3 >= s) w[4 * s4 + 3] = fmaf(-err, u.w, w[4 * s4 + 3]);
    }
    const bool own = (q == k);
    w[s] = own ? wh : w[s];
    e_out[s] = own ? ev : e_out[s];
    loss = own ? fmaf(e * e, hrd2[jj], loss) : loss;
    cw[s >> 2] |= own ? (((uint32_t)qv) << (8 * (s & 3))) : 0u;
  }
  }

  if (active) {
    uint8_t* crow = codes_sw + (int64_t)r * n + i1;
    float* ehi = Err_hi + (int64_t)r * kBlock;
    float* elo = Err_lo + (int64_t)r * kBlock;
#pragma unroll
    for (int s = 0; s < NS; ++s) {
      const int c = L * s + q;
      if (c < bsz) {
        crow[c] = (uint8_t)((cw[s >> 2] >> (8 * (s & 3))) & 0xFFu);
        wrow[c] = w[s];
      }
      float h, l;
      tf32_split(e_out[s], h, l);
      ehi[c] = h;
      elo[c] = l;
    }
  }
  if (row_loss) {
#pragma unroll
    for (int o = 1; o < L; o <<= 1) loss += __shfl_xor_sync(0xffffffffu, loss, o);
    if (active && q == 0) row_loss[r] += loss;
  }
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
  for (int j = threadIdx.x; j < n; j += blockDim.x) {
    crow[j] = codes_sw[(int64_t)r * n + j];
    if (Wq) srow[j] = Wf[(int64_t)r * n + j];
  }
  __syncthreads();
  for (int c = threadIdx.x; c < n; c += blockDim.x) {
    const int k = pos[c];
    codes[(int64_t)r * n + c] = crow[k];
    if (Wq) Wq[(int64_t)r * n + c] = srow[k];
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
  return align_up(sizeof(float) * rows * n, 256) +
         4 * align_up(sizeof(float) * rows * kBlock, 256) + align_up((size_t)rows * n, 256) +
         align_up(sizeof(int32_t) * n, 256) + 2 * align_up(sizeof(float) * n * ut_ld(n), 256);
}

cudaError_t launch_quantize_layer(const void* W, int wt, int64_t rows64, int64_t n64,
                                  const float* U, const int32_t* perm, const uint8_t* dead,
                                  int bits, int group_size, int sym, uint8_t* codes,
                                  float* scales, uint8_t* zeros, int32_t* g_idx, float* Wq,
                                  float* row_loss, void* ws, cudaStream_t s) {
  const int rows = (int)rows64, n = (int)n64;
  SweepWs w = carve(ws, rows64, n64);
  const float maxq = (float)((1 << bits) - 1);
  const int per_row = group_size <= 0;
  const int G = per_row ? 1 : (n + group_size - 1) / group_size;
  const int gmode = per_row ? 0 : (group_size >= kBlock ? 1 : 2);
  cudaError_t e;

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
  const int sweep_ctas = (rows * kSweepLanes + kSweepThreads - 1) / kSweepThreads;
  const int sms = num_sms();

  // operands of the lazy update on the tensor cores; with a row stride that
  // is a multiple of 16 bytes the update lands in Wf by TMA reduce-add
  CUtensorMap mEh[2], mEl[2], mUh, mUl, mW;
  const bool reduce = (n % 4) == 0;
  if (n > kBlock) {
    ut_split_kernel<<<dim3((unsigned)((w.ldut + 31) / 32), (unsigned)((n + 31) / 32)), 256, 0, s>>>(
        U, n, w.ldut, w.UT_hi, w.UT_lo);
    note_launch();
    for (int b = 0; b < 2; ++b)
      if (!make_tma_2d(&mEh[b], w.Err_hi[b], false, rows, kBlock, kBlock, 32, 128) ||
          !make_tma_2d(&mEl[b], w.Err_lo[b], false, rows, kBlock, kBlock, 32, 128))
        return cudaErrorInvalidValue;
    if (!make_tma_2d(&mUh, w.UT_hi, false, n, n, w.ldut, 32, 128) ||
        !make_tma_2d(&mUl, w.UT_lo, false, n, n, w.ldut, 32, 128))
      return cudaErrorInvalidValue;
    if (reduce) {
      if (!make_tma_2d(&mW, w.Wf, false, rows, n, n, 32, 32)) return cudaErrorInvalidValue;
      if ((e = cudaFuncSetAttribute(panel_gemm2_kernel<SweepTrailItems, true>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)pg2_smem_bytes(true))) != cudaSuccess)
        return e;
    } else {
      mW = mUh;  // not read by the read-modify-write epilogue
      if ((e = cudaFuncSetAttribute(panel_gemm2_kernel<SweepTrailItems, false>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)pg2_smem_bytes(false))) != cudaSuccess)
        return e;
    }
  }
  auto trail = [&](int blk, int i1, int c0, int c1, int max_grid, cudaStream_t st) {
    const SweepTrailItems dec{w.Wf, rows, n, i1, c0, c1};
    int chunk = 1, units = 0;
    pg2_plan(dec, max_grid, chunk, units);
    const int grid = std::min(units, max_grid);
    const int eb = blk & 1;
    if (reduce)
      panel_gemm2_kernel<SweepTrailItems, true><<<grid, kPg2Threads, pg2_smem_bytes(true), st>>>(
          mEh[eb], mEl[eb], mUh, mUl, mW, mW, dec, chunk, units, nullptr, 0, nullptr);
    else
      panel_gemm2_kernel<SweepTrailItems, false><<<grid, kPg2Threads, pg2_smem_bytes(false), st>>>(
          mEh[eb], mEl[eb], mUh, mUl, mW, mW, dec, chunk, units, nullptr, 0, nullptr);
    note_launch();
  };

  // Look-ahead.  After block b is swept, only block b+1's columns are
  // updated on the caller's stream (the "near" update, which the next sweep
  // waits for); the update of every later column ("far") runs on the side
  // stream, on part of the SMs, while block b+1 is swept.  Each column block
  // still receives its updates in block order -- far(0), ..., far(c-2),
  // near(c-1) for block c -- because near(b) waits for far(b-1); the err
  // terms alternate between two buffers, and sweep(b+2) (after near(b+1),
  // after far(b)) is the next writer of far(b)'s buffer.
  SideStream side{};
  const bool lookahead = n > 2 * kBlock && side_stream(&side);
  std::unique_lock<std::mutex> side_guard(side_lock(), std::defer_lock);
  // SMs left to the far update: the sweep's CTAs (up to two per SM) keep the rest
  const int far_grid = std::max(sms / 4, sms - (sweep_ctas + 1) / 2);
  if (lookahead) {
    side_guard.lock();
    if ((e = cudaEventRecord(side.ev[0], s)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(side.s, side.ev[0], 0)) != cudaSuccess)
      return e;
  }
  bool far_pending = false;  // far(b-1) was issued and near(b) must wait for it
  for (int i1 = 0, blk = 0; i1 < n; i1 += kBlock, ++blk) {
    const int bsz = std::min(kBlock, n - i1);
    const int i2 = i1 + bsz;
    const int eb = blk & 1;
#define GPTQ_SWEEP_LAUNCH(GSV)                                                                 \
  sweep_block_kernel<GSV><<<sweep_ctas, kSweepThreads, us_smem, s>>>(                          \
      w.Wf, rows, n, U, i1, bsz, maxq, sym, group_size, G, w.Err_hi[eb], w.Err_lo[eb],         \
      w.codes_sw, scales, zeros, row_loss)
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
    if (i2 >= n) break;  // bsz == 128 below: only the last block is short
    if (!lookahead) {
      trail(blk, i1, i2, n, sms, s);
      continue;
    }
    const int near_end = std::min(i2 + kBlock, n);
    if (near_end < n) {
      // far(b) needs block b's err terms: fork after the sweep
      if ((e = cudaEventRecord(side.ev[0], s)) != cudaSuccess ||
          (e = cudaStreamWaitEvent(side.s, side.ev[0], 0)) != cudaSuccess)
        return e;
    }
    if (far_pending && (e = cudaStreamWaitEvent(s, side.ev[1], 0)) != cudaSuccess) return e;
    trail(blk, i1, i2, near_end, sms, s);
    far_pending = false;
    if (near_end < n) {
      trail(blk, i1, near_end, n, far_grid, side.s);
      if ((e = cudaEventRecord(side.ev[1], side.s)) != cudaSuccess) return e;
      far_pending = true;
    }
  }
  if (lookahead) {  // join: everything on the side stream precedes what follows on s
    if ((e = cudaEventRecord(side.ev[1], side.s)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(s, side.ev[1], 0)) != cudaSuccess)
      return e;
    side_guard.unlock();
  }
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

}  // namespace gptq
