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

#include "gemm_f32.cuh"
#include "gptq_internal.cuh"

namespace gptq {
namespace {

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct SweepWs {
  float* Wf;          // rows x n, sweep order; after the sweep holds w_hat
  float* Err;         // rows x 128
  uint8_t* codes_sw;  // rows x n, sweep order
  int32_t* pos;       // n: sweep position of each original column
};

SweepWs carve(void* ws, int64_t rows, int64_t n) {
  char* p = static_cast<char*>(ws);
  SweepWs w;
  w.Wf = reinterpret_cast<float*>(p);
  p += align_up(sizeof(float) * rows * n, 256);
  w.Err = reinterpret_cast<float*>(p);
  p += align_up(sizeof(float) * rows * kBlock, 256);
  w.codes_sw = reinterpret_cast<uint8_t*>(p);
  p += align_up((size_t)rows * n, 256);
  w.pos = reinterpret_cast<int32_t*>(p);
  return w;
}

// The ruler for values spanning [mn, mx]: range stretched to include 0
// ([-1, 1] when flat), scale = (xmax - xmin) / maxq, zero = rint(-xmin / scale).
__device__ __forceinline__ void fit_ruler(float mn, float mx, float maxq, float& scale,
                                          float& zf) {
  float xmin = fminf(mn, 0.f), xmax = fmaxf(mx, 0.f);
  if (xmin == 0.f && xmax == 0.f) {
    xmin = -1.f;
    xmax = 1.f;
  }
  scale = __fdiv_rn(xmax - xmin, maxq);
  zf = rintf(__fdiv_rn(-xmin, scale));
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
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
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
    const uint8_t* __restrict__ dead, float* __restrict__ Wf, int per_row, float maxq,
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
      fit_ruler(mn, mx, maxq, scale, zf);
      scales[r] = scale;
      zeros[r] = (uint8_t)zf;
    }
  }
  if (row_loss && threadIdx.x == 0) row_loss[r] = 0.f;
}

// One block [i1, i1 + bsz) of the sweep.  One warp per row; lane l holds
// block columns l, l+32, l+64, l+96.  Column jj is rounded by its owner lane,
// the error term is broadcast, and every lane repairs its later columns with
// row jj of U's diagonal block (shared memory).
//   gmode 0: per-row ruler (already in scales / zeros)
//   gmode 1: groups of >= 128 columns (a multiple of 128): fitted at a block
//            start that is a group start, from the current Wf
//   gmode 2: groups of 32 or 64 columns inside the block
template <int GMODE>
__global__ void __launch_bounds__(256) sweep_block_kernel(
    float* __restrict__ Wf, int rows, int n, const float* __restrict__ U, int i1, int bsz,
    float maxq, int gsize, int G, float* __restrict__ Err, uint8_t* __restrict__ codes_sw,
    float* __restrict__ scales, uint8_t* __restrict__ zeros, float* __restrict__ row_loss) {
  extern __shared__ float Us[];  // [128][128]: U[i1 + a][i1 + b]
  for (int i = threadIdx.x; i < kBlock * kBlock; i += blockDim.x) {
    const int a = i / kBlock, b = i % kBlock;
    Us[i] = (a < bsz && b < bsz) ? U[(int64_t)(i1 + a) * n + i1 + b] : 0.f;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;

  for (int r = warp; r < rows; r += nwarps) {
    float* wrow = Wf + (int64_t)r * n + i1;
    float w[4];
#pragma unroll
    for (int s = 0; s < 4; ++s) w[s] = (lane + 32 * s < bsz) ? wrow[lane + 32 * s] : 0.f;

    float scale = 0.f, zf = 0.f;
    if (GMODE == 0) {
      scale = scales[r];
      zf = (float)zeros[r];
    } else if (GMODE == 1) {
      const int g = i1 / gsize;
      if (i1 % gsize == 0) {
        const int end = min(i1 + gsize, n);
        float mn = INFINITY, mx = -INFINITY;
        for (int c = i1 + lane; c < end; c += 32) {
          const float v = Wf[(int64_t)r * n + c];
          mn = fminf(mn, v);
          mx = fmaxf(mx, v);
        }
        fit_ruler(warp_min(mn), warp_max(mx), maxq, scale, zf);
        if (lane == 0) {
          scales[(int64_t)r * G + g] = scale;
          zeros[(int64_t)r * G + g] = (uint8_t)zf;
        }
      } else {
        scale = scales[(int64_t)r * G + g];
        zf = (float)zeros[(int64_t)r * G + g];
      }
    }

    float q_out[4] = {0.f, 0.f, 0.f, 0.f}, wq_out[4] = {0.f, 0.f, 0.f, 0.f},
          e_out[4] = {0.f, 0.f, 0.f, 0.f};
    float loss = 0.f;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      if (32 * s >= bsz) break;
      if (GMODE == 2 && (32 * s) % gsize == 0) {
        // group [32 s, 32 s + gsize) of the block, current (repaired) values
        float mn = INFINITY, mx = -INFINITY;
#pragma unroll
        for (int s2 = s; s2 < 4; ++s2) {
          if (32 * (s2 - s) < gsize && lane + 32 * s2 < bsz) {
            mn = fminf(mn, w[s2]);
            mx = fmaxf(mx, w[s2]);
          }
        }
        fit_ruler(warp_min(mn), warp_max(mx), maxq, scale, zf);
        if (lane == 0) {
          const int g = (i1 + 32 * s) / gsize;
          scales[(int64_t)r * G + g] = scale;
          zeros[(int64_t)r * G + g] = (uint8_t)zf;
        }
      }
#pragma unroll 4
      for (int l = 0; l < 32; ++l) {
        const int jj = 32 * s + l;
        if (jj >= bsz) break;
        float err = 0.f;
        if (lane == l) {
          const float x = w[s];
          float q = rintf(__fdiv_rn(x, scale)) + zf;
          q = fminf(fmaxf(q, 0.f), maxq);
          const float wh = __fmul_rn(scale, q - zf);
          const float e = x - wh;
          const float d = Us[jj * kBlock + jj];
          err = __fdiv_rn(e, d);
          loss += __fdiv_rn(e * e, 2.f * d * d);
          q_out[s] = q;
          wq_out[s] = wh;
          e_out[s] = err;
        }
        err = __shfl_sync(0xffffffffu, err, l);
        const float* urow = Us + jj * kBlock;
#pragma unroll
        for (int s2 = s; s2 < 4; ++s2) w[s2] = fmaf(-err, urow[32 * s2 + lane], w[s2]);
      }
    }
    uint8_t* crow = codes_sw + (int64_t)r * n + i1;
    float* erow = Err + (int64_t)r * kBlock;
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      const int c = lane + 32 * s;
      if (c < bsz) {
        crow[c] = (uint8_t)q_out[s];
        wrow[c] = wq_out[s];
      }
      erow[c] = e_out[s];
    }
    if (row_loss) {
      loss = warp_sum(loss);
      if (lane == 0) row_loss[r] += loss;
    }
  }
}

// Wf[:, i2:] -= Err(rows x K) * U[i1:i1+K, i2:]   (grid: col tiles x row tiles)
__global__ void __launch_bounds__(256) sweep_trailing_kernel(float* __restrict__ Wf, int rows,
                                                             int n, const float* __restrict__ U,
                                                             const float* __restrict__ Err, int i1,
                                                             int i2, int K) {
  __shared__ __align__(16) float sm[kTileSmemFloats];
  const int c0 = blockIdx.x * kTileM, r0 = blockIdx.y * kTileM;
  float* C = Wf + (int64_t)r0 * n + i2 + c0;
  const float* P = Err + (int64_t)r0 * kBlock;
  const float* Q = U + (int64_t)i1 * n + i2 + c0;
  tile_sub<false>(C, n, P, kBlock, Q, n, min(kTileM, rows - r0), min(kTileM, n - i2 - c0), K, sm);
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

size_t quantize_workspace_bytes(int64_t rows, int64_t n) {
  return align_up(sizeof(float) * rows * n, 256) + align_up(sizeof(float) * rows * kBlock, 256) +
         align_up((size_t)rows * n, 256) + align_up(sizeof(int32_t) * n, 256);
}

cudaError_t launch_quantize_layer(const void* W, int wt, int64_t rows64, int64_t n64,
                                  const float* U, const int32_t* perm, const uint8_t* dead,
                                  int bits, int group_size, uint8_t* codes, float* scales,
                                  uint8_t* zeros, int32_t* g_idx, float* Wq, float* row_loss,
                                  void* ws, cudaStream_t s) {
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
        static_cast<const __nv_bfloat16*>(W), n, perm, dead, w.Wf, per_row, maxq, scales, zeros,
        row_loss);
    note_launch();
  } else {
    if ((e = set_smem(gather_w_kernel<float>, row_smem)) != cudaSuccess) return e;
    gather_w_kernel<float><<<rows, 256, row_smem, s>>>(static_cast<const float*>(W), n, perm,
                                                       dead, w.Wf, per_row, maxq, scales, zeros,
                                                       row_loss);
    note_launch();
  }

  const size_t us_smem = sizeof(float) * kBlock * kBlock;
  if ((e = set_smem(sweep_block_kernel<0>, us_smem)) != cudaSuccess) return e;
  if ((e = set_smem(sweep_block_kernel<1>, us_smem)) != cudaSuccess) return e;
  if ((e = set_smem(sweep_block_kernel<2>, us_smem)) != cudaSuccess) return e;
  const int sweep_ctas = std::min((rows + 7) / 8, 3 * num_sms());
  for (int i1 = 0; i1 < n; i1 += kBlock) {
    const int bsz = std::min(kBlock, n - i1);
    const int i2 = i1 + bsz;
    if (gmode == 0)
      sweep_block_kernel<0><<<sweep_ctas, 256, us_smem, s>>>(
          w.Wf, rows, n, U, i1, bsz, maxq, group_size, G, w.Err, w.codes_sw, scales, zeros,
          row_loss);
    else if (gmode == 1)
      sweep_block_kernel<1><<<sweep_ctas, 256, us_smem, s>>>(
          w.Wf, rows, n, U, i1, bsz, maxq, group_size, G, w.Err, w.codes_sw, scales, zeros,
          row_loss);
    else
      sweep_block_kernel<2><<<sweep_ctas, 256, us_smem, s>>>(
          w.Wf, rows, n, U, i1, bsz, maxq, group_size, G, w.Err, w.codes_sw, scales, zeros,
          row_loss);
    note_launch();
    if (i2 < n) {
      dim3 grid((n - i2 + kTileM - 1) / kTileM, (rows + kTileM - 1) / kTileM);
      sweep_trailing_kernel<<<grid, 256, 0, s>>>(w.Wf, rows, n, U, w.Err, i1, i2, bsz);
      note_launch();
    }
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
