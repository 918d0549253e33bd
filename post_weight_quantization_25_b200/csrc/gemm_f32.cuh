// fp32 CUDA-core tile update shared by the Cholesky/inverse and the sweep's
// lazy block update: one 128 x 128 tile of C per 256-thread CTA,
//     C[m][c] -= sum_{t < K} P[m][t] * Q(t, c),
// with P row-major (t contiguous) and Q either K-major (Q(t,c) = Q[c][t]) or
// N-major (Q(t,c) = Q[t][c]).  Plain FFMA in fp32: both users need fp32
// accuracy (page "GPTQ, with the code open", section "Paper vs. code": TF32
// is switched off because the Cholesky chain needs full 32-bit precision).
#pragma once
#include <cstdint>

namespace gptq {

constexpr int kTileM = 128;
constexpr int kTileBK = 16;
constexpr int kTileLD = kTileM + 4;
constexpr int kTileSmemFloats = 2 * kTileBK * kTileLD;

// Rows of C/P at or past `mext`, and columns at or past `cext`, are neither
// read nor written.  K may be any value >= 0.  Must be called by all 256
// threads of the CTA; `smem` holds kTileSmemFloats floats.
template <bool Q_KMAJOR>
__device__ __forceinline__ void tile_sub(float* __restrict__ C, int64_t ldc,
                                         const float* __restrict__ P, int64_t ldp,
                                         const float* __restrict__ Q, int64_t ldq, int mext,
                                         int cext, int K, float* smem) {
  float* Ps = smem;                        // [kTileBK][kTileLD], Ps[t][m]
  float* Qs = smem + kTileBK * kTileLD;    // [kTileBK][kTileLD], Qs[t][c]
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  for (int k0 = 0; k0 < K; k0 += kTileBK) {
    // P chunk -> Ps[t][m]; 16 consecutive threads read 16 consecutive t of one row
#pragma unroll
    for (int r = 0; r < (kTileM * kTileBK) / 256; ++r) {
      const int i = tid + 256 * r;
      const int m = i / kTileBK, t = i % kTileBK;
      float v = 0.f;
      if (m < mext && k0 + t < K) v = __ldg(P + (int64_t)m * ldp + k0 + t);
      Ps[t * kTileLD + m] = v;
    }
#pragma unroll
    for (int r = 0; r < (kTileM * kTileBK) / 256; ++r) {
      const int i = tid + 256 * r;
      float v = 0.f;
      if (Q_KMAJOR) {
        const int c = i / kTileBK, t = i % kTileBK;
        if (c < cext && k0 + t < K) v = __ldg(Q + (int64_t)c * ldq + k0 + t);
        Qs[t * kTileLD + c] = v;
      } else {
        const int t = i / kTileM, c = i % kTileM;
        if (c < cext && k0 + t < K) v = __ldg(Q + (int64_t)(k0 + t) * ldq + c);
        Qs[t * kTileLD + c] = v;
      }
    }
    __syncthreads();
#pragma unroll
    for (int t = 0; t < kTileBK; ++t) {
      const float4 a0 = *reinterpret_cast<const float4*>(&Ps[t * kTileLD + ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&Ps[t * kTileLD + 64 + ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Qs[t * kTileLD + tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Qs[t * kTileLD + 64 + tx * 4]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int m = (i < 4) ? (ty * 4 + i) : (64 + ty * 4 + i - 4);
    if (m >= mext) continue;
    float* crow = C + (int64_t)m * ldc;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int c = (j < 4) ? (tx * 4 + j) : (64 + tx * 4 + j - 4);
      if (c < cext) crow[c] -= acc[i][j];
    }
  }
}

}  // namespace gptq
