// Packed storage of tick indices and dequantization.
//
// Page "GPTQ, with the code open", section "What quantization is, and why
// anyone bothers": a weight is stored as the index of its tick plus, once per
// row (or group), the ruler; turning it back into a number is one multiply,
// w_hat = scale (q - zero).  The bit layout is this library's own:
//   int4: column 8i+k  -> bits [4k, 4k+4) of 32-bit word i of the row
//   int3: column 32i+k -> bits [3k, 3k+3) of the 96-bit little-endian word
//         made of 32-bit words 3i, 3i+1, 3i+2 of the row.
// All kernels are HBM-bound streaming passes: each thread owns one 32-code
// group (128-bit loads of codes, 128-bit stores of int4 words).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "gptq_internal.cuh"

namespace gptq {
namespace {

__device__ __forceinline__ uint32_t pack8_int4(uint2 c) {
  uint32_t w = 0;
#pragma unroll
  for (int k = 0; k < 4; ++k) w |= ((c.x >> (8 * k)) & 0xFu) << (4 * k);
#pragma unroll
  for (int k = 0; k < 4; ++k) w |= ((c.y >> (8 * k)) & 0xFu) << (4 * (k + 4));
  return w;
}

// One thread per 32 codes (n % 32 == 0): two 16-byte loads, one 16-byte store.
__global__ void pack_int4_vec_kernel(const uint8_t* __restrict__ codes, int64_t groups_per_row,
                                     int64_t total, int64_t n, uint32_t* __restrict__ out) {
  const int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (g >= total) return;
  const int64_t r = g / groups_per_row, i = g % groups_per_row;
  const uint4* src = reinterpret_cast<const uint4*>(codes + r * n + 32 * i);
  const uint4 a = src[0], b = src[1];
  uint4 w;
  w.x = pack8_int4(make_uint2(a.x, a.y));
  w.y = pack8_int4(make_uint2(a.z, a.w));
  w.z = pack8_int4(make_uint2(b.x, b.y));
  w.w = pack8_int4(make_uint2(b.z, b.w));
  *reinterpret_cast<uint4*>(out + r * (n / 8) + 4 * i) = w;
}

// One thread per 8 codes (n % 8 == 0, any alignment of the row).
__global__ void pack_int4_kernel(const uint8_t* __restrict__ codes, int64_t words_per_row,
                                 int64_t total, int64_t n, uint32_t* __restrict__ out) {
  const int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (g >= total) return;
  const int64_t r = g / words_per_row, i = g % words_per_row;
  const uint8_t* c = codes + r * n + 8 * i;
  uint32_t w = 0;
#pragma unroll
  for (int k = 0; k < 8; ++k) w |= ((uint32_t)c[k] & 0xFu) << (4 * k);
  out[r * words_per_row + i] = w;
}

// One thread per 32 codes -> 3 words.
__global__ void pack_int3_kernel(const uint8_t* __restrict__ codes, int64_t groups_per_row,
                                 int64_t total, int64_t n, int vec, uint32_t* __restrict__ out) {
  const int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (g >= total) return;
  const int64_t r = g / groups_per_row, i = g % groups_per_row;
  const uint8_t* c = codes + r * n + 32 * i;
  uint32_t q[32];
  if (vec) {
    const uint4 a = reinterpret_cast<const uint4*>(c)[0];
    const uint4 b = reinterpret_cast<const uint4*>(c)[1];
    const uint32_t v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int k = 0; k < 32; ++k) q[k] = (v[k >> 2] >> (8 * (k & 3))) & 7u;
  } else {
#pragma unroll
    for (int k = 0; k < 32; ++k) q[k] = c[k] & 7u;
  }
  uint32_t w0 = 0, w1 = 0, w2 = 0;
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    const int bit = 3 * k;  // compile-time after unrolling
    if (bit + 3 <= 32) {
      w0 |= q[k] << bit;
    } else if (bit < 32) {
      w0 |= q[k] << bit;
      w1 |= q[k] >> (32 - bit);
    } else if (bit + 3 <= 64) {
      w1 |= q[k] << (bit - 32);
    } else if (bit < 64) {
      w1 |= q[k] << (bit - 32);
      w2 |= q[k] >> (64 - bit);
    } else {
      w2 |= q[k] << (bit - 64);
    }
  }
  uint32_t* o = out + r * (3 * (n / 32)) + 3 * i;
  o[0] = w0;
  o[1] = w1;
  o[2] = w2;
}

__device__ __forceinline__ int group_of(int64_t c, int group_size, const int32_t* g_idx) {
  if (g_idx) return g_idx[c];
  return group_size > 0 ? (int)(c / group_size) : 0;
}

// One thread per 8 consecutive values of a row: an int4 word, or a quarter
// (24 bits) of an int3 word triple, so each thread writes 16 contiguous bytes
// (bf16) or 32 (fp32) and a warp's stores are coalesced.
template <int BITS, bool BF16>
__global__ void dequant_kernel(const uint32_t* __restrict__ packed, int64_t units_per_row,
                               int64_t total, int64_t n, const float* __restrict__ scales,
                               const uint8_t* __restrict__ zeros, int group_size, int64_t G,
                               const int32_t* __restrict__ g_idx, void* __restrict__ out) {
  const int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (g >= total) return;
  const int64_t r = g / units_per_row, j = g % units_per_row;  // values [8 j, 8 j + 8)
  const float* srow = scales + r * G;
  const uint8_t* zrow = zeros + r * G;
  uint32_t bits24;  // 8 codes, code k in bits [BITS k, BITS k + BITS)
  if (BITS == 4) {
    bits24 = packed[r * units_per_row + j];
  } else {
    // column 32 i + k sits in bits [3 k, 3 k + 3) of words 3i..3i+2 (little-endian)
    const uint32_t* p = packed + r * (3 * (n / 32)) + 3 * (j >> 2);
    switch (j & 3) {
      case 0: bits24 = p[0] & 0xFFFFFFu; break;
      case 1: bits24 = (p[0] >> 24) | ((p[1] & 0xFFFFu) << 8); break;
      case 2: bits24 = (p[1] >> 16) | ((p[2] & 0xFFu) << 16); break;
      default: bits24 = p[2] >> 8; break;
    }
  }
  const int64_t c0 = 8 * j;
  float v[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int gi = group_of(c0 + k, group_size, g_idx);
    const float q = (float)((bits24 >> (BITS * k)) & ((1u << BITS) - 1u));
    v[k] = __fmul_rn(srow[gi], q - (float)zrow[gi]);
  }
  if (BF16) {
    __nv_bfloat16* o = static_cast<__nv_bfloat16*>(out) + r * n + c0;
    if ((reinterpret_cast<uintptr_t>(o) & 15) == 0) {
      __align__(16) __nv_bfloat16 t[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) t[k] = __float2bfloat16_rn(v[k]);
      *reinterpret_cast<uint4*>(o) = *reinterpret_cast<const uint4*>(t);
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) o[k] = __float2bfloat16_rn(v[k]);
    }
  } else {
    float* o = static_cast<float*>(out) + r * n + c0;
    if ((reinterpret_cast<uintptr_t>(o) & 15) == 0) {
      reinterpret_cast<float4*>(o)[0] = make_float4(v[0], v[1], v[2], v[3]);
      reinterpret_cast<float4*>(o)[1] = make_float4(v[4], v[5], v[6], v[7]);
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) o[k] = v[k];
    }
  }
}

// 8 codes of row `prow` starting at column 8 j (int4: word j; int3: the
// quarter j % 4 of word triple j / 4), code k in bits [BITS k, BITS k + BITS).
template <int BITS>
__device__ __forceinline__ uint32_t codes8(const uint32_t* __restrict__ prow, int64_t j) {
  if (BITS == 4) return prow[j];
  const uint32_t* p = prow + 3 * (j >> 2);
  switch (j & 3) {
    case 0: return p[0] & 0xFFFFFFu;
    case 1: return (p[0] >> 24) | ((p[1] & 0xFFFFu) << 8);
    case 2: return (p[1] >> 16) | ((p[2] & 0xFFu) << 16);
    default: return p[2] >> 8;
  }
}

// y[b][r] = sum_c w_hat[r][c] x[b][c] for B activation vectors, w_hat[r][c] =
// scale (code - zero) dequantized on the fly (the same single fp32 multiply
// as dequant_kernel) and never written out.  A CTA owns kMvRowsPerCta rows
// (kMvRowsPerWarp per warp); their rulers (scale, zero) are staged in shared
// memory once, x and each column's group a chunk of kMvChunk columns at a
// time.  Lane l of a warp takes the 8-column units l, l + 32, ... of the
// chunk, so a warp's code loads are contiguous.  Without g_idx the 8 columns
// of a unit share one group (group sizes are >= 32), so a unit reads one
// ruler.  fp32 accumulation per lane, then a shuffle reduction.
constexpr int kMvThreads = 256;
constexpr int kMvRowsPerWarp = 4;
constexpr int kMvRowsPerCta = (kMvThreads / 32) * kMvRowsPerWarp;
constexpr int kMvChunk = 1024;
constexpr int64_t kMvMaxRulerBytes = 96 * 1024;  // staged rulers per CTA; past that, L1

template <int BITS, int B, bool XBF16>
__global__ void __launch_bounds__(kMvThreads) dequant_matvec_kernel(
    const uint32_t* __restrict__ packed, int64_t rows, int64_t n,
    const float* __restrict__ scales, const uint8_t* __restrict__ zeros, int group_size,
    int64_t G, const int32_t* __restrict__ g_idx, const int32_t* __restrict__ perm,
    const void* __restrict__ x, int64_t ldx, float* __restrict__ y, int64_t ldy) {
  __shared__ __align__(16) float xs[B][kMvChunk];
  __shared__ __align__(16) int gs[kMvChunk];
  extern __shared__ float2 rul[];  // (scale, zero) of the CTA's rows, if staged
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row0 = (int64_t)blockIdx.x * kMvRowsPerCta;
  const int64_t rbase = row0 + warp * kMvRowsPerWarp;
  const int64_t wpr = n * BITS / 32;  // packed words per row
  const bool staged = (int64_t)kMvRowsPerCta * G * 8 <= kMvMaxRulerBytes;
  if (staged) {
    for (int64_t i = threadIdx.x; i < (int64_t)kMvRowsPerCta * G; i += kMvThreads) {
      const int64_t r = row0 + i / G;
      rul[i] = r < rows ? make_float2(scales[row0 * G + i], (float)zeros[row0 * G + i])
                        : make_float2(0.f, 0.f);
    }
  }
  float acc[kMvRowsPerWarp][B];
#pragma unroll
  for (int rr = 0; rr < kMvRowsPerWarp; ++rr)
#pragma unroll
    for (int b = 0; b < B; ++b) acc[rr][b] = 0.f;
  for (int64_t c0 = 0; c0 < n; c0 += kMvChunk) {
    const int cn = (int)min((int64_t)kMvChunk, n - c0);
    __syncthreads();  // the previous chunk has been consumed (and the rulers staged)
    for (int i = threadIdx.x; i < cn; i += kMvThreads) {
      // column c0 + i of the packed row multiplies x[perm[c0 + i]] (codes in
      // sweep order) or x[c0 + i] (original order)
      const int64_t xc = perm ? (int64_t)perm[c0 + i] : c0 + i;
#pragma unroll
      for (int b = 0; b < B; ++b) {
        const int64_t xi = (int64_t)b * ldx + xc;
        xs[b][i] = XBF16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(x)[xi])
                         : static_cast<const float*>(x)[xi];
      }
      gs[i] = group_of(c0 + i, group_size, g_idx);
    }
    __syncthreads();
    const int units = cn / 8;  // n % 8 == 0 (int4) or n % 32 == 0 (int3)
    // every code word this lane needs in the chunk, loaded up front so the
    // loads are all in flight together (a chunk has at most 128 units: 4 per lane)
    constexpr int kUPL = kMvChunk / 8 / 32;
    uint32_t cw[kMvRowsPerWarp][kUPL];
#pragma unroll
    for (int rr = 0; rr < kMvRowsPerWarp; ++rr) {
      const int64_t r = rbase + rr;
      const uint32_t* prow = packed + (r < rows ? r : 0) * wpr;
#pragma unroll
      for (int j = 0; j < kUPL; ++j) {
        const int u = lane + 32 * j;
        cw[rr][j] = (r < rows && u < units) ? codes8<BITS>(prow, c0 / 8 + u) : 0u;
      }
    }
#pragma unroll
    for (int rr = 0; rr < kMvRowsPerWarp; ++rr) {
      const int64_t r = rbase + rr;
      if (r >= rows) break;  // warp-uniform
      const float2* rrow = rul + (r - row0) * G;
      const float* srow = scales + r * G;
      const uint8_t* zrow = zeros + r * G;
#pragma unroll
      for (int j = 0; j < kUPL; ++j) {
        const int u = lane + 32 * j;
        if (u >= units) break;
        const uint32_t bits24 = cw[rr][j];
        float sc[8], zr[8];
        if (g_idx) {
          const int4 ga = *reinterpret_cast<const int4*>(gs + 8 * u);
          const int4 gb = *reinterpret_cast<const int4*>(gs + 8 * u + 4);
          const int gi[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float2 sz = staged ? rrow[gi[k]] : make_float2(srow[gi[k]], (float)zrow[gi[k]]);
            sc[k] = sz.x;
            zr[k] = sz.y;
          }
        } else {
          const int g0 = gs[8 * u];
          const float2 sz = staged ? rrow[g0] : make_float2(srow[g0], (float)zrow[g0]);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            sc[k] = sz.x;
            zr[k] = sz.y;
          }
        }
        float wq[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float q = (float)((bits24 >> (BITS * k)) & ((1u << BITS) - 1u));
          wq[k] = __fmul_rn(sc[k], q - zr[k]);
        }
#pragma unroll
        for (int b = 0; b < B; ++b) {
          const float4 xa = *reinterpret_cast<const float4*>(&xs[b][8 * u]);
          const float4 xb = *reinterpret_cast<const float4*>(&xs[b][8 * u + 4]);
          float t = acc[rr][b];
          t = fmaf(wq[0], xa.x, t);
          t = fmaf(wq[1], xa.y, t);
          t = fmaf(wq[2], xa.z, t);
          t = fmaf(wq[3], xa.w, t);
          t = fmaf(wq[4], xb.x, t);
          t = fmaf(wq[5], xb.y, t);
          t = fmaf(wq[6], xb.z, t);
          t = fmaf(wq[7], xb.w, t);
          acc[rr][b] = t;
        }
      }
    }
  }
#pragma unroll
  for (int rr = 0; rr < kMvRowsPerWarp; ++rr) {
    const int64_t r = rbase + rr;
#pragma unroll
    for (int b = 0; b < B; ++b) {
      float v = acc[rr][b];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0 && r < rows) y[(int64_t)b * ldy + r] = v;
    }
  }
}

unsigned blocks_for(int64_t total, int threads) { return (unsigned)((total + threads - 1) / threads); }

}  // namespace

cudaError_t launch_pack_int4(const uint8_t* codes, int64_t rows, int64_t n, uint32_t* out,
                             cudaStream_t s) {
  if (rows == 0) return cudaSuccess;
  const bool vec = (n % 32 == 0) && (reinterpret_cast<uintptr_t>(codes) % 16 == 0) &&
                   (reinterpret_cast<uintptr_t>(out) % 16 == 0);
  if (vec) {
    const int64_t total = rows * (n / 32);
    pack_int4_vec_kernel<<<blocks_for(total, 256), 256, 0, s>>>(codes, n / 32, total, n, out);
    note_launch();
  } else {
    const int64_t total = rows * (n / 8);
    pack_int4_kernel<<<blocks_for(total, 256), 256, 0, s>>>(codes, n / 8, total, n, out);
    note_launch();
  }
  return cudaGetLastError();
}

cudaError_t launch_pack_int3(const uint8_t* codes, int64_t rows, int64_t n, uint32_t* out,
                             cudaStream_t s) {
  if (rows == 0) return cudaSuccess;
  const int vec = (reinterpret_cast<uintptr_t>(codes) % 16 == 0) ? 1 : 0;
  const int64_t total = rows * (n / 32);
  pack_int3_kernel<<<blocks_for(total, 256), 256, 0, s>>>(codes, n / 32, total, n, vec, out);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_dequant(const uint32_t* packed, int bits, int64_t rows, int64_t n,
                           const float* scales, const uint8_t* zeros, int group_size,
                           int64_t n_groups, const int32_t* g_idx, void* out, int out_bf16,
                           cudaStream_t s) {
  if (rows == 0) return cudaSuccess;
  if (bits == 4) {
    const int64_t upr = n / 8, total = rows * upr;
    if (out_bf16)
      dequant_kernel<4, true><<<blocks_for(total, 256), 256, 0, s>>>(
          packed, upr, total, n, scales, zeros, group_size, n_groups, g_idx, out);
    else
      dequant_kernel<4, false><<<blocks_for(total, 256), 256, 0, s>>>(
          packed, upr, total, n, scales, zeros, group_size, n_groups, g_idx, out);
  } else {
    const int64_t upr = n / 8, total = rows * upr;  // n % 32 == 0 for int3
    if (out_bf16)
      dequant_kernel<3, true><<<blocks_for(total, 256), 256, 0, s>>>(
          packed, upr, total, n, scales, zeros, group_size, n_groups, g_idx, out);
    else
      dequant_kernel<3, false><<<blocks_for(total, 256), 256, 0, s>>>(
          packed, upr, total, n, scales, zeros, group_size, n_groups, g_idx, out);
  }
  note_launch();
  return cudaGetLastError();
}

}  // namespace gptq

namespace gptq {
namespace {
// dst[r][k] = src[r][perm[k]]: one CTA per row, the row staged in shared memory.
__global__ void __launch_bounds__(256) gather_columns_u8_kernel(const uint8_t* __restrict__ src,
                                                                int64_t n,
                                                                const int32_t* __restrict__ perm,
                                                                uint8_t* __restrict__ dst) {
  extern __shared__ uint8_t srow[];
  const int64_t r = blockIdx.x;
  for (int64_t c = threadIdx.x; c < n; c += blockDim.x) srow[c] = src[r * n + c];
  __syncthreads();
  for (int64_t k = threadIdx.x; k < n; k += blockDim.x) dst[r * n + k] = srow[perm[k]];
}

template <int BITS, int B>
void mv_launch(const uint32_t* packed, int64_t rows, int64_t n, const float* scales,
               const uint8_t* zeros, int group_size, int64_t G, const int32_t* g_idx,
               const int32_t* perm, const void* x, int x_bf16, int64_t ldx, float* y, int64_t ldy,
               cudaStream_t s) {
  const unsigned grid = (unsigned)((rows + kMvRowsPerCta - 1) / kMvRowsPerCta);
  const int64_t rb = (int64_t)kMvRowsPerCta * G * 8;
  const size_t dyn = rb <= kMvMaxRulerBytes ? (size_t)rb : 0;
  if (x_bf16) {
    cudaFuncSetAttribute(dequant_matvec_kernel<BITS, B, true>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMvMaxRulerBytes);
    dequant_matvec_kernel<BITS, B, true><<<grid, kMvThreads, dyn, s>>>(
        packed, rows, n, scales, zeros, group_size, G, g_idx, perm, x, ldx, y, ldy);
  } else {
    cudaFuncSetAttribute(dequant_matvec_kernel<BITS, B, false>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMvMaxRulerBytes);
    dequant_matvec_kernel<BITS, B, false><<<grid, kMvThreads, dyn, s>>>(
        packed, rows, n, scales, zeros, group_size, G, g_idx, perm, x, ldx, y, ldy);
  }
  note_launch();
}
template <int BITS>
void mv_batch(int b, const uint32_t* packed, int64_t rows, int64_t n, const float* scales,
              const uint8_t* zeros, int group_size, int64_t G, const int32_t* g_idx,
              const int32_t* perm, const void* x, int x_bf16, int64_t ldx, float* y, int64_t ldy,
              cudaStream_t s) {
  switch (b) {
    case 8: mv_launch<BITS, 8>(packed, rows, n, scales, zeros, group_size, G, g_idx, perm, x, x_bf16, ldx, y, ldy, s); break;
    case 4: mv_launch<BITS, 4>(packed, rows, n, scales, zeros, group_size, G, g_idx, perm, x, x_bf16, ldx, y, ldy, s); break;
    case 2: mv_launch<BITS, 2>(packed, rows, n, scales, zeros, group_size, G, g_idx, perm, x, x_bf16, ldx, y, ldy, s); break;
    default: mv_launch<BITS, 1>(packed, rows, n, scales, zeros, group_size, G, g_idx, perm, x, x_bf16, ldx, y, ldy, s); break;
  }
}
}  // namespace

cudaError_t launch_gather_columns_u8(const uint8_t* src, int64_t rows, int64_t n,
                                     const int32_t* perm, uint8_t* dst, cudaStream_t s) {
  if (rows == 0) return cudaSuccess;
  if ((size_t)n > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(
        gather_columns_u8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)n);
    if (e != cudaSuccess) return e;
  }
  gather_columns_u8_kernel<<<(unsigned)rows, 256, (size_t)n, s>>>(src, n, perm, dst);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_dequant_matvec(const uint32_t* packed, int bits, int64_t rows, int64_t n,
                                  const float* scales, const uint8_t* zeros, int group_size,
                                  int64_t n_groups, const int32_t* g_idx, const int32_t* perm,
                                  const void* x, int x_bf16, int64_t batch, float* y,
                                  cudaStream_t s) {
  if (rows == 0 || batch == 0) return cudaSuccess;
  const size_t esz = x_bf16 ? 2 : 4;
  // batches of 8, 4, 2, 1 vectors per launch
  for (int64_t b0 = 0; b0 < batch;) {
    const int64_t left = batch - b0;
    const int b = left >= 8 ? 8 : left >= 4 ? 4 : left >= 2 ? 2 : 1;
    const void* xb = static_cast<const char*>(x) + (size_t)b0 * (size_t)n * esz;
    float* yb = y + b0 * rows;
    if (bits == 4)
      mv_batch<4>(b, packed, rows, n, scales, zeros, group_size, n_groups, g_idx, perm, xb,
                  x_bf16, n, yb, rows, s);
    else
      mv_batch<3>(b, packed, rows, n, scales, zeros, group_size, n_groups, g_idx, perm, xb,
                  x_bf16, n, yb, rows, s);
    b0 += b;
  }
  return cudaGetLastError();
}

}  // namespace gptq
