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
