// Packed storage of tick indices, dequantization, and the consumer of the
// packed codes (dequant x activation).
//
// Page "GPTQ, with the code open", section "What quantization is, and why
// anyone bothers": a weight is stored as the index of its tick plus, once per
// row (or group), the ruler; turning it back into a number is one multiply,
// w_hat = scale (q - zero).  The bit layout is this library's own:
//   int4: column 8i+k  -> bits [4k, 4k+4) of 32-bit word i of the row
//   int3: column 32i+k -> bits [3k, 3k+3) of the 96-bit little-endian word
//         made of 32-bit words 3i, 3i+1, 3i+2 of the row.
// Packing and dequantization are HBM-bound streaming passes (a thread owns a
// 32-code group or 8 values: 128-bit loads and stores).  The dequant x
// activation kernels follow further down: one on the FP32 pipe, one on the
// tensor cores (mma.sync with exact bf16 (q - zero) operands).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "gptq_internal.cuh"
#include "sm100_ptx.cuh"

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
    v[k] = index_ok(gi, G, kCheckGroupIndex) ? __fmul_rn(srow[gi], q - (float)zrow[gi]) : 0.f;
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

// The same dequantization with one CTA per RPC rows: the rows' rulers are
// staged once in shared memory as (scale, zero) pairs, so each value costs
// one shared-memory read for its ruler instead of two global ones, and the
// group index of 8 columns comes in two 16-byte loads that serve all RPC
// rows (g_idx is read once per RPC rows, not once per row).  Same
// arithmetic and bytes out as dequant_kernel.
constexpr int kDqRowThreads = 128;
constexpr int kDqRowMaxG = 2048;   // rulers staged per CTA (16 KB of shared memory)
constexpr int kDqRowsPerCta = 4;   // RPC when RPC x G rulers fit

template <int BITS, bool BF16, int RPC>
__global__ void __launch_bounds__(kDqRowThreads) dequant_row_kernel(
    const uint32_t* __restrict__ packed, int64_t rows, int64_t n, const float* __restrict__ scales,
    const uint8_t* __restrict__ zeros, int group_size, int64_t G,
    const int32_t* __restrict__ g_idx, void* __restrict__ out) {
  __shared__ float2 rul[kDqRowMaxG];   // [RPC][G]
  const int64_t r0 = (int64_t)blockIdx.x * RPC;
  const int nr = (int)(rows - r0 < RPC ? rows - r0 : RPC);
  // the rows r0 .. r0 + nr - 1 are contiguous in scales and zeros
  for (int64_t e = threadIdx.x; e < nr * G; e += kDqRowThreads)
    rul[e] = make_float2(scales[r0 * G + e], (float)zeros[r0 * G + e]);
  __syncthreads();
  const int64_t upr = n / 8;
  for (int64_t j = threadIdx.x; j < upr; j += kDqRowThreads) {
    const int64_t c0 = 8 * j;
    int gi[8];
    if (g_idx) {
      const int4 ga = __ldg(reinterpret_cast<const int4*>(g_idx + c0));
      const int4 gb = __ldg(reinterpret_cast<const int4*>(g_idx + c0) + 1);
      gi[0] = ga.x; gi[1] = ga.y; gi[2] = ga.z; gi[3] = ga.w;
      gi[4] = gb.x; gi[5] = gb.y; gi[6] = gb.z; gi[7] = gb.w;
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) gi[k] = group_size > 0 ? (int)((c0 + k) / group_size) : 0;
    }
#pragma unroll
    for (int rho = 0; rho < RPC; ++rho) {
      if (rho >= nr) break;
      const int64_t r = r0 + rho;
      const uint32_t* prow = packed + r * (n * BITS / 32);
      uint32_t bits24;
      if (BITS == 4) {
        bits24 = prow[j];
      } else {
        const uint32_t* p = prow + 3 * (j >> 2);
        switch (j & 3) {
          case 0: bits24 = p[0] & 0xFFFFFFu; break;
          case 1: bits24 = (p[0] >> 24) | ((p[1] & 0xFFFFu) << 8); break;
          case 2: bits24 = (p[1] >> 16) | ((p[2] & 0xFFu) << 16); break;
          default: bits24 = p[2] >> 8; break;
        }
      }
      const float2* rr = rul + rho * G;
      float v[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float q = (float)((bits24 >> (BITS * k)) & ((1u << BITS) - 1u));
        if (index_ok(gi[k], G, kCheckGroupIndex)) {
          const float2 sz = rr[gi[k]];
          v[k] = __fmul_rn(sz.x, q - sz.y);
        } else {
          v[k] = 0.f;
        }
      }
      if (BF16) {
        __align__(16) __nv_bfloat16 t[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) t[k] = __float2bfloat16_rn(v[k]);
        *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(out) + r * n + c0) =
            *reinterpret_cast<const uint4*>(t);
      } else {
        float* o = static_cast<float*>(out) + r * n + c0;
        reinterpret_cast<float4*>(o)[0] = make_float4(v[0], v[1], v[2], v[3]);
        reinterpret_cast<float4*>(o)[1] = make_float4(v[4], v[5], v[6], v[7]);
      }
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
      int64_t xc = perm ? (int64_t)perm[c0 + i] : c0 + i;
      if (!index_ok(xc, n, kCheckPermutation)) xc = 0;
#pragma unroll
      for (int b = 0; b < B; ++b) {
        const int64_t xi = (int64_t)b * ldx + xc;
        xs[b][i] = XBF16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(x)[xi])
                         : static_cast<const float*>(x)[xi];
      }
      const int gsel = group_of(c0 + i, group_size, g_idx);
      gs[i] = index_ok(gsel, G, kCheckGroupIndex) ? gsel : 0;
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

// ---------------------------------------------------------------------------
// The same product for codes in the ORIGINAL column order with a per-column
// group index g_idx (act-order layers stored without re-ordering).  Here the
// 8 columns of a code word belong to unrelated groups, so every weight needs
// its own (scale, zero) and the per-group factoring of the tensor-core
// kernel does not apply.  The cost is then the ruler lookup, and the layout
// below makes it one conflict-free shared-memory read per weight:
//   * lane = row: a warp owns 32 rows and walks columns; the column (hence
//     its group g_idx[c] and its activations) is the same for every lane, so
//     those reads are broadcasts, and lane l reads the ruler of row l,
//     group g at rul[l * rpitch + g] with an odd pitch (distinct banks);
//   * a CTA is 8 warps on the same 32 rows, each warp taking 128 of every
//     1024-column chunk; each warp stages its 32 x 128 codes with coalesced
//     16-byte cp.async copies, double-buffered (the next chunk's codes load
//     while this one's are used); piece k of row l sits in slot
//     k ^ ((l >> 1) & 3) of the row's four 16-byte slots, so that the lanes'
//     16-byte reads of their own rows do not conflict;
//   * w_hat = scale * (q - zero) as one fp32 multiply of the exact q - zero,
//     formed as (2^23 + q) - (2^23 + zero) from the code's bits;
//   * each lane keeps 4 interleaved partial sums per vector (column k of a
//     code word goes to sum k % 4), the 8 warps' sums meet in shared memory
//     in a fixed order: y is the same from run to run.
// Requires packed 16-byte aligned, n % 32 == 0 (int4) or n % 128 == 0
// (int3), so that every staged piece is a whole, aligned 16 bytes.
constexpr int kGxWarps = 8;
constexpr int kGxChunk = 1024;
constexpr int kGxSlice = kGxChunk / kGxWarps;     // 128 columns per warp per chunk
constexpr int kGxPitchW = 16;                     // code tile row pitch in words (64 B)
constexpr int kGxTileWords = 32 * kGxPitchW;
constexpr int64_t kGxMaxRulerBytes = 112 * 1024;  // staged rulers per CTA; past that, L1

template <int B>
__host__ __device__ constexpr size_t gx_fixed_bytes() {
  return sizeof(uint32_t) * kGxWarps * 2 * kGxTileWords + 2 * sizeof(float) * B * kGxChunk +
         2 * sizeof(int) * kGxChunk + sizeof(float) * kGxWarps * B * 32;
}
constexpr int kGxPer = kGxChunk / (kGxWarps * 32);  // columns of a chunk each thread stages

template <int BITS, int B, bool XBF16, bool STAGED>
__global__ void __launch_bounds__(kGxWarps * 32) dequant_matvec_gidx_kernel(
    const uint32_t* __restrict__ packed, int64_t rows, int64_t n,
    const float* __restrict__ scales, const uint8_t* __restrict__ zeros, int64_t G, int rpitch,
    const int32_t* __restrict__ g_idx, const void* __restrict__ x, int64_t ldx,
    float* __restrict__ y, int64_t ldy) {
  extern __shared__ __align__(16) uint32_t gx_smem[];
  uint32_t* tiles = gx_smem;                                               // [warp][2][32][pitch]
  float* xs2 = reinterpret_cast<float*>(tiles + kGxWarps * 2 * kGxTileWords);  // [2][B][chunk]
  int* gs2 = reinterpret_cast<int*>(xs2 + 2 * B * kGxChunk);              // [2][chunk]
  float* red = reinterpret_cast<float*>(gs2 + 2 * kGxChunk);              // [warp][B][32]
  float2* rul = reinterpret_cast<float2*>(red + kGxWarps * B * 32);      // [32][rpitch]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row0 = (int64_t)blockIdx.x * 32;
  const int64_t r = row0 + lane;
  const int64_t wpr = n * BITS / 32;  // packed words per row
  constexpr int kWords = kGxSlice * BITS / 32;   // words of a row per slice: 16 or 12
  constexpr int kPieces = kWords / 4;            // 16-byte pieces per row: 4 or 3
  constexpr float kMagic = 8388608.f;            // 2^23
  if (STAGED) {
    // the CTA's rows' rulers are contiguous in scales / zeros: element i of
    // that range is (row i / G, group i % G); four loads in flight per thread
    const int Gi = (int)G, tot = 32 * Gi;
    const int64_t live = (min(rows - row0, (int64_t)32)) * G;
    const float* sbase = scales + row0 * G;
    const uint8_t* zbase = zeros + row0 * G;
    for (int i0 = threadIdx.x; i0 < tot; i0 += 4 * kGxWarps * 32) {
      float sv[4], zv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * kGxWarps * 32;
        const bool ok = i < live;
        sv[u] = ok ? __ldg(sbase + i) : 0.f;
        zv[u] = ok ? (float)__ldg(zbase + i) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * kGxWarps * 32;
        if (i < tot) {
          const int rr = i / Gi;
          rul[rr * rpitch + (i - rr * Gi)] = make_float2(sv[u], kMagic + zv[u]);
        }
      }
    }
  }
  const float* srow = scales + min(r, rows - 1) * G;
  const uint8_t* zrow = zeros + min(r, rows - 1) * G;
  // stage this warp's slice of chunk c0 into buffer buf
  auto stage_codes = [&](int64_t c0, int buf) {
    uint32_t* t = tiles + (warp * 2 + buf) * kGxTileWords;
    const int64_t col = c0 + (int64_t)warp * kGxSlice;
#pragma unroll
    for (int k = 0; k < kPieces; ++k) {
      const int i = lane + 32 * k;
      const int rr = i / kPieces, part = i % kPieces;
      const int64_t pc = col + (int64_t)part * (128 / kPieces);  // first column of the piece
      const bool ok = row0 + rr < rows && pc < n;
      const uint32_t* src = ok ? packed + (row0 + rr) * wpr + col * BITS / 32 + 4 * part : packed;
      ptx::cp_async_16z(t + rr * kGxPitchW + 4 * (part ^ ((rr >> 1) & 3)), src, ok ? 16 : 0);
    }
  };
  // this thread's columns i = tid + 256 j of a chunk: activations and groups
  // are loaded into registers one chunk ahead and stored after the chunk's
  // work, so their load latency hides behind it
  float xr[kGxPer][B];
  int gr[kGxPer];
  auto load_side = [&](int64_t c0) {
#pragma unroll
    for (int j = 0; j < kGxPer; ++j) {
      const int64_t c = c0 + threadIdx.x + kGxWarps * 32 * j;
      const bool ok = c < n;
      gr[j] = ok ? __ldg(g_idx + c) : 0;
      if (!index_ok(gr[j], G, kCheckGroupIndex)) gr[j] = 0;
#pragma unroll
      for (int b = 0; b < B; ++b) {
        const int64_t xi = (int64_t)b * ldx + (ok ? c : 0);
        xr[j][b] = !ok ? 0.f
                 : XBF16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(x)[xi])
                         : __ldg(static_cast<const float*>(x) + xi);
      }
    }
  };
  auto store_side = [&](int sb) {
#pragma unroll
    for (int j = 0; j < kGxPer; ++j) {
      const int i = threadIdx.x + kGxWarps * 32 * j;
      gs2[sb * kGxChunk + i] = gr[j];
#pragma unroll
      for (int b = 0; b < B; ++b) xs2[(sb * B + b) * kGxChunk + i] = xr[j][b];
    }
  };
  float acc[B][4];
#pragma unroll
  for (int b = 0; b < B; ++b)
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[b][k] = 0.f;
  stage_codes(0, 0);
  ptx::cp_async_commit();
  load_side(0);
  store_side(0);
  int buf = 0;
  for (int64_t c0 = 0; c0 < n; c0 += kGxChunk, buf ^= 1) {
    const int cn = (int)min((int64_t)kGxChunk, n - c0);
    const bool more = c0 + kGxChunk < n;
    __syncwarp();  // every lane is done reading the tile the next copies overwrite
    if (more) {
      stage_codes(c0 + kGxChunk, buf ^ 1);
      load_side(c0 + kGxChunk);
    }
    ptx::cp_async_commit();
    ptx::cp_async_wait<1>();  // this thread's pieces of chunk c0 have landed
    __syncthreads();          // ... and every other thread's, with chunk c0's xs and gs
    const float* xs = xs2 + buf * B * kGxChunk;
    const int* gs = gs2 + buf * kGxChunk;
    const uint32_t* t = tiles + (warp * 2 + buf) * kGxTileWords + lane * kGxPitchW;
    uint32_t w[kWords];
#pragma unroll
    for (int k = 0; k < kPieces; ++k) {
      const uint4 v = *reinterpret_cast<const uint4*>(t + 4 * (k ^ ((lane >> 1) & 3)));
      w[4 * k] = v.x;
      w[4 * k + 1] = v.y;
      w[4 * k + 2] = v.z;
      w[4 * k + 3] = v.w;
    }
    const int cb0 = warp * kGxSlice;
    const float2* rrow = rul + lane * rpitch;
#pragma unroll
    for (int u = 0; u < kGxSlice / 8; ++u) {
      const int cb = cb0 + 8 * u;
      if (cb >= cn) break;  // warp-uniform (n % 32 == 0: whole units)
      uint32_t bits24;
      if (BITS == 4) {
        bits24 = w[u];
      } else {
        const int j = u >> 2;
        bits24 = (u & 3) == 0 ? w[3 * j]
               : (u & 3) == 1 ? __funnelshift_r(w[3 * j], w[3 * j + 1], 24)
               : (u & 3) == 2 ? __funnelshift_r(w[3 * j + 1], w[3 * j + 2], 16)
                              : (w[3 * j + 2] >> 8);
      }
      const int4 ga = *reinterpret_cast<const int4*>(gs + cb);
      const int4 gb = *reinterpret_cast<const int4*>(gs + cb + 4);
      const int gi[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
      float wq[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float2 sz = STAGED ? rrow[gi[k]] : make_float2(__ldg(srow + gi[k]),
                                                             kMagic + (float)__ldg(zrow + gi[k]));
        const float q = __uint_as_float(0x4B000000u | ((bits24 >> (BITS * k)) & ((1u << BITS) - 1u)));
        wq[k] = __fmul_rn(sz.x, q - sz.y);
      }
#pragma unroll
      for (int b = 0; b < B; ++b) {
        const float4 xa = *reinterpret_cast<const float4*>(xs + b * kGxChunk + cb);
        const float4 xb = *reinterpret_cast<const float4*>(xs + b * kGxChunk + cb + 4);
        acc[b][0] = fmaf(wq[0], xa.x, acc[b][0]);
        acc[b][1] = fmaf(wq[1], xa.y, acc[b][1]);
        acc[b][2] = fmaf(wq[2], xa.z, acc[b][2]);
        acc[b][3] = fmaf(wq[3], xa.w, acc[b][3]);
        acc[b][0] = fmaf(wq[4], xb.x, acc[b][0]);
        acc[b][1] = fmaf(wq[5], xb.y, acc[b][1]);
        acc[b][2] = fmaf(wq[6], xb.z, acc[b][2]);
        acc[b][3] = fmaf(wq[7], xb.w, acc[b][3]);
      }
    }
    // the next chunk's side buffer: last read during the previous chunk, which
    // every thread finished before this chunk's barrier
    if (more) store_side(buf ^ 1);
  }
  ptx::cp_async_wait_all();
#pragma unroll
  for (int b = 0; b < B; ++b)
    red[(warp * B + b) * 32 + lane] = (acc[b][0] + acc[b][1]) + (acc[b][2] + acc[b][3]);
  __syncthreads();
  // fixed-order sum over the 8 warps: thread (b, l) for b < B
  if (threadIdx.x < B * 32) {
    const int b = threadIdx.x >> 5, l = threadIdx.x & 31;
    float v[kGxWarps];
#pragma unroll
    for (int k = 0; k < kGxWarps; ++k) v[k] = red[(k * B + b) * 32 + l];
    const float s = ((v[0] + v[1]) + (v[2] + v[3])) + ((v[4] + v[5]) + (v[6] + v[7]));
    if (row0 + l < rows) y[(int64_t)b * ldy + row0 + l] = s;
  }
}

template <int BITS, int B>
void gx_launch(const uint32_t* packed, int64_t rows, int64_t n, const float* scales,
               const uint8_t* zeros, int64_t G, const int32_t* g_idx, const void* x, int x_bf16,
               int64_t ldx, float* y, int64_t ldy, cudaStream_t s) {
  static_assert(kGxWarps == 8, "the fixed-order sum is written for 8 warps");
  const unsigned grid = (unsigned)((rows + 31) / 32);
  const int rpitch = (int)(G | 1);
  const int64_t rb = (int64_t)32 * rpitch * 8;
  const bool staged = rb <= kGxMaxRulerBytes;
  const size_t dyn = gx_fixed_bytes<B>() + (staged ? (size_t)rb : 0);
#define GX_GO(XB, ST)                                                                          \
  {                                                                                            \
    auto k = dequant_matvec_gidx_kernel<BITS, B, XB, ST>;                                      \
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);           \
    k<<<grid, kGxWarps * 32, dyn, s>>>(packed, rows, n, scales, zeros, G, rpitch, g_idx, x, ldx, \
                                       y, ldy);                                                \
  }
  if (x_bf16) {
    if (staged) GX_GO(true, true) else GX_GO(true, false)
  } else {
    if (staged) GX_GO(false, true) else GX_GO(false, false)
  }
#undef GX_GO
  note_launch();
}
template <int BITS>
void gx_batch(int b, const uint32_t* packed, int64_t rows, int64_t n, const float* scales,
              const uint8_t* zeros, int64_t G, const int32_t* g_idx, const void* x, int x_bf16,
              int64_t ldx, float* y, int64_t ldy, cudaStream_t s) {
  switch (b) {
    case 8: gx_launch<BITS, 8>(packed, rows, n, scales, zeros, G, g_idx, x, x_bf16, ldx, y, ldy, s); break;
    case 4: gx_launch<BITS, 4>(packed, rows, n, scales, zeros, G, g_idx, x, x_bf16, ldx, y, ldy, s); break;
    case 2: gx_launch<BITS, 2>(packed, rows, n, scales, zeros, G, g_idx, x, x_bf16, ldx, y, ldy, s); break;
    default: gx_launch<BITS, 1>(packed, rows, n, scales, zeros, G, g_idx, x, x_bf16, ldx, y, ldy, s); break;
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
  // one CTA per row when the rulers fit its shared memory and every row's
  // output starts 16-byte aligned (and g_idx, if given, is 16-byte aligned)
  const bool row_form = n_groups <= kDqRowMaxG && (n * (out_bf16 ? 2 : 4)) % 16 == 0 &&
                        reinterpret_cast<uintptr_t>(out) % 16 == 0 &&
                        (!g_idx || reinterpret_cast<uintptr_t>(g_idx) % 16 == 0) &&
                        rows <= 0x7fffffff;
  if (row_form) {
    // RPC rows per CTA when their rulers fit the staged table
    const bool multi = n_groups * kDqRowsPerCta <= kDqRowMaxG;
    const int rpc = multi ? kDqRowsPerCta : 1;
    const unsigned grid = (unsigned)((rows + rpc - 1) / rpc);
#define GPTQ_DQ_ROW(B, F, R)                                                              \
  dequant_row_kernel<B, F, R><<<grid, kDqRowThreads, 0, s>>>(packed, rows, n, scales, zeros, \
                                                             group_size, n_groups, g_idx, out)
    if (bits == 4 && out_bf16) {
      if (multi) GPTQ_DQ_ROW(4, true, kDqRowsPerCta); else GPTQ_DQ_ROW(4, true, 1);
    } else if (bits == 4) {
      if (multi) GPTQ_DQ_ROW(4, false, kDqRowsPerCta); else GPTQ_DQ_ROW(4, false, 1);
    } else if (out_bf16) {
      if (multi) GPTQ_DQ_ROW(3, true, kDqRowsPerCta); else GPTQ_DQ_ROW(3, true, 1);
    } else {
      if (multi) GPTQ_DQ_ROW(3, false, kDqRowsPerCta); else GPTQ_DQ_ROW(3, false, 1);
    }
#undef GPTQ_DQ_ROW
    note_launch();
    return cudaGetLastError();
  }
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
  for (int64_t k = threadIdx.x; k < n; k += blockDim.x) {
    const int32_t pk = perm[k];
    dst[r * n + k] = index_ok(pk, n, kCheckPermutation) ? srow[pk] : 0;
  }
}

// ---------------------------------------------------------------------------
// int4 codes x bf16 activations on the tensor cores (mma.sync, register
// operands).  Decode-size batches (1..8 vectors) make this a skinny product:
// on the FP32 pipe the dequantize + FMA per weight costs ~3.4 instructions,
// more issue slots than the 0.5 byte of HBM it reads, and at 8 vectors it is
// ALU-bound outright.  Here each pair of codes becomes an exact bf16x2 pair
// (q - zero) with one shift + LOP3 (magic 128.0) and one bf16x2 subtract, and
// the dot with all 8 vector slots is one m16n8k16 MMA per 256 weights, so
// every batch size up to 8 costs the same instructions.
//
// Exactness: q - zero (|.| < 128) and x (bf16) are exact bf16 operands, so
// every product is exact in fp32; partial sums are fp32 (tensor-core
// accumulation), then scaled by the group's scale with one FMA: y = sum over
// groups of scale * sum (q - zero) x.
//
// Work: CTA (tile, h) takes 16 rows (the MMA's M) and half h of the
// 128-column slices; its warps take slices in turn and their partial sums
// are added in a fixed order.  Each warp streams its slices' codes through a
// private ring of kDqStages shared-memory slots with cp.async (each thread
// copies and later reads back its own 16-byte pieces), so a warp keeps
// kDqStages - 1 slices of code loads in flight without holding registers.  The two halves meet in y by atomic adds onto
// zeros: fp32 addition of two terms is commutative, so y is the same
// whichever half lands first.  Thread (g = lane / 4, t = lane % 4) holds
// rows g and g + 8; in a slice, MMA pair j (j = 0..3) covers 32-column block
// bj with the thread contributing word wj of it:
//   block mode  (group_size a multiple of 128, or per row): bj = t, wj = j --
//               one 16-byte load per row, the 4 blocks of a slice share a group;
//   interleaved (group_size 32 or 64): bj = j, wj = t -- four 4-byte loads
//               per row, each MMA pair stays inside one 32-column block, so a
//               group's scale applies to its own partial sum.
// From word w (8 codes, column 8 wj + i of the block in bits 4i..4i+3) the
// k-slots are paired as (i, i + 4): ((w >> 4i) & 0x000F000F) | 0x43004300 is
// the bf16 pair (128 + q_i, 128 + q_{i+4}): OR-ing a small integer into the
// mantissa of a power of two and subtracting that power is the classic
// "magic number" integer-to-float conversion (for int4 / int8 weights on GPUs
// it is described in Kim et al., "Who Says Elephants Can't Run: Bringing Large
// Scale MoE Models into Cloud Scale Production", 2022).  A prep kernel writes x once per
// call in that pairing (and in sweep order when a perm is given), so the MMA
// B fragments load straight from it, and zeroes y.

__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The four bf16 pairs (128 + q_i, 128 + q_{i+4}), i = 0..3, of 8 codes:
// int4: a 32-bit word, code i in bits 4i..4i+3; int3: 24 bits, code i in
// bits 3i..3i+2, first spread so that codes i and i + 4 sit 16 bits apart.
template <int BITS>
__device__ __forceinline__ uint4 code_pairs(uint32_t w) {
  constexpr uint32_t kMagic = 0x43004300u;
  if constexpr (BITS == 4) {
    constexpr uint32_t kMask = 0x000F000Fu;
    return make_uint4((w & kMask) | kMagic, ((w >> 4) & kMask) | kMagic,
                      ((w >> 8) & kMask) | kMagic, ((w >> 12) & kMask) | kMagic);
  } else {
    constexpr uint32_t kMask = 0x00070007u;
    const uint32_t sp = (w & 0xFFFu) | ((w >> 12) << 16);  // codes 4..7 -> bits 16..27
    return make_uint4((sp & kMask) | kMagic, ((sp >> 3) & kMask) | kMagic,
                      ((sp >> 6) & kMask) | kMagic, ((sp >> 9) & kMask) | kMagic);
  }
}

// Two MMAs for 8 codes per row: codes wa (row g) and wb (row g + 8) with
// their zero pairs za / zb; xp holds the 8 activations of vector g in pair
// order (x0, x4), (x1, x5), (x2, x6), (x3, x7).
template <int BITS>
__device__ __forceinline__ void mma_word(float (&c)[4], uint32_t wa, uint32_t wb, uint32_t za,
                                         uint32_t zb, const uint4& xp) {
  const uint4 a = code_pairs<BITS>(wa), b = code_pairs<BITS>(wb);
  mma_bf16_16816(c, bf16x2_sub(a.x, za), bf16x2_sub(b.x, zb), bf16x2_sub(a.y, za),
                 bf16x2_sub(b.y, zb), xp.x, xp.y);
  mma_bf16_16816(c, bf16x2_sub(a.z, za), bf16x2_sub(b.z, zb), bf16x2_sub(a.w, za),
                 bf16x2_sub(b.w, zb), xp.z, xp.w);
}

// int3: quarter q (codes 8q .. 8q + 7) of a 32-code block stored in words
// w0, w1, w2 (little-endian 96 bits); bits above the quarter are ignored.
__device__ __forceinline__ uint32_t int3_quarter(uint32_t w0, uint32_t w1, uint32_t w2, int q) {
  switch (q) {
    case 0: return w0;
    case 1: return __funnelshift_r(w0, w1, 24);
    case 2: return __funnelshift_r(w1, w2, 16);
    default: return w2 >> 8;
  }
}

__device__ __forceinline__ uint32_t zero_pair(uint8_t z) {
  return 0x43004300u | (uint32_t)z | ((uint32_t)z << 16);
}

constexpr int kDqWarps = 4;    // warps per CTA
constexpr int kDqStages = 5;   // code slices a warp keeps in flight (cp.async ring)
constexpr int kDqMinBlocks = 8;
constexpr int kDqSplit = 2;    // column halves per row tile (two atomic adds per output)
// bytes between the 16 code rows of a staged slice: 64 (int4 block mode: each
// thread reads back its own 16-byte pieces, conflict-free) or 80 (the 4-byte
// reads of the other modes: 8 rows x 4 words land on distinct banks)
template <int BITS, bool kInterleaved>
__host__ __device__ constexpr int dq_pitch() { return BITS == 4 && !kInterleaved ? 64 : 80; }

// The non-code operands of one slice for one thread: activations of its
// block(s) and the rulers of its rows.
// (block mode: one ruler per row for the slice; interleaved: one per block)
template <bool kInterleaved>
struct DqSide {
  static constexpr int kR = kInterleaved ? 4 : 1;
  uint4 xq[4];
  float fa[kR], fb[kR];
  uint32_t za[kR], zb[kR];
};

// gshift = log2(group_size), or 31 for one group per row.  kFull: every
// block of slice s is inside the row (no masking).
template <bool kInterleaved, bool kFull>
__device__ __forceinline__ void dq_side(DqSide<kInterleaved>& d, int s, int nblk, int t, int gshift,
                                        const __nv_bfloat16* xr, const float* sa, const float* sb,
                                        const uint8_t* za_row, const uint8_t* zb_row) {
  if constexpr (!kInterleaved) {
    const int blk = 4 * s + t;
    const bool ok = kFull || blk < nblk;
    const uint4* xv = reinterpret_cast<const uint4*>(xr + 32 * blk);
#pragma unroll
    for (int j = 0; j < 4; ++j) d.xq[j] = ok ? __ldg(xv + j) : make_uint4(0, 0, 0, 0);
    const int grp = (128 * s) >> gshift;  // one group for the whole slice
    d.fa[0] = __ldg(sa + grp);
    d.fb[0] = __ldg(sb + grp);
    d.za[0] = zero_pair(__ldg(za_row + grp));
    d.zb[0] = zero_pair(__ldg(zb_row + grp));
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int blk = 4 * s + j;
      const bool ok = kFull || blk < nblk;
      d.xq[j] = ok ? __ldg(reinterpret_cast<const uint4*>(xr + 32 * blk + 8 * t))
                   : make_uint4(0, 0, 0, 0);
      const int grp = ok ? (32 * blk) >> gshift : 0;
      d.fa[j] = __ldg(sa + grp);
      d.fb[j] = __ldg(sb + grp);
      d.za[j] = zero_pair(__ldg(za_row + grp));
      d.zb[j] = zero_pair(__ldg(zb_row + grp));
    }
  }
}

// `st`: this warp's staged slice (16 rows x pitch bytes of codes): int4,
// 16 words per row (block b = words 4b .. 4b + 3); int3, 12 words per row
// (block b = words 3b .. 3b + 2).
template <int BITS, bool kInterleaved>
__device__ __forceinline__ void dq_slice(float (&Y)[4], const uint8_t* st,
                                         const DqSide<kInterleaved>& d, int g, int t) {
  constexpr int P = dq_pitch<BITS, kInterleaved>();
  const uint32_t* ra = reinterpret_cast<const uint32_t*>(st + g * P);
  const uint32_t* rb = reinterpret_cast<const uint32_t*>(st + (g + 8) * P);
  if constexpr (!kInterleaved) {
    uint32_t wa[4], wb[4];
    if constexpr (BITS == 4) {
      const uint4 qa = *reinterpret_cast<const uint4*>(ra + 4 * t);
      const uint4 qb = *reinterpret_cast<const uint4*>(rb + 4 * t);
      wa[0] = qa.x; wa[1] = qa.y; wa[2] = qa.z; wa[3] = qa.w;
      wb[0] = qb.x; wb[1] = qb.y; wb[2] = qb.z; wb[3] = qb.w;
    } else {
      const uint32_t a0 = ra[3 * t], a1 = ra[3 * t + 1], a2 = ra[3 * t + 2];
      const uint32_t b0 = rb[3 * t], b1 = rb[3 * t + 1], b2 = rb[3 * t + 2];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        wa[q] = int3_quarter(a0, a1, a2, q);
        wb[q] = int3_quarter(b0, b1, b2, q);
      }
    }
    float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < 4; ++j) mma_word<BITS>(c, wa[j], wb[j], d.za[0], d.zb[0], d.xq[j]);
    Y[0] = fmaf(d.fa[0], c[0], Y[0]);
    Y[1] = fmaf(d.fa[0], c[1], Y[1]);
    Y[2] = fmaf(d.fb[0], c[2], Y[2]);
    Y[3] = fmaf(d.fb[0], c[3], Y[3]);
  } else {
    // blocks past the row end hold zero x, so their terms vanish
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t wa, wb;
      if constexpr (BITS == 4) {
        wa = ra[4 * j + t];
        wb = rb[4 * j + t];
      } else {
        // quarter t of block j: words 3j + (3t) / 4 and the next
        const int w0 = 3 * j + (3 * t) / 4;
        const uint32_t a_lo = ra[w0], b_lo = rb[w0];
        const uint32_t a_hi = t == 1 || t == 2 ? ra[w0 + 1] : 0u;
        const uint32_t b_hi = t == 1 || t == 2 ? rb[w0 + 1] : 0u;
        wa = t == 0 ? a_lo : t == 1 ? __funnelshift_r(a_lo, a_hi, 24)
                           : t == 2 ? __funnelshift_r(a_lo, a_hi, 16) : a_lo >> 8;
        wb = t == 0 ? b_lo : t == 1 ? __funnelshift_r(b_lo, b_hi, 24)
                           : t == 2 ? __funnelshift_r(b_lo, b_hi, 16) : b_lo >> 8;
      }
      float c[4] = {0.f, 0.f, 0.f, 0.f};
      mma_word<BITS>(c, wa, wb, d.za[j], d.zb[j], d.xq[j]);
      Y[0] = fmaf(d.fa[j], c[0], Y[0]);
      Y[1] = fmaf(d.fa[j], c[1], Y[1]);
      Y[2] = fmaf(d.fb[j], c[2], Y[2]);
      Y[3] = fmaf(d.fb[j], c[3], Y[3]);
    }
  }
}

template <int BITS, bool kInterleaved>
__global__ void __launch_bounds__(kDqWarps * 32, kDqMinBlocks) dequant_mma_kernel(
    const uint32_t* __restrict__ packed, int64_t rows, int64_t n,
    const float* __restrict__ scales, const uint8_t* __restrict__ zeros, int gshift, int64_t G,
    const __nv_bfloat16* __restrict__ xp, int nb, float* __restrict__ y, int64_t ldy) {
  constexpr int P = dq_pitch<BITS, kInterleaved>();
  // int3 pieces are read by other lanes than the ones that stage them
  constexpr bool kShared = kInterleaved || BITS == 3;
  constexpr int kStageBytes = 16 * P;
  __shared__ __align__(16) uint8_t ring[kDqWarps][kDqStages][kStageBytes];
  __shared__ float red[kDqWarps][16][9];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;
  const int64_t r0 = (int64_t)blockIdx.x * 16;
  // rows past the end read the last row (valid memory) and are not stored
  const int64_t ra = min(r0 + g, rows - 1), rb = min(r0 + g + 8, rows - 1);
  const int64_t wpr = n * BITS / 32;  // words per row
  const uint32_t* pa = packed + ra * wpr;
  const uint32_t* pb = packed + rb * wpr;
  const float* sa = scales + ra * G;
  const float* sb = scales + rb * G;
  const uint8_t* za_row = zeros + ra * G;
  const uint8_t* zb_row = zeros + rb * G;
  // vector slots past nb repeat a real vector; their outputs are not stored
  const __nv_bfloat16* xr = xp + (int64_t)(g % nb) * n;
  const int nblk = (int)(n / 32), nsl = (nblk + 3) / 4, nfull = nblk / 4;
  const int per = (nsl + kDqSplit - 1) / kDqSplit;
  const int s_lo = (int)blockIdx.y * per, s_hi = min(nsl, s_lo + per);
  // this warp's slices: first + k kDqWarps, k = 0 .. K - 1
  const int first = s_lo + warp;
  const int K = first < s_hi ? (s_hi - first + kDqWarps - 1) / kDqWarps : 0;
  uint8_t* myring = &ring[warp][0][0];
  // int4: each thread stages 16 bytes (its block) of rows g and g + 8 per
  // slice; int3: 4-byte words t, t + 4, t + 8 of the slice's 12 per row (rows
  // are only 4-byte aligned), words past the row's end not copied
  auto issue = [&](int k) {
    if (k < K) {
      const int sl = first + k * kDqWarps;
      uint8_t* st = myring + (k % kDqStages) * kStageBytes;
      if constexpr (BITS == 4) {
        const int blk = 4 * sl + t;
        if (blk < nblk) {
          ptx::cp_async_16(st + g * P + 16 * t, pa + 4 * blk);
          ptx::cp_async_16(st + (g + 8) * P + 16 * t, pb + 4 * blk);
        }
      } else {
        const int nw = 3 * min(4, nblk - 4 * sl);  // words of this slice in a row
#pragma unroll
        for (int i = 0; i < 3; ++i) {
          const int wdx = t + 4 * i;
          if (wdx < nw) {
            ptx::cp_async_4(st + g * P + 4 * wdx, pa + 12 * sl + wdx, 4);
            ptx::cp_async_4(st + (g + 8) * P + 4 * wdx, pb + 12 * sl + wdx, 4);
          }
        }
      }
    }
    ptx::cp_async_commit();
  };
  auto side = [&](DqSide<kInterleaved>& d, int k) {
    const int s = first + k * kDqWarps;
    if (s < nfull)
      dq_side<kInterleaved, true>(d, s, nblk, t, gshift, xr, sa, sb, za_row, zb_row);
    else
      dq_side<kInterleaved, false>(d, s, nblk, t, gshift, xr, sa, sb, za_row, zb_row);
  };
#pragma unroll
  for (int k = 0; k < kDqStages - 1; ++k) issue(k);
  float Y[4] = {0.f, 0.f, 0.f, 0.f};
  for (int k = 0; k < K; ++k) {
    if (kShared) __syncwarp();  // every lane is done with the slot refilled next
    issue(k + kDqStages - 1);
    ptx::cp_async_wait<kDqStages - 1>();  // slice k has landed (this thread's part)
    if (kShared) __syncwarp();            // ... and every other lane's part
    DqSide<kInterleaved> cur;
    side(cur, k);
    dq_slice<BITS, kInterleaved>(Y, myring + (k % kDqStages) * kStageBytes, cur, g, t);
  }
  ptx::cp_async_wait<0>();
  red[warp][g][2 * t] = Y[0];
  red[warp][g][2 * t + 1] = Y[1];
  red[warp][g + 8][2 * t] = Y[2];
  red[warp][g + 8][2 * t + 1] = Y[3];
  __syncthreads();
  for (int i = threadIdx.x; i < 128; i += kDqWarps * 32) {
    const int b = i >> 4, rr = i & 15;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kDqWarps; ++w) v += red[w][rr][b];
    if (b < nb && r0 + rr < rows) atomicAdd(y + (int64_t)b * ldy + r0 + rr, v);
  }
}

// xp[b][8w + 2i] = x[b][c(8w + i)], xp[b][8w + 2i + 1] = x[b][c(8w + i + 4)]
// (i = 0..3) with c(k) = perm[k] (sweep order) or k; and y[0 .. ny) = 0.
__global__ void dq_prep_kernel(const __nv_bfloat16* __restrict__ x, int64_t n, int64_t nwords,
                               const int32_t* __restrict__ perm, __nv_bfloat16* __restrict__ xp,
                               float* __restrict__ y, int64_t ny) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < nwords; i += stride) {
    const int64_t b = i / (n / 8), w = i % (n / 8);
    const __nv_bfloat16* xb = x + b * n;
    __align__(16) __nv_bfloat16 o[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int64_t c0 = 8 * w + k, c1 = 8 * w + k + 4;
      int64_t s0 = perm ? perm[c0] : c0, s1 = perm ? perm[c1] : c1;
      if (!index_ok(s0, n, kCheckPermutation)) s0 = 0;
      if (!index_ok(s1, n, kCheckPermutation)) s1 = 0;
      o[2 * k] = xb[s0];
      o[2 * k + 1] = xb[s1];
    }
    *reinterpret_cast<uint4*>(xp + b * n + 8 * w) = *reinterpret_cast<const uint4*>(o);
  }
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < ny; i += stride) y[i] = 0.f;
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

size_t dequant_matvec_workspace_bytes(int64_t batch, int64_t n) {
  return ((size_t)batch * (size_t)n * sizeof(__nv_bfloat16) + 255) / 256 * 256;
}

cudaError_t launch_dequant_matvec(const uint32_t* packed, int bits, int64_t rows, int64_t n,
                                  const float* scales, const uint8_t* zeros, int group_size,
                                  int64_t n_groups, const int32_t* g_idx, const int32_t* perm,
                                  const void* x, int x_bf16, int64_t batch, float* y,
                                  void* ws, cudaStream_t s) {
  if (rows == 0 || batch == 0) return cudaSuccess;
  // the tensor-core path: int4 / int3, bf16 activations, groups that are runs of
  // 32 k consecutive columns, 16-byte aligned code rows and activations
  // group sizes: one per row, or a power of two >= 32 (a shift finds the group)
  const bool pow2 = group_size >= 32 && (group_size & (group_size - 1)) == 0;
  const bool mma = x_bf16 && !g_idx && n % 32 == 0 && (group_size <= 0 || pow2) &&
                   reinterpret_cast<uintptr_t>(packed) % (bits == 4 ? 16 : 4) == 0;
  if (mma) {
    // x in MMA pair order (and sweep order under perm), in the caller's workspace
    __nv_bfloat16* xp = static_cast<__nv_bfloat16*>(ws);
    const int64_t nwords = batch * (n / 8), ny = batch * rows;
    const int64_t work = std::max(nwords, ny);
    const unsigned pgrid = (unsigned)std::min<int64_t>((work + 255) / 256, (int64_t)num_sms() * 8);
    dq_prep_kernel<<<pgrid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x), n, nwords, perm,
                                         xp, y, ny);
    note_launch();
    const bool inter = group_size > 0 && group_size < 128;
    int gshift = 31;
    if (group_size > 0)
      for (gshift = 0; (1 << gshift) < group_size; ++gshift) {
      }
    const dim3 grid((unsigned)((rows + 15) / 16), kDqSplit);
    for (int64_t b0 = 0; b0 < batch; b0 += 8) {
      const int nb = (int)(batch - b0 < 8 ? batch - b0 : 8);
      const __nv_bfloat16* xb = xp + b0 * n;
      float* yb = y + b0 * rows;
      if (bits == 4 && inter)
        dequant_mma_kernel<4, true><<<grid, kDqWarps * 32, 0, s>>>(
            packed, rows, n, scales, zeros, gshift, n_groups, xb, nb, yb, rows);
      else if (bits == 4)
        dequant_mma_kernel<4, false><<<grid, kDqWarps * 32, 0, s>>>(
            packed, rows, n, scales, zeros, gshift, n_groups, xb, nb, yb, rows);
      else if (inter)
        dequant_mma_kernel<3, true><<<grid, kDqWarps * 32, 0, s>>>(
            packed, rows, n, scales, zeros, gshift, n_groups, xb, nb, yb, rows);
      else
        dequant_mma_kernel<3, false><<<grid, kDqWarps * 32, 0, s>>>(
            packed, rows, n, scales, zeros, gshift, n_groups, xb, nb, yb, rows);
      note_launch();
    }
    return cudaGetLastError();
  }
  const size_t esz = x_bf16 ? 2 : 4;
  // original column order with g_idx: the row-per-lane kernel, where its
  // 16-byte staging applies
  const bool gx = g_idx && reinterpret_cast<uintptr_t>(packed) % 16 == 0 &&
                  (bits == 4 ? n % 32 == 0 : n % 128 == 0);
  // batches of 8, 4, 2, 1 vectors per launch
  for (int64_t b0 = 0; b0 < batch;) {
    const int64_t left = batch - b0;
    const int b = left >= 8 ? 8 : left >= 4 ? 4 : left >= 2 ? 2 : 1;
    const void* xb = static_cast<const char*>(x) + (size_t)b0 * (size_t)n * esz;
    float* yb = y + b0 * rows;
    if (gx && bits == 4)
      gx_batch<4>(b, packed, rows, n, scales, zeros, n_groups, g_idx, xb, x_bf16, n, yb, rows, s);
    else if (gx)
      gx_batch<3>(b, packed, rows, n, scales, zeros, n_groups, g_idx, xb, x_bf16, n, yb, rows, s);
    else if (bits == 4)
      mv_batch<4>(b, packed, rows, n, scales, zeros, group_size, n_groups, g_idx, perm, xb,
                  x_bf16, n, yb, rows, s);
    else
      mv_batch<3>(b, packed, rows, n, scales, zeros, group_size, n_groups, g_idx, perm, xb,
                  x_bf16, n, yb, rows, s);
    b0 += b;
  }
  return cudaGetLastError();
}

uint32_t take_device_checks_pack() { return take_unit_device_checks(); }

}  // namespace gptq
