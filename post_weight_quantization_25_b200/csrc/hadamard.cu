// Random-sign blocked Hadamard rotation (fast Walsh-Hadamard transform).
//
// Page "Post-Training Quantization: Calibration, GPTQ and Why Rotations Help",
// section "Rotations: making outliers disappear": a Hadamard matrix scaled to
// a rotation spreads one large entry over all entries; the activations get
// the rotation and the weights its inverse, so the layer's product is
// unchanged.  Here R = blockdiag(H_b / sqrt(b)) diag(s) with Sylvester's H_b
// (b a power of two, 32 <= b <= 1024) and per-feature signs s: X' = R X acts
// on the columns of X (features x tokens), W' = W R^T on the rows of W.
//
// Both are HBM-bound passes (one read, one write per element); the transform
// itself is log2(b) butterfly stages in fp32 registers, never a matrix
// product.  A warp holds one block of b = 32 VPL values, lane l holding
// elements l + 32 i: the stages over the high index bits (strides 32 .. b/2)
// run inside each lane, the five over the low bits (strides 1 .. 16) through
// shfl_xor -- or, in the column kernel for b = 1024, inside each lane again
// after the warp re-reads its column from shared memory as elements 32 l + i.
// The order of butterfly stages does not change the result's definition
// (they commute), only the fp32 rounding.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <type_traits>

#include "gptq_internal.cuh"

namespace gptq {
namespace {

__device__ __forceinline__ float to_f(const float* p) { return *p; }
__device__ __forceinline__ float to_f(const __nv_bfloat16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ void from_f(float* p, float v) { *p = v; }
__device__ __forceinline__ void from_f(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

template <int VPL>
__device__ __forceinline__ void fwht_warp(float (&v)[VPL], int lane) {
#pragma unroll
  for (int h = 1; h < VPL; h <<= 1)
#pragma unroll
    for (int i = 0; i < VPL; ++i)
      if ((i & h) == 0) {
        const float a = v[i], b = v[i + h];
        v[i] = a + b;
        v[i + h] = a - b;
      }
  // partner lane l ^ m: the lower lane keeps v + o, the upper one o - v,
  // i.e. o + sgn v with sgn = -1 on the upper lane (one FMA, exact product)
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const float sgn = (lane & m) ? -1.f : 1.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) v[i] = fmaf(sgn, v[i], __shfl_xor_sync(0xffffffffu, v[i], m));
  }
}

// Butterflies over the index bits of i inside one lane (v[i] holds element
// base + stride * i of the block, for any base and stride).
template <int N>
__device__ __forceinline__ void fwht_lane(float (&v)[N]) {
#pragma unroll
  for (int h = 1; h < N; h <<= 1)
#pragma unroll
    for (int i = 0; i < N; ++i)
      if ((i & h) == 0) {
        const float a = v[i], b = v[i + h];
        v[i] = a + b;
        v[i + h] = a - b;
      }
}

// W' = W R^T: each row's blocks of b contiguous elements, one warp per block
// (in == out is allowed: a warp reads its whole block before writing it).
constexpr int kRowsWarps = 8;

template <int VPL, typename TI, typename TO>
__global__ void __launch_bounds__(kRowsWarps * 32) hadamard_rows_kernel(
    const TI* in, int64_t ld_in, TO* out, int64_t ld_out, int64_t rows, int64_t nblk,
    const float* __restrict__ signs, float scale) {
  const int lane = threadIdx.x & 31;
  const int64_t seg = (int64_t)blockIdx.x * kRowsWarps + (threadIdx.x >> 5);
  if (seg >= rows * nblk) return;  // whole warps
  const int64_t r = seg / nblk, c0 = (seg % nblk) * (32 * VPL);
  const TI* p = in + r * ld_in + c0;
  float v[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) v[i] = to_f(p + lane + 32 * i) * __ldg(signs + c0 + lane + 32 * i);
  fwht_warp<VPL>(v, lane);
  TO* q = out + r * ld_out + c0;
#pragma unroll
  for (int i = 0; i < VPL; ++i) from_f(q + lane + 32 * i, v[i] * scale);
}

// X' = R X: a CTA stages b features x kColsTok tokens in shared memory
// (pitch kColsTok + 1 floats, token index XOR-swizzled for b = 1024: the row
// loads and the column passes of the warps land on distinct banks, at most
// two-way in the second pass), then warp w transforms token column w
// (in == out is allowed: the tile is read in full before it is written).
// 32 tokens per tile: each feature row is read and written as 64-byte
// pieces of bf16 (measured 0.90 against 0.97 ms with 16-token tiles on the
// 28672 x 16384 rotation, same results)
constexpr int kColsTok = 32;

// The same row transform with 16-byte accesses, for blocks of 256 or more
// with 16-byte aligned rows: lane l holds elements 256 c + 8 l + j of the
// block (c < VPL / 8, j < 8) in v[8 c + j], so a warp moves 512 (bf16) or
// 1024 (fp32) contiguous bytes per access.  fwht_warp runs its butterflies
// over the register index (element bits 0-2 and 8-9) and the lane index
// (element bits 3-7): the same transform, in a different stage order.
template <typename T>
__device__ __forceinline__ void load8(const T* p, float (&d)[8]) {
  if constexpr (sizeof(T) == 2) {
    const uint4 raw = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&raw);
#pragma unroll
    for (int j = 0; j < 8; ++j) d[j] = __bfloat162float(e[j]);
  } else {
    const float4 a = reinterpret_cast<const float4*>(p)[0];
    const float4 b = reinterpret_cast<const float4*>(p)[1];
    d[0] = a.x; d[1] = a.y; d[2] = a.z; d[3] = a.w;
    d[4] = b.x; d[5] = b.y; d[6] = b.z; d[7] = b.w;
  }
}
template <typename T>
__device__ __forceinline__ void store8(T* p, const float (&d)[8]) {
  if constexpr (sizeof(T) == 2) {
    __align__(16) __nv_bfloat16 e[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) e[j] = __float2bfloat16_rn(d[j]);
    *reinterpret_cast<uint4*>(p) = *reinterpret_cast<const uint4*>(e);
  } else {
    reinterpret_cast<float4*>(p)[0] = make_float4(d[0], d[1], d[2], d[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(d[4], d[5], d[6], d[7]);
  }
}

template <int VPL, typename TI, typename TO>
__global__ void __launch_bounds__(kRowsWarps * 32) hadamard_rows_vec_kernel(
    const TI* in, int64_t ld_in, TO* out, int64_t ld_out, int64_t rows, int64_t nblk,
    const float* __restrict__ signs, float scale) {
  static_assert(VPL % 8 == 0, "chunks of 8 values per lane");
  const int lane = threadIdx.x & 31;
  const int64_t seg = (int64_t)blockIdx.x * kRowsWarps + (threadIdx.x >> 5);
  if (seg >= rows * nblk) return;  // whole warps
  const int64_t r = seg / nblk, c0 = (seg % nblk) * (32 * VPL);
  const TI* p = in + r * ld_in + c0;
  float v[VPL];
#pragma unroll
  for (int c = 0; c < VPL / 8; ++c) {
    float d[8], sg[8];
    load8(p + 256 * c + 8 * lane, d);
    load8(signs + c0 + 256 * c + 8 * lane, sg);
#pragma unroll
    for (int j = 0; j < 8; ++j) v[8 * c + j] = d[j] * sg[j];
  }
  fwht_warp<VPL>(v, lane);
  TO* q = out + r * ld_out + c0;
#pragma unroll
  for (int c = 0; c < VPL / 8; ++c) {
    float d[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) d[j] = v[8 * c + j] * scale;
    store8(q + 256 * c + 8 * lane, d);
  }
}

template <int VPL, typename TI, typename TO>
__global__ void __launch_bounds__(kColsTok * 32) hadamard_cols_kernel(
    const TI* in, int64_t ld_in, TO* out, int64_t ld_out, int64_t ntok,
    const float* __restrict__ signs, float scale, int vec_in, int vec_out) {
  constexpr int B = 32 * VPL, P = kColsTok + 1, NT = kColsTok * 32;
  constexpr int VI = 16 / (int)sizeof(TI), VO = 16 / (int)sizeof(TO);  // per 16 bytes
  extern __shared__ float tile[];  // B x P
  // element (f, t) of the tile; for b = 1024 the token index is XOR-swizzled
  // by the feature's 32-block, so that both column passes below (lane l on
  // features l + 32 i, then on 32 l + i) read their 32 values from distinct
  // banks (at most two-way in the second)
  auto at = [](int f, int t) {
    return VPL == 32 ? f * P + (t ^ ((f >> 5) & (kColsTok - 1))) : f * P + t;
  };
  const int64_t f0 = (int64_t)blockIdx.y * B, t0 = (int64_t)blockIdx.x * kColsTok;
  const int tt = (int)(ntok - t0 < kColsTok ? ntok - t0 : kColsTok);
  const int tid = threadIdx.x;
  if (vec_in && tt == kColsTok) {
    // 16-byte loads: thread -> (feature row, vector of VI tokens)
    constexpr int kPer = kColsTok / VI;
    for (int idx = tid; idx < B * kPer; idx += NT) {
      const int f = idx / kPer, c = idx % kPer;
      const uint4 raw = *reinterpret_cast<const uint4*>(in + (f0 + f) * ld_in + t0 + c * VI);
      const TI* e = reinterpret_cast<const TI*>(&raw);
      const float sg = __ldg(signs + f0 + f);
#pragma unroll
      for (int j = 0; j < VI; ++j) tile[at(f, c * VI + j)] = to_f(e + j) * sg;
    }
  } else {
    const int tc = tid % kColsTok, fr = tid / kColsTok;
    for (int f = fr; f < B; f += NT / kColsTok) {
      const float sg = __ldg(signs + f0 + f);
      tile[at(f, tc)] = tc < tt ? to_f(in + (f0 + f) * ld_in + t0 + tc) * sg : 0.f;
    }
  }
  __syncthreads();
  const int w = tid >> 5, lane = tid & 31;
  float v[VPL];
  if constexpr (VPL == 32) {
    // no shuffles: the high index bits in registers (lane l: features
    // l + 32 i), back to the tile, then the low bits (lane l: 32 l + i)
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = tile[at(lane + 32 * i, w)];
    fwht_lane<32>(v);
#pragma unroll
    for (int i = 0; i < 32; ++i) tile[at(lane + 32 * i, w)] = v[i];
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = tile[at(32 * lane + i, w)];
    fwht_lane<32>(v);
#pragma unroll
    for (int i = 0; i < 32; ++i) tile[at(32 * lane + i, w)] = v[i] * scale;
  } else {
#pragma unroll
    for (int i = 0; i < VPL; ++i) v[i] = tile[at(lane + 32 * i, w)];
    fwht_warp<VPL>(v, lane);
#pragma unroll
    for (int i = 0; i < VPL; ++i) tile[at(lane + 32 * i, w)] = v[i] * scale;
  }
  __syncthreads();
  if (vec_out && tt == kColsTok) {
    constexpr int kPer = kColsTok / VO;
    for (int idx = tid; idx < B * kPer; idx += NT) {
      const int f = idx / kPer, c = idx % kPer;
      uint4 raw;
      TO* e = reinterpret_cast<TO*>(&raw);
#pragma unroll
      for (int j = 0; j < VO; ++j) from_f(e + j, tile[at(f, c * VO + j)]);
      *reinterpret_cast<uint4*>(out + (f0 + f) * ld_out + t0 + c * VO) = raw;
    }
  } else {
    const int tc = tid % kColsTok, fr = tid / kColsTok;
    for (int f = fr; f < B; f += NT / kColsTok)
      if (tc < tt) from_f(out + (f0 + f) * ld_out + t0 + tc, tile[at(f, tc)]);
  }
}

// R X for blocks of 1024 features with bf16 input and output, 64 tokens per
// CTA: the tile is staged as bf16 token pairs (one 32-bit word per feature
// and pair), so each feature row moves as one 128-byte piece; the fp32
// values between the two passes go through a per-warp scratch instead of the
// tile.  Warp w transforms token pairs w and w + 16, one token at a time,
// with the same operations in the same order as hadamard_cols_kernel<32>
// (signs, high index bits, low index bits, scale, one rounding to bf16), so
// the results are the same bit for bit.  Full 64-token tiles only.
constexpr int kC64Tok = 64;
constexpr int kC64Warps = 16;
constexpr int kC64WP = 33;                 // words per tile row (32 pairs + 1: no bank conflicts)
constexpr size_t kC64Smem =
    sizeof(uint32_t) * 1024 * kC64WP + sizeof(float) * kC64Warps * 32 * 33 + sizeof(float) * 1024;

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__global__ void __launch_bounds__(kC64Warps * 32) hadamard_cols1024_bf16_kernel(
    const __nv_bfloat16* in, int64_t ld_in, __nv_bfloat16* out, int64_t ld_out,
    const float* __restrict__ signs, float scale) {
  extern __shared__ __align__(16) uint32_t c64_smem[];
  uint32_t* tile = c64_smem;                                       // [1024][kC64WP]
  float* scr_all = reinterpret_cast<float*>(tile + 1024 * kC64WP); // [warp][32][33]
  float* sgn = scr_all + kC64Warps * 32 * 33;                      // [1024]
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int64_t f0 = (int64_t)blockIdx.y * 1024, t0 = (int64_t)blockIdx.x * kC64Tok;
  for (int f = tid; f < 1024; f += kC64Warps * 32) sgn[f] = __ldg(signs + f0 + f);
  // load: piece p = (row p / 8, 8 tokens 8 (p % 8) ..): 16 bytes from global,
  // four words into the row (a warp covers 4 rows x 128 bytes)
#pragma unroll 4
  for (int j = 0; j < 1024 * 8 / (kC64Warps * 32); ++j) {
    const int p = tid + kC64Warps * 32 * j;
    const int f = p >> 3, c = p & 7;
    const uint4 v = *reinterpret_cast<const uint4*>(in + (f0 + f) * ld_in + t0 + 8 * c);
    uint32_t* d = tile + f * kC64WP + 4 * c;
    d[0] = v.x;
    d[1] = v.y;
    d[2] = v.z;
    d[3] = v.w;
  }
  __syncthreads();
  float* scr = scr_all + w * 32 * 33;
  for (int kp = 0; kp < 2; ++kp) {
    const int k = w + kC64Warps * kp;   // token pair 2k, 2k + 1
    float res[2][32];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      float v[32];
      // pass one: lane l holds features l + 32 i (high index bits in registers)
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const uint32_t word = tile[(lane + 32 * i) * kC64WP + k];
        v[i] = (half ? bf16_hi(word) : bf16_lo(word)) * sgn[lane + 32 * i];
      }
      fwht_lane<32>(v);
#pragma unroll
      for (int i = 0; i < 32; ++i) scr[i * 33 + lane] = v[i];
      __syncwarp();
      // pass two: lane l holds features 32 l + i (low index bits)
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = scr[lane * 33 + i];
      fwht_lane<32>(v);
#pragma unroll
      for (int i = 0; i < 32; ++i) scr[lane * 33 + i] = v[i] * scale;
      __syncwarp();
      // back to lane l holding features l + 32 i
#pragma unroll
      for (int i = 0; i < 32; ++i) res[half][i] = scr[i * 33 + lane];
      __syncwarp();
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const uint32_t lo = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(res[0][i]));
      const uint32_t hi = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(res[1][i]));
      tile[(lane + 32 * i) * kC64WP + k] = lo | (hi << 16);
    }
  }
  __syncthreads();
#pragma unroll 4
  for (int j = 0; j < 1024 * 8 / (kC64Warps * 32); ++j) {
    const int p = tid + kC64Warps * 32 * j;
    const int f = p >> 3, c = p & 7;
    const uint32_t* s = tile + f * kC64WP + 4 * c;
    *reinterpret_cast<uint4*>(out + (f0 + f) * ld_out + t0 + 8 * c) = make_uint4(s[0], s[1], s[2], s[3]);
  }
}

unsigned cdiv(int64_t a, int64_t b) { return (unsigned)((a + b - 1) / b); }

template <int VPL, typename TI, typename TO>
cudaError_t rows_launch(const void* in, int64_t ld_in, void* out, int64_t ld_out, int64_t rows,
                        int64_t n, const float* signs, float scale, cudaStream_t s) {
  const int64_t nblk = n / (32 * VPL);
  const bool vec = VPL % 8 == 0 && reinterpret_cast<uintptr_t>(in) % 16 == 0 &&
                   reinterpret_cast<uintptr_t>(out) % 16 == 0 &&
                   reinterpret_cast<uintptr_t>(signs) % 16 == 0 &&
                   ((size_t)ld_in * sizeof(TI)) % 16 == 0 && ((size_t)ld_out * sizeof(TO)) % 16 == 0;
  if constexpr (VPL % 8 == 0) {
    if (vec) {
      hadamard_rows_vec_kernel<VPL, TI, TO><<<cdiv(rows * nblk, kRowsWarps), kRowsWarps * 32, 0, s>>>(
          static_cast<const TI*>(in), ld_in, static_cast<TO*>(out), ld_out, rows, nblk, signs,
          scale);
      note_launch();
      return cudaGetLastError();
    }
  }
  hadamard_rows_kernel<VPL, TI, TO><<<cdiv(rows * nblk, kRowsWarps), kRowsWarps * 32, 0, s>>>(
      static_cast<const TI*>(in), ld_in, static_cast<TO*>(out), ld_out, rows, nblk, signs, scale);
  note_launch();
  return cudaGetLastError();
}

template <int VPL, typename TI, typename TO>
cudaError_t cols_launch(const void* in, int64_t ld_in, void* out, int64_t ld_out, int64_t n,
                        int64_t ntok, const float* signs, float scale, cudaStream_t s) {
  constexpr int B = 32 * VPL;
  if constexpr (VPL == 32 && std::is_same<TI, __nv_bfloat16>::value &&
                std::is_same<TO, __nv_bfloat16>::value) {
    // whole 64-token tiles by the bf16-tile kernel, the rest (if any) below
    const int64_t nfull = ntok / kC64Tok * kC64Tok;
    const bool ok = nfull > 0 && reinterpret_cast<uintptr_t>(in) % 16 == 0 &&
                    reinterpret_cast<uintptr_t>(out) % 16 == 0 && (ld_in * 2) % 16 == 0 &&
                    (ld_out * 2) % 16 == 0;
    if (ok) {
      cudaError_t e = cudaFuncSetAttribute(hadamard_cols1024_bf16_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)kC64Smem);
      if (e != cudaSuccess) return e;
      const dim3 grid((unsigned)(nfull / kC64Tok), (unsigned)(n / 1024));
      hadamard_cols1024_bf16_kernel<<<grid, kC64Warps * 32, kC64Smem, s>>>(
          static_cast<const __nv_bfloat16*>(in), ld_in, static_cast<__nv_bfloat16*>(out), ld_out,
          signs, scale);
      note_launch();
      if ((e = cudaGetLastError()) != cudaSuccess || nfull == ntok) return e;
      in = static_cast<const __nv_bfloat16*>(in) + nfull;
      out = static_cast<__nv_bfloat16*>(out) + nfull;
      ntok -= nfull;
    }
  }
  const size_t smem = (size_t)B * (kColsTok + 1) * sizeof(float);
  if (smem > 48 * 1024) {
    const cudaError_t e = cudaFuncSetAttribute(hadamard_cols_kernel<VPL, TI, TO>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               (int)smem);
    if (e != cudaSuccess) return e;
  }
  // 16-byte row pieces when every tile's token start is 16-byte aligned
  const int vec_in = (reinterpret_cast<uintptr_t>(in) % 16 == 0) &&
                     ((size_t)ld_in * sizeof(TI)) % 16 == 0;
  const int vec_out = (reinterpret_cast<uintptr_t>(out) % 16 == 0) &&
                      ((size_t)ld_out * sizeof(TO)) % 16 == 0;
  const dim3 grid(cdiv(ntok, kColsTok), (unsigned)(n / B));
  hadamard_cols_kernel<VPL, TI, TO><<<grid, kColsTok * 32, smem, s>>>(
      static_cast<const TI*>(in), ld_in, static_cast<TO*>(out), ld_out, ntok, signs, scale,
      vec_in, vec_out);
  note_launch();
  return cudaGetLastError();
}

template <int VPL>
cudaError_t dispatch(bool cols, int in_bf16, int out_bf16, const void* in, int64_t ld_in,
                     void* out, int64_t ld_out, int64_t a, int64_t b, const float* signs,
                     float scale, cudaStream_t s) {
  using BF = __nv_bfloat16;
  if (cols) {
    if (in_bf16 && out_bf16) return cols_launch<VPL, BF, BF>(in, ld_in, out, ld_out, a, b, signs, scale, s);
    if (in_bf16) return cols_launch<VPL, BF, float>(in, ld_in, out, ld_out, a, b, signs, scale, s);
    if (out_bf16) return cols_launch<VPL, float, BF>(in, ld_in, out, ld_out, a, b, signs, scale, s);
    return cols_launch<VPL, float, float>(in, ld_in, out, ld_out, a, b, signs, scale, s);
  }
  if (in_bf16 && out_bf16) return rows_launch<VPL, BF, BF>(in, ld_in, out, ld_out, a, b, signs, scale, s);
  if (in_bf16) return rows_launch<VPL, BF, float>(in, ld_in, out, ld_out, a, b, signs, scale, s);
  if (out_bf16) return rows_launch<VPL, float, BF>(in, ld_in, out, ld_out, a, b, signs, scale, s);
  return rows_launch<VPL, float, float>(in, ld_in, out, ld_out, a, b, signs, scale, s);
}

}  // namespace

cudaError_t launch_hadamard(bool cols, int block, int in_bf16, int out_bf16, const void* in,
                            int64_t ld_in, void* out, int64_t ld_out, int64_t a, int64_t b,
                            const float* signs, cudaStream_t s) {
  // 1 / sqrt(block): exact for block = 4^k (a power of two), else rounded
  const float scale = (float)(1.0 / std::sqrt((double)block));
  switch (block) {
    case 32: return dispatch<1>(cols, in_bf16, out_bf16, in, ld_in, out, ld_out, a, b, signs, scale, s);
    case 64: return dispatch<2>(cols, in_bf16, out_bf16, in, ld_in, out, ld_out, a, b, signs, scale, s);
    case 128: return dispatch<4>(cols, in_bf16, out_bf16, in, ld_in, out, ld_out, a, b, signs, scale, s);
    case 256: return dispatch<8>(cols, in_bf16, out_bf16, in, ld_in, out, ld_out, a, b, signs, scale, s);
    case 512: return dispatch<16>(cols, in_bf16, out_bf16, in, ld_in, out, ld_out, a, b, signs, scale, s);
    case 1024: return dispatch<32>(cols, in_bf16, out_bf16, in, ld_in, out, ld_out, a, b, signs, scale, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace gptq
