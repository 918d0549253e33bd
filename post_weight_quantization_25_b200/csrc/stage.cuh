// Staging a 128 x 128 fp32 block from global memory into shared memory with
// many loads in flight per thread (the naive one-load-per-iteration loop is
// bound by L2 latency, roughly 128 serialized round trips per CTA).
#pragma once
#include <cstdint>

namespace gptq {

// For every element (r, c) of the 128 x 128 block whose top-left corner is
// `src` (row stride `ld` floats) calls store(r, c, v), where v is the element
// if r < vr, c < vc (and c <= r when `lower`), else `pad(r, c)`.
// NT threads cooperate; each keeps 8 float4 loads in flight.  `vec` says that
// src and ld allow 16-byte loads.
template <int NT, class Store, class Pad>
__device__ __forceinline__ void stage_block_128(const float* __restrict__ src, int64_t ld, int vr,
                                                int vc, bool lower, bool vec, Store store,
                                                Pad pad) {
  constexpr int kF4 = 128 * 128 / 4;  // float4 slots in the block
  for (int f0 = 0; f0 < kF4; f0 += 8 * NT) {
    float4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int f = f0 + u * NT + (int)threadIdx.x;
      const int r = f >> 5, c = (f & 31) * 4;
      v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (f < kF4 && r < vr && c < vc && (!lower || c <= r)) {
        const float* s = src + (int64_t)r * ld + c;
        if (vec && c + 3 < vc) {
          v[u] = *reinterpret_cast<const float4*>(s);
        } else {
          v[u].x = s[0];
          if (c + 1 < vc) v[u].y = s[1];
          if (c + 2 < vc) v[u].z = s[2];
          if (c + 3 < vc) v[u].w = s[3];
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int f = f0 + u * NT + (int)threadIdx.x;
      if (f >= kF4) continue;
      const int r = f >> 5, c = (f & 31) * 4;
      const float e[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int cc = c + k;
        const bool inside = r < vr && cc < vc && (!lower || cc <= r);
        store(r, cc, inside ? e[k] : pad(r, cc));
      }
    }
  }
}

}  // namespace gptq
