// Correctly rounded binary32 division a / b by Markstein's method, for use on
// latency-critical chains where b is reused (the ruler's scale, fixed for a
// whole group of columns).
//
// Method: P. Markstein, "Computation of elementary functions on the IBM
// RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990; also J.-M.
// Muller et al., "Handbook of Floating-Point Arithmetic", 2nd ed., ch. 4
// (division with a fused multiply-add).  With y = RN(1/b) and a quotient q
// within one ulp of a/b, the remainder r = a - b q is exact in binary32 and
// RN(q + r y) = RN(a / b).  Starting from q0 = RN(a y), one correction step
// brings q within one ulp, and a second one rounds correctly.
//
// Domain: b positive and normal, a / b neither overflowing nor needing
// gradual underflow of the remainder; md_prepare() rescales b (and, per
// call, a) by an exact power of two so that any positive normal or
// subnormal b is covered.  A GPU test compares the result with CUDA's IEEE
// division bit for bit, including quotients next to half-integers.
#pragma once

namespace gptq {

struct MDiv {
  float b;   // rescaled divisor
  float y;   // RN(1 / b)
  float sa;  // power of two applied to the dividend
};

__device__ __forceinline__ MDiv md_prepare(float b) {
  MDiv m;
  m.sa = (b < 0x1p-64f) ? 0x1p64f : ((b > 0x1p64f) ? 0x1p-64f : 1.f);
  m.b = b * m.sa;
  m.y = __frcp_rn(m.b);
  return m;
}

__device__ __forceinline__ float md_div(float a, const MDiv& m) {
  const float x = a * m.sa;  // exact: power-of-two rescaling in range
  const float q0 = x * m.y;
  const float r0 = fmaf(-m.b, q0, x);
  const float q1 = fmaf(r0, m.y, q0);
  const float r1 = fmaf(-m.b, q1, x);
  return fmaf(r1, m.y, q1);
}

}  // namespace gptq
