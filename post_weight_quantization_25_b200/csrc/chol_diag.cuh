// The two latency-critical steps of one 128-wide Cholesky panel.
//
//  chol_diag_kernel    one CTA factors the panel's diagonal block A_pp = L L^T
//                      and inverts L's four 32 x 32 diagonal leaves.
//  panel_apply_kernel  every vector of the panel (a row of A below the block,
//                      or a row of the inverse's right-hand side) is solved,
//                      x = v L^-T, as four dense 32-column stages:
//                          x_j = (v_j - sum_{k<j} x_k L_jk^T) Li_jj^T,
//                      so no vector walks 128 dependent substitution steps.
//
// The diagonal block sits in shared memory and is worked in 32 x 32 leaves.
// For leaf j one warp factors the leaf in registers (right-looking, unscaled
// LDL^T, four columns per step: each lane runs the 4 x 4 block's recurrence
// itself, rows exchange 16-byte values through shared memory; square roots
// at the end), the rows
// below it are solved against the leaf by substitution (one thread per row),
// and the remaining lower block takes the rank-32 update from a transposed
// copy of the solved rows (16-byte loads, 8 x 4 register tiles).  At the end
// four warps invert the four leaves at once (one lane per column).
// Every product is an fp32 FMA; no step uses reduced precision.
#pragma once
#include <cstdint>

#include "sm100_ptx.cuh"

namespace gptq {

constexpr int kDiagThreads = 256;
constexpr int kDP = 129;   // row pitch (floats) of the block S
constexpr int kXP = 132;   // row pitch of XT (transposed solved rows)
constexpr int kTP = 36;    // row pitch of a transposed 32 x 32 leaf
// S[128][kDP] | XT[32][kXP] | LTl[32][kTP] | rinv[128] | yb[32], zb[32] (float4) | fail
constexpr size_t kDiagSmemBytes =
    sizeof(float) * (128 * kDP + 32 * kXP + 32 * kTP + 128 + 256) + 16 + 16;  // + the fail flag

// Outputs of chol_diag_kernel, in the Cholesky workspace:
//   Lt[k][c]     = L[c][k]           (128 x 128; only the 32 x 32 blocks with
//                                     block(k) < block(c) are written, the
//                                     ones the apply reads)
//   LiT[j][t][c] = (L_jj^-1)[c][t]   (4 leaves of 32 x 32, zero for t > c)
constexpr int kDiagOutFloats = 128 * 128 + 4 * 32 * 32;

// 1/d: hardware estimate and one Newton step (a multiplier needs no more)
__device__ __forceinline__ float recip_nr(float d) {
  const float r0 = ptx::rcp_approx(d);
  return fmaf(fmaf(-d, r0, 1.f), r0, r0);
}

// One warp: factor the 32 x 32 leaf at (c0, c0) of S in place (lower part);
// writes 1 / L_kk to rinv[c0 + k] and the leaf transposed to LTl[t][m] =
// L[c0+m][c0+t].  Returns (warp-uniform) the 1-based index of the first
// non-positive or non-finite pivot within the leaf, or 0.
//
// Right-looking unscaled LDL^T, four columns per step.  Lane i holds row i.
// For the panel of columns J..J+3 every lane reads the panel's 4 x 4
// diagonal block (rows J..J+3, published in shared memory) and runs the
// same short recurrence: pivots d_t and multipliers M_st = z_st / d_t, with
//     z_i = y_i M^-T:  z_i0 = y_i0,  z_i1 = y_i1 - M10 z_i0,
//                      z_i2 = y_i2 - M20 z_i0 - M21 z_i1,
//                      z_i3 = y_i3 - M30 z_i0 - M31 z_i1 - M32 z_i2
// for its own row's panel entries y_i (z_ss = d_s for the panel rows, so
// every lane sees the same pivots).  z_i stays in the row (the unscaled L
// entries), the rows publish z, and the trailing entries take
//     a_ik -= sum_t (z_it / d_t) z_kt,
// the panel's next four columns first so they can be published early.
// Square roots come at the end: L_ik = z_ik / sqrt(d_k), L_kk = sqrt(d_k).
__device__ __forceinline__ int leaf_factor(float* S, float* rinv, float* LTl, float4* yb,
                                           float4* zb, int c0, int lane) {
  float a[32];
#pragma unroll
  for (int k = 0; k < 32; ++k) a[k] = (k <= lane) ? S[(c0 + lane) * kDP + c0 + k] : 0.f;
  int first_bad = 0;
  yb[lane] = make_float4(a[0], a[1], a[2], a[3]);
#pragma unroll
  for (int J = 0; J < 32; J += 4) {
    __syncwarp();
    // the panel's diagonal block, then the shared recurrence
    const float4 r0 = yb[J], r1 = yb[J + 1], r2 = yb[J + 2], r3 = yb[J + 3];
    const float d0 = r0.x;
    const float i0 = recip_nr(d0);
    const float M10 = r1.x * i0, M20 = r2.x * i0, M30 = r3.x * i0;
    const float d1 = fmaf(-M10, r1.x, r1.y);                 // z_11
    const float i1 = recip_nr(d1);
    const float z21 = fmaf(-M10, r2.x, r2.y);
    const float z31 = fmaf(-M10, r3.x, r3.y);
    const float M21 = z21 * i1, M31 = z31 * i1;
    const float d2 = fmaf(-M21, z21, fmaf(-M20, r2.x, r2.z));  // z_22
    const float i2 = recip_nr(d2);
    const float z32 = fmaf(-M21, z31, fmaf(-M20, r3.x, r3.z));
    const float M32 = z32 * i2;
    const float d3 = fmaf(-M32, z32, fmaf(-M31, z31, fmaf(-M30, r3.x, r3.w)));  // z_33
    const float i3 = recip_nr(d3);
    const float dv[4] = {d0, d1, d2, d3};
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const bool badj = !(dv[t] > 0.f) || !isfinite(dv[t]);
      first_bad = (first_bad == 0 && badj) ? (J + t + 1) : first_bad;
    }
    // this row's z (for the panel rows this reproduces the pivots above)
    const float z0 = a[J];
    const float z1 = fmaf(-M10, z0, a[J + 1]);
    const float z2 = fmaf(-M21, z1, fmaf(-M20, z0, a[J + 2]));
    const float z3 = fmaf(-M32, z2, fmaf(-M31, z1, fmaf(-M30, z0, a[J + 3])));
    a[J] = z0;
    a[J + 1] = z1;
    a[J + 2] = z2;
    a[J + 3] = z3;
    if (J + 4 < 32) {
      zb[lane] = make_float4(z0, z1, z2, z3);
      const float m0 = z0 * i0, m1 = z1 * i1, m2 = z2 * i2, m3 = z3 * i3;
      __syncwarp();
      float4 zk[32];
#pragma unroll
      for (int k = J + 4; k < 32; ++k) zk[k] = zb[k];
      // the next panel's columns first, then publish them
#pragma unroll
      for (int k = J + 4; k < J + 8; ++k)
        a[k] = fmaf(-m3, zk[k].w, fmaf(-m2, zk[k].z, fmaf(-m1, zk[k].y, fmaf(-m0, zk[k].x, a[k]))));
      yb[lane] = make_float4(a[J + 4], a[J + 5], a[J + 6], a[J + 7]);
#pragma unroll
      for (int k = J + 8; k < 32; ++k)
        a[k] = fmaf(-m3, zk[k].w, fmaf(-m2, zk[k].z, fmaf(-m1, zk[k].y, fmaf(-m0, zk[k].x, a[k]))));
    }
  }
  if (first_bad) return first_bad;
  // L_ik = a_ik / sqrt(d_k), L_kk = sqrt(d_k)
  float dd = 1.f;
#pragma unroll
  for (int k = 0; k < 32; ++k)
    if (k == lane) dd = a[k];
  const float rs = __frsqrt_rn(dd);
  rinv[c0 + lane] = rs;
  const float lkk = __fsqrt_rn(dd);
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    const float rk = __shfl_sync(0xffffffffu, rs, k);
    const float l = (k < lane) ? a[k] * rk : ((k == lane) ? lkk : 0.f);
    if (k <= lane) S[(c0 + lane) * kDP + c0 + k] = l;
    LTl[k * kTP + lane] = l;   // zero above the diagonal of the transpose
  }
  return 0;
}

// One warp: column `lane` of the inverse of the 32 x 32 lower leaf at
// (c0, c0) of S, written as row `lane` of LiT: LiT[lane][m] = Li[m][lane].
__device__ __forceinline__ void leaf_inverse(const float* S, const float* rinv, float* LiT,
                                             int c0, int lane) {
  float x[32];
#pragma unroll
  for (int m = 0; m < 32; ++m) x[m] = (m == lane) ? 1.f : 0.f;
#pragma unroll
  for (int t = 0; t < 32; ++t) {
    const float xt = x[t] * rinv[c0 + t];
    x[t] = xt;
#pragma unroll
    for (int m = t + 1; m < 32; ++m) x[m] = fmaf(-S[(c0 + m) * kDP + c0 + t], xt, x[m]);
  }
  float4* dst = reinterpret_cast<float4*>(LiT + lane * 32);
#pragma unroll
  for (int q = 0; q < 8; ++q)
    dst[q] = make_float4(4 * q + 0 >= lane ? x[4 * q + 0] : 0.f, 4 * q + 1 >= lane ? x[4 * q + 1] : 0.f,
                         4 * q + 2 >= lane ? x[4 * q + 2] : 0.f, 4 * q + 3 >= lane ? x[4 * q + 3] : 0.f);
}

// Threads 0 .. kDiagThreads - 1 synchronise on barrier `bar` (0:
// __syncthreads, else a named barrier of kDiagThreads threads).
__device__ __forceinline__ void diag_sync(int bar) {
  if (bar == 0)
    __syncthreads();
  else
    ptx::named_bar_sync(bar, kDiagThreads);
}

// Factor the diagonal block of panel p of the n x n lower matrix A and
// invert its leaves; writes Lt and LiT (layouts above) to `out`.  Rows and
// columns past a short last panel are identity padding.  On a failed pivot
// sets *info = n - (global index of the pivot in A), if no failure was
// recorded before, and returns.  Run by threads 0 .. kDiagThreads - 1 (tid)
// with kDiagSmemBytes of shared memory at dsm.
__device__ __forceinline__ void chol_diag_body(const float* __restrict__ A, int n, int p,
                                               float* __restrict__ out,
                                               int32_t* __restrict__ info, float* dsm, int tid,
                                               int bar) {
  float* S = dsm;                    // [128][kDP]  the block, becomes L
  float* XT = S + 128 * kDP;         // [32][kXP]   XT[k][r] = solved row r, column k of the leaf
  XT = reinterpret_cast<float*>((reinterpret_cast<uintptr_t>(XT) + 15) & ~uintptr_t(15));
  float* LTl = XT + 32 * kXP;        // [32][kTP]   current leaf, transposed
  float* rinv = LTl + 32 * kTP;      // [128]       1 / L_kk
  float4* yb = reinterpret_cast<float4*>(rinv + 128);  // [32] leaf panel rows
  float4* zb = yb + 32;                                 // [32] leaf z values
  volatile int* fail = reinterpret_cast<volatile int*>(zb + 32);
  const int kb = p * 128;
  const int bs = min(128, n - kb);
  const int lane = tid & 31, warp = tid >> 5;

  // stage the lower block (async copies, all in flight at once); rows past
  // bs are the identity; entries above the diagonal are never read
  if ((n % 4) == 0) {
    // 16-byte loads (rows start 16-byte aligned, bs is a multiple of 4), four
    // in flight per thread before their stores into the odd-pitched block
    constexpr int kIt = 128 * 32 / kDiagThreads;
#pragma unroll 1
    for (int i0 = 0; i0 < kIt; i0 += 4) {
      float4 v[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int f = tid + kDiagThreads * (i0 + i);
        const int r = f >> 5, c = (f & 31) * 4;
        v[i] = (c <= r && r < bs)
                   ? __ldcg(reinterpret_cast<const float4*>(A + (int64_t)(kb + r) * n + kb + c))
                   : make_float4(r == c, r == c + 1, r == c + 2, r == c + 3);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int f = tid + kDiagThreads * (i0 + i);
        const int r = f >> 5, c = (f & 31) * 4;
        if (c > r) continue;
        float* d = S + r * kDP + c;
        d[0] = v[i].x;
        d[1] = v[i].y;
        d[2] = v[i].z;
        d[3] = v[i].w;
      }
    }
  } else {
    for (int f = tid; f < 128 * 32; f += kDiagThreads) {
      const int r = f >> 5, c = (f & 31) * 4;
      if (c > r) continue;
      if (r >= bs) {
#pragma unroll
        for (int i = 0; i < 4; ++i) S[r * kDP + c + i] = (r == c + i) ? 1.f : 0.f;
        continue;
      }
      const float* src = A + (int64_t)(kb + r) * n + kb + c;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        ptx::cp_async_4(S + r * kDP + c + i, (c + i < bs) ? src + i : src, (c + i < bs) ? 4 : 0);
    }
    ptx::cp_async_wait_all();
  }
  if (tid == 0) *fail = 0;
  diag_sync(bar);

  for (int j = 0; j < 4; ++j) {
    const int c0 = 32 * j;
    if (warp == 0) {
      const int fb = leaf_factor(S, rinv, LTl, yb, zb, c0, lane);
      if (fb && lane == 0) *fail = c0 + fb;
    }
    diag_sync(bar);
    const int fl = *fail;
    if (fl) {
      if (tid == 0) atomicCAS(info, 0, n - (kb + fl - 1));
      return;
    }
    const int base = c0 + 32;
    const int rem = 128 - base;
    if (rem == 0) break;
    // rows below the leaf: x <- x L_jj^-T by substitution, one thread per row;
    // the leaf's columns come from LTl as 16-byte broadcasts
    if (tid < rem) {
      const int r = base + tid;
      float x[32];
#pragma unroll
      for (int k = 0; k < 32; ++k) x[k] = S[r * kDP + c0 + k];
#pragma unroll
      for (int t = 0; t < 32; ++t) {
        const float xt = x[t] * rinv[c0 + t];
        x[t] = xt;
        const float4* lt = reinterpret_cast<const float4*>(LTl + t * kTP);
#pragma unroll
        for (int q = (t + 1) / 4; q < 8; ++q) {
          const float4 l4 = lt[q];
          if (4 * q + 0 > t) x[4 * q + 0] = fmaf(-xt, l4.x, x[4 * q + 0]);
          if (4 * q + 1 > t) x[4 * q + 1] = fmaf(-xt, l4.y, x[4 * q + 1]);
          if (4 * q + 2 > t) x[4 * q + 2] = fmaf(-xt, l4.z, x[4 * q + 2]);
          if (4 * q + 3 > t) x[4 * q + 3] = fmaf(-xt, l4.w, x[4 * q + 3]);
        }
      }
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        S[r * kDP + c0 + k] = x[k];
        XT[k * kXP + (r - base)] = x[k];
      }
    }
    diag_sync(bar);
    // rank-32 update of the remaining lower block: 8-row x 4-column tiles
    // (ti, tj) with 4 tj <= 8 ti + 7; rows past bs are identity padding
    {
      const int mt = rem / 8;                 // row tiles
      const int ntiles = mt * (mt + 1);       // sum over ti of (2 ti + 2)
      for (int t = tid; t < ntiles; t += kDiagThreads) {
        int ti = 0;
        while ((ti + 1) * (ti + 2) <= t) ++ti;
        const int tj = t - ti * (ti + 1);
        const int rl = 8 * ti, sl = 4 * tj;   // local to base
        float acc[8][4];
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int q = 0; q < 4; ++q) acc[i][q] = 0.f;
#pragma unroll 4
        for (int k = 0; k < 32; ++k) {
          const float4 r4a = *reinterpret_cast<const float4*>(XT + k * kXP + rl);
          const float4 r4b = *reinterpret_cast<const float4*>(XT + k * kXP + rl + 4);
          const float4 s4 = *reinterpret_cast<const float4*>(XT + k * kXP + sl);
          const float ra[8] = {r4a.x, r4a.y, r4a.z, r4a.w, r4b.x, r4b.y, r4b.z, r4b.w};
          const float sa[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
          for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[i][q] = fmaf(ra[i], sa[q], acc[i][q]);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = base + rl + i;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int s = base + sl + q;
            if (s <= r && r < bs) S[r * kDP + s] -= acc[i][q];
          }
        }
      }
    }
    diag_sync(bar);
  }

  // ---- outputs: the four leaf inverses (warps 0-3) beside the blocks of
  // L transposed that the apply reads (warps 4-7): the six 32 x 32 blocks
  // (kb, jb), kb < jb, of Lt (rows k of block kb, columns c of block jb);
  // the rest of Lt is never read and is not written
  float* Lt = out;
  float* LiT = out + 128 * 128;
  if (warp < 4) {
    leaf_inverse(S, rinv, LiT + warp * 32 * 32, 32 * warp, lane);
  } else {
    for (int f = tid - 128; f < 6 * 32 * 8; f += kDiagThreads - 128) {
      const int b = f >> 8, r = (f >> 3) & 31, q = f & 7;
      const int kb = b < 3 ? 0 : (b < 5 ? 1 : 2);
      const int jb = b < 3 ? b + 1 : (b < 5 ? b - 1 : 3);
      const int k = 32 * kb + r, c = 32 * jb + 4 * q;   // k < c: below the diagonal of L
      float4 o;
      o.x = S[(c + 0) * kDP + k];
      o.y = S[(c + 1) * kDP + k];
      o.z = S[(c + 2) * kDP + k];
      o.w = S[(c + 3) * kDP + k];
      *reinterpret_cast<float4*>(Lt + k * 128 + c) = o;
    }
  }
}

__global__ void __launch_bounds__(kDiagThreads) chol_diag_kernel(const float* __restrict__ A,
                                                                 int n, int p,
                                                                 float* __restrict__ out,
                                                                 int32_t* __restrict__ info) {
  if (*(volatile int32_t*)info != 0) return;
  extern __shared__ __align__(16) float dsm[];
  chol_diag_body(A, n, p, out, info, dsm, threadIdx.x, 0);
}

// x = v L^-T for every vector of panel p: vectors [0, nA) are rows
// kb+bs+v of A, vectors [nA, nA + kb + bs) are rows v - nA of RT (both
// restricted to the panel's columns [kb, kb + bs)).  The result goes, split
// into its TF32 part and remainder, to row g (row pitch ldpb) of PBh / PBl (g = the vector's
// row in A or RT); RT rows also get x written back.
// 32 vectors per CTA; stage j: thread (v, cq) = (tid / 8, tid % 8) owns
// columns 32 j + 4 cq .. + 3 of vector v.
constexpr int kApplyThreads = 256;
constexpr int kApplyVecs = 32;
constexpr int kVP = 132;  // row pitch of the vector tile
constexpr size_t kApplySmemBytes =
    sizeof(float) * (128 * 128 + 4 * 32 * 32 + 2 * kApplyVecs * kVP);

// Vectors [v0, v0 + kApplyVecs) of panel p, by threads 0 .. kApplyThreads - 1
// (tid) with kApplySmemBytes of shared memory at asmem; barrier as diag_sync.
__device__ __forceinline__ void panel_apply_body(
    const float* __restrict__ A, float* __restrict__ RT, int n, int p,
    const float* __restrict__ diag_out, float* __restrict__ PBh, float* __restrict__ PBl, int ldpb,
    float* asmem, int tid, int v0, int bar) {
  static_assert(kApplyThreads == kDiagThreads, "the apply shares the diagonal step's barrier");
  float* Lt = asmem;                         // [128][128]
  float* LiT = Lt + 128 * 128;               // [4][32][32]
  float* X = LiT + 4 * 32 * 32;              // [32][kVP]  vectors, solved in place
  float* Y = X + kApplyVecs * kVP;           // [32][kVP]  stage scratch
  const int kb = p * 128;
  const int bs = min(128, n - kb);
  const int nA = n - kb - bs;
  const int nvec = nA + kb + bs;
  if (v0 >= nvec) return;
  // everything staged with async copies, all in flight at once.  Of L^T only
  // the six 32 x 32 blocks (kb, jb), kb < jb, are read (stage jb takes rows
  // k < 32 jb of its columns); the inverted leaves in full
  for (int f = tid; f < 6 * 32 * 8; f += kApplyThreads) {
    const int b = f >> 8, r = (f >> 3) & 31, q = f & 7;
    const int kb = b < 3 ? 0 : (b < 5 ? 1 : 2);
    const int jb = b < 3 ? b + 1 : (b < 5 ? b - 1 : 3);
    const int off = (32 * kb + r) * 128 + 32 * jb + 4 * q;
    ptx::cp_async_16(asmem + off, diag_out + off);
  }
  for (int f = tid; f < 4 * 32 * 32 / 4; f += kApplyThreads)
    ptx::cp_async_16(LiT + 4 * f, diag_out + 128 * 128 + 4 * f);
  if ((n % 4) == 0) {
    // rows start 16-byte aligned and bs is a multiple of 4: 16-byte copies
    for (int f = tid; f < kApplyVecs * 32; f += kApplyThreads) {
      const int vi = f >> 5, k = (f & 31) * 4;
      const int v = v0 + vi;
      const bool ok = v < nvec && k < bs;
      const float* row = (v < nA) ? (A + (int64_t)(kb + bs + v) * n + kb)
                                  : (RT + (int64_t)min(v - nA, n - 1) * n + kb);
      ptx::cp_async_16z(X + vi * kVP + k, ok ? row + k : A, ok ? 16 : 0);
    }
  } else {
    for (int f = tid; f < kApplyVecs * 128; f += kApplyThreads) {
      const int vi = f >> 7, k = f & 127;
      const int v = v0 + vi;
      const bool ok = v < nvec && k < bs;
      const float* row = (v < nA) ? (A + (int64_t)(kb + bs + v) * n + kb)
                                  : (RT + (int64_t)min(v - nA, n - 1) * n + kb);
      ptx::cp_async_4(X + vi * kVP + k, ok ? row + k : A, ok ? 4 : 0);
    }
  }
  ptx::cp_async_wait_all();
  diag_sync(bar);
  const int vi = tid >> 3, cq = tid & 7;
  float* xr = X + vi * kVP;
  for (int j = 0; j < 4; ++j) {
    const int cb = 32 * j + 4 * cq;
    // y = v_j - sum_{k < 32 j} x_k L[cb + i][k]
    float y0 = xr[cb], y1 = xr[cb + 1], y2 = xr[cb + 2], y3 = xr[cb + 3];
    // eight k at a time: their loads are issued together, then the FMAs
    // (still in k order)
#pragma unroll 1
    for (int k0 = 0; k0 < 32 * j; k0 += 8) {
      const float4 xa = *reinterpret_cast<const float4*>(xr + k0);
      const float4 xb = *reinterpret_cast<const float4*>(xr + k0 + 4);
      const float xk[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
      float4 l4[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) l4[i] = *reinterpret_cast<const float4*>(Lt + (k0 + i) * 128 + cb);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        y0 = fmaf(-xk[i], l4[i].x, y0);
        y1 = fmaf(-xk[i], l4[i].y, y1);
        y2 = fmaf(-xk[i], l4[i].z, y2);
        y3 = fmaf(-xk[i], l4[i].w, y3);
      }
    }
    *reinterpret_cast<float4*>(Y + vi * kVP + 4 * cq) = make_float4(y0, y1, y2, y3);
    diag_sync(bar);
    // x_j = y Li_jj^T: x[c] = sum_{t <= c} y[t] Li[c][t] = sum_t y[t] LiT[t][c]
    const float* yr = Y + vi * kVP;
    const float* lit = LiT + j * 32 * 32 + 4 * cq;
    float z0 = 0.f, z1 = 0.f, z2 = 0.f, z3 = 0.f;
#pragma unroll
    for (int t0 = 0; t0 < 32; t0 += 8) {
      const float4 ya = *reinterpret_cast<const float4*>(yr + t0);
      const float4 yb = *reinterpret_cast<const float4*>(yr + t0 + 4);
      const float yt[8] = {ya.x, ya.y, ya.z, ya.w, yb.x, yb.y, yb.z, yb.w};
      float4 l4[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) l4[i] = *reinterpret_cast<const float4*>(lit + (t0 + i) * 32);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        z0 = fmaf(yt[i], l4[i].x, z0);
        z1 = fmaf(yt[i], l4[i].y, z1);
        z2 = fmaf(yt[i], l4[i].z, z2);
        z3 = fmaf(yt[i], l4[i].w, z3);
      }
    }
    *reinterpret_cast<float4*>(xr + cb) = make_float4(z0, z1, z2, z3);
    diag_sync(bar);
  }
  // outputs
  for (int f = tid; f < kApplyVecs * 32; f += kApplyThreads) {
    const int vv = f >> 5, c4 = (f & 31) * 4;
    const int v = v0 + vv;
    if (v >= nvec) continue;
    const bool is_rt = v >= nA;
    const int64_t g = is_rt ? (int64_t)(v - nA) : (int64_t)(kb + bs + v);
    float4 x4 = *reinterpret_cast<const float4*>(X + vv * kVP + c4);
    float xv[4] = {x4.x, x4.y, x4.z, x4.w};
    float hv[4], lv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (c4 + i >= bs) xv[i] = 0.f;
      hv[i] = ptx::tf32_hi(xv[i]);
      lv[i] = xv[i] - hv[i];
    }
    *reinterpret_cast<float4*>(PBh + g * ldpb + c4) = make_float4(hv[0], hv[1], hv[2], hv[3]);
    *reinterpret_cast<float4*>(PBl + g * ldpb + c4) = make_float4(lv[0], lv[1], lv[2], lv[3]);
    if (is_rt) {
      float* rt = RT + g * n + kb;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (c4 + i < bs) rt[c4 + i] = xv[i];
    }
  }
}

__global__ void __launch_bounds__(kApplyThreads) panel_apply_kernel(
    const float* __restrict__ A, float* __restrict__ RT, int n, int p,
    const float* __restrict__ diag_out, float* __restrict__ PBh, float* __restrict__ PBl, int ldpb,
    const int32_t* __restrict__ info) {
  if (*(volatile const int32_t*)info != 0) return;
  extern __shared__ __align__(16) float asmem[];
  panel_apply_body(A, RT, n, p, diag_out, PBh, PBl, ldpb, asmem, threadIdx.x,
                   blockIdx.x * kApplyVecs, 0);
}

}  // namespace gptq
