// Preparation of H and the upper Cholesky factor U of the damped inverse.
//
// Page "GPTQ, with the code open":
//  * section "Paper vs. code": silent inputs (diag(H) == 0) are dead, their
//    diagonal is set to 1; act-order sorts the columns by descending
//    diag(H); 1 % of mean(diag H) is added to the diagonal;
//  * section "From one repair to a whole model": a Cholesky factorisation
//    whose rows hold every entry of the shrinking inverses [H_F^-1] -- the
//    upper factor U with H'^-1 = U^T U; U[j][j]^2 = [H_F^-1]_jj for
//    F = {j, ..., n-1}.
//
// Route taken here (one factorisation and one triangular inverse instead of
// the pages' Cholesky -> inverse -> Cholesky): with J the index reversal,
// factor J H' J = L L^T (lower L), invert M = L^-1, and U = J M J.  Because
// H' = (J L J)(J L J)^T with J L J upper, (J L J)^-1 = J M J is the upper
// factor of H'^-1, and that factor is unique.
//
// Both the factorisation and the inverse run right-looking over 128-wide
// panels p = 0, 1, ...:
//   (a) factor the diagonal block L_pp                         (1 CTA)
//   (b) apply L_pp^-1 to every vector that needs it: the panel rows below
//       (-> L_ip, the triangular solve) and the block row p of the inverse's
//       right-hand side (-> M_p., forward substitution)       (one warp per vector)
//   (c) rank-128 updates of the trailing lower matrix and of the remaining
//       right-hand side rows                                   (fp32 tiles)
// The inverse is kept transposed (RT = M^T) in U's own buffer, so that every
// vector in (b) and every operand in (c) is a contiguous row segment; at the
// end U = J M J = (J RT J)^T is one in-place anti-transpose of that buffer.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>

#include "gptq_internal.cuh"
#include "panel_gemm.cuh"
#include "stage.cuh"

namespace gptq {
namespace {

constexpr int kPanel = kBlock;  // 128
constexpr int kPadLD = kPanel + 1;
constexpr int32_t kInfoTimeout = -2;  // `info` value when a device wait gave up

struct CholWs {
  float* A;       // n x n, lower part used: J P^T H P J + lambda I
  float* dprime;  // n: diag(H) with dead entries set to 1
  double* lam;    // 1: damping
  float* PBh;     // n x 128: the current panel's solved vectors, TF32 part
  float* PBl;     // n x 128: remainder
};

constexpr size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Workspace bytes for order n (also sizes the built-in scratch of the
// allocation-free entry point below, hence constexpr).
constexpr size_t chol_ws_bytes(int64_t n) {
  return align_up(sizeof(float) * n * n, 256) + align_up(sizeof(float) * n, 256) + 256 +
         2 * align_up(sizeof(float) * n * kPanel, 256);
}

CholWs carve(void* ws, int64_t n) {
  char* p = static_cast<char*>(ws);
  CholWs w;
  w.A = reinterpret_cast<float*>(p);
  p += align_up(sizeof(float) * n * n, 256);
  w.dprime = reinterpret_cast<float*>(p);
  p += align_up(sizeof(float) * n, 256);
  w.lam = reinterpret_cast<double*>(p);
  p += 256;
  w.PBh = reinterpret_cast<float*>(p);
  p += align_up(sizeof(float) * n * kPanel, 256);
  w.PBl = reinterpret_cast<float*>(p);
  return w;
}

// ---------------------------------------------------------------- preparation
__global__ void __launch_bounds__(1024) diag_prep_kernel(const float* __restrict__ H, int n,
                                                         float percdamp, uint8_t* __restrict__ dead,
                                                         float* __restrict__ dprime,
                                                         double* __restrict__ lam,
                                                         int32_t* __restrict__ info) {
  __shared__ double part[32];
  double sum = 0.0;
  bool bad = false;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    const float d = H[(int64_t)i * n + i];
    const bool is_dead = (d == 0.f);
    const float dd = is_dead ? 1.f : d;
    bad |= !isfinite(d);
    dead[i] = is_dead ? 1 : 0;
    dprime[i] = dd;
    sum += (double)dd;
  }
  if (__syncthreads_or(bad) && threadIdx.x == 0) atomicCAS(info, 0, -1);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = sum;
  __syncthreads();
  if (threadIdx.x < 32) {
    double v = (threadIdx.x < (blockDim.x >> 5)) ? part[threadIdx.x] : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (threadIdx.x == 0) *lam = (double)percdamp * (v / (double)n);
  }
}

// Stable descending order of dprime: position of i = #{j: d_j > d_i} +
// #{j < i: d_j == d_i}.  NaN keys rank as -inf so the result is always a
// permutation (a NaN diagonal is reported through info anyway).
__device__ __forceinline__ float rank_key(float d) { return isnan(d) ? -INFINITY : d; }

__global__ void __launch_bounds__(256) actorder_rank_kernel(const float* __restrict__ dprime,
                                                            int n, int32_t* __restrict__ perm) {
  __shared__ float keys[2048];
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const float ki = (i < n) ? rank_key(dprime[i]) : 0.f;
  int pos = 0;
  for (int t0 = 0; t0 < n; t0 += 2048) {
    const int cnt = min(2048, n - t0);
    for (int j = threadIdx.x; j < cnt; j += blockDim.x) keys[j] = rank_key(dprime[t0 + j]);
    __syncthreads();
    if (i < n) {
      for (int j = 0; j < cnt; ++j) {
        const float kj = keys[j];
        pos += (kj > ki) || (kj == ki && t0 + j < i);
      }
    }
    __syncthreads();
  }
  if (i < n) perm[pos] = i;
}

__global__ void iota_kernel(int32_t* __restrict__ perm, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) perm[i] = i;
}

// A[a][b] (b <= a) = H[p(n-1-a)][p(n-1-b)] (+ lambda on the diagonal, dead -> 1 + lambda).
// One CTA per output row; the source row of H is staged in shared memory.
__global__ void __launch_bounds__(256) gather_reversed_kernel(
    const float* __restrict__ H, int n, const int32_t* __restrict__ perm,
    const uint8_t* __restrict__ dead, const double* __restrict__ lam, float* __restrict__ A) {
  extern __shared__ float hrow[];
  const int a = blockIdx.x;
  const int pa = perm ? perm[n - 1 - a] : (n - 1 - a);
  const float* src = H + (int64_t)pa * n;
  for (int j = threadIdx.x; j < n; j += blockDim.x) hrow[j] = src[j];
  __syncthreads();
  const float lf = (float)(*lam);
  float* dst = A + (int64_t)a * n;
  for (int b = threadIdx.x; b <= a; b += blockDim.x) {
    const int pb = perm ? perm[n - 1 - b] : (n - 1 - b);
    float v = hrow[pb];
    if (b == a) v = (dead[pa] ? 1.f : v) + lf;
    dst[b] = v;
  }
}

__global__ void set_diag_one_kernel(float* __restrict__ M, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) M[(int64_t)i * n + i] = 1.f;
}

// ---------------------------------------------------------------- panel (a)
// Factor the diagonal block of panel p in place (lower part of A).
//
// Blocked over four 32-column sub-panels, block kept in shared memory:
//  (1) one warp factors the 32 x 32 diagonal sub-block in registers (lane i
//      holds row i): per column one shuffle for the pivot, then the column's
//      entries are shuffled to the lanes that need them -- no barriers;
//  (2) the rows below it solve against that factor in parallel (one thread
//      per row, 32 entries in registers, the factor read as broadcasts);
//  (3) all threads subtract the rank-32 product from the remaining lower
//      block with 4 x 4 register tiles.
__device__ __forceinline__ float chol_elem(const float* S, int r, int c) {
  return S[r * kPadLD + c];
}

__global__ void __launch_bounds__(256) chol_diag_kernel(float* __restrict__ A, int n, int p,
                                                        int32_t* __restrict__ info) {
  if (*(volatile int32_t*)info != 0) return;
  extern __shared__ float dyn_smem[];
  float* S = dyn_smem;                     // [128][kPadLD]
  float* rdiag = dyn_smem + kPanel * kPadLD;  // [128]
  __shared__ int fail;
  const int kb = p * kPanel;
  const int bs = min(kPanel, n - kb);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool vec = (n % 4) == 0;
  // stage the lower block (identity padding), 8 float4 loads in flight per thread
  for (int f0 = 0; f0 < kPanel * kPanel / 4; f0 += 8 * 256) {
    float4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int f = f0 + u * 256 + tid;
      const int r = f >> 5, c = (f & 31) * 4;
      v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r < bs && c <= r) {
        const float* src = A + (int64_t)(kb + r) * n + kb + c;
        if (vec && c + 3 < bs) {
          v[u] = *reinterpret_cast<const float4*>(src);
        } else {
          v[u].x = src[0];
          if (c + 1 < bs) v[u].y = src[1];
          if (c + 2 < bs) v[u].z = src[2];
          if (c + 3 < bs) v[u].w = src[3];
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int f = f0 + u * 256 + tid;
      const int r = f >> 5, c = (f & 31) * 4;
      float* d = S + r * kPadLD + c;
      d[0] = (r == c) ? (r < bs ? v[u].x : 1.f) : v[u].x;
      d[1] = (r == c + 1) ? (r < bs ? v[u].y : 1.f) : v[u].y;
      d[2] = (r == c + 2) ? (r < bs ? v[u].z : 1.f) : v[u].z;
      d[3] = (r == c + 3) ? (r < bs ? v[u].w : 1.f) : v[u].w;
    }
  }
  if (tid == 0) fail = 0;
  __syncthreads();

  for (int c0 = 0; c0 < bs; c0 += 32) {
    // (1) 32 x 32 diagonal sub-block, one warp, registers.  Unscaled
    // (LDL^T-like) right-looking form: step j publishes column j as it
    // stands (colj[k] = a_kj) and every lane i > j applies
    // a_ik -= (a_ij / d_j) a_kj; the column entries are read from shared
    // memory with independent loads issued ahead of the FMAs, so a step is
    // one short dependency chain.  Square roots come at the end:
    // L_ik = a_ik / sqrt(d_k), L_kk = sqrt(d_k).
    if (warp == 0) {
      float* colj = rdiag + kPanel;  // 32 floats of scratch after rdiag
      float a[32];
#pragma unroll
      for (int k = 0; k < 32; ++k) a[k] = (k <= lane) ? chol_elem(S, c0 + lane, c0 + k) : 0.f;
      bool bad = false;
      int first_bad = 0;
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        colj[lane] = (lane >= j) ? a[j] : 0.f;
        __syncwarp();
        const float d = colj[j];
        // failure bookkeeping by selects (no branch inside the unrolled loop);
        // once bad, the results are discarded
        const bool badj = !(d > 0.f) || !isfinite(d);
        first_bad = (!bad && badj) ? (c0 + j + 1) : first_bad;
        bad = bad || badj;
        float ck[32];
#pragma unroll
        for (int k = 0; k < 32; ++k) ck[k] = (k > j) ? colj[k] : 0.f;
        // 1/d: hardware estimate plus one Newton step (fp32 accurate to ~1
        // ulp, which is all a multiplier of the factorisation needs)
        const float r0 = ptx::rcp_approx(d);
        const float rd = fmaf(fmaf(-d, r0, 1.f), r0, r0);
        const float lij = (lane > j) ? a[j] * rd : 0.f;
#pragma unroll
        for (int k = 0; k < 32; ++k)
          if (k > j) a[k] = fmaf(-lij, ck[k], a[k]);
        __syncwarp();
      }
      if (bad && lane == 0) fail = first_bad;
      if (!bad) {
        // pivots d_k = a_kk; scale row `lane` by 1/sqrt(d_k)
#pragma unroll
        for (int k = 0; k < 32; ++k)
          if (k == lane) colj[lane] = a[k];
        __syncwarp();
        const float rs_own = 1.f / sqrtf(colj[lane]);
        rdiag[c0 + lane] = rs_own;  // 1 / L_kk for the solve below
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          if (k < lane) S[(c0 + lane) * kPadLD + c0 + k] = a[k] * rdiag[c0 + k];
          if (k == lane) S[(c0 + lane) * kPadLD + c0 + k] = sqrtf(a[k]);
        }
      }
    }
    __syncthreads();
    if (fail) {
      if (tid == 0) atomicCAS(info, 0, n - (kb + fail - 1));
      return;
    }
    // (2) rows below the sub-block: x <- x L_sub^-T, one thread per row
    const int rem = bs - c0 - 32;
    if (tid < rem) {
      const int r = c0 + 32 + tid;
      float x[32];
#pragma unroll
      for (int k = 0; k < 32; ++k) x[k] = chol_elem(S, r, c0 + k);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        x[j] *= rdiag[c0 + j];
#pragma unroll
        for (int k = 0; k < 32; ++k)
          if (k > j) x[k] = fmaf(-x[j], chol_elem(S, c0 + k, c0 + j), x[k]);
      }
#pragma unroll
      for (int k = 0; k < 32; ++k) S[r * kPadLD + c0 + k] = x[k];
    }
    __syncthreads();
    // (3) trailing lower block [c0+32, bs)^2 -= rank-32 product, 4 x 4 tiles
    if (rem > 0) {
      const int mt = (rem + 3) / 4;
      const int ntiles = mt * (mt + 1) / 2;
      const int base = c0 + 32;
      for (int t = tid; t < ntiles; t += blockDim.x) {
        int ti = (int)((sqrtf(8.f * (float)t + 1.f) - 1.f) * 0.5f);
        while ((ti + 1) * (ti + 2) / 2 <= t) ++ti;
        while (ti * (ti + 1) / 2 > t) --ti;
        const int tj = t - ti * (ti + 1) / 2;
        const int r0 = base + 4 * ti, s0 = base + 4 * tj;
        float acc[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 8
        for (int k = 0; k < 32; ++k) {
          float ra[4], sa[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) ra[i] = chol_elem(S, min(r0 + i, kPanel - 1), c0 + k);
#pragma unroll
          for (int j = 0; j < 4; ++j) sa[j] = chol_elem(S, min(s0 + j, kPanel - 1), c0 + k);
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(ra[i], sa[j], acc[i][j]);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j)
            if (r0 + i < bs && s0 + j < bs) S[(r0 + i) * kPadLD + s0 + j] -= acc[i][j];
      }
    }
    __syncthreads();
  }
  for (int i = tid; i < bs * kPanel; i += blockDim.x) {
    const int rr = i / kPanel, c = i % kPanel;
    if (c <= rr) A[(int64_t)(kb + rr) * n + kb + c] = S[rr * kPadLD + c];
  }
}

// ---------------------------------------------------------------- panel (b)
// v <- L_pp^-1 v for every vector: the rows of A below the panel
// (restricted to the panel's columns) and rows [0, kb + bs) of RT.
// Four lanes (a quad) per vector, eight vectors per warp; lane q holds
// entries q, q+4, ..., q+124 (slot s = entry / 4).  Step j: the owner lane
// (j % 4) scales entry j by 1/L_jj, the quad shares it, and every lane
// subtracts it times column j of L from its later entries.  Shared memory
// holds Lq[j][q][s] = L[4 s + q][j] (pitch 36 floats: float4 reads, no bank
// conflicts); unrolled over j so finished slots cost nothing.
constexpr int kSolveThreads = 128;
constexpr int kLqPitch = 36;
constexpr int kLqRow = 4 * kLqPitch;
constexpr size_t kSolveSmemBytes = sizeof(float) * (kPanel * kLqRow + kPanel);

// Every solved vector is also written, split into its TF32 part and the
// remainder, to row `g` of the panel buffer PBh / PBl (g = the vector's row
// in A or RT), the operand of the tensor-core trailing update.  Rows of A
// below the panel are not written back: only the trailing update reads them.
__global__ void __launch_bounds__(kSolveThreads) panel_solve_kernel(
    float* __restrict__ A, float* __restrict__ RT, int n, int p, float* __restrict__ PBh,
    float* __restrict__ PBl, const int32_t* __restrict__ info) {
  if (*(volatile const int32_t*)info != 0) return;
  extern __shared__ __align__(16) float dyn_smem[];
  float* Lq = dyn_smem;
  float* rdiag = dyn_smem + kPanel * kLqRow;
  const int kb = p * kPanel;
  const int bs = min(kPanel, n - kb);
  stage_block_128<kSolveThreads>(
      A + (int64_t)kb * n + kb, n, bs, bs, /*lower=*/true, (n % 4) == 0,
      [&](int r, int c, float v) { Lq[c * kLqRow + (r & 3) * kLqPitch + (r >> 2)] = v; },
      [](int r, int c) { return (r == c) ? 1.f : 0.f; });
  __syncthreads();
  for (int i = threadIdx.x; i < kPanel; i += blockDim.x)
    rdiag[i] = 1.f / Lq[i * kLqRow + (i & 3) * kLqPitch + (i >> 2)];
  __syncthreads();

  const int q = threadIdx.x & 3;
  const int lane = threadIdx.x & 31;
  const int nA = n - kb - bs;
  const int nvec = nA + kb + bs;
  const int quads = (gridDim.x * blockDim.x) >> 2;
  const float* lq_lane = Lq + q * kLqPitch;
  // `base` is the warp's first vector: uniform across the warp, so the whole
  // warp stays in the loop together (the shuffles need all 32 lanes)
  for (int base = (blockIdx.x * blockDim.x + (threadIdx.x & ~31)) >> 2; base < nvec;
       base += quads) {
    const int v0 = base + (lane >> 2);
    const bool active = v0 < nvec;
    float* vec = !active ? nullptr
                 : (v0 < nA) ? (A + (int64_t)(kb + bs + v0) * n + kb)
                             : (RT + (int64_t)(v0 - nA) * n + kb);
    float x[32];
#pragma unroll
    for (int s = 0; s < 32; ++s) {
      const int c = 4 * s + q;
      x[s] = (active && c < bs) ? vec[c] : 0.f;
    }
#pragma unroll
    for (int s = 0; s < 32; ++s) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        // no early exit for a short panel: entries past bs are 0 and the
        // padded factor is the identity there, so those steps change nothing
        const int j = 4 * s + k;
        const float yv = x[s] * rdiag[j];
        const float y = __shfl_sync(0xffffffffu, yv, k, 4);
        const float* lcol = lq_lane + j * kLqRow;
#pragma unroll
        for (int s4 = s >> 2; s4 < 8; ++s4) {
          const float4 l4 = *reinterpret_cast<const float4*>(lcol + 4 * s4);
          if (4 * s4 + 0 >= s) x[4 * s4 + 0] = fmaf(-l4.x, y, x[4 * s4 + 0]);
          if (4 * s4 + 1 >= s) x[4 * s4 + 1] = fmaf(-l4.y, y, x[4 * s4 + 1]);
          if (4 * s4 + 2 >= s) x[4 * s4 + 2] = fmaf(-l4.z, y, x[4 * s4 + 2]);
          if (4 * s4 + 3 >= s) x[4 * s4 + 3] = fmaf(-l4.w, y, x[4 * s4 + 3]);
        }
        x[s] = (q == k) ? y : x[s];
      }
    }
    if (active) {
      const bool is_rt = v0 >= nA;
      const int64_t g = is_rt ? (int64_t)(v0 - nA) : (int64_t)(kb + bs + v0);
      float* ph = PBh + g * kPanel;
      float* pl = PBl + g * kPanel;
#pragma unroll
      for (int s = 0; s < 32; ++s) {
        const int c = 4 * s + q;
        const float xv = (c < bs) ? x[s] : 0.f;
        if (is_rt && c < bs) vec[c] = xv;
        float h, l;
        tf32_split(xv, h, l);
        ph[c] = h;
        pl[c] = l;
      }
    }
  }
}

// The trailing update of panel p as tiles for the tensor-core panel GEMM.
// Tiles [0, T1): lower tiles (rb, sb), p < sb <= rb, of A -= L_p L_p^T;
// tiles [T1, T1+T2): RT[cb][rb] -= RT[cb][p] L[rb][p]^T, cb <= p < rb.
// Both operands are rows of the panel buffer (P = rows of the C tile's row
// block, Q = rows of its column block).
struct CholTrailDecoder {
  float* A;
  float* RT;
  int n, p, nblk;
  __device__ PgTile tile(int bx, int) const {
    PgTile t;
    const int m = nblk - p - 1;
    const int T1 = m * (m + 1) / 2;
    int idx = bx;
    t.ldc = n;
    t.pkx = 0;
    t.qkx = 0;
    if (idx < T1) {
      int rr = (int)((sqrtf(8.f * (float)idx + 1.f) - 1.f) * 0.5f);
      while ((rr + 1) * (rr + 2) / 2 <= idx) ++rr;
      while (rr * (rr + 1) / 2 > idx) --rr;
      const int ss = idx - rr * (rr + 1) / 2;
      const int rb = p + 1 + rr, sb = p + 1 + ss;
      t.C = A + (int64_t)rb * kPanel * n + (int64_t)sb * kPanel;
      t.prow = rb * kPanel;
      t.qrow = sb * kPanel;
      t.mext = min(kPanel, n - rb * kPanel);
      t.cext = min(kPanel, n - sb * kPanel);
    } else {
      idx -= T1;
      const int cb = idx / m, rb = p + 1 + idx % m;
      t.C = RT + (int64_t)cb * kPanel * n + (int64_t)rb * kPanel;
      t.prow = cb * kPanel;
      t.qrow = rb * kPanel;
      t.mext = kPanel;
      t.cext = min(kPanel, n - rb * kPanel);
    }
    t.valid = 1;
    return t;
  }
};

// ---------------------------------------------------------------- finish
// In place: U[i][j] <- U[n-1-j][n-1-i] (an involution; it maps the upper
// triangle onto itself and the zero lower triangle onto itself).
// Tiled form for n % 32 == 0: tile (I, J) swaps with (nt-1-J, nt-1-I).
__global__ void __launch_bounds__(256) anti_transpose_tiles_kernel(float* __restrict__ U, int n) {
  __shared__ float T0[32][33];
  __shared__ float T1[32][33];
  const int nt = n / 32;
  const int I = blockIdx.y, J = blockIdx.x;
  if (I > J || I + J > nt - 1) return;
  const int I2 = nt - 1 - J, J2 = nt - 1 - I;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
  for (int a = ty; a < 32; a += 8) {
    T0[a][tx] = U[(int64_t)(32 * I + a) * n + 32 * J + tx];
    T1[a][tx] = U[(int64_t)(32 * I2 + a) * n + 32 * J2 + tx];
  }
  __syncthreads();
  for (int a = ty; a < 32; a += 8) {
    U[(int64_t)(32 * I + a) * n + 32 * J + tx] = T1[31 - tx][31 - a];
    U[(int64_t)(32 * I2 + a) * n + 32 * J2 + tx] = T0[31 - tx][31 - a];
  }
}

__global__ void anti_transpose_elems_kernel(float* __restrict__ U, int n) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  const int i = blockIdx.y;
  if (j >= n || i > j || i + j >= n - 1) return;
  const int64_t a = (int64_t)i * n + j;
  const int64_t b = (int64_t)(n - 1 - j) * n + (n - 1 - i);
  const float va = U[a], vb = U[b];
  U[a] = vb;
  U[b] = va;
}

}  // namespace

size_t cholesky_workspace_bytes(int64_t n) { return chol_ws_bytes(n); }

cudaError_t launch_cholesky_inverse(const float* H, int64_t n64, float percdamp, int actorder,
                                    float* U, int32_t* perm, uint8_t* dead, int32_t* info,
                                    void* ws, cudaStream_t s) {
  const int n = (int)n64;
  CholWs w = carve(ws, n64);
  cudaError_t e;
  if ((e = cudaMemsetAsync(info, 0, sizeof(int32_t), s)) != cudaSuccess) return e;
  diag_prep_kernel<<<1, 1024, 0, s>>>(H, n, percdamp, dead, w.dprime, w.lam, info);
  note_launch();
  int32_t* perm_used = nullptr;
  if (actorder) {
    actorder_rank_kernel<<<(n + 255) / 256, 256, 0, s>>>(w.dprime, n, perm);
    note_launch();
    perm_used = perm;
  } else if (perm) {
    iota_kernel<<<(n + 255) / 256, 256, 0, s>>>(perm, n);
    note_launch();
  }
  const size_t row_smem = sizeof(float) * (size_t)n;
  if (row_smem > 48 * 1024) {
    if ((e = cudaFuncSetAttribute(gather_reversed_kernel,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, (int)row_smem)) !=
        cudaSuccess)
      return e;
  }
  gather_reversed_kernel<<<n, 256, row_smem, s>>>(H, n, perm_used, dead, w.lam, w.A);
  note_launch();
  if ((e = cudaMemsetAsync(U, 0, sizeof(float) * (size_t)n * n, s)) != cudaSuccess) return e;
  set_diag_one_kernel<<<(n + 255) / 256, 256, 0, s>>>(U, n);
  note_launch();

  const int nblk = (n + kPanel - 1) / kPanel;
  const int sms = num_sms();
  const size_t diag_smem = sizeof(float) * (kPanel * kPadLD + 2 * kPanel);
  const size_t solve_smem = kSolveSmemBytes;
  if ((e = cudaFuncSetAttribute(chol_diag_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)diag_smem)) != cudaSuccess ||
      (e = cudaFuncSetAttribute(panel_solve_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)solve_smem)) != cudaSuccess)
    return e;
  // one quad per vector (n vectors per panel), capped at 3 resident CTAs per SM
  const int solve_ctas = std::min((4 * n + kSolveThreads - 1) / kSolveThreads, 3 * sms);
  CUtensorMap mPh, mPl;
  if (nblk > 1) {
    if (!make_tma_2d(&mPh, w.PBh, false, n, kPanel, kPanel, 32, 128) ||
        !make_tma_2d(&mPl, w.PBl, false, n, kPanel, kPanel, 32, 128))
      return cudaErrorInvalidValue;
    if ((e = cudaFuncSetAttribute(panel_gemm_kernel<CholTrailDecoder>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)kPgSmemBytes)) != cudaSuccess)
      return e;
  }
  for (int p = 0; p < nblk; ++p) {
    chol_diag_kernel<<<1, 256, diag_smem, s>>>(w.A, n, p, info);
    note_launch();
    panel_solve_kernel<<<solve_ctas, kSolveThreads, solve_smem, s>>>(w.A, U, n, p, w.PBh, w.PBl,
                                                                      info);
    note_launch();
    const int m = nblk - p - 1;
    const int tiles = m * (m + 1) / 2 + (p + 1) * m;
    if (tiles > 0) {
      const CholTrailDecoder dec{w.A, U, n, p, nblk};
      panel_gemm_kernel<CholTrailDecoder><<<tiles, kPgThreads, kPgSmemBytes, s>>>(
          mPh, mPl, mPh, mPl, dec, info, kInfoTimeout, info);
      note_launch();
    }
  }
  if (n % 32 == 0) {
    const int nt = n / 32;
    anti_transpose_tiles_kernel<<<dim3(nt, (nt + 1) / 2), 256, 0, s>>>(U, n);
    note_launch();
  } else {
    anti_transpose_elems_kernel<<<dim3((n + 255) / 256, n), 256, 0, s>>>(U, n);
    note_launch();
  }
  return cudaGetLastError();
}

}  // namespace gptq

// ---------------------------------------------------------------------------
// Allocation-free variant of gptq_cholesky_inverse.
//
// Some callers cannot allocate device memory at the time they quantize: a
// host program that hands out all device memory from its own fixed pool and
// forbids allocation once it is running (a serving process, a plugin inside
// another runtime) can neither call cudaMalloc nor give this library a
// workspace.  For them the factorisation's scratch lives in the array below,
// which is part of the library image: every GPU that loads the library holds
// these bytes until the process exits.
//
// Limit: n <= kNoAllocMaxN (2048), i.e. the scratch of one 2048 x 2048
// factorisation, 18.9 MB.  Larger n is rejected with GPTQ_ERR_WORKSPACE.
//
// The array's name in host code is only a host-side stand-in, not a device
// address.  The device address is looked up with cudaGetSymbolAddress once
// per device, with that device current, by the first call made on it; that
// first call should therefore come before any stream capture.  Every call
// shares the one array: calls whose kernels overlap on the GPU (on different
// streams, or from different threads) race on it and must be serialised by
// the caller.  Nothing in the array has to start at zero: every byte a call
// reads is written earlier in that same call.
#include <mutex>

namespace {

constexpr int64_t kNoAllocMaxN = 2048;
constexpr size_t kNoAllocBytes = gptq::chol_ws_bytes(kNoAllocMaxN);
constexpr int kNoAllocMaxDevices = 64;

static __device__ __align__(256) unsigned char g_chol_scratch[kNoAllocBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kNoAllocMaxDevices] = {};

}  // namespace

extern "C" gptq_status gptq_cholesky_inverse_noalloc(const float* H, int64_t n, float percdamp,
                                                     int actorder, float* U, int32_t* perm,
                                                     uint8_t* dead, int32_t* info, void* stream) {
  if (!H || !U || !dead || !info || n <= 0) return GPTQ_ERR_INVALID_ARG;
  if (actorder && !perm) return GPTQ_ERR_INVALID_ARG;
  if (!(percdamp >= 0.f)) return GPTQ_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(H) % 4 != 0 || reinterpret_cast<uintptr_t>(U) % 16 != 0)
    return GPTQ_ERR_INVALID_ARG;
  if (n > kNoAllocMaxN || gptq::cholesky_workspace_bytes(n) > kNoAllocBytes)
    return GPTQ_ERR_WORKSPACE;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GPTQ_ERR_CUDA;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return GPTQ_ERR_UNSUPPORTED;
  void* ws = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_chol_scratch) != cudaSuccess || !p) return GPTQ_ERR_CUDA;
      g_scratch_addr[dev] = p;
    }
    ws = g_scratch_addr[dev];
  }
  const cudaError_t e = gptq::launch_cholesky_inverse(H, n, percdamp, actorder, U, perm, dead,
                                                      info, ws, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}
