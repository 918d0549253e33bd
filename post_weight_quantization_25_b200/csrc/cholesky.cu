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
//   (a) factor the diagonal block L_pp, invert its 32 x 32 leaves  (1 CTA)
//   (b) apply L_pp^-1 to every vector that needs it: the panel rows below
//       (-> L_ip) and the block row p of the inverse's right-hand side
//       (-> M_p.), in four dense 32-column stages (fp32 FMA)
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
#include "chol_diag.cuh"
#include "panel_gemm.cuh"
#include "persist.cuh"

namespace gptq {
namespace {

constexpr int kPanel = kBlock;  // 128
constexpr int32_t kInfoTimeout = -2;  // `info` value when a device wait gave up

// Two-level blocking for large n: inside a super-panel of kSuperPanelCols
// columns the trailing updates are rank-128 (one per panel) and stop at the
// super-panel's end; the columns past it are updated once per super-panel
// with all its panels' vectors (K up to kSuperPanelCols), so the trailing
// matrix is read and written once per super-panel instead of once per panel.
// Smaller n uses one level (the super-panel is the panel).
constexpr int kSuperPanelCols = 1024;
constexpr int64_t kTwoLevelMinN = 8192;
constexpr int64_t super_panel_cols(int64_t n) {
  return n >= kTwoLevelMinN ? kSuperPanelCols : kPanel;
}

struct CholWs {
  float* A;       // n x n, lower part used: J P^T H P J + lambda I
  float* dprime;  // n: diag(H) with dead entries set to 1
  double* lam;    // 1: damping
  float* PBh[2];  // n x SP: a super-panel's solved vectors, TF32 part (super-panels alternate)
  float* PBl[2];  // n x SP: remainder
  float* Dout[2];  // the diagonal step's outputs (L^T of the block, inverted leaves), by panel parity
  uint32_t* ctr;   // the persistent factorisation's counters
};

constexpr size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Workspace bytes for order n (also sizes the built-in scratch of the
// allocation-free entry point below, hence constexpr).
// counters of the persistent factorisation: [0] next task, tile[nblk][nblk]
// (panels applied), vdone[2][nblk] (apply chunks done, by panel parity),
// tdone[nblk] (update tasks done per panel), ddone[nblk] (diagonal factored)
constexpr size_t chol_ctr_bytes(int64_t n) {
  const int64_t nb = (n + kPanel - 1) / kPanel;
  return align_up(sizeof(uint32_t) * (size_t)(1 + nb * nb + 4 * nb), 256);
}
constexpr size_t chol_ws_bytes(int64_t n) {
  return align_up(sizeof(float) * n * n, 256) + align_up(sizeof(float) * n, 256) + 256 +
         4 * align_up(sizeof(float) * n * super_panel_cols(n), 256) +
         2 * align_up(sizeof(float) * kDiagOutFloats, 256) + chol_ctr_bytes(n);
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
  const int64_t sp = super_panel_cols(n);
  for (int b = 0; b < 2; ++b) {
    w.PBh[b] = reinterpret_cast<float*>(p);
    p += align_up(sizeof(float) * n * sp, 256);
    w.PBl[b] = reinterpret_cast<float*>(p);
    p += align_up(sizeof(float) * n * sp, 256);
  }
  for (int b = 0; b < 2; ++b) {
    w.Dout[b] = reinterpret_cast<float*>(p);
    p += align_up(sizeof(float) * kDiagOutFloats, 256);
  }
  w.ctr = reinterpret_cast<uint32_t*>(p);
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

// Eight threads (consecutive lanes) count for each key, over every eighth
// other key, and their counts are summed: a CTA of 256 threads ranks 32 keys.
constexpr int kRankSplit = 8;
constexpr int kRankKeysPerCta = 256 / kRankSplit;
__global__ void __launch_bounds__(256) actorder_rank_kernel(const float* __restrict__ dprime,
                                                            int n, int32_t* __restrict__ perm) {
  __shared__ float keys[2048];
  const int i = blockIdx.x * kRankKeysPerCta + threadIdx.x / kRankSplit;
  const int sub = threadIdx.x % kRankSplit;
  const float ki = (i < n) ? rank_key(dprime[i]) : 0.f;
  int pos = 0;
  for (int t0 = 0; t0 < n; t0 += 2048) {
    const int cnt = min(2048, n - t0);
    for (int j = threadIdx.x; j < cnt; j += blockDim.x) keys[j] = rank_key(dprime[t0 + j]);
    __syncthreads();
    if (i < n) {
      for (int j = sub; j < cnt; j += kRankSplit) {
        const float kj = keys[j];
        pos += (kj > ki) || (kj == ki && t0 + j < i);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int o = 1; o < kRankSplit; o <<= 1) pos += __shfl_xor_sync(0xffffffffu, pos, o);
  if (i < n && sub == 0) perm[pos] = i;
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
  float* dst = A + (int64_t)a * n;
  // 16-byte row loads and four-column outputs where the rows allow it
  const bool v4 = (n % 4) == 0 && reinterpret_cast<uintptr_t>(H) % 16 == 0 &&
                  reinterpret_cast<uintptr_t>(A) % 16 == 0 &&
                  (!perm || reinterpret_cast<uintptr_t>(perm) % 16 == 0);
  if (v4) {
    for (int j = threadIdx.x; j < n / 4; j += blockDim.x)
      reinterpret_cast<float4*>(hrow)[j] = reinterpret_cast<const float4*>(src)[j];
  } else {
    for (int j = threadIdx.x; j < n; j += blockDim.x) hrow[j] = src[j];
  }
  __syncthreads();
  const float lf = (float)(*lam);
  const float diag = dead[pa] ? 1.f : hrow[pa];
  // columns [0, 4 nv) four at a time: column b + i takes perm[n - 1 - b - i],
  // i.e. the 16-byte group perm[n - 4 - b .. n - 1 - b] read backwards
  const int nv = v4 ? (a + 1) / 4 : 0;
  for (int b4 = threadIdx.x; b4 < nv; b4 += blockDim.x) {
    const int b = 4 * b4;
    int4 q;
    if (perm)
      q = *reinterpret_cast<const int4*>(perm + (n - 4 - b));
    else
      q = make_int4(n - 4 - b, n - 3 - b, n - 2 - b, n - 1 - b);
    float4 v = make_float4(hrow[q.w], hrow[q.z], hrow[q.y], hrow[q.x]);
    if (b + 3 == a) v.w = diag + lf;
    *reinterpret_cast<float4*>(dst + b) = v;
  }
  for (int b = 4 * nv + threadIdx.x; b <= a; b += blockDim.x) {
    const int pb = perm ? perm[n - 1 - b] : (n - 1 - b);
    const float v = (b == a) ? diag + lf : hrow[pb];
    dst[b] = v;
  }
}

__global__ void set_diag_one_kernel(float* __restrict__ M, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) M[(int64_t)i * n + i] = 1.f;
}

// ---------------------------------------------------------------- panel (a), (b)
// chol_diag_kernel and panel_apply_kernel (chol_diag.cuh).

// The trailing update of panel p as items for the tensor-core panel GEMM.
// Item R (a 128-row block, P = its rows of the panel buffer):
//   R > p:  lower tiles A[R][S] -= L_Rp L_Sp^T for p < S <= R   (R - p tiles)
//   R <= p: tiles RT[R][S] -= RT[R][p] L_Sp^T for p < S < nblk  (nblk-1-p tiles)
// In both cases the Q rows (the panel buffer rows of block S) and the C
// tiles run over consecutive blocks from S = p + 1.
struct CholTrailItems {
  float* A;
  float* RT;
  int n, p, nblk;
  int cb_lo, cb_hi;  // column blocks [cb_lo, cb_hi) of this launch
  int pk;            // column of panel p's vectors in the super-panel buffer
  // row block R updates column blocks [p + 1, R] of A (R > p) or
  // [p + 1, nblk) of RT (R <= p), clipped to the window
  __host__ __device__ int col_lo() const { return cb_lo > p + 1 ? cb_lo : p + 1; }
  __host__ __device__ int col_hi(int R) const {
    const int h = R > p ? R + 1 : nblk;
    return h < cb_hi ? h : cb_hi;
  }
  __host__ __device__ int num_items() const { return nblk; }
  __host__ __device__ int item_nq(int R) const {
    const int q = col_hi(R) - col_lo();
    return q > 0 ? q : 0;
  }
  __device__ PgItem item(int R) const {
    PgItem I;
    const int c0 = col_lo() * kPanel;
    I.C0 = (R > p ? A : RT) + (int64_t)R * kPanel * n + c0;
    I.ldc = n;
    I.cmap = R > p ? 0 : 1;
    I.cx0 = c0;
    I.cy0 = R * kPanel;
    I.prow = R * kPanel;
    I.pkx = pk;
    I.qrow0 = c0;
    I.qkx = pk;
    I.nq = item_nq(R);
    I.mext = min(kPanel, n - R * kPanel);
    I.cext_last = min(kPanel, n - c0 - kPanel * (I.nq - 1));
    I.nkb = kPanel / 32;
    return I;
  }
};

// The update past a finished super-panel [P0, P1) (panels), for the column
// blocks [cb_lo, cb_hi) at or past P1, with all its panels' vectors at once
// (stream_gemm_kernel):
//   R >= P1: lower tiles A[R][S] -= sum_{P0 <= p < P1} L_Rp L_Sp^T, P1 <= S <= R
//   R <  P1: tiles RT[R][S] -= sum_{max(P0, R) <= p < P1} RT[R][p] L_Sp^T, S >= P1
// (a row block inside the super-panel is a right-hand-side row only for the
// panels at or after it, so its K range starts there).
struct CholSuperItems {
  float* A;
  float* RT;
  int n, P0, P1, nblk;
  int cb_lo, cb_hi;
  __host__ __device__ int col_lo() const { return cb_lo > P1 ? cb_lo : P1; }
  __host__ __device__ int col_hi(int R) const {
    const int h = R >= P1 ? R + 1 : nblk;
    return h < cb_hi ? h : cb_hi;
  }
  __host__ __device__ int num_items() const { return nblk; }
  __host__ __device__ int item_nq(int R) const {
    const int q = col_hi(R) - col_lo();
    return q > 0 ? q : 0;
  }
  __device__ PgItem item(int R) const {
    PgItem I;
    const int c0 = col_lo() * kPanel;
    const int kp0 = R >= P1 ? P0 : (R > P0 ? R : P0);  // first panel that reaches row block R
    I.C0 = (R >= P1 ? A : RT) + (int64_t)R * kPanel * n + c0;
    I.ldc = n;
    I.cmap = R >= P1 ? 0 : 1;
    I.cx0 = c0;
    I.cy0 = R * kPanel;
    I.prow = R * kPanel;
    I.pkx = (kp0 - P0) * kPanel;
    I.qrow0 = c0;
    I.qkx = I.pkx;
    I.nq = item_nq(R);
    I.mext = min(kPanel, n - R * kPanel);
    I.cext_last = min(kPanel, n - c0 - kPanel * (I.nq - 1));
    I.nkb = (P1 - kp0) * (kPanel / 32);
    return I;
  }
};

// ---------------------------------------------------------------- persistent form
// For 3 <= nblk and n a multiple of 128 below the two-level width, one launch
// runs every panel's steps as tasks that CTAs (one per SM) take from a global
// counter.  For each panel p the queue holds, in this order:
//   D(p)      the diagonal block of panel p (chol_diag_body, 256 threads)
//   F(p - 1)  the trailing update by panel p - 1 of the column blocks past
//             p (up to kCpChunk tiles per task), which runs beside D(p)
//   A(p, k)   the apply of L_pp^-1 to vectors [32 k, 32 k + 32) of the panel
//             (panel_apply_body); the rows of block p + 1 come first
//   N(p)      the update by panel p of column block p + 1 (one tile per task,
//             the diagonal tile (p + 1, p + 1) first)
// so the chain from one diagonal block to the next is D(p), the apply of the
// next block's 128 rows and one tile update; the rest of each panel's apply
// and update runs on the other SMs.  Counters in global memory (zeroed per
// launch) carry the dependencies:
//   tile[R][S]   panels applied to tile (R, S) of A (R >= S) or RT (R < S);
//                before panel p it must read p (A) or p - R (RT)
//   vdone[b][R]  apply chunks done for row block R by the panels of parity b
//   tdone[p]     update tasks of panel p done (the panel-vector buffer and the
//                diagonal outputs of parity p & 1 are reused by panel p + 2)
//   ddone[p]     D(p) done
// Every task comes after the tasks it waits for in the queue order, so the
// waits end; each tile gets its updates in panel order, so the result does
// not depend on the timing.  Once `info` holds an error the tasks skip their
// work and only publish their counters.
constexpr int kCpChunk = 4;   // tiles per far-update task at most
constexpr int kCpBar = 1;     // named barrier of the diagonal and apply tasks

struct CholPersistArgs {
  float* A;
  float* RT;
  int n, nblk;
  float* Dout0;
  float* Dout1;
  float* PBh0;
  float* PBl0;
  float* PBh1;
  float* PBl1;
  uint32_t* ctr;
  int32_t* info;
  const int32_t* gate;
  uint64_t limit_ns;
};

struct CpTask {
  int kind;    // 0 diagonal, 1 apply, 2 update
  int p;       // panel
  int R;       // update: row block
  int c0, c1;  // update: column blocks [c0, c1)
  int k;       // apply: chunk of 32 vectors
};

__host__ __device__ inline int cp_ceil4(int x) { return (x + kCpChunk - 1) / kCpChunk; }

// far tasks of panel q (its column blocks past q + 1): A row blocks
// R in [q + 2, nblk) take ceil((R - q - 1) / 4) tasks, RT row blocks R <= q
// take ceil((nblk - q - 2) / 4) each
__host__ __device__ inline int cp_far_tasks(int nblk, int q) {
  const int m = nblk - q - 2;
  if (q < 0 || m <= 0) return 0;
  const int a = m / 4, r = m % 4;
  return 2 * a * (a + 1) + r * (a + 1) + (q + 1) * cp_ceil4(m);
}
__host__ __device__ inline int cp_near_tasks(int nblk, int p) { return p + 1 < nblk ? nblk : 0; }
__host__ __device__ inline int cp_update_tasks(int nblk, int p) {
  return cp_near_tasks(nblk, p) + cp_far_tasks(nblk, p);
}
__host__ __device__ inline int cp_step_tasks(int nblk, int n, int p) {
  return 1 + cp_far_tasks(nblk, p - 1) + n / 32 + cp_near_tasks(nblk, p);
}
__host__ __device__ inline int cp_total(int nblk, int n) {
  int t = 0;
  for (int p = 0; p < nblk; ++p) t += cp_step_tasks(nblk, n, p);
  return t;
}

__host__ __device__ inline CpTask cp_decode(int nblk, int n, int t) {
  CpTask k;
  k.R = k.c0 = k.c1 = k.k = 0;
  for (int p = 0;; ++p) {
    k.p = p;
    if (t == 0) {
      k.kind = 0;
      return k;
    }
    t -= 1;
    const int nF = cp_far_tasks(nblk, p - 1);
    if (t < nF) {
      const int q = p - 1;
      k.kind = 2;
      k.p = q;
      // A row blocks first (their column block q + 2 feeds the next diagonal)
      for (int R = q + 2; R < nblk; ++R) {
        const int ch = cp_ceil4(R - q - 1);
        if (t < ch) {
          k.R = R;
          k.c0 = q + 2 + kCpChunk * t;
          k.c1 = min(k.c0 + kCpChunk, R + 1);
          return k;
        }
        t -= ch;
      }
      const int per = cp_ceil4(nblk - q - 2);
      k.R = t / per;
      k.c0 = q + 2 + kCpChunk * (t % per);
      k.c1 = min(k.c0 + kCpChunk, nblk);
      return k;
    }
    t -= nF;
    if (t < n / 32) {
      k.kind = 1;
      k.k = t;
      return k;
    }
    t -= n / 32;
    const int nN = cp_near_tasks(nblk, p);
    if (t < nN) {
      k.kind = 2;
      k.R = t == 0 ? p + 1 : (t - 1 < p + 1 ? t - 1 : t);
      k.c0 = p + 1;
      k.c1 = p + 2;
      return k;
    }
    t -= nN;
  }
}

// The diagonal and apply tasks (inlined: as separate calls they measured
// slower, 52k against 48k cycles for the diagonal block's four leaves)
__device__ __forceinline__ void cp_diag_task(const float* A, int n, int p, float* out, int32_t* info,
                                          float* sm, int tid) {
  chol_diag_body(A, n, p, out, info, sm, tid, kCpBar);
}
__device__ __forceinline__ void cp_apply_task(const float* A, float* RT, int n, int p,
                                           const float* dout, float* PBh, float* PBl, float* sm,
                                           int tid, int v0) {
  panel_apply_body(A, RT, n, p, dout, PBh, PBl, kPanel, sm, tid, v0, kCpBar);
}

__global__ void __launch_bounds__(kPg2Threads, 1)
    chol_persist_kernel(const __grid_constant__ CUtensorMap mPh0,
                        const __grid_constant__ CUtensorMap mPl0,
                        const __grid_constant__ CUtensorMap mPh1,
                        const __grid_constant__ CUtensorMap mPl1,
                        const __grid_constant__ CUtensorMap mA,
                        const __grid_constant__ CUtensorMap mRT, const CholPersistArgs a) {
  extern __shared__ uint8_t smem_raw[];
  constexpr int32_t kTimeout = kInfoTimeout;
  PersistCta cta;
  cta.init(smem_raw, a.limit_ns);
  volatile int* abort_flag = cta.abort_flag();
  volatile int* skip_flag = cta.skip_slot();
  const uint64_t kLimit = a.limit_ns;
  const int nblk = a.nblk, n = a.n;
  uint32_t* tile = a.ctr + 1;
  uint32_t* vdone = tile + nblk * nblk;
  uint32_t* tdone = vdone + 2 * nblk;
  uint32_t* ddone = tdone + nblk;
  const int tid = threadIdx.x;
  if (tid == 0 && !ptx::gate_wait_bounded(a.gate, kLimit))
    persist_abort(abort_flag, a.info, kTimeout);
  const int total = cp_total(nblk, n);

  // thread 0: wait for *f >= v (bounded); false on timeout or abort
  auto wait_ge = [&](const uint32_t* f, uint32_t v) {
    return ptx::flag_wait_bounded(f, v, abort_flag, kLimit);
  };

  while (true) {
    const int t = cta.next_task(a.ctr, total);
    if (t < 0) break;
    const CpTask k = cp_decode(nblk, n, t);
    const int p = k.p;
    if (k.kind == 0 || k.kind == 1) {
      // ------------------------------------------- diagonal or apply task
      int R0 = 0, R1 = 0;   // apply: the chunk's row blocks (at most two)
      if (k.kind == 1) {
        const int nA = n - (p + 1) * kPanel;
        const int v0 = 32 * k.k;
        R0 = v0 < nA ? p + 1 + v0 / kPanel : (v0 - nA) / kPanel;
        const int v1 = v0 + 31;
        R1 = v1 < nA ? p + 1 + v1 / kPanel : (v1 - nA) / kPanel;
      }
      if (tid == 0) {
        bool ok = true;
        if (k.kind == 0) {
          ok = wait_ge(&tile[p * nblk + p], (uint32_t)p);
        } else {
          ok = wait_ge(&ddone[p], 1u);
          // the chunk's rows of column block p have every earlier panel
          for (int R = R0; R <= R1 && ok; ++R)
            ok = wait_ge(&tile[R * nblk + p], (uint32_t)(R > p ? p : p - R));
        }
        // the buffers of parity p & 1 are free once panel p - 2's updates are done
        if (ok && p >= 2) ok = wait_ge(&tdone[p - 2], (uint32_t)cp_update_tasks(nblk, p - 2));
        if (!ok) persist_abort(abort_flag, a.info, kTimeout);
        fence_proxy_async_global();
        *skip_flag = *(volatile int32_t*)a.info != 0;
      }
      __syncthreads();
      if (*abort_flag) continue;
      if (!*skip_flag && tid < kDiagThreads) {
        float* sm = reinterpret_cast<float*>(cta.smem);
        if (k.kind == 0)
          cp_diag_task(a.A, n, p, (p & 1) ? a.Dout1 : a.Dout0, a.info, sm, tid);
        else
          cp_apply_task(a.A, a.RT, n, p, (p & 1) ? a.Dout1 : a.Dout0, (p & 1) ? a.PBh1 : a.PBh0,
                        (p & 1) ? a.PBl1 : a.PBl0, sm, tid, 32 * k.k);
        // shared memory the next task's TMA loads overwrite, and the panel
        // vectors other CTAs read by TMA, are ordered before the async proxy
        asm volatile("fence.proxy.async;" ::: "memory");
      }
      __syncthreads();
      if (tid == 0) {
        __threadfence();
        if (k.kind == 0) {
          ptx::st_release_gpu(&ddone[p], 1u);
        } else {
          atomicAdd(&vdone[(p & 1) * nblk + R0], 1u);
          if (R1 != R0) atomicAdd(&vdone[(p & 1) * nblk + R1], 1u);
        }
      }
      continue;
    }
    // ------------------------------------------------------------ update task
    const int R = k.R;
    const uint32_t vneed = (uint32_t)(4 * (p / 2 + 1));   // apply chunks of block R, parity p & 1
    if (tid == 0) {
      bool ok = wait_ge(&vdone[(p & 1) * nblk + R], vneed);
      for (int S = k.c0; S < k.c1 && ok; ++S) ok = wait_ge(&vdone[(p & 1) * nblk + S], vneed);
      for (int S = k.c0; S < k.c1 && ok; ++S)
        ok = wait_ge(&tile[R * nblk + S], (uint32_t)(R >= S ? p : p - R));
      if (!ok) persist_abort(abort_flag, a.info, kTimeout);
      fence_proxy_async_global();
      *skip_flag = *(volatile int32_t*)a.info != 0;
    }
    __syncthreads();
    if (*abort_flag) continue;
    if (!*skip_flag) {
      PgItem I;
      const int c0 = k.c0 * kPanel;
      I.C0 = (R > p ? a.A : a.RT) + (int64_t)R * kPanel * n + c0;
      I.ldc = n;
      I.cmap = R > p ? 0 : 1;
      I.cx0 = c0;
      I.cy0 = R * kPanel;
      I.prow = R * kPanel;
      I.pkx = 0;
      I.qrow0 = c0;
      I.qkx = 0;
      I.nq = k.c1 - k.c0;
      I.mext = min(kPanel, n - R * kPanel);
      I.cext_last = min(kPanel, n - c0 - kPanel * (I.nq - 1));
      I.nkb = kPanel / 32;
      if (p & 1)
        cta.update(I, mPh1, mPl1, mPh1, mPl1, mA, mRT, a.info, kTimeout);
      else
        cta.update(I, mPh0, mPl0, mPh0, mPl0, mA, mRT, a.info, kTimeout);
    }
    __syncthreads();
    if (tid == 0 && !*abort_flag) {
      __threadfence();
      for (int S = k.c0; S < k.c1; ++S)
        ptx::st_release_gpu(&tile[R * nblk + S], (uint32_t)(R >= S ? p + 1 : p - R + 1));
      atomicAdd(&tdone[p], 1u);
    }
  }
  cta.teardown();
}

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
                                    void* ws, cudaStream_t s, cudaStream_t side_s) {
  const int n = (int)n64;
  CholWs w = carve(ws, n64);
  cudaError_t e;
  if ((e = cudaMemsetAsync(info, 0, sizeof(int32_t), s)) != cudaSuccess) return e;
  diag_prep_kernel<<<1, 1024, 0, s>>>(H, n, percdamp, dead, w.dprime, w.lam, info);
  note_launch();
  int32_t* perm_used = nullptr;
  if (actorder) {
    actorder_rank_kernel<<<(n + kRankKeysPerCta - 1) / kRankKeysPerCta, 256, 0, s>>>(w.dprime, n,
                                                                                   perm);
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
  if ((e = cudaFuncSetAttribute(chol_diag_kernel,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kDiagSmemBytes)) != cudaSuccess ||
      (e = cudaFuncSetAttribute(panel_apply_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kApplySmemBytes)) != cudaSuccess)
    return e;
  const int apply_ctas = (n + kApplyVecs - 1) / kApplyVecs;  // n vectors per panel
  const int SPW = (int)super_panel_cols(n);  // super-panel columns (kPanel: one level)
  const int npan = SPW / kPanel;             // panels per super-panel
  // operands of the trailing updates; with a row stride that is a multiple
  // of 16 bytes the updates land in A and RT by TMA reduce-add
  CUtensorMap mPh[2], mPl[2], mA, mRT;
  const bool reduce = (n % 4) == 0;
  if (nblk > 1) {
    for (int b = 0; b < 2; ++b)
      if (!make_tma_2d(&mPh[b], w.PBh[b], false, n, SPW, SPW, 32, 128) ||
          !make_tma_2d(&mPl[b], w.PBl[b], false, n, SPW, SPW, 32, 128))
        return cudaErrorInvalidValue;
    if (reduce) {
      if (!make_tma_2d(&mA, w.A, false, n, n, n, 32, 32) ||
          !make_tma_2d(&mRT, U, false, n, n, n, 32, 32))
        return cudaErrorInvalidValue;
    } else {
      mA = mRT = mPh[0];  // not read by the read-modify-write epilogue
    }
    if ((e = cudaFuncSetAttribute(reduce ? (const void*)panel_gemm2_kernel<CholTrailItems, true>
                                         : (const void*)panel_gemm2_kernel<CholTrailItems, false>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)pg2_smem_bytes(reduce))) != cudaSuccess)
      return e;
    if (npan > 1 &&
        (e = cudaFuncSetAttribute(reduce ? (const void*)stream_gemm_kernel<CholSuperItems, true>
                                         : (const void*)stream_gemm_kernel<CholSuperItems, false>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)sg_smem_bytes(reduce))) != cudaSuccess)
      return e;
  }
  // Widths that are a multiple of 128 below the two-level width: one
  // persistent launch, with or without a side stream (at n = 4096 it measured
  // 1.856 ms against 1.898 ms for the launch-by-launch form with its
  // look-ahead stream); other widths launch panel by panel.
  const bool persist = reduce && n % kPanel == 0 && nblk >= 3 && npan == 1;
  if (persist) {
    if ((e = cudaMemsetAsync(w.ctr, 0, chol_ctr_bytes(n64), s)) != cudaSuccess) return e;
    const WaitGate pg = current_wait_gate();
    CholPersistArgs a;
    a.A = w.A;
    a.RT = U;
    a.n = n;
    a.nblk = nblk;
    a.Dout0 = w.Dout[0];
    a.Dout1 = w.Dout[1];
    a.PBh0 = w.PBh[0];
    a.PBl0 = w.PBl[0];
    a.PBh1 = w.PBh[1];
    a.PBl1 = w.PBl[1];
    a.ctr = w.ctr;
    a.info = info;
    a.gate = pg.gate;
    a.limit_ns = pg.limit_ns;
    const size_t smem = pg2_smem_bytes(true);
    static_assert(kDiagSmemBytes <= (size_t)kPg2PBytes + kPg2QStages * kPg2QStageBytes &&
                      kApplySmemBytes <= (size_t)kPg2PBytes + kPg2QStages * kPg2QStageBytes,
                  "the diagonal and apply tasks reuse the update's shared memory");
    if ((e = cudaFuncSetAttribute(chol_persist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)smem)) != cudaSuccess)
      return e;
    const int grid = std::min(sms, cp_total(nblk, n));
    chol_persist_kernel<<<grid, kPg2Threads, smem, s>>>(mPh[0], mPl[0], mPh[1], mPl[1], mA, mRT,
                                                        a);
    note_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  } else {
  const WaitGate wg = current_wait_gate();
  // rank-128 update by panel p (buffer b, column pk) of column blocks [cb_lo, cb_hi)
  auto trail = [&](int b, int p, int pk, int cb_lo, int cb_hi, cudaStream_t st) -> cudaError_t {
    const CholTrailItems dec{w.A, U, n, p, nblk, cb_lo, cb_hi, pk};
    int chunk = 1, units = 0;
    pg2_plan(dec, sms, chunk, units);
    if (units == 0) return cudaSuccess;
    const int grid = std::min(units, sms);
    if (reduce)
      panel_gemm2_kernel<CholTrailItems, true><<<grid, kPg2Threads, pg2_smem_bytes(true), st>>>(
          mPh[b], mPl[b], mPh[b], mPl[b], mA, mRT, dec, chunk, units, info, kInfoTimeout, info,
          wg.gate, wg.limit_ns);
    else
      panel_gemm2_kernel<CholTrailItems, false><<<grid, kPg2Threads, pg2_smem_bytes(false), st>>>(
          mPh[b], mPl[b], mPh[b], mPl[b], mA, mRT, dec, chunk, units, info, kInfoTimeout, info,
          wg.gate, wg.limit_ns);
    note_launch();
    return cudaGetLastError();
  };
  // the update past the super-panel [P0, P1) of column blocks [cb_lo, cb_hi)
  auto past = [&](int b, int P0, int P1, int cb_lo, int cb_hi, cudaStream_t st) -> cudaError_t {
    if (npan == 1) return trail(b, P0, 0, cb_lo, cb_hi, st);
    const CholSuperItems dec{w.A, U, n, P0, P1, nblk, cb_lo, cb_hi};
    const int units = sg_units(dec);
    if (units == 0) return cudaSuccess;
    const int grid = std::min(units, sms);
    if (reduce)
      stream_gemm_kernel<CholSuperItems, true><<<grid, kPg2Threads, sg_smem_bytes(true), st>>>(
          mPh[b], mPl[b], mPh[b], mPl[b], mA, mRT, dec, units, info, kInfoTimeout, info, wg.gate,
          wg.limit_ns);
    else
      stream_gemm_kernel<CholSuperItems, false><<<grid, kPg2Threads, sg_smem_bytes(false), st>>>(
          mPh[b], mPl[b], mPh[b], mPl[b], mA, mRT, dec, units, info, kInfoTimeout, info, wg.gate,
          wg.limit_ns);
    note_launch();
    return cudaGetLastError();
  };
  // Look-ahead (when the caller gives a side stream): the trailing update of
  // panel p is split into the next panel's column block (near, on the
  // caller's stream, so panel p + 1 can be factored at once) and the rest
  // (far, on the side stream, overlapping the factorisation of panel p + 1).
  // Inside a super-panel the updates stop at its end; after its last panel
  // the update past it is split the same way.  Every element still receives
  // its updates in a fixed order: each near update waits for the far update
  // issued before it.  Super-panels alternate between the two halves of the
  // panel-vector buffer; the next writer of a half (the first panel two
  // super-panels on) runs after the caller's stream has waited for the last
  // far update that reads it.  Without a side stream everything runs on s.
  SideEvents side;
  const bool ahead = nblk > 2 && side_s != nullptr && side_s != s;
  if (ahead && !side.create()) return cudaErrorMemoryAllocation;
  bool far_pending = false, past_pending = false;
  for (int P0 = 0, sp = 0; P0 < nblk; P0 += npan, ++sp) {
    const int P1 = std::min(P0 + npan, nblk);
    const int b = sp & 1;
    for (int p = P0; p < P1; ++p) {
      const int pk = (p - P0) * kPanel;
      chol_diag_kernel<<<1, kDiagThreads, kDiagSmemBytes, s>>>(w.A, n, p, w.Dout[0], info);
      note_launch();
      panel_apply_kernel<<<apply_ctas, kApplyThreads, kApplySmemBytes, s>>>(
          w.A, U, n, p, w.Dout[0], w.PBh[b] + pk, w.PBl[b] + pk, SPW, info);
      note_launch();
      if (p + 1 >= nblk) break;
      const bool inside = p + 1 < P1;      // more panels of this super-panel follow
      const int end = inside ? P1 : nblk;  // column blocks this panel's update reaches
      if (!ahead) {
        if ((e = inside ? trail(b, p, pk, p + 1, end, s) : past(b, P0, P1, p + 1, end, s)) !=
            cudaSuccess)
          return e;
        continue;
      }
      if (p + 2 < end) {
        // side: far(p) after apply(p) (and after the earlier far updates, in stream order)
        if ((e = cudaEventRecord(side.ev[0], s)) != cudaSuccess ||
            (e = cudaStreamWaitEvent(side_s, side.ev[0], 0)) != cudaSuccess)
          return e;
      }
      // caller's stream: near(p) after the far update issued before it has landed
      if (far_pending) {
        if ((e = cudaStreamWaitEvent(s, side.ev[1], 0)) != cudaSuccess) return e;
        far_pending = false;
      }
      if (past_pending) {
        if ((e = cudaStreamWaitEvent(s, side.ev[2], 0)) != cudaSuccess) return e;
        past_pending = false;
      }
      if ((e = inside ? trail(b, p, pk, p + 1, p + 2, s) : past(b, P0, P1, p + 1, p + 2, s)) !=
          cudaSuccess)
        return e;
      if (p + 2 < end) {
        if ((e = inside ? trail(b, p, pk, p + 2, end, side_s)
                        : past(b, P0, P1, p + 2, end, side_s)) != cudaSuccess)
          return e;
        if ((e = cudaEventRecord(side.ev[inside ? 1 : 2], side_s)) != cudaSuccess) return e;
        (inside ? far_pending : past_pending) = true;
      }
    }
  }
  if (ahead) {
    // join: every far update before the caller's stream goes on
    if ((e = cudaEventRecord(side.ev[1], side_s)) != cudaSuccess ||
        (e = cudaStreamWaitEvent(s, side.ev[1], 0)) != cudaSuccess)
      return e;
  }
  }  // launch by launch
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
// factorisation, 21.1 MB.  Larger n is rejected with GPTQ_ERR_WORKSPACE.
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
  const gptq::NvtxScope nvtx("gptq_cholesky_inverse_noalloc");
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
                                                      info, ws, static_cast<cudaStream_t>(stream),
                                                      nullptr);
  return e == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA;
}
