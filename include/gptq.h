/*
 * gptq.h -- C ABI of libgptq_b200.so, a GPTQ layer-wise weight quantizer for
 * NVIDIA B200 (sm_100a).
 *
 * The method is the one described on the web page "GPTQ, with the code open"
 * (modelfoundations.com/notes/gptq): per linear layer, accumulate the
 * calibration Hessian H = 2 X X^T; zero dead inputs, optionally reorder the
 * columns by descending diag(H) ("act-order"), add 1 % of the mean diagonal
 * ("damping"); take the upper Cholesky factor U of H^-1; sweep the columns
 * left to right, rounding each to an asymmetric min-max grid ("ruler") and
 * spreading its rounding error over the columns not yet quantized, with the
 * repairs past the current block of 128 columns deferred to one product per
 * block; store tick indices plus a per-row or per-group ruler.
 *
 * Conventions shared by every entry point:
 *  - Every pointer argument is DEVICE memory owned by the caller unless the
 *    comment says otherwise.  The library allocates no device memory (every
 *    scratch buffer is a caller workspace sized by gptq_workspace_size),
 *    creates no stream, and keeps no state between calls apart from the
 *    launch counter read by gptq_launch_count, the calling thread's wait
 *    gate (gptq_set_wait_gate, a test hook), a per-device cache of one
 *    occupancy query and, in the debug build only, the words of failed
 *    index checks (gptq_device_checks).  A call given a side stream creates four CUDA events
 *    for its enqueue and destroys them before it returns.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the
 *    legacy default stream).  The returned status covers argument checks and
 *    kernel launches only.  Numerical failures and device-side wait timeouts
 *    are written to the caller's device `info` word (0 = no failure).
 *  - Matrices are row-major and dense: a rows x cols matrix has its element
 *    (r, c) at offset r*ld + c, with ld = cols unless a leading dimension is
 *    passed.
 *  - n (input features, columns of W, size of H) indexes the SWEEP ORDER
 *    after act-order wherever the comment says "sweep order".
 */
#ifndef GPTQ_B200_H
#define GPTQ_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GPTQ_OK = 0,
  GPTQ_ERR_INVALID_ARG = 1,  /* null pointer, bad size, misaligned buffer      */
  GPTQ_ERR_UNSUPPORTED = 2,  /* valid request this build does not implement    */
  GPTQ_ERR_WORKSPACE = 3,    /* workspace smaller than gptq_workspace_size()   */
  GPTQ_ERR_CUDA = 4,         /* a CUDA runtime call or kernel launch failed    */
  GPTQ_ERR_TIMEOUT = 5       /* (device `info` value) a bounded wait ran out   */
} gptq_status;

typedef enum { GPTQ_BF16 = 0, GPTQ_F32 = 1 } gptq_dtype;

/* Quantizer settings (page "What is GPTQ", table "Key settings"; page "GPTQ,
 * with the code open", section "Paper vs. code").
 *   bits        2..8; the packers handle 3 and 4.
 *   group_size  -1 = one ruler per row, fitted before the sweep on the
 *               unrepaired weights; otherwise a new ruler every group_size
 *               columns of the sweep order, fitted when the sweep reaches the
 *               group's first column, on the current (repaired) weights.
 *               Supported: 32, 64, 128 or any multiple of 128.
 *   percdamp    damping as a fraction of mean(diag H); 0.01 in the pages.
 *   block       lazy-update block; must be 128.
 *   actorder    nonzero: sweep columns in order of descending diag(H).
 *   sym         0: asymmetric min-max ruler (the default in the pages);
 *               1: the opt-in symmetric ruler -- range [-m, m] with
 *               m = max(|min|, |max|), scale = 2m / (2^b - 1), zero point on
 *               the middle tick 2^(b-1).  Any other value: invalid. */
typedef struct {
  int bits;
  int group_size;
  float percdamp;
  int block;
  int actorder;
  int sym;
} gptq_config;

typedef enum {
  GPTQ_OP_HESSIAN = 0,
  GPTQ_OP_CHOLESKY = 1,
  GPTQ_OP_QUANTIZE = 2,
  GPTQ_OP_DEQUANT_MATVEC = 3
} gptq_op;

/* Bytes of device workspace `op` needs for these sizes (0 is possible).
 * rows/n/ntok as in the calls below (for GPTQ_OP_DEQUANT_MATVEC, rows is the
 * number of activation vectors, `batch`); xt is the calibration dtype
 * (hessian only); cfg may be NULL except for GPTQ_OP_QUANTIZE.  Host
 * pointer `bytes`.  Workspaces are 256-byte aligned; their contents on entry
 * do not matter. */
gptq_status gptq_workspace_size(int op, int64_t rows, int64_t n, int64_t ntok, gptq_dtype xt,
                                const gptq_config* cfg, size_t* bytes);

/* H += alpha * X X^T     (page "GPTQ, with the code open", section "Measuring
 * damage where it matters": H = 2 X X^T; section "Paper vs. code": H is built
 * up over calibration batches -- call once per batch; alpha = 2 gives the sum
 * form).
 *   H      n x n fp32.  Must be symmetric on entry (e.g. zeroed); on return
 *          it is symmetric: the upper triangle is accumulated and mirrored.
 *   X      n x ntok, features x tokens, row stride ldx elements (ldx >= ntok),
 *          dtype xt.  bf16: the products are exact in fp32 and summed in fp32
 *          on the tensor cores.  fp32: each value is split into two bf16
 *          parts hi + lo and H gets hi hi^T + hi lo^T + lo hi^T.
 *          Requirements: X 16-byte aligned, ldx * sizeof(element) a multiple
 *          of 16 bytes; H 16-byte aligned.
 *   token_major  must be 0.
 *   ws     workspace of gptq_workspace_size(GPTQ_OP_HESSIAN, 0, n, ntok, xt)
 *          bytes: counters of the ordered reduction (below), and for fp32 X
 *          the bf16 parts.
 *   info   optional device int32: set to GPTQ_ERR_TIMEOUT if a pipeline wait
 *          inside the kernel gave up (then H is incomplete).  Not cleared.
 * The result is reproducible bit for bit: the tokens are cut into chunks
 * (for parallelism) and the chunks of each output tile are added into H in
 * chunk order, one chunk at a time.  Calls that overlap on the GPU must not
 * share a workspace or an H. */
gptq_status gptq_hessian_accumulate(float* H, const void* X, gptq_dtype xt, int64_t n,
                                    int64_t ntok, int64_t ldx, int token_major, float alpha,
                                    void* ws, size_t ws_bytes, int32_t* info, void* stream);

/* Preparation and the upper Cholesky factor of the damped inverse
 * (page "GPTQ, with the code open", sections "From one repair to a whole
 * model" and "Paper vs. code"):
 *   dead[i]  = diag(H)_i == 0; such diagonal entries are set to 1 (their
 *              weight columns are zeroed by gptq_quantize_layer);
 *   perm     = identity, or with actorder a stable sort of the columns by
 *              descending diag(H) (after the dead fix): perm[k] is the
 *              original column quantized k-th;
 *   H'       = H[perm][:, perm] + lambda I, lambda = percdamp * mean(diag H);
 *   U        n x n fp32, upper triangular (strict lower part written as 0),
 *              in sweep order, with H'^-1 = U^T U.
 * H (n x n fp32, symmetric) is read, not modified.
 * perm may be NULL only when actorder == 0.  dead: uint8[n].
 * info (device int32, required): 0 on success; k > 0 if H' was found not
 * positive definite at sweep position k - 1 (the factorisation runs from the
 * last sweep position towards the first, so this is the highest failing
 * position); -1 if diag(H) holds a NaN or an infinity; -2 if a bounded wait
 * inside a tensor-core kernel gave up.  On failure U is
 * undefined.  ws: gptq_workspace_size(GPTQ_OP_CHOLESKY, 0, n, 0, .., NULL).
 * side_stream: NULL (or equal to stream) runs everything on `stream`.
 * Otherwise a second stream of the caller's, used for look-ahead: the part
 * of each panel's trailing update that the next panel does not need runs
 * there, overlapping the next panel's factorisation; the call leaves
 * `stream` ordered after all of it.  The caller must not use side_stream for
 * anything that may run between the call's enqueue and the completion of
 * its work on `stream`; results are identical either way. */
gptq_status gptq_cholesky_inverse(const float* H, int64_t n, float percdamp, int actorder,
                                  float* U, int32_t* perm, uint8_t* dead, int32_t* info,
                                  void* ws, size_t ws_bytes, void* stream, void* side_stream);

/* gptq_cholesky_inverse for callers that cannot allocate device memory.
 * The pages have no counterpart of this entry point; it exists for host
 * programs that own all device memory in a fixed pool and forbid allocation
 * while running, so they can neither call cudaMalloc nor pass a workspace.
 * Same arguments, results and `info` contract as gptq_cholesky_inverse, minus
 * the workspace and the side stream: the scratch is a 21.1 MB array built
 * into the library, so n must be <= 2048 (larger n returns
 * GPTQ_ERR_WORKSPACE), and everything runs on `stream`.  The library looks
 * up that array's device address once per device, in the first call made with
 * that device current; make that first call before any stream capture.  All
 * calls share the array: calls that overlap on the GPU race on it, so the
 * caller must serialise them (e.g. one stream).  No call allocates device
 * memory or creates a stream or an event. */
gptq_status gptq_cholesky_inverse_noalloc(const float* H, int64_t n, float percdamp,
                                          int actorder, float* U, int32_t* perm, uint8_t* dead,
                                          int32_t* info, void* stream);

/* The column sweep with lazy block updates (page "GPTQ, with the code open",
 * sections "The repair rule", "From one repair to a whole model" and "What
 * quantization is, and why anyone bothers").  For each column j of the sweep
 * order, for every row:
 *   scale = (xmax - xmin) / (2^bits - 1), zero = rint(-xmin / scale) with
 *   [xmin, xmax] the ruler's range stretched to include 0 ([-1, 1] if flat);
 *   q = clamp(rint(w / scale) + zero, 0, 2^bits - 1);  w_hat = scale (q - zero);
 *   err = (w - w_hat) / U[j][j];  W[:, j+1:] -= err * U[j, j+1:]
 * with the update past the current 128-column block applied once per block.
 * All arithmetic is fp32 with IEEE division and round-half-to-even.  The
 * result is reproducible bit for bit.
 *   W        rows x n in wt (original column order); not modified.
 *   U, perm, dead  from gptq_cholesky_inverse (perm may be NULL = identity).
 *   codes    uint8 rows x n, ORIGINAL column order.
 *   scales   fp32 rows x G, zeros uint8 rows x G, G = ceil(n / group_size)
 *            (1 for per-row rulers), in sweep order of the groups.
 *   g_idx    optional int32[n]: group of each original column.
 *   Wq       optional fp32 rows x n, original order: the dequantized weights.
 *   row_loss optional fp32[rows]: sum over columns of (w - w_hat)^2 / (2 U_jj^2).
 *   ws       gptq_workspace_size(GPTQ_OP_QUANTIZE, rows, n, 0, .., cfg).
 *   info     optional device int32, set to 0 by the call, then to -2 if a
 *            bounded wait inside a tensor-core kernel gave up (the outputs
 *            are then undefined).
 *   side_stream  as for gptq_cholesky_inverse: NULL runs everything on
 *            `stream`; a second stream lets the lazy update of the columns
 *            past the next block overlap the next block's sweep. */
gptq_status gptq_quantize_layer(const void* W, gptq_dtype wt, int64_t rows, int64_t n,
                                const float* U, const int32_t* perm, const uint8_t* dead,
                                const gptq_config* cfg, uint8_t* codes, float* scales,
                                uint8_t* zeros, int32_t* g_idx, float* Wq, float* row_loss,
                                void* ws, size_t ws_bytes, int32_t* info, void* stream,
                                void* side_stream);

/* Packed storage of tick indices (page "GPTQ, with the code open", section
 * "What quantization is, and why anyone bothers": store the tick index).  The
 * bit layout is this library's own:
 *   int4: column 8i+k of a row -> bits [4k, 4k+4) of uint32 word i of the row
 *         (n % 8 == 0; out is rows x n/8).
 *   int3: column 32i+k -> bits [3k, 3k+3) of the 96-bit little-endian word
 *         formed by uint32 words 3i, 3i+1, 3i+2 of the row (n % 32 == 0; out is
 *         rows x 3n/32).  Codes are masked to their low 4 (3) bits. */
gptq_status gptq_pack_int4(const uint8_t* codes, int64_t rows, int64_t n, uint32_t* out,
                           void* stream);
gptq_status gptq_pack_int3(const uint8_t* codes, int64_t rows, int64_t n, uint32_t* out,
                           void* stream);

/* w_hat[r][c] = scale[r][G(c)] * (code[r][c] - zero[r][G(c)])  -- one fp32
 * multiply (section "What quantization is, and why anyone bothers": turning
 * an integer back into a number is one multiply); ot = GPTQ_BF16 rounds that
 * fp32 value to bfloat16, half to even.  G(c) = g_idx[c] if g_idx is given,
 * else c / group_size, or 0 when group_size <= 0.  packed in the layout of
 * gptq_pack_int4 / gptq_pack_int3 (bits 4 or 3); scales fp32 and zeros uint8
 * are rows x G with row stride G = ceil(n / group_size) (1 if per row) --
 * pass n_groups explicitly when g_idx is used.  out: rows x n of ot. */
gptq_status gptq_dequant(const uint32_t* packed, int bits, int64_t rows, int64_t n,
                         const float* scales, const uint8_t* zeros, int group_size,
                         int64_t n_groups, const int32_t* g_idx, void* out, gptq_dtype ot,
                         void* stream);

/* The consumer of the packed codes: y = x w_hat^T for `batch` activation
 * vectors, with w_hat dequantized on the fly and never stored (page "GPTQ,
 * with the code open", section "Claims & evidence": the faster generation
 * comes from custom kernels at batch size 1, where reading the weights
 * dominates -- packed codes are 8 / bits times smaller than fp32, 4 / bits
 * times smaller than bf16).
 * Two kernels serve it.  int4 or int3 codes with bf16 x, no g_idx,
 * n % 32 == 0, group_size a power of two >= 32 (or per row), packed 16-byte
 * (int4) or 4-byte (int3) aligned and zero points < 128: the tensor-core kernel, which multiplies exact bf16
 * (q - zero) pairs with x in fp32 MMA accumulators, scales each group's sum
 * once, and adds the two column halves of every output onto zeros (two
 * terms, so the result does not depend on their order).  It first writes x
 * (gathered by perm, if given) into the workspace as batch x n bf16, and
 * zeroes y.  Codes in original order with g_idx (int4 with n % 32 == 0, or
 * int3 with n % 128 == 0, packed 16-byte aligned): a kernel with one row
 * per lane, each weight's own (scale, zero) read from shared memory, four
 * partial sums per lane and vector added over the warps in a fixed order.
 * Everything else: the FP32-pipe kernel, one rounded FMA per term.  Every
 * path gives the same y from run to run.
 *   packed, scales, zeros, group_size, n_groups, g_idx: exactly as for
 *          gptq_dequant (same layout, same single-multiply w_hat).
 *   perm   NULL, or (with g_idx NULL) the sweep order of an act-order layer:
 *          the packed rows then hold the codes in sweep order (column k is
 *          original column perm[k], see gptq_gather_columns_u8), so every
 *          group is a run of group_size consecutive columns, and column k
 *          multiplies x[b][perm[k]].  Reading rulers per run instead of per
 *          column is what makes act-order layers fast here.
 *   x      batch x n activations, row-major, xt = GPTQ_BF16 or GPTQ_F32.
 *   y      batch x rows fp32 (written), y[b][r] = sum_c w_hat[r][c] x[b][c],
 *          summed in fp32.
 *   ws     gptq_workspace_size(GPTQ_OP_DEQUANT_MATVEC, batch, n, ...) bytes.
 * batch >= 0 (any size; launched in groups of 8, 4, 2, 1).  Errors as for
 * gptq_dequant; perm together with g_idx is invalid. */
gptq_status gptq_dequant_matvec(const uint32_t* packed, int bits, int64_t rows, int64_t n,
                                const float* scales, const uint8_t* zeros, int group_size,
                                int64_t n_groups, const int32_t* g_idx, const int32_t* perm,
                                const void* x, gptq_dtype xt, int64_t batch, float* y,
                                void* ws, size_t ws_bytes, void* stream);

/* dst[r][k] = src[r][perm[k]] for a rows x n byte matrix (device pointers;
 * perm int32[n], a permutation of 0..n-1).  With the `perm` of
 * gptq_cholesky_inverse it turns codes in original column order into codes
 * in sweep order, for packing and gptq_dequant_matvec.  src and dst must not
 * overlap. */
gptq_status gptq_gather_columns_u8(const uint8_t* src, int64_t rows, int64_t n,
                                   const int32_t* perm, uint8_t* dst, void* stream);

/* Random-sign blocked Hadamard rotation R = blockdiag(H_b / sqrt(b)) diag(s)
 * (page "Post-Training Quantization: Calibration, GPTQ and Why Rotations
 * Help", section "Rotations: making outliers disappear": rotate the
 * activations, give the weights the inverse rotation, and the layer's product
 * is unchanged while outliers are spread over all entries).  H_b is
 * Sylvester's Hadamard matrix, H[i][j] = (-1)^popcount(i & j); block b is a
 * power of two in [32, 1024] (else GPTQ_ERR_UNSUPPORTED) and divides n;
 * signs: n floats, +1 or -1 (device).  Computed in fp32 by a fast
 * Walsh-Hadamard transform (log2 b butterfly stages), rounded once to ot
 * (bf16: half to even).
 *
 * gptq_hadamard_rows: W' = W R^T for W rows x n (row stride ld_in elements):
 *   out[r][kb + j] = (1/sqrt(b)) sum_i H_b[j][i] s[kb + i] in[r][kb + i].
 * gptq_hadamard_cols: X' = R X for X n x ntok (row stride ld_in elements):
 *   out[kb + j][t] = (1/sqrt(b)) sum_i H_b[j][i] s[kb + i] in[kb + i][t].
 * in / out: device pointers of type it / ot (GPTQ_BF16 or GPTQ_F32), either
 * the same buffer (same type and stride: in place) or non-overlapping; the
 * caller owns both.  Strides must cover a row (ld >= n, resp. ntok).  Zero
 * rows or tokens: nothing is done. */
gptq_status gptq_hadamard_rows(const void* in, gptq_dtype it, int64_t rows, int64_t n,
                               int64_t ld_in, const float* signs, int block, void* out,
                               gptq_dtype ot, int64_t ld_out, void* stream);
gptq_status gptq_hadamard_cols(const void* in, gptq_dtype it, int64_t n, int64_t ntok,
                               int64_t ld_in, const float* signs, int block, void* out,
                               gptq_dtype ot, int64_t ld_out, void* stream);

/* Static string for a status code (host). */
const char* gptq_status_string(int status);

/* Diagnostics (host): number of kernels this library has enqueued in this
 * process so far. */
int64_t gptq_launch_count(void);

/* Test hook for the bounded waits (host).  Every wait inside the library's
 * tensor-core kernels (gptq_hessian_accumulate, the trailing updates of
 * gptq_cholesky_inverse and gptq_quantize_layer) gives up after 1 s and
 * reports through the call's `info` word instead of hanging.  To exercise
 * that path, a test passes a device int32 `gate` that holds 0 and a short
 * limit_ns (1..1e9): every such kernel that the calling host thread enqueues
 * afterwards first waits for *gate != 0 with nothing in flight, gives up
 * after limit_ns, and the call reports its timeout as documented.  gate =
 * NULL restores the normal behaviour (limit_ns ignored).  The setting
 * belongs to the calling host thread only.  Returns GPTQ_ERR_INVALID_ARG for
 * a limit out of range. */
gptq_status gptq_set_wait_gate(const int32_t* gate, int64_t limit_ns);

/* Debug builds only (host; no counterpart in the pages).  The library can be
 * built a second time as libgptq_b200_debug.so with device-side index checks
 * (python -m post_weight_quantization_25_b200.build --debug): every kernel
 * that indexes with a caller-supplied group index (g_idx of gptq_dequant,
 * gptq_dequant_matvec) or permutation (perm of gptq_quantize_layer,
 * gptq_gather_columns_u8, gptq_dequant_matvec) tests each index against its
 * range first, does not use one that is out of range (the value it would
 * have produced is left 0, so those outputs are undefined), and records the
 * kind of check that failed.  gptq_device_checks waits for the device
 * (cudaDeviceSynchronize), writes the recorded kinds to *flags (host) as a
 * bit set -- 1: a group index out of [0, n_groups), 2: a permutation entry
 * out of [0, n) -- and clears them.  Release builds do no such checks (those
 * indices are the caller's to keep in range) and return GPTQ_ERR_UNSUPPORTED;
 * a debug build returns GPTQ_ERR_INVALID_ARG for flags = NULL. */
gptq_status gptq_device_checks(uint32_t* flags);

/* Self-test of the division the sweep uses to round w / scale (a
 * correctly rounded binary32 division by Markstein's FMA method, with the
 * reciprocal of the divisor computed once per ruler): out[i] = a[i] / b[i]
 * for b[i] > 0.  Device arrays of `count` floats.  The result must equal
 * IEEE round-to-nearest division bit for bit; the tests check that. */
gptq_status gptq_selftest_division(const float* a, const float* b, int64_t count, float* out,
                                   void* stream);

#ifdef __cplusplus
}
#endif

#endif /* GPTQ_B200_H */
