// C ABI of libgptq_b200.so: argument checks, workspace layout, launches.
// See include/gptq.h for the contract of every entry point.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "gptq_internal.cuh"

namespace gptq {

int num_sms() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms > 0 ? sms : 148;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver entry point is looked up through the runtime, so the library
// does not link libcuda directly and loads on machines without a GPU.
static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

bool make_tma_2d(CUtensorMap* map, const void* base, bool bf16, int64_t rows, int64_t cols,
                 int64_t ld, uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const int64_t esz = bf16 ? 2 : 4;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * esz)};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
             const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static std::atomic<long long> g_launches{0};

bool SideEvents::create() {
  for (auto& e : ev)
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
      e = nullptr;
      return false;
    }
  return true;
}

SideEvents::~SideEvents() {
  for (auto& e : ev)
    if (e) cudaEventDestroy(e);
}

namespace {
thread_local WaitGate t_gate = {nullptr, (uint64_t)kGridWaitLimitNs};
}  // namespace

WaitGate current_wait_gate() { return t_gate; }

void set_wait_gate(const int32_t* gate, uint64_t limit_ns) {
  t_gate.gate = gate;
  t_gate.limit_ns = gate ? limit_ns : (uint64_t)kGridWaitLimitNs;
}

void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

}  // namespace gptq

namespace {

constexpr int64_t kMaxN = 57344;       // a row of H / W is staged in shared memory
constexpr int64_t kMaxRows = 1 << 24;

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

gptq_status cuda_status(cudaError_t e) { return e == cudaSuccess ? GPTQ_OK : GPTQ_ERR_CUDA; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// [split-K turnstile flags | fp32 input only: bf16 hi part | bf16 lo part]
size_t hessian_flags_bytes(int64_t n) { return align_up(gptq::syrk_flag_bytes(n), 256); }

size_t hessian_split_bytes(int64_t n, int64_t ntok) {
  const int64_t ld = (ntok + 7) / 8 * 8;
  return align_up(sizeof(uint16_t) * (size_t)n * ld, 256);
}

size_t hessian_ws(int64_t n, int64_t ntok, gptq_dtype xt) {
  return hessian_flags_bytes(n) + (xt == GPTQ_F32 ? 2 * hessian_split_bytes(n, ntok) : 0);
}

gptq_status check_cfg(const gptq_config* cfg) {
  if (!cfg) return GPTQ_ERR_INVALID_ARG;
  if (cfg->bits < 2 || cfg->bits > 8) return GPTQ_ERR_INVALID_ARG;
  if (cfg->sym != 0 && cfg->sym != 1) return GPTQ_ERR_INVALID_ARG;
  if (cfg->block != gptq::kBlock) return GPTQ_ERR_UNSUPPORTED;
  const int g = cfg->group_size;
  if (g == 0 || g < -1) return GPTQ_ERR_INVALID_ARG;
  if (g > 0 && !(g == 32 || g == 64 || g % gptq::kBlock == 0)) return GPTQ_ERR_UNSUPPORTED;
  return GPTQ_OK;
}

}  // namespace

extern "C" {

int64_t gptq_launch_count(void) { return gptq::g_launches.load(std::memory_order_relaxed); }

gptq_status gptq_set_wait_gate(const int32_t* gate, int64_t limit_ns) {
  if (gate && (limit_ns <= 0 || limit_ns > gptq::kGridWaitLimitNs)) return GPTQ_ERR_INVALID_ARG;
  gptq::set_wait_gate(gate, (uint64_t)limit_ns);
  return GPTQ_OK;
}

gptq_status gptq_selftest_division(const float* a, const float* b, int64_t count, float* out,
                                   void* stream) {
  if (count < 0) return GPTQ_ERR_INVALID_ARG;
  if (count == 0) return GPTQ_OK;
  if (!a || !b || !out) return GPTQ_ERR_INVALID_ARG;
  return cuda_status(
      gptq::launch_selftest_division(a, b, count, out, static_cast<cudaStream_t>(stream)));
}

gptq_status gptq_device_checks(uint32_t* flags) {
#ifdef GPTQ_DEVICE_CHECKS
  if (!flags) return GPTQ_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return GPTQ_ERR_CUDA;
  const uint32_t v = gptq::take_device_checks_pack() | gptq::take_device_checks_sweep();
  if (v == ~0u) return GPTQ_ERR_CUDA;
  *flags = v;
  return GPTQ_OK;
#else
  (void)flags;
  return GPTQ_ERR_UNSUPPORTED;
#endif
}

const char* gptq_status_string(int status) {
  switch (status) {
    case GPTQ_OK: return "ok";
    case GPTQ_ERR_INVALID_ARG: return "invalid argument";
    case GPTQ_ERR_UNSUPPORTED: return "unsupported request";
    case GPTQ_ERR_WORKSPACE: return "workspace too small";
    case GPTQ_ERR_CUDA: return "CUDA error";
    case GPTQ_ERR_TIMEOUT: return "device wait timed out";
    default: return "unknown status";
  }
}

gptq_status gptq_workspace_size(int op, int64_t rows, int64_t n, int64_t ntok, gptq_dtype xt,
                                const gptq_config* cfg, size_t* bytes) {
  if (!bytes || n <= 0 || n > kMaxN) return GPTQ_ERR_INVALID_ARG;
  switch (op) {
    case GPTQ_OP_HESSIAN:
      if (ntok < 0) return GPTQ_ERR_INVALID_ARG;
      *bytes = hessian_ws(n, ntok, xt);
      return GPTQ_OK;
    case GPTQ_OP_CHOLESKY:
      *bytes = gptq::cholesky_workspace_bytes(n);
      return GPTQ_OK;
    case GPTQ_OP_QUANTIZE: {
      if (rows < 0 || rows > kMaxRows) return GPTQ_ERR_INVALID_ARG;
      const gptq_status st = check_cfg(cfg);
      if (st != GPTQ_OK) return st;
      *bytes = gptq::quantize_workspace_bytes(rows, n);
      return GPTQ_OK;
    }
    case GPTQ_OP_DEQUANT_MATVEC:
      if (rows < 0) return GPTQ_ERR_INVALID_ARG;
      *bytes = gptq::dequant_matvec_workspace_bytes(rows, n);
      return GPTQ_OK;
    default:
      return GPTQ_ERR_INVALID_ARG;
  }
}

gptq_status gptq_hessian_accumulate(float* H, const void* X, gptq_dtype xt, int64_t n,
                                    int64_t ntok, int64_t ldx, int token_major, float alpha,
                                    void* ws, size_t ws_bytes, int32_t* info, void* stream) {
  const gptq::NvtxScope nvtx("gptq_hessian_accumulate");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!H || n <= 0 || n > kMaxN || ntok < 0 || ldx < ntok) return GPTQ_ERR_INVALID_ARG;
  if (xt != GPTQ_BF16 && xt != GPTQ_F32) return GPTQ_ERR_INVALID_ARG;
  if (token_major) return GPTQ_ERR_UNSUPPORTED;
  if (!aligned(H, 16)) return GPTQ_ERR_INVALID_ARG;
  if (ntok == 0) return GPTQ_OK;
  if (!X) return GPTQ_ERR_INVALID_ARG;
  const size_t need = hessian_ws(n, ntok, xt);
  if (!ws || ws_bytes < need) return GPTQ_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return GPTQ_ERR_INVALID_ARG;
  void* flags = ws;
  cudaError_t e;
  if (xt == GPTQ_BF16) {
    if (!aligned(X, 16) || (ldx * 2) % 16 != 0) return GPTQ_ERR_INVALID_ARG;
    if ((e = gptq::launch_syrk_bf16(H, n, X, X, ntok, ldx, alpha, info, flags, s)) !=
        cudaSuccess)
      return cuda_status(e);
  } else {
    if (!aligned(X, 4)) return GPTQ_ERR_INVALID_ARG;
    const int64_t ld = (ntok + 7) / 8 * 8;
    char* hi = static_cast<char*>(ws) + hessian_flags_bytes(n);
    char* lo = hi + hessian_split_bytes(n, ntok);
    if ((e = gptq::launch_split_bf16(static_cast<const float*>(X), n, ntok, ldx, hi, lo, ld, s)) !=
        cudaSuccess)
      return cuda_status(e);
    // hi hi^T + hi lo^T + lo hi^T  (lo lo^T is below fp32 resolution of the sum)
    if ((e = gptq::launch_syrk_bf16(H, n, hi, hi, ntok, ld, alpha, info, flags, s)) !=
            cudaSuccess ||
        (e = gptq::launch_syrk_bf16(H, n, hi, lo, ntok, ld, alpha, info, flags, s)) !=
            cudaSuccess ||
        (e = gptq::launch_syrk_bf16(H, n, lo, hi, ntok, ld, alpha, info, flags, s)) !=
            cudaSuccess)
      return cuda_status(e);
  }
  return cuda_status(gptq::launch_mirror_upper(H, n, s));
}

gptq_status gptq_cholesky_inverse(const float* H, int64_t n, float percdamp, int actorder,
                                  float* U, int32_t* perm, uint8_t* dead, int32_t* info,
                                  void* ws, size_t ws_bytes, void* stream, void* side_stream) {
  const gptq::NvtxScope nvtx("gptq_cholesky_inverse");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!H || !U || !dead || !info || n <= 0 || n > kMaxN) return GPTQ_ERR_INVALID_ARG;
  if (actorder && !perm) return GPTQ_ERR_INVALID_ARG;
  if (!(percdamp >= 0.f)) return GPTQ_ERR_INVALID_ARG;
  if (!ws || ws_bytes < gptq::cholesky_workspace_bytes(n)) return GPTQ_ERR_WORKSPACE;
  if (!aligned(ws, 256) || !aligned(H, 4) || !aligned(U, 16)) return GPTQ_ERR_INVALID_ARG;
  return cuda_status(gptq::launch_cholesky_inverse(H, n, percdamp, actorder, U, perm, dead, info,
                                                   ws, s, static_cast<cudaStream_t>(side_stream)));
}

gptq_status gptq_quantize_layer(const void* W, gptq_dtype wt, int64_t rows, int64_t n,
                                const float* U, const int32_t* perm, const uint8_t* dead,
                                const gptq_config* cfg, uint8_t* codes, float* scales,
                                uint8_t* zeros, int32_t* g_idx, float* Wq, float* row_loss,
                                void* ws, size_t ws_bytes, int32_t* info, void* stream,
                                void* side_stream) {
  const gptq::NvtxScope nvtx("gptq_quantize_layer");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const gptq_status st = check_cfg(cfg);
  if (st != GPTQ_OK) return st;
  if (n <= 0 || n > kMaxN || rows < 0 || rows > kMaxRows) return GPTQ_ERR_INVALID_ARG;
  if (wt != GPTQ_BF16 && wt != GPTQ_F32) return GPTQ_ERR_INVALID_ARG;
  if (rows == 0) return GPTQ_OK;
  if (!W || !U || !dead || !codes || !scales || !zeros) return GPTQ_ERR_INVALID_ARG;
  if (!ws || ws_bytes < gptq::quantize_workspace_bytes(rows, n)) return GPTQ_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return GPTQ_ERR_INVALID_ARG;
  return cuda_status(gptq::launch_quantize_layer(W, wt, rows, n, U, perm, dead, cfg->bits,
                                                 cfg->group_size, cfg->sym, codes, scales, zeros,
                                                 g_idx, Wq, row_loss, ws, info, s,
                                                 static_cast<cudaStream_t>(side_stream)));
}

gptq_status gptq_pack_int4(const uint8_t* codes, int64_t rows, int64_t n, uint32_t* out,
                           void* stream) {
  const gptq::NvtxScope nvtx("gptq_pack_int4");
  if (rows < 0 || n <= 0 || n % 8 != 0) return GPTQ_ERR_INVALID_ARG;
  if (rows == 0) return GPTQ_OK;
  if (!codes || !out || !aligned(out, 4)) return GPTQ_ERR_INVALID_ARG;
  return cuda_status(gptq::launch_pack_int4(codes, rows, n, out, static_cast<cudaStream_t>(stream)));
}

gptq_status gptq_pack_int3(const uint8_t* codes, int64_t rows, int64_t n, uint32_t* out,
                           void* stream) {
  const gptq::NvtxScope nvtx("gptq_pack_int3");
  if (rows < 0 || n <= 0 || n % 32 != 0) return GPTQ_ERR_INVALID_ARG;
  if (rows == 0) return GPTQ_OK;
  if (!codes || !out || !aligned(out, 4)) return GPTQ_ERR_INVALID_ARG;
  return cuda_status(gptq::launch_pack_int3(codes, rows, n, out, static_cast<cudaStream_t>(stream)));
}

gptq_status gptq_dequant(const uint32_t* packed, int bits, int64_t rows, int64_t n,
                         const float* scales, const uint8_t* zeros, int group_size,
                         int64_t n_groups, const int32_t* g_idx, void* out, gptq_dtype ot,
                         void* stream) {
  const gptq::NvtxScope nvtx("gptq_dequant");
  if (bits != 3 && bits != 4) return GPTQ_ERR_UNSUPPORTED;
  if (rows < 0 || n <= 0) return GPTQ_ERR_INVALID_ARG;
  if ((bits == 4 && n % 8) || (bits == 3 && n % 32)) return GPTQ_ERR_INVALID_ARG;
  if (ot != GPTQ_BF16 && ot != GPTQ_F32) return GPTQ_ERR_INVALID_ARG;
  const int64_t Gdef = group_size > 0 ? (n + group_size - 1) / group_size : 1;
  const int64_t G = n_groups > 0 ? n_groups : Gdef;
  if (!g_idx && G < Gdef) return GPTQ_ERR_INVALID_ARG;
  if (rows == 0) return GPTQ_OK;
  if (!packed || !scales || !zeros || !out || !aligned(packed, 4) || !aligned(scales, 4))
    return GPTQ_ERR_INVALID_ARG;
  return cuda_status(gptq::launch_dequant(packed, bits, rows, n, scales, zeros, group_size, G,
                                          g_idx, out, ot == GPTQ_BF16 ? 1 : 0,
                                          static_cast<cudaStream_t>(stream)));
}

gptq_status gptq_dequant_matvec(const uint32_t* packed, int bits, int64_t rows, int64_t n,
                                const float* scales, const uint8_t* zeros, int group_size,
                                int64_t n_groups, const int32_t* g_idx, const int32_t* perm,
                                const void* x, gptq_dtype xt, int64_t batch, float* y,
                                void* ws, size_t ws_bytes, void* stream) {
  const gptq::NvtxScope nvtx("gptq_dequant_matvec");
  if (bits != 3 && bits != 4) return GPTQ_ERR_UNSUPPORTED;
  if (rows < 0 || n <= 0 || batch < 0) return GPTQ_ERR_INVALID_ARG;
  if ((bits == 4 && n % 8) || (bits == 3 && n % 32)) return GPTQ_ERR_INVALID_ARG;
  if (xt != GPTQ_BF16 && xt != GPTQ_F32) return GPTQ_ERR_INVALID_ARG;
  if (perm && g_idx) return GPTQ_ERR_INVALID_ARG;
  const int64_t Gdef = group_size > 0 ? (n + group_size - 1) / group_size : 1;
  const int64_t G = n_groups > 0 ? n_groups : Gdef;
  if (!g_idx && G < Gdef) return GPTQ_ERR_INVALID_ARG;
  if (rows == 0 || batch == 0) return GPTQ_OK;
  if (!packed || !scales || !zeros || !x || !y || !aligned(packed, 4) || !aligned(scales, 4) ||
      !aligned(y, 4) || !aligned(x, xt == GPTQ_BF16 ? 2 : 4))
    return GPTQ_ERR_INVALID_ARG;
  if (!ws || ws_bytes < gptq::dequant_matvec_workspace_bytes(batch, n))
    return GPTQ_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return GPTQ_ERR_INVALID_ARG;
  return cuda_status(gptq::launch_dequant_matvec(packed, bits, rows, n, scales, zeros,
                                                 group_size, G, g_idx, perm, x,
                                                 xt == GPTQ_BF16 ? 1 : 0, batch, y, ws,
                                                 static_cast<cudaStream_t>(stream)));
}

gptq_status gptq_gather_columns_u8(const uint8_t* src, int64_t rows, int64_t n,
                                   const int32_t* perm, uint8_t* dst, void* stream) {
  const gptq::NvtxScope nvtx("gptq_gather_columns_u8");
  if (rows < 0 || n <= 0 || n > kMaxN) return GPTQ_ERR_INVALID_ARG;
  if (rows == 0) return GPTQ_OK;
  if (!src || !perm || !dst || src == dst) return GPTQ_ERR_INVALID_ARG;
  return cuda_status(gptq::launch_gather_columns_u8(src, rows, n, perm, dst,
                                                    static_cast<cudaStream_t>(stream)));
}

static gptq_status hadamard_common(bool cols, const void* in, gptq_dtype it, int64_t a,
                                   int64_t b, int64_t n, int64_t ld_in, const float* signs,
                                   int block, void* out, gptq_dtype ot, int64_t ld_out,
                                   void* stream) {
  if (block < 32 || block > 1024 || (block & (block - 1))) return GPTQ_ERR_UNSUPPORTED;
  if ((it != GPTQ_BF16 && it != GPTQ_F32) || (ot != GPTQ_BF16 && ot != GPTQ_F32))
    return GPTQ_ERR_INVALID_ARG;
  if (a < 0 || b < 0 || n <= 0 || n % block) return GPTQ_ERR_INVALID_ARG;
  const int64_t inner = cols ? b : n;  // contiguous extent of a row
  if (ld_in < inner || ld_out < inner) return GPTQ_ERR_INVALID_ARG;
  if (a == 0 || b == 0) return GPTQ_OK;
  if (!in || !out || !signs || !aligned(signs, 4) || !aligned(in, it == GPTQ_BF16 ? 2 : 4) ||
      !aligned(out, ot == GPTQ_BF16 ? 2 : 4))
    return GPTQ_ERR_INVALID_ARG;
  if (in == out && (it != ot || ld_in != ld_out)) return GPTQ_ERR_INVALID_ARG;
  return cuda_status(gptq::launch_hadamard(cols, block, it == GPTQ_BF16, ot == GPTQ_BF16, in,
                                           ld_in, out, ld_out, a, b, signs,
                                           static_cast<cudaStream_t>(stream)));
}

gptq_status gptq_hadamard_rows(const void* in, gptq_dtype it, int64_t rows, int64_t n,
                               int64_t ld_in, const float* signs, int block, void* out,
                               gptq_dtype ot, int64_t ld_out, void* stream) {
  const gptq::NvtxScope nvtx("gptq_hadamard_rows");
  return hadamard_common(false, in, it, rows, n, n, ld_in, signs, block, out, ot, ld_out, stream);
}

gptq_status gptq_hadamard_cols(const void* in, gptq_dtype it, int64_t n, int64_t ntok,
                               int64_t ld_in, const float* signs, int block, void* out,
                               gptq_dtype ot, int64_t ld_out, void* stream) {
  const gptq::NvtxScope nvtx("gptq_hadamard_cols");
  return hadamard_common(true, in, it, n, ntok, n, ld_in, signs, block, out, ot, ld_out, stream);
}

}  // extern "C"
