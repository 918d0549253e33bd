"""GPTQ layer-wise weight quantizer for NVIDIA B200 -- Python binding.

Every function named ``gptq_*`` here marshals torch tensors into the C entry
point of the same name in ``libgptq_b200.so`` (declared in include/gptq.h)
and raises ``GptqError`` on a non-OK status.  All the arithmetic runs in the
library's CUDA kernels; PyTorch only provides device memory and streams.

``quantize_linear`` chains the calls for one linear layer, the way the page
"GPTQ, with the code open" describes the method: H from the calibration
inputs, the Cholesky factor of the damped inverse, the column sweep, packed
codes.
"""
from __future__ import annotations

import ctypes
import dataclasses

import torch

from . import _lib
from ._lib import (GPTQ_BF16, GPTQ_F32, GPTQ_OP_CHOLESKY, GPTQ_OP_DEQUANT_MATVEC, GPTQ_OP_HESSIAN,
                   GPTQ_OP_QUANTIZE, GptqConfig)

__all__ = ["GptqError", "GptqConfig", "LayerPipeline", "gptq_workspace_size",
           "gptq_hadamard_rows", "gptq_hadamard_cols", "gptq_hessian_accumulate",
           "gptq_cholesky_inverse", "gptq_quantize_layer", "gptq_pack_int4", "gptq_pack_int3",
           "gptq_dequant", "gptq_dequant_matvec", "gptq_gather_columns_u8", "gptq_status_string",
           "make_config", "gptq_set_wait_gate", "gptq_launch_count",
           "QuantizedLinear",
           "quantize_linear", "LayerQuantizer", "library"]


class GptqError(RuntimeError):
    pass


def library() -> ctypes.CDLL:
    return _lib.load()


def debug_library() -> ctypes.CDLL:
    """libgptq_b200_debug.so: the same entry points with device-side checks
    of caller-supplied indices (build it with ``build(debug=True)``)."""
    return _lib.load(_lib.DEBUG_LIB_PATH)


def gptq_device_checks(lib: ctypes.CDLL | None = None) -> int:
    """The index checks that failed since the last read, as a bit set (1: a
    group index out of range, 2: a permutation entry out of range), then
    cleared; waits for the device.  Debug library only."""
    lib = debug_library() if lib is None else lib
    flags = ctypes.c_uint32(0)
    _check(lib.gptq_device_checks(ctypes.byref(flags)), "gptq_device_checks")
    return int(flags.value)


def gptq_status_string(status: int) -> str:
    return library().gptq_status_string(int(status)).decode()


def gptq_launch_count() -> int:
    """Kernels the library has enqueued in this process so far."""
    return int(library().gptq_launch_count())


def gptq_set_wait_gate(gate: torch.Tensor | None, limit_ns: int = 1_000_000_000) -> None:
    """Test hook of the bounded device waits (see include/gptq.h): with a
    device int32 ``gate`` holding 0, the tensor-core kernels this thread
    enqueues next wait for it and give up after ``limit_ns``; None restores
    the normal behaviour."""
    if gate is not None:
        _need_cuda(gate)
        if gate.dtype != torch.int32:
            raise GptqError("gate must be a device int32 tensor")
    _check(library().gptq_set_wait_gate(_p(gate), int(limit_ns)), "gptq_set_wait_gate")


def _check(status: int, what: str) -> None:
    if status != 0:
        raise GptqError(f"{what}: {gptq_status_string(status)} (status {status})")


def _p(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _side(side_stream) -> int | None:
    """A second stream for look-ahead, or None (one stream)."""
    return None if side_stream is None else side_stream.cuda_stream


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return GPTQ_BF16
    if dt == torch.float32:
        return GPTQ_F32
    raise GptqError(f"unsupported dtype {dt} (bf16 or fp32)")


def _need_cuda(*ts) -> None:
    for t in ts:
        if t is not None and not t.is_cuda:
            raise GptqError("tensors must live on the GPU")


def make_config(bits=4, group_size=128, percdamp=0.01, actorder=False, block=128,
                sym=False) -> GptqConfig:
    return GptqConfig(int(bits), int(group_size), float(percdamp), int(block), int(bool(actorder)),
                      int(bool(sym)))


def gptq_workspace_size(op: int, rows: int, n: int, ntok: int = 0,
                        xdtype: torch.dtype = torch.bfloat16, cfg: GptqConfig | None = None) -> int:
    out = ctypes.c_size_t(0)
    st = library().gptq_workspace_size(int(op), int(rows), int(n), int(ntok), _dtype_code(xdtype),
                                       ctypes.byref(cfg) if cfg is not None else None,
                                       ctypes.byref(out))
    _check(st, "gptq_workspace_size")
    return int(out.value)


def _workspace(nbytes: int, device, ws):
    if nbytes == 0:
        return ws
    if ws is not None and ws.numel() >= nbytes:
        return ws
    return torch.empty(nbytes + 256, dtype=torch.uint8, device=device)


def _aligned_ptr(ws) -> tuple[int | None, int]:
    if ws is None:
        return None, 0
    p = ws.data_ptr()
    off = (-p) % 256
    return p + off, ws.numel() - off


def gptq_hessian_accumulate(H: torch.Tensor, X: torch.Tensor, alpha: float = 2.0, ws=None,
                            info: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """H += alpha * X X^T for X (n features x N tokens, bf16 or fp32); returns H."""
    _need_cuda(H, X, info)
    n, ntok = X.shape
    if H.dtype != torch.float32 or H.shape != (n, n) or not H.is_contiguous():
        raise GptqError("H must be a contiguous n x n float32 tensor")
    if X.stride(1) != 1:
        raise GptqError("X must have contiguous rows (tokens)")
    need = gptq_workspace_size(GPTQ_OP_HESSIAN, 0, n, ntok, X.dtype)
    ws = _workspace(need, X.device, ws)
    wp, wn = _aligned_ptr(ws)
    st = library().gptq_hessian_accumulate(_p(H), _p(X), _dtype_code(X.dtype), n, ntok,
                                           X.stride(0), 0, float(alpha), wp, wn, _p(info),
                                           _stream(stream))
    _check(st, "gptq_hessian_accumulate")
    return H


def gptq_cholesky_inverse(H: torch.Tensor, percdamp: float = 0.01, actorder: bool = False,
                          U=None, perm=None, dead=None, info=None, ws=None, stream=None,
                          side_stream=None):
    """Dead inputs, act-order, damping and U (upper, H'^-1 = U^T U).
    Returns (U, perm, dead, info); info is a device int32 (0 = success).
    side_stream: a second torch.cuda.Stream for the look-ahead (same result)."""
    _need_cuda(H)
    n = H.shape[0]
    dev = H.device
    U = torch.empty(n, n, dtype=torch.float32, device=dev) if U is None else U
    perm = torch.empty(n, dtype=torch.int32, device=dev) if perm is None else perm
    dead = torch.empty(n, dtype=torch.uint8, device=dev) if dead is None else dead
    info = torch.empty(1, dtype=torch.int32, device=dev) if info is None else info
    need = gptq_workspace_size(GPTQ_OP_CHOLESKY, 0, n)
    ws = _workspace(need, dev, ws)
    wp, wn = _aligned_ptr(ws)
    st = library().gptq_cholesky_inverse(_p(H), n, float(percdamp), int(bool(actorder)), _p(U),
                                         _p(perm), _p(dead), _p(info), wp, wn, _stream(stream),
                                         _side(side_stream))
    _check(st, "gptq_cholesky_inverse")
    return U, perm, dead, info


def gptq_cholesky_inverse_noalloc(H: torch.Tensor, percdamp: float, actorder: bool, U, perm,
                                  dead, info, stream=None):
    """gptq_cholesky_inverse for callers that cannot allocate device memory:
    every output buffer is the caller's and the scratch is built into the
    library (n <= 2048).  Nothing is allocated here either."""
    _need_cuda(H, U, perm, dead, info)
    n = H.shape[0]
    st = library().gptq_cholesky_inverse_noalloc(_p(H), n, float(percdamp), int(bool(actorder)),
                                                 _p(U), _p(perm), _p(dead), _p(info),
                                                 _stream(stream))
    _check(st, "gptq_cholesky_inverse_noalloc")
    return U, perm, dead, info


def gptq_quantize_layer(W: torch.Tensor, U: torch.Tensor, perm, dead, cfg: GptqConfig,
                        codes=None, scales=None, zeros=None, g_idx=None, Wq=None, row_loss=None,
                        want_g_idx: bool = True, want_wq: bool = False, want_loss: bool = False,
                        ws=None, info=None, stream=None, side_stream=None) -> dict:
    """The column sweep.  Returns dict(codes, scales, zeros, g_idx, Wq, row_loss).
    info: optional device int32 (set to 0, or -2 if a device wait gave up);
    side_stream: a second torch.cuda.Stream for the look-ahead (same result)."""
    _need_cuda(W, U, perm, dead)
    rows, n = W.shape
    if not W.is_contiguous():
        raise GptqError("W must be contiguous")
    dev = W.device
    G = 1 if cfg.group_size <= 0 else (n + cfg.group_size - 1) // cfg.group_size
    codes = torch.empty(rows, n, dtype=torch.uint8, device=dev) if codes is None else codes
    scales = torch.empty(rows, G, dtype=torch.float32, device=dev) if scales is None else scales
    zeros = torch.empty(rows, G, dtype=torch.uint8, device=dev) if zeros is None else zeros
    if g_idx is None and want_g_idx:
        g_idx = torch.empty(n, dtype=torch.int32, device=dev)
    if Wq is None and want_wq:
        Wq = torch.empty(rows, n, dtype=torch.float32, device=dev)
    if row_loss is None and want_loss:
        row_loss = torch.empty(rows, dtype=torch.float32, device=dev)
    need = gptq_workspace_size(GPTQ_OP_QUANTIZE, rows, n, 0, torch.bfloat16, cfg)
    ws = _workspace(need, dev, ws)
    wp, wn = _aligned_ptr(ws)
    st = library().gptq_quantize_layer(_p(W), _dtype_code(W.dtype), rows, n, _p(U), _p(perm),
                                       _p(dead), ctypes.byref(cfg), _p(codes), _p(scales),
                                       _p(zeros), _p(g_idx), _p(Wq), _p(row_loss), wp, wn,
                                       _p(info), _stream(stream), _side(side_stream))
    _check(st, "gptq_quantize_layer")
    return {"codes": codes, "scales": scales, "zeros": zeros, "g_idx": g_idx, "Wq": Wq,
            "row_loss": row_loss}


def gptq_pack_int4(codes: torch.Tensor, out=None, stream=None) -> torch.Tensor:
    _need_cuda(codes)
    rows, n = codes.shape
    out = torch.empty(rows, n // 8, dtype=torch.int32, device=codes.device) if out is None else out
    _check(library().gptq_pack_int4(_p(codes), rows, n, _p(out), _stream(stream)),
           "gptq_pack_int4")
    return out


def gptq_pack_int3(codes: torch.Tensor, out=None, stream=None) -> torch.Tensor:
    _need_cuda(codes)
    rows, n = codes.shape
    out = (torch.empty(rows, 3 * n // 32, dtype=torch.int32, device=codes.device)
           if out is None else out)
    _check(library().gptq_pack_int3(_p(codes), rows, n, _p(out), _stream(stream)),
           "gptq_pack_int3")
    return out


def gptq_dequant(packed: torch.Tensor, bits: int, n: int, scales: torch.Tensor,
                 zeros: torch.Tensor, group_size: int = -1, g_idx=None,
                 out_dtype: torch.dtype = torch.float32, out=None, stream=None) -> torch.Tensor:
    _need_cuda(packed, scales, zeros, g_idx)
    rows = packed.shape[0]
    out = torch.empty(rows, n, dtype=out_dtype, device=packed.device) if out is None else out
    st = library().gptq_dequant(_p(packed), int(bits), rows, int(n), _p(scales), _p(zeros),
                                int(group_size), scales.shape[1], _p(g_idx), _p(out),
                                _dtype_code(out.dtype), _stream(stream))
    _check(st, "gptq_dequant")
    return out


def gptq_gather_columns_u8(src: torch.Tensor, perm: torch.Tensor, out=None,
                           stream=None) -> torch.Tensor:
    """out[r][k] = src[r][perm[k]] (uint8 rows x n): codes into sweep order."""
    _need_cuda(src, perm)
    rows, n = src.shape
    out = torch.empty_like(src) if out is None else out
    _check(library().gptq_gather_columns_u8(_p(src), rows, n, _p(perm), _p(out), _stream(stream)),
           "gptq_gather_columns_u8")
    return out


def gptq_dequant_matvec(packed: torch.Tensor, bits: int, n: int, scales: torch.Tensor,
                        zeros: torch.Tensor, x: torch.Tensor, group_size: int = -1, g_idx=None,
                        perm=None, out=None, ws=None, stream=None) -> torch.Tensor:
    """y = x w_hat^T with w_hat dequantized on the fly from the packed codes.
    x: (batch, n) or (n,) bf16/fp32 on the GPU; returns (batch, rows) fp32
    (or (rows,) for a 1-D x).  perm: the codes are packed in sweep order
    (see gptq_gather_columns_u8) and column k multiplies x[perm[k]]."""
    _need_cuda(packed, scales, zeros, g_idx, perm, x)
    rows = packed.shape[0]
    x2 = x.reshape(1, -1) if x.dim() == 1 else x
    if x2.shape[1] != n or not x2.is_contiguous():
        raise GptqError("x must be a contiguous (batch, n) tensor")
    batch = x2.shape[0]
    out = torch.empty(batch, rows, dtype=torch.float32, device=packed.device) if out is None else out
    need = gptq_workspace_size(GPTQ_OP_DEQUANT_MATVEC, batch, n)
    ws = _workspace(need, packed.device, ws)
    wp, wn = _aligned_ptr(ws)
    st = library().gptq_dequant_matvec(_p(packed), int(bits), rows, int(n), _p(scales), _p(zeros),
                                       int(group_size), scales.shape[1], _p(g_idx), _p(perm),
                                       _p(x2), _dtype_code(x2.dtype), batch, _p(out), wp, wn,
                                       _stream(stream))
    _check(st, "gptq_dequant_matvec")
    return out.reshape(-1) if x.dim() == 1 else out


def _hadamard(cols: bool, x: torch.Tensor, signs: torch.Tensor, block: int, out, out_dtype,
              stream):
    _need_cuda(x, signs)
    if x.dim() != 2 or x.stride(1) != 1:
        raise GptqError("x must be a 2-D tensor with contiguous rows")
    if signs.dtype != torch.float32 or not signs.is_contiguous():
        raise GptqError("signs must be a contiguous float32 tensor")
    a, b = x.shape
    if out is None:
        out = torch.empty(a, b, dtype=out_dtype or x.dtype, device=x.device)
    if out.dim() != 2 or out.shape != x.shape or out.stride(1) != 1:
        raise GptqError("out must match x, with contiguous rows")
    fn = library().gptq_hadamard_cols if cols else library().gptq_hadamard_rows
    st = fn(_p(x), _dtype_code(x.dtype), a, b, x.stride(0), _p(signs), int(block), _p(out),
            _dtype_code(out.dtype), out.stride(0), _stream(stream))
    _check(st, "gptq_hadamard_cols" if cols else "gptq_hadamard_rows")
    return out


def gptq_hadamard_rows(W: torch.Tensor, signs: torch.Tensor, block: int = 1024, out=None,
                       out_dtype=None, stream=None) -> torch.Tensor:
    """W' = W R^T with R = blockdiag(H_b / sqrt(b)) diag(signs), along the rows
    of W (rows x n).  out may be W itself (in place)."""
    return _hadamard(False, W, signs, block, out, out_dtype, stream)


def gptq_hadamard_cols(X: torch.Tensor, signs: torch.Tensor, block: int = 1024, out=None,
                       out_dtype=None, stream=None) -> torch.Tensor:
    """X' = R X along the first axis of X (n x ntok).  out may be X itself."""
    return _hadamard(True, X, signs, block, out, out_dtype, stream)


@dataclasses.dataclass
class QuantizedLinear:
    packed: torch.Tensor
    scales: torch.Tensor
    zeros: torch.Tensor
    g_idx: torch.Tensor | None
    perm: torch.Tensor
    bits: int
    group_size: int
    n: int
    codes: torch.Tensor
    info: torch.Tensor
    H: torch.Tensor | None = None
    U: torch.Tensor | None = None
    Wq: torch.Tensor | None = None
    row_loss: torch.Tensor | None = None


def quantize_linear(W: torch.Tensor, X=None, H: torch.Tensor | None = None, bits: int = 4,
                    group_size: int = 128, percdamp: float = 0.01, actorder: bool = False,
                    alpha: float = 2.0, want_wq: bool = False, want_loss: bool = False,
                    keep_factors: bool = False, sym: bool = False,
                    stream=None) -> QuantizedLinear:
    """GPTQ for one linear layer W (rows x n).  X: one calibration tensor
    (n x N) or an iterable of batches; or pass a ready Hessian H."""
    _need_cuda(W)
    rows, n = W.shape
    if H is None:
        if X is None:
            raise GptqError("give calibration inputs X or a Hessian H")
        H = torch.zeros(n, n, dtype=torch.float32, device=W.device)
        batches = [X] if isinstance(X, torch.Tensor) else X
        for xb in batches:
            gptq_hessian_accumulate(H, xb, alpha, stream=stream)
    cfg = make_config(bits, group_size, percdamp, actorder, sym=sym)
    U, perm, dead, info = gptq_cholesky_inverse(H, percdamp, actorder, stream=stream)
    q = gptq_quantize_layer(W, U, perm, dead, cfg, want_wq=want_wq, want_loss=want_loss,
                            stream=stream)
    if bits == 4 and n % 8 == 0:
        packed = gptq_pack_int4(q["codes"], stream=stream)
    elif bits == 3 and n % 32 == 0:
        packed = gptq_pack_int3(q["codes"], stream=stream)
    else:
        packed = q["codes"]
    return QuantizedLinear(packed, q["scales"], q["zeros"], q["g_idx"], perm, bits, group_size, n,
                           q["codes"], info, H if keep_factors else None,
                           U if keep_factors else None, q["Wq"], q["row_loss"])


class LayerQuantizer:
    """Repeated GPTQ of one layer shape with every buffer allocated once.

    ``run(W, X)`` enqueues the whole hot path on one stream, in order:
    H = 0, H += 2 X X^T, dead inputs / act-order / damping / U, the column
    sweep, packing, and dequantization to ``out_dtype``.  Outputs stay in the
    attributes (``H``, ``U``, ``perm``, ``dead``, ``info``, ``codes``,
    ``scales``, ``zeros``, ``g_idx``, ``packed``, ``deq`` and, if asked for,
    ``Wq`` and ``row_loss``).  ``events``: six CUDA events recorded around the
    five stages, for timing.  ``side``: the quantizer's own second stream,
    given to the factorisation and the sweep for their look-ahead
    (``lookahead=False``: everything on the caller's stream; same results).
    """

    STAGES = ("hessian", "cholesky_inverse", "sweep", "pack", "dequant")

    def __init__(self, rows: int, n: int, ntok: int, bits: int = 4, group_size: int = 128,
                 percdamp: float = 0.01, actorder: bool = False,
                 x_dtype: torch.dtype = torch.bfloat16, w_dtype: torch.dtype = torch.bfloat16,
                 out_dtype: torch.dtype = torch.bfloat16, want_wq: bool = False,
                 want_loss: bool = False, sym: bool = False, device=None,
                 lookahead: bool = True):
        if bits == 4 and n % 8:
            raise GptqError("int4 packing needs n % 8 == 0")
        if bits == 3 and n % 32:
            raise GptqError("int3 packing needs n % 32 == 0")
        if bits not in (3, 4):
            raise GptqError("packed storage is int3 or int4")
        dev = torch.device("cuda") if device is None else torch.device(device)
        self.rows, self.n, self.ntok, self.bits = rows, n, ntok, bits
        self.group_size, self.percdamp, self.actorder = group_size, percdamp, actorder
        self.cfg = make_config(bits, group_size, percdamp, actorder, sym=sym)
        G = 1 if group_size <= 0 else (n + group_size - 1) // group_size
        f32 = torch.float32
        self.H = torch.empty(n, n, dtype=f32, device=dev)
        self.U = torch.empty(n, n, dtype=f32, device=dev)
        self.perm = torch.empty(n, dtype=torch.int32, device=dev)
        self.dead = torch.empty(n, dtype=torch.uint8, device=dev)
        self.info = torch.zeros(1, dtype=torch.int32, device=dev)
        self.info_h = torch.zeros(1, dtype=torch.int32, device=dev)
        self.info_q = torch.zeros(1, dtype=torch.int32, device=dev)
        self.side = torch.cuda.Stream(dev) if lookahead else None
        self.codes = torch.empty(rows, n, dtype=torch.uint8, device=dev)
        self.scales = torch.empty(rows, G, dtype=f32, device=dev)
        self.zeros = torch.empty(rows, G, dtype=torch.uint8, device=dev)
        self.g_idx = torch.empty(n, dtype=torch.int32, device=dev)
        self.packed = torch.empty(rows, n * bits // 32, dtype=torch.int32, device=dev)
        self.deq = torch.empty(rows, n, dtype=out_dtype, device=dev)
        self.Wq = torch.empty(rows, n, dtype=f32, device=dev) if want_wq else None
        self.row_loss = torch.empty(rows, dtype=f32, device=dev) if want_loss else None
        self.ws_h = _workspace(gptq_workspace_size(GPTQ_OP_HESSIAN, 0, n, ntok, x_dtype), dev,
                               None)
        self.ws_c = _workspace(gptq_workspace_size(GPTQ_OP_CHOLESKY, 0, n), dev, None)
        self.ws_q = _workspace(gptq_workspace_size(GPTQ_OP_QUANTIZE, rows, n, 0, w_dtype,
                                                   self.cfg), dev, None)
        self._pack = gptq_pack_int4 if bits == 4 else gptq_pack_int3
        self.x_dtype, self.w_dtype = x_dtype, w_dtype
        self._stage = None        # run_streamed: two device staging buffers, device W, events

    def hessian(self, X: torch.Tensor, stream, mark=None) -> None:
        """H = 0, H += 2 X X^T on `stream`; mark(0) / mark(1) around the
        accumulation."""
        with torch.cuda.stream(stream):
            self.H.zero_()
        if mark:
            mark(0)
        gptq_hessian_accumulate(self.H, X, 2.0, ws=self.ws_h, info=self.info_h, stream=stream)
        if mark:
            mark(1)

    def finish(self, W: torch.Tensor, stream, mark=None) -> None:
        """Everything after the Hessian, on `stream`: U, the sweep, packing,
        dequantization.  mark(i) is called after stage i (2..5)."""
        gptq_cholesky_inverse(self.H, self.percdamp, self.actorder, self.U, self.perm, self.dead,
                              self.info, ws=self.ws_c, stream=stream, side_stream=self.side)
        if mark:
            mark(2)
        gptq_quantize_layer(W, self.U, self.perm, self.dead, self.cfg, self.codes, self.scales,
                            self.zeros, self.g_idx, self.Wq, self.row_loss, ws=self.ws_q,
                            info=self.info_q, stream=stream, side_stream=self.side)
        if mark:
            mark(3)
        self._pack(self.codes, self.packed, stream=stream)
        if mark:
            mark(4)
        gptq_dequant(self.packed, self.bits, self.n, self.scales, self.zeros, self.group_size,
                     self.g_idx, self.deq.dtype, out=self.deq, stream=stream)
        if mark:
            mark(5)

    def run_streamed(self, W_host: torch.Tensor, X_batches, stream=None):
        """The whole layer from inputs in (pinned) host memory: W and the
        calibration batches X_b (each n x N_b, contiguous) are copied in on a
        copy stream while H accumulates batch by batch on ``stream`` (page
        "GPTQ, with the code open", section "Paper vs. code": H is a sum over
        calibration batches), so the host-to-device copies overlap the
        Hessian.  Two device staging buffers of the largest batch take turns;
        a buffer is refilled only after the accumulation that read it.  The
        result equals ``run`` on the concatenated X up to the fp32 order of
        the Hessian's sums.

        Consecutive calls overlap: a call's copies wait only for the last
        reads of the buffers they overwrite (a staging buffer's previous
        accumulation, the device W's previous sweep), so they can run while
        the previous call's factorisation and sweep finish.  The host
        tensors must stay alive and unchanged until the copies are done (for
        example until ``stream`` has reached this call's end)."""
        s = torch.cuda.current_stream() if stream is None else stream
        dev = self.H.device
        if len(X_batches) == 0:
            raise GptqError("no calibration batch")
        for Xb in X_batches:
            if Xb.dim() != 2 or Xb.shape[0] != self.n or not Xb.is_contiguous() \
                    or Xb.dtype != self.x_dtype:
                raise GptqError("each batch must be a contiguous n x N_b tensor of the layer's "
                                "input dtype")
        if W_host.shape != (self.rows, self.n) or W_host.dtype != self.w_dtype:
            raise GptqError("W must be rows x n in the layer's weight dtype")
        nb = max(int(Xb.shape[1]) for Xb in X_batches)
        st = self._stage
        if st is None or st["cap"] < nb:
            st = {"cap": nb,
                  "buf": [torch.empty(self.n * nb, dtype=self.x_dtype, device=dev)
                          for _ in range(2)],
                  "W": torch.empty(self.rows, self.n, dtype=self.w_dtype, device=dev),
                  "copy": torch.cuda.Stream(dev),
                  "ev_w": torch.cuda.Event(), "ev_w_free": torch.cuda.Event(),
                  "ev_copied": [torch.cuda.Event(), torch.cuda.Event()],
                  "ev_used": [torch.cuda.Event(), torch.cuda.Event()]}
            if self._stage is not None:
                # new buffers: the old ones may still be read on s
                ev = torch.cuda.Event()
                ev.record(s)
                st["copy"].wait_event(ev)
            self._stage = st
        cs = st["copy"]
        # each staging buffer is overwritten once the accumulation that read
        # it last is done, W once the previous call's sweep has read it
        # (events never recorded yet make these waits no-ops).  W goes after
        # the first two batches, so that the copy stream does not hold those
        # behind the previous call's sweep.
        with torch.cuda.stream(s):
            self.H.zero_()
        w_after = min(1, len(X_batches) - 1)
        for i, Xb in enumerate(X_batches):
            slot = i % 2
            cs.wait_event(st["ev_used"][slot])
            dst = st["buf"][slot][: self.n * Xb.shape[1]].view(self.n, Xb.shape[1])
            with torch.cuda.stream(cs):
                dst.copy_(Xb, non_blocking=True)
            st["ev_copied"][slot].record(cs)
            if i == w_after:
                cs.wait_event(st["ev_w_free"])
                with torch.cuda.stream(cs):
                    st["W"].copy_(W_host, non_blocking=True)
                st["ev_w"].record(cs)
            s.wait_event(st["ev_copied"][slot])
            gptq_hessian_accumulate(self.H, dst, 2.0, ws=self.ws_h, info=self.info_h, stream=s)
            st["ev_used"][slot].record(s)
        s.wait_event(st["ev_w"])
        self.finish(st["W"], s)
        st["ev_w_free"].record(s)
        return self

    def run(self, W: torch.Tensor, X: torch.Tensor, stream=None, events=None):
        s = torch.cuda.current_stream() if stream is None else stream
        ev = events

        def mark(i):
            if ev is not None:
                ev[i].record(s)

        self.hessian(X, s, mark)
        self.finish(W, s, mark)
        return self

    def check_info(self) -> None:
        """Raises GptqError if a device status word reports a failure (syncs)."""
        ci, hi, qi = int(self.info.item()), int(self.info_h.item()), int(self.info_q.item())
        if ci != 0 or hi != 0 or qi != 0:
            raise GptqError(f"device status: cholesky info {ci}, hessian info {hi}, "
                            f"sweep info {qi}")


class LayerPipeline:
    """GPTQ of a sequence of linears, one layer at a time (page "GPTQ, with
    the code open", section "From one repair to a whole model": each layer is
    repaired from its own inputs and Hessian), with the Hessian of linear
    l + 1 accumulating on one stream while linear l is factored, swept,
    packed and dequantized on another.  The Hessian is tensor-core bound and
    the rest a chain of small dependent launches, so the two overlap on the
    SMs the chain leaves idle.

    ``shapes``: (rows, n) per linear; every linear sees ``ntok`` tokens.
    One LayerQuantizer per linear holds that linear's buffers and outputs
    (``layers[l]``).  ``run(Ws, Xs)`` enqueues everything and makes the
    caller's stream wait for the last linear.

    Measured on a 7B decoder block (7 linears, 65536 tokens each) the overlap
    gains nothing (0.96 to 1.00 of the one-stream time): the Hessian's
    persistent grid holds every SM, so the factorisation's and the sweep's
    kernels only get SMs when it ends.  So ``run`` uses the one-stream order
    unless ``overlap=True`` is asked for.
    """

    def __init__(self, shapes, ntok: int, bits: int = 4, group_size: int = 128,
                 percdamp: float = 0.01, actorder: bool = False, sym: bool = False,
                 x_dtype: torch.dtype = torch.bfloat16, w_dtype: torch.dtype = torch.bfloat16,
                 out_dtype: torch.dtype = torch.bfloat16, want_wq: bool = False,
                 want_loss: bool = False, device=None):
        dev = torch.device("cuda") if device is None else torch.device(device)
        self.layers = [LayerQuantizer(rows, n, ntok, bits, group_size, percdamp, actorder,
                                      x_dtype, w_dtype, out_dtype, want_wq, want_loss, sym=sym,
                                      device=dev)
                       for rows, n in shapes]
        self.s_h = torch.cuda.Stream(dev)
        self.s_q = torch.cuda.Stream(dev)
        self.ev_h = [torch.cuda.Event() for _ in shapes]
        self.ev_start = torch.cuda.Event()
        self.ev_done = torch.cuda.Event()

    def run(self, Ws, Xs, stream=None, overlap: bool = False):
        """overlap=False (the default) runs the work one linear after another
        on the caller's stream; overlap=True puts each next Hessian on a
        second stream (same results)."""
        s = torch.cuda.current_stream() if stream is None else stream
        if len(Ws) != len(self.layers) or len(Xs) != len(self.layers):
            raise GptqError("one W and one X per linear")
        if not overlap:
            for q, W, X in zip(self.layers, Ws, Xs):
                q.hessian(X, s)
                q.finish(W, s)
            return self
        self.ev_start.record(s)
        self.s_h.wait_event(self.ev_start)
        self.s_q.wait_event(self.ev_start)
        L = len(self.layers)
        for l in range(L + 1):
            if l < L:
                self.layers[l].hessian(Xs[l], self.s_h)
                self.ev_h[l].record(self.s_h)
            if l >= 1:
                self.s_q.wait_event(self.ev_h[l - 1])
                self.layers[l - 1].finish(Ws[l - 1], self.s_q)
        self.ev_done.record(self.s_q)
        s.wait_event(self.ev_done)
        return self

    def check_info(self) -> None:
        for q in self.layers:
            q.check_info()


# ----------------------------------------------------------------- checkpoint / resume
# Page "GPTQ, with the code open", section "From one repair to a whole model":
# a model is quantized one layer at a time, each from its own inputs.  For a
# long run over many linears, each finished linear's stored result is written
# to its own file, and a restarted run skips the linears whose files exist.

STORED_KEYS = ("packed", "scales", "zeros", "g_idx", "perm")


def save_quantized(path: str, outputs: dict, meta: dict) -> None:
    """Write one linear's stored result (host copies of ``STORED_KEYS`` and
    ``meta``) to ``path``.  The file appears only once it is complete: it is
    written under a temporary name and renamed, so an interrupted run leaves
    no partial result that a resumed run would take for a finished one."""
    import os
    blob = {k: outputs[k].detach().cpu() for k in STORED_KEYS if outputs.get(k) is not None}
    blob["meta"] = dict(meta)
    tmp = path + ".partial"
    torch.save(blob, tmp)
    os.replace(tmp, path)


def load_quantized(path: str) -> dict:
    return torch.load(path, map_location="cpu", weights_only=True)


def quantize_linears(names, quantize, out_dir: str, resume: bool = True) -> list:
    """Quantize the linears ``names`` in order with ``quantize(name) ->
    (outputs, meta)`` (``outputs`` holds at least ``packed``, ``scales`` and
    ``zeros`` of that linear), storing each under ``out_dir/<name>.pt``.  With
    ``resume``, a linear whose file already exists is not quantized again.
    Returns the names quantized by this call."""
    import os
    os.makedirs(out_dir, exist_ok=True)
    done = []
    for name in names:
        path = os.path.join(out_dir, f"{name}.pt")
        if resume and os.path.exists(path):
            continue
        outputs, meta = quantize(name)
        save_quantized(path, outputs, meta)
        done.append(name)
    return done


def layer_quantizer_outputs(lq: "LayerQuantizer") -> tuple:
    """(outputs, meta) of a LayerQuantizer after ``run``, for
    quantize_linears: checks ``info`` first (a failed linear is not stored)."""
    lq.check_info()
    outputs = {"packed": lq.packed, "scales": lq.scales, "zeros": lq.zeros,
               "g_idx": lq.g_idx if lq.actorder else None,
               "perm": lq.perm if lq.actorder else None}
    meta = {"rows": lq.rows, "n": lq.n, "bits": lq.bits, "group_size": lq.group_size,
            "actorder": bool(lq.actorder), "percdamp": lq.percdamp}
    return outputs, meta
