"""Seeded synthetic inputs for the GPTQ layer quantizer.

This module only draws random tensors with the shapes and distributions of
the workloads below; it holds none of the quantizer's arithmetic, and both
the CUDA path's tests/benchmark and the CPU oracle's tests take their inputs
from it.  The oracle receives the exact bytes the GPU receives (bf16 values
widened exactly to fp32), so no random-number parity is needed between
devices.

Workloads (W is rows x n, X is n features x N tokens):

* ``layer256``   W 256x256 fp32 N(0, 0.02^2); X 256x2048 fp32 N(0,1);
  4-bit per-row ruler; damping 1 %; block 128; no act-order.
* ``q_proj_7b``  W 4096x4096 bf16 N(0, 0.02^2); X 4096x262144 bf16 N(0,1)
  (128 sequences x 2048 tokens) with 8 fixed outlier channels scaled x20;
  4-bit, group 128, act-order.
* ``down_proj_7b`` W 4096x11008 bf16 N(0, 0.015^2); X 11008x131072 bf16,
  0.5 * Student-t(3); 3-bit, group 128; damping 1 %; block 128.
* ``stack_7b``   32 blocks x {q,k,v,o 4096x4096; gate,up 11008x4096;
  down 4096x11008} bf16 N(0, 0.02^2), one seeded X of 65536 tokens N(0,1)
  per linear; 4-bit, group 128; layers in order.
* ``down_proj_70b`` W 8192x28672 bf16 N(0, 0.01^2); X 28672x65536 N(0,1)
  with round(0.001 n) outlier channels x50; W and X rotated by a random-sign
  normalised Hadamard in blocks of 1024 (computed in fp32, rounded to bf16);
  4-bit, group 128, act-order.

Seed of tensor t of workload c (1-based, in the order above): 1000 c + t,
t = 0 weights, 1 calibration inputs, 2 outlier channels, 3 rotation signs;
``stack_7b`` linear l of block b uses 4000 + 10 b + l + 100000 t.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int
    rows: int
    n: int
    ntok: int
    w_dtype: torch.dtype
    x_dtype: torch.dtype
    w_std: float
    bits: int
    group_size: int
    actorder: bool
    percdamp: float = 0.01
    block: int = 128
    x_kind: str = "normal"        # "normal" | "student_t3"
    x_scale: float = 1.0
    outliers: int = 0
    outlier_gain: float = 1.0
    hadamard_block: int = 0

    @property
    def weights(self) -> int:
        return self.rows * self.n


WORKLOADS = {
    "layer256": Workload("layer256", 1, 256, 256, 2048, torch.float32, torch.float32,
                         0.02, 4, -1, False),
    "q_proj_7b": Workload("q_proj_7b", 2, 4096, 4096, 262144, torch.bfloat16, torch.bfloat16,
                          0.02, 4, 128, True, outliers=8, outlier_gain=20.0),
    "down_proj_7b": Workload("down_proj_7b", 3, 4096, 11008, 131072, torch.bfloat16,
                             torch.bfloat16, 0.015, 3, 128, False, x_kind="student_t3",
                             x_scale=0.5),
    "down_proj_70b": Workload("down_proj_70b", 5, 8192, 28672, 65536, torch.bfloat16,
                              torch.bfloat16, 0.01, 4, 128, True, outliers=29,
                              outlier_gain=50.0, hadamard_block=1024),
}

# (name, rows, n) of the seven linears of one 7B decoder block
STACK_7B_LINEARS = (("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096),
                    ("o", 4096, 4096), ("gate", 11008, 4096), ("up", 11008, 4096),
                    ("down", 4096, 11008))


def stack_7b_workload(block: int, linear: int, ntok: int = 65536) -> Workload:
    name, rows, n = STACK_7B_LINEARS[linear]
    return Workload(f"stack_7b.b{block}.{name}", 4, rows, n, ntok, torch.bfloat16,
                    torch.bfloat16, 0.02, 4, 128, False)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _seed(wl: Workload, t: int) -> int:
    if wl.index == 4:
        b, lin = wl.name.split(".")[1:3]
        idx = [x[0] for x in STACK_7B_LINEARS].index(lin)
        return 4000 + 10 * int(b[1:]) + idx + 100000 * t
    return 1000 * wl.index + t


def make_weights(wl: Workload, device="cpu", rows: int | None = None) -> torch.Tensor:
    """W (rows x n) in the workload's dtype; ``rows`` takes the first rows only."""
    r = wl.rows if rows is None else rows
    g = _gen(_seed(wl, 0), device)
    W = torch.randn(wl.rows, wl.n, generator=g, device=device, dtype=torch.float32) * wl.w_std
    return W[:r].to(wl.w_dtype).contiguous()


def outlier_channels(wl: Workload, device="cpu") -> torch.Tensor:
    g = _gen(_seed(wl, 2), "cpu")
    return torch.randperm(wl.n, generator=g)[:wl.outliers].to(device)


def make_calibration(wl: Workload, device="cpu", ntok: int | None = None,
                     row_chunk: int = 1024) -> torch.Tensor:
    """X (n x N) in the workload's dtype, drawn row chunk by row chunk."""
    N = wl.ntok if ntok is None else ntok
    g = _gen(_seed(wl, 1), device)
    X = torch.empty(wl.n, N, device=device, dtype=wl.x_dtype)
    for r0 in range(0, wl.n, row_chunk):
        r1 = min(r0 + row_chunk, wl.n)
        if wl.x_kind == "normal":
            blk = torch.randn(r1 - r0, N, generator=g, device=device, dtype=torch.float32)
        elif wl.x_kind == "student_t3":
            z = torch.randn(r1 - r0, N, generator=g, device=device, dtype=torch.float32)
            chi = torch.zeros_like(z)
            for _ in range(3):
                chi += torch.randn(r1 - r0, N, generator=g, device=device,
                                   dtype=torch.float32) ** 2
            blk = z / torch.sqrt(chi / 3.0)
        else:
            raise ValueError(wl.x_kind)
        X[r0:r1] = (blk * wl.x_scale).to(wl.x_dtype)
    if wl.outliers:
        idx = outlier_channels(wl, device)
        X[idx] = (X[idx].float() * wl.outlier_gain).to(wl.x_dtype)
    return X


def hadamard_signs(wl: Workload, device="cpu") -> torch.Tensor:
    g = _gen(_seed(wl, 3), "cpu")
    return (torch.randint(0, 2, (wl.n,), generator=g) * 2 - 1).to(device, torch.float32)


def rotate_inputs(wl: Workload, W: torch.Tensor, X: torch.Tensor):
    """Random-sign normalised Hadamard rotation R = blockdiag(H_b / sqrt(b)) diag(s):
    X' = R X and W' = W R^T, computed in fp32 and rounded to the workload's
    dtypes.  This is input preparation for the workload, ahead of the
    quantizer."""
    b = wl.hadamard_block
    if not b:
        return W, X
    dev = X.device
    Hb = torch.ones(1, 1, device=dev)
    while Hb.shape[0] < b:
        Hb = torch.cat([torch.cat([Hb, Hb], 1), torch.cat([Hb, -Hb], 1)], 0)
    Hb = Hb / math.sqrt(b)
    s = hadamard_signs(wl, dev)
    nb = wl.n // b
    Xr = torch.empty_like(X)
    for i in range(nb):
        sl = slice(i * b, (i + 1) * b)
        Xr[sl] = (Hb @ (X[sl].float() * s[sl, None])).to(X.dtype)
    Wr = torch.empty_like(W)
    Wf = W.float()
    for i in range(nb):
        sl = slice(i * b, (i + 1) * b)
        Wr[:, sl] = ((Wf[:, sl] * s[None, sl]) @ Hb.T).to(W.dtype)
    return Wr, Xr


def make_inputs(wl: Workload, device="cpu", rows: int | None = None, ntok: int | None = None):
    W = make_weights(wl, device, rows)
    X = make_calibration(wl, device, ntok)
    if wl.hadamard_block:
        W, X = rotate_inputs(wl, W, X)
    return W, X


def identity_calibration(n: int, copies: int, gains=None, dtype=torch.bfloat16,
                         device="cpu") -> torch.Tensor:
    """X = diag(gains) [I I ... I] (n x copies*n): its Hessian is diagonal."""
    X = torch.eye(n, device=device, dtype=torch.float32).repeat(1, copies)
    if gains is not None:
        X = X * torch.as_tensor(gains, dtype=torch.float32, device=device)[:, None]
    return X.to(dtype)


def random_layer(rows: int, n: int, ntok: int, seed: int, w_std: float = 0.02,
                 dtype=torch.float32, device="cpu", dead=(), correlated: float = 0.0):
    """A small seeded layer for parity tests: W ~ N(0, w_std^2), X ~ N(0,1)
    (optionally mixed with a shared component so inputs correlate), with the
    listed input channels silenced."""
    g = _gen(seed, device)
    W = torch.randn(rows, n, generator=g, device=device) * w_std
    X = torch.randn(n, ntok, generator=g, device=device)
    if correlated:
        shared = torch.randn(1, ntok, generator=g, device=device)
        X = (1 - correlated) * X + correlated * shared
    for c in dead:
        X[c] = 0
    return W.to(dtype).contiguous(), X.to(dtype).contiguous()
