"""gptq_cholesky_inverse_noalloc: the factorisation for callers that cannot
allocate device memory (a host program that owns all device memory in a fixed
pool and forbids allocation while it runs).  Its scratch is built into the
library, so it must give the same U / perm / dead / info as the workspace
entry point, call after call, while the shared scratch keeps the previous
call's contents.

This file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import post_weight_quantization_25_b200 as G
import workloads
from oracle import gptq_oracle as O

pytestmark = pytest.mark.gpu


def _spd(n, seed):
    _, X = workloads.random_layer(1, n, 2 * n + 64, seed=seed, correlated=0.3,
                                  dead=(n // 3,))
    return torch.from_numpy(O.hessian(X.double().numpy()).astype(np.float32)).cuda()


def _buffers(n):
    return (torch.empty(n, n, dtype=torch.float32, device="cuda"),
            torch.empty(n, dtype=torch.int32, device="cuda"),
            torch.empty(n, dtype=torch.uint8, device="cuda"),
            torch.empty(1, dtype=torch.int32, device="cuda"))


def _noalloc(H, actorder):
    lib = G.library()
    n = H.shape[0]
    U, perm, dead, info = _buffers(n)
    st = lib.gptq_cholesky_inverse_noalloc(
        ctypes.c_void_p(H.data_ptr()), n, ctypes.c_float(0.01), int(actorder),
        ctypes.c_void_p(U.data_ptr()), ctypes.c_void_p(perm.data_ptr()),
        ctypes.c_void_p(dead.data_ptr()), ctypes.c_void_p(info.data_ptr()),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, G.gptq_status_string(st)
    return U, perm, dead, info


def test_noalloc_matches_workspace_entry_point_twice_in_a_row():
    cases = [(2048, True, 7), (300, True, 8), (640, False, 9)]
    for n, act, seed in cases:
        H = _spd(n, seed)
        U0, p0, d0, i0 = G.gptq_cholesky_inverse(H, 0.01, act)
        U1, p1, d1, i1 = _noalloc(H, act)
        torch.cuda.synchronize()
        assert int(i0.item()) == 0 and int(i1.item()) == 0
        assert torch.equal(p0, p1) and torch.equal(d0, d1)
        a, b = U0.double(), U1.double()
        assert float(torch.linalg.norm(a - b) / torch.linalg.norm(a)) <= 1e-4


def test_noalloc_rejects_sizes_past_its_scratch():
    lib = G.library()
    n = 2049
    H = torch.eye(n, device="cuda")
    U, perm, dead, info = _buffers(n)
    st = lib.gptq_cholesky_inverse_noalloc(
        ctypes.c_void_p(H.data_ptr()), n, ctypes.c_float(0.01), 1,
        ctypes.c_void_p(U.data_ptr()), ctypes.c_void_p(perm.data_ptr()),
        ctypes.c_void_p(dead.data_ptr()), ctypes.c_void_p(info.data_ptr()), None)
    assert st == 3          # GPTQ_ERR_WORKSPACE: larger than the built-in scratch
