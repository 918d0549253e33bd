"""gptq_cholesky_inverse_noalloc: the factorisation for callers that cannot
allocate device memory (a host program that owns all device memory in a fixed
pool and forbids allocation while it runs).  Its scratch is an array built
into the library and shared by every call, so a call must not depend on what
the previous call left there.

The checks: two no-alloc calls in a row on different inputs (the larger one
first, so the scratch holds another problem's data when the second starts)
give bit for bit what the workspace entry point gives on the same inputs,
and one of them matches the fp64 oracle's factor.

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


@pytest.mark.parametrize("first,second", [((2048, True, 7), (300, True, 8)),
                                          ((1000, False, 9), (640, False, 10))])
def test_noalloc_twice_in_a_row_equals_workspace_entry_point(first, second):
    inputs = [(_spd(n, seed), act) for n, act, seed in (first, second)]
    # two calls back to back on the same stream: the second starts with the
    # first one's data in the shared scratch
    got = [_noalloc(H, act) for H, act in inputs]
    torch.cuda.synchronize()
    for (H, act), (U1, p1, d1, i1) in zip(inputs, got):
        U0, p0, d0, i0 = G.gptq_cholesky_inverse(H, 0.01, act)
        torch.cuda.synchronize()
        assert int(i0.item()) == 0 and int(i1.item()) == 0
        assert torch.equal(p0, p1) and torch.equal(d0, d1)
        assert torch.equal(U0, U1)
    # the second call's factor against the oracle's (the pages' route, fp64)
    H, act = inputs[1]
    U1, p1, _, _ = got[1]
    prep = O.prepare(H.cpu().double().numpy(), np.zeros((1, H.shape[0])), 0.01, act,
                     forced_perm=p1.cpu().numpy().astype(np.int64) if act else None)
    Uo = O.upper_cholesky_of_inverse(prep["Hp"])
    rel = np.linalg.norm(U1.cpu().double().numpy() - Uo) / np.linalg.norm(Uo)
    assert rel <= 1e-4, rel


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
