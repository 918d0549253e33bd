"""The rounding decision of the sweep, q = clamp(rint(w / scale) + zero),
must be taken exactly as binary32 IEEE division would take it (the pages'
implementation runs in full fp32; the oracle takes the decision in binary32).

The sweep computes w / scale with Markstein's FMA division and a reciprocal
of the scale computed once per ruler; these tests check that primitive bit
for bit against IEEE division, and the end-to-end codes on weights placed on
and next to the half-integer rounding boundaries.
"""
import ctypes

import numpy as np
import pytest
import torch

import post_weight_quantization_25_b200 as G
import workloads
from oracle import gptq_oracle as O

pytestmark = pytest.mark.gpu


def _gpu_div(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    ad = torch.from_numpy(a.astype(np.float32)).cuda()
    bd = torch.from_numpy(b.astype(np.float32)).cuda()
    out = torch.empty_like(ad)
    st = G.library().gptq_selftest_division(ctypes.c_void_p(ad.data_ptr()),
                                            ctypes.c_void_p(bd.data_ptr()), ad.numel(),
                                            ctypes.c_void_p(out.data_ptr()), None)
    assert st == 0
    torch.cuda.synchronize()
    return out.cpu().numpy()


def _check(a, b):
    a = a.astype(np.float32)
    b = b.astype(np.float32)
    got = _gpu_div(a, b)
    ref = (a / b).astype(np.float32)  # numpy binary32 division: IEEE round to nearest
    bad = ~((got == ref) | (np.isnan(got) & np.isnan(ref)))
    assert not bad.any(), (a[bad][:5], b[bad][:5], got[bad][:5], ref[bad][:5])


def test_division_random_pairs():
    rng = np.random.default_rng(2024)
    m = 1 << 22
    a = (rng.choice([-1.0, 1.0], m) * 10.0 ** rng.uniform(-9, 3, m)).astype(np.float32)
    b = (10.0 ** rng.uniform(-8, 1, m)).astype(np.float32)
    _check(a, b)
    # random bit patterns over whole binades of the divisor
    bb = rng.integers(0x30000000, 0x42000000, m, dtype=np.uint32).view(np.float32)
    aa = (rng.standard_normal(m) * 0.05).astype(np.float32)
    _check(aa, bb)


def test_division_near_half_integers():
    rng = np.random.default_rng(7)
    m = 1 << 20
    b = (10.0 ** rng.uniform(-6, 0, m)).astype(np.float32)
    k = rng.integers(-300, 300, m).astype(np.float32)
    a0 = ((k + np.float32(0.5)) * b).astype(np.float32)
    for steps in (-3, -2, -1, 0, 1, 2, 3):
        a = a0.copy()
        direction = np.float32(np.inf) if steps > 0 else np.float32(-np.inf)
        for _ in range(abs(steps)):
            a = np.nextafter(a, direction).astype(np.float32)
        _check(a, b)


def test_division_extreme_divisors():
    rng = np.random.default_rng(3)
    m = 1 << 16
    for lo, hi in ((1e-38, 1e-30), (1e-25, 1e-18), (1e18, 1e25)):
        b = (10.0 ** rng.uniform(np.log10(lo), np.log10(hi), m)).astype(np.float32)
        a = (b * rng.uniform(-300, 300, m)).astype(np.float32)
        _check(a, b)
    _check(np.zeros(8, np.float32), np.full(8, 0.25, np.float32))


@pytest.mark.parametrize("bits,g", [(4, -1), (3, 128), (4, 32)])
def test_codes_on_rounding_boundaries_match_oracle(bits, g):
    """H is diagonal, so GPTQ is round-to-nearest; weights sit on and within
    three ulps of the half-integer boundaries of their ruler.  The GPU codes
    must equal the oracle's binary32 decisions exactly."""
    rng = np.random.default_rng(11 + bits + max(g, 0))
    rows, n = 48, 256
    maxq = 2 ** bits - 1
    W = np.zeros((rows, n), dtype=np.float32)
    gs = n if g <= 0 else g
    for r in range(rows):
        for g0 in range(0, n, gs):
            lo = np.float32(-rng.uniform(0.01, 0.05))
            hi = np.float32(rng.uniform(0.01, 0.05))
            scale, zero = O.fit_grid(lo, hi, bits)
            k = rng.integers(0, maxq, gs - 2).astype(np.float32)
            vals = ((k - np.float32(zero) + np.float32(0.5)) * scale).astype(np.float32)
            shift = rng.integers(-3, 4, gs - 2)
            for i in range(gs - 2):
                d = np.float32(np.inf) if shift[i] > 0 else np.float32(-np.inf)
                for _ in range(abs(int(shift[i]))):
                    vals[i] = np.nextafter(vals[i], d)
            vals = np.clip(vals, lo, hi)
            W[r, g0:g0 + gs] = np.concatenate([[lo, hi], vals])
    X = workloads.identity_calibration(n, 2, dtype=torch.bfloat16)
    Wt = torch.from_numpy(W).cuda()
    H = torch.zeros(n, n, device="cuda")
    G.gptq_hessian_accumulate(H, X.cuda())
    cfg = G.make_config(bits, g, 0.01, False)
    U, perm, dead, info = G.gptq_cholesky_inverse(H, 0.01, False)
    q = G.gptq_quantize_layer(Wt, U, perm, dead, cfg)
    torch.cuda.synchronize()
    ref = O.rtn(W.astype(np.float64), bits, g)
    assert np.array_equal(q["codes"].cpu().numpy().astype(np.int64), ref["codes"])
    assert np.array_equal(q["scales"].cpu().numpy(), ref["scales"])
