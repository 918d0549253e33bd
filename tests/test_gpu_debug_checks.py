"""The debug build (libgptq_b200_debug.so, device-side index checks).

Kernels that index with caller-supplied group indices or permutations test
each index first in this build: an index out of range is not used, its
outputs are left 0 (or undefined where documented), and gptq_device_checks
reports which kind of check failed.  Every out-of-range index below is
caught by those checks before any memory access, so nothing here reads or
writes outside a buffer.  Clean calls report nothing and give the release
library's results bit for bit.

The binding's calls are routed to the debug library for the duration of
each test.
"""
import numpy as np
import pytest
import torch

import post_weight_quantization_25_b200 as G
from post_weight_quantization_25_b200 import _lib

pytestmark = pytest.mark.gpu


@pytest.fixture
def debug_lib():
    import os
    if not os.path.exists(_lib.DEBUG_LIB_PATH):
        from post_weight_quantization_25_b200 import build
        build.build(debug=True)
    release = _lib.load()
    dbg = _lib.load(_lib.DEBUG_LIB_PATH)
    _lib._LIB = dbg
    try:
        assert G.gptq_device_checks(dbg) == 0
        yield dbg
    finally:
        torch.cuda.synchronize()
        _lib._LIB = release


def _codes(rows, n, bits, G_, seed):
    rng = np.random.default_rng(seed)
    codes = torch.from_numpy(rng.integers(0, 2 ** bits, (rows, n)).astype(np.uint8)).cuda()
    scales = torch.from_numpy(rng.uniform(1e-3, 0.1, (rows, G_)).astype(np.float32)).cuda()
    zeros = torch.from_numpy(rng.integers(0, 2 ** bits, (rows, G_)).astype(np.uint8)).cuda()
    return codes, scales, zeros


@pytest.mark.parametrize("bits,out_dtype,offset", [(4, torch.bfloat16, 0), (3, torch.float32, 0),
                                                   (4, torch.float32, 1)])
def test_dequant_reports_group_indices_out_of_range(debug_lib, bits, out_dtype, offset):
    """One CTA per row (aligned output) and one thread per 8 values (an
    output one element off 16-byte alignment)."""
    rows, n, g = 24, 512, 64
    codes, scales, zeros = _codes(rows, n, bits, n // g, 5 + bits)
    packed = (G.gptq_pack_int4 if bits == 4 else G.gptq_pack_int3)(codes)
    rng = np.random.default_rng(11)
    gidx = rng.integers(0, n // g, n).astype(np.int32)
    # the reference: the release library on a clean g_idx
    _lib._LIB = _lib.load()
    ref = G.gptq_dequant(packed, bits, n, scales, zeros, g, torch.from_numpy(gidx).cuda(),
                         out_dtype)
    torch.cuda.synchronize()
    _lib._LIB = debug_lib
    buf = torch.full((rows * n + offset,), 7.0, dtype=out_dtype, device="cuda")
    out = buf[offset:].view(rows, n)
    # a clean call: same values as the release library, nothing reported
    G.gptq_dequant(packed, bits, n, scales, zeros, g, torch.from_numpy(gidx).cuda(), out_dtype,
                   out=out)
    assert G.gptq_device_checks(debug_lib) == 0
    assert torch.equal(out, ref)
    bad = gidx.copy()
    bad[[3, 100, 511]] = [n // g + 3, -1, 1 << 20]
    G.gptq_dequant(packed, bits, n, scales, zeros, g, torch.from_numpy(bad).cuda(), out_dtype,
                   out=out)
    assert G.gptq_device_checks(debug_lib) == 1
    good = np.ones(n, dtype=bool)
    good[[3, 100, 511]] = False
    assert torch.equal(out[:, torch.from_numpy(good).cuda()], ref[:, torch.from_numpy(good).cuda()])
    assert torch.all(out[:, [3, 100, 511]] == 0)
    assert G.gptq_device_checks(debug_lib) == 0          # read and cleared


def test_gather_columns_reports_a_permutation_out_of_range(debug_lib):
    rows, n = 9, 300
    codes, _, _ = _codes(rows, n, 4, 1, 3)
    perm = np.random.default_rng(4).permutation(n).astype(np.int32)
    ref = codes[:, torch.from_numpy(perm.astype(np.int64)).cuda()]
    out = G.gptq_gather_columns_u8(codes, torch.from_numpy(perm).cuda())
    assert G.gptq_device_checks(debug_lib) == 0 and torch.equal(out, ref)
    perm[[0, 150]] = [n, -7]
    out = G.gptq_gather_columns_u8(codes, torch.from_numpy(perm).cuda())
    assert G.gptq_device_checks(debug_lib) == 2
    keep = torch.ones(n, dtype=torch.bool, device="cuda")
    keep[[0, 150]] = False
    assert torch.equal(out[:, keep], ref[:, keep]) and torch.all(out[:, [0, 150]] == 0)


def test_dequant_matvec_reports_bad_indices(debug_lib):
    """The g_idx kernel and the tensor-core kernel's permuted activations."""
    rows, n, g = 40, 1024, 128
    codes, scales, zeros = _codes(rows, n, 4, n // g, 8)
    packed = G.gptq_pack_int4(codes)
    x = torch.randn(2, n, device="cuda").to(torch.bfloat16)
    gidx = torch.from_numpy(np.random.default_rng(2).integers(0, n // g, n).astype(np.int32))
    G.gptq_dequant_matvec(packed, 4, n, scales, zeros, x, g, gidx.cuda())
    assert G.gptq_device_checks(debug_lib) == 0
    gidx[17] = n // g
    y = G.gptq_dequant_matvec(packed, 4, n, scales, zeros, x, g, gidx.cuda())
    assert G.gptq_device_checks(debug_lib) == 1 and bool(torch.isfinite(y).all())
    perm = torch.from_numpy(np.random.default_rng(3).permutation(n).astype(np.int32))
    G.gptq_dequant_matvec(packed, 4, n, scales, zeros, x, g, perm=perm.cuda())
    assert G.gptq_device_checks(debug_lib) == 0
    perm[5] = n + 1
    y = G.gptq_dequant_matvec(packed, 4, n, scales, zeros, x, g, perm=perm.cuda())
    assert G.gptq_device_checks(debug_lib) == 2 and bool(torch.isfinite(y).all())


def test_quantize_layer_reports_a_permutation_out_of_range(debug_lib):
    """The weight gather, the position map and the un-permute of the sweep."""
    import workloads
    rows, n = 16, 256
    W, X = workloads.random_layer(rows, n, 704, seed=21, dtype=torch.bfloat16, correlated=0.3)
    Wd = W.cuda()
    H = torch.zeros(n, n, device="cuda")
    G.gptq_hessian_accumulate(H, X.cuda())
    U, perm, dead, info = G.gptq_cholesky_inverse(H, 0.01, True)
    torch.cuda.synchronize()
    assert int(info.item()) == 0
    cfg = G.make_config(4, 128, 0.01, True)
    clean = G.gptq_quantize_layer(Wd, U, perm, dead, cfg)
    assert G.gptq_device_checks(debug_lib) == 0
    bad = perm.clone()
    bad[10] = n + 2
    G.gptq_quantize_layer(Wd, U, bad, dead, cfg)
    assert G.gptq_device_checks(debug_lib) & 2
    # the context is still usable, and a clean call repeats the clean results
    again = G.gptq_quantize_layer(Wd, U, perm, dead, cfg)
    assert G.gptq_device_checks(debug_lib) == 0
    for k, a in clean.items():
        if isinstance(a, torch.Tensor):
            assert torch.equal(a, again[k]), k
