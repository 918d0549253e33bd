"""CUDA path vs the fp64 oracle, element by element, on seeded inputs.

Every call goes through the C ABI (the ctypes binding).  Sizes span several
128-wide tiles with ragged tails; the tolerances are the agreed ones: H
relative Frobenius <= 1e-4, codes identical except at rounding ties (replayed
and counted), objective relative <= 1e-3, per-row scales <= 1e-6, group
scales <= 1e-4, packing and dequant bit-exact.
"""
import numpy as np
import pytest
import torch

import post_weight_quantization_25_b200 as G
import workloads
from oracle import gptq_oracle as O

from gpu_util import compare_layer, device_x, gpu_layer, to_np

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------------ storage
@pytest.mark.parametrize("bits,rows,n,g,use_gidx", [
    (4, 7, 64, 16, False), (4, 33, 256, 128, True), (4, 5, 24, -1, False),
    (3, 9, 96, 32, False), (3, 17, 256, 128, True), (3, 3, 32, -1, False)])
def test_pack_and_dequant_bit_exact(bits, rows, n, g, use_gidx):
    rng = np.random.default_rng(bits * 1000 + n)
    codes = rng.integers(0, 2 ** bits, (rows, n))
    G_ = 1 if g <= 0 else (n + g - 1) // g
    scales = rng.uniform(1e-4, 0.2, (rows, G_)).astype(np.float32)
    zeros = rng.integers(0, 2 ** bits, (rows, G_))
    gidx = rng.integers(0, G_, n) if use_gidx else None
    cd = torch.from_numpy(codes.astype(np.uint8)).cuda()
    packed = G.gptq_pack_int4(cd) if bits == 4 else G.gptq_pack_int3(cd)
    ref = O.pack_int4(codes) if bits == 4 else O.pack_int3(codes)
    got = packed.cpu().numpy().view(np.uint32)
    assert np.array_equal(got, ref)
    sd = torch.from_numpy(scales).cuda()
    zd = torch.from_numpy(zeros.astype(np.uint8)).cuda()
    gd = torch.from_numpy(gidx.astype(np.int32)).cuda() if use_gidx else None
    w32 = G.gptq_dequant(packed, bits, n, sd, zd, g, gd, torch.float32)
    ref32 = O.dequant(ref, bits, n, scales, zeros, g, gidx)
    assert np.array_equal(w32.cpu().numpy(), ref32)
    w16 = G.gptq_dequant(packed, bits, n, sd, zd, g, gd, torch.bfloat16)
    ref16 = O.dequant(ref, bits, n, scales, zeros, g, gidx, out="bf16")
    assert np.array_equal(w16.view(torch.int16).cpu().numpy().view(np.uint16), ref16)


@pytest.mark.parametrize("bits,rows,n,g,use_gidx,batch,xdt", [
    (4, 7, 64, 16, False, 1, torch.float32), (4, 33, 256, 128, True, 3, torch.bfloat16),
    (4, 130, 1032, -1, False, 8, torch.bfloat16), (3, 9, 96, 32, False, 2, torch.float32),
    (3, 17, 2080, 128, True, 11, torch.bfloat16), (4, 1, 8, -1, False, 1, torch.float32),
    # original order with g_idx on the row-per-lane kernel: several 1024-column
    # chunks with a ragged last one, rows past a 32-row tile, fp32 and bf16 x,
    # int3 (n % 128 == 0), and 512 groups (rulers read through L1, not staged)
    (4, 70, 1056, 32, True, 8, torch.float32), (3, 45, 2176, 64, True, 5, torch.bfloat16),
    (4, 40, 2048, 4, True, 2, torch.bfloat16), (4, 33, 3072, 128, True, 1, torch.bfloat16)])
def test_dequant_matvec_matches_oracle(bits, rows, n, g, use_gidx, batch, xdt):
    """y = x w_hat^T with w_hat dequantized on the fly, within mv_bound."""
    rng = np.random.default_rng(bits * 7 + n + batch)
    codes = rng.integers(0, 2 ** bits, (rows, n))
    G_ = 1 if g <= 0 else (n + g - 1) // g
    scales = rng.uniform(1e-4, 0.2, (rows, G_)).astype(np.float32)
    zeros = rng.integers(0, 2 ** bits, (rows, G_))
    gidx = rng.integers(0, G_, n) if use_gidx else None
    cd = torch.from_numpy(codes.astype(np.uint8)).cuda()
    packed = G.gptq_pack_int4(cd) if bits == 4 else G.gptq_pack_int3(cd)
    x = torch.randn(batch, n, generator=torch.Generator().manual_seed(n)).to(xdt)
    y = G.gptq_dequant_matvec(packed, bits, n, torch.from_numpy(scales).cuda(),
                              torch.from_numpy(zeros.astype(np.uint8)).cuda(), x.cuda(), g,
                              torch.from_numpy(gidx.astype(np.int32)).cuda() if use_gidx else None)
    ref_packed = O.pack_int4(codes) if bits == 4 else O.pack_int3(codes)
    yo, mag = O.dequant_matvec(ref_packed, bits, n, scales, zeros, x.float().numpy(), g, gidx)
    err = np.abs(y.cpu().numpy().astype(np.float64) - yo)
    bound = mv_bound(n, mag)
    assert np.all(err <= bound), float(np.max(err / bound))


def mv_bound(n, mag):
    """Rounding bound of gptq_dequant_matvec against the fp64 product with
    binary32 w_hat.  FP32-pipe kernel: each lane sums n/32 rounded FMA terms,
    then five shuffle levels.  Row-per-lane g_idx kernel: each of a lane's
    four partial sums takes n/32 rounded FMA terms (8 warps share the
    columns), then two levels over the four sums and three over the warps.  Tensor-core kernel (int4, bf16 x): the products
    (q - zero) x are exact; at most 8 MMA accumulations of 16 products per
    128-column slice (<= 16 roundings, internal order unknown), one FMA by the
    scale, n/512 slice sums per warp, 3 levels over 8 warps, plus one rounding
    for scale (q - zero) versus the binary32 w_hat.  Both depths are below
    n/32 + 24; the bound doubles that first-order figure."""
    return 2 * (n / 32 + 24) * 2.0 ** -24 * mag + 1e-30


@pytest.mark.parametrize("bits", [4, 3])
@pytest.mark.parametrize("rows,n,g,batch,use_perm", [
    (33, 1056, 32, 3, False), (100, 2048, 128, 8, True), (16, 4096, -1, 1, False),
    (5, 96, 32, 9, True), (47, 640, 64, 2, False), (18, 1024, 256, 5, False),
    (257, 4224, 128, 1, True), (9, 160, 32, 2, False)])
def test_dequant_matvec_tensor_core_path(bits, rows, n, g, batch, use_perm):
    """int4 / int3 codes x bf16 activations with contiguous groups run on the
    MMA kernel: one prep launch (x in pair / sweep order, y zeroed), then one
    launch per 8 vectors.
    Ragged row tiles (rows % 16), partial 128-column slices (n % 128), group
    sizes 32 / 64 (per-block scales), 128 / 256 / per row (per-slice scales),
    batches past 8, and extreme codes against extreme zero points."""
    rng = np.random.default_rng(rows * 31 + n + batch + bits)
    top = 2 ** bits - 1
    codes = rng.integers(0, top + 1, (rows, n))
    codes[0, : n // 2] = top
    codes[-1, : n // 3] = 0
    G_ = 1 if g <= 0 else n // g
    scales = rng.uniform(1e-4, 0.2, (rows, G_)).astype(np.float32)
    zeros = rng.integers(0, top + 1, (rows, G_))
    zeros[0, :] = 0
    zeros[-1, :] = top
    perm = rng.permutation(n) if use_perm else None
    pack = G.gptq_pack_int4 if bits == 4 else G.gptq_pack_int3
    packed = pack(torch.from_numpy(codes.astype(np.uint8)).cuda())
    x = torch.randn(batch, n, generator=torch.Generator().manual_seed(rows)).to(torch.bfloat16)
    before = G.gptq_launch_count()
    y = G.gptq_dequant_matvec(packed, bits, n, torch.from_numpy(scales).cuda(),
                              torch.from_numpy(zeros.astype(np.uint8)).cuda(), x.cuda(), g,
                              perm=torch.from_numpy(perm.astype(np.int32)).cuda()
                              if use_perm else None)
    torch.cuda.synchronize()
    assert G.gptq_launch_count() - before == 1 + (batch + 7) // 8  # x prep + one per 8 vectors
    ref_packed = O.pack_int4(codes) if bits == 4 else O.pack_int3(codes)
    yo, mag = O.dequant_matvec(ref_packed, bits, n, scales, zeros, x.float().numpy(), g,
                               perm=perm)
    err = np.abs(y.cpu().numpy().astype(np.float64) - yo)
    bound = mv_bound(n, mag)
    assert np.all(err <= bound), float(np.max(err / bound))


@pytest.mark.parametrize("bits,rows,n,g,batch", [(4, 40, 1024, 128, 1), (3, 33, 2048, 128, 4),
                                                 (4, 7, 256, 32, 8)])
def test_dequant_matvec_in_sweep_order(bits, rows, n, g, batch):
    """Act-order layers: the codes gathered into sweep order (bit exact), packed,
    and multiplied with x[perm] -- the same y as the original-order product."""
    rng = np.random.default_rng(bits + rows + n)
    codes = rng.integers(0, 2 ** bits, (rows, n))
    perm = rng.permutation(n)
    G_ = n // g
    scales = rng.uniform(1e-4, 0.2, (rows, G_)).astype(np.float32)
    zeros = rng.integers(0, 2 ** bits, (rows, G_))
    gidx = np.empty(n, dtype=np.int64)
    gidx[perm] = np.arange(n) // g          # group of original column c
    cd = torch.from_numpy(codes.astype(np.uint8)).cuda()
    pd = torch.from_numpy(perm.astype(np.int32)).cuda()
    csw = G.gptq_gather_columns_u8(cd, pd)
    assert np.array_equal(csw.cpu().numpy(), codes[:, perm].astype(np.uint8))
    pk = G.gptq_pack_int4(csw) if bits == 4 else G.gptq_pack_int3(csw)
    x = torch.randn(batch, n, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    sd = torch.from_numpy(scales).cuda()
    zd = torch.from_numpy(zeros.astype(np.uint8)).cuda()
    y = G.gptq_dequant_matvec(pk, bits, n, sd, zd, x.cuda(), g, perm=pd)
    ref_sw = O.pack_int4(codes[:, perm]) if bits == 4 else O.pack_int3(codes[:, perm])
    yo, mag = O.dequant_matvec(ref_sw, bits, n, scales, zeros, x.float().numpy(), g, perm=perm)
    err = np.abs(y.cpu().numpy().astype(np.float64) - yo)
    assert np.all(err <= mv_bound(n, mag))
    # the same product in original column order with g_idx
    ref_o = O.pack_int4(codes) if bits == 4 else O.pack_int3(codes)
    yo2, _ = O.dequant_matvec(ref_o, bits, n, scales, zeros, x.float().numpy(), g, gidx)
    np.testing.assert_allclose(yo, yo2, rtol=0, atol=1e-12 * float(np.max(mag)))


def test_pack_int4_unaligned_row_length():
    rng = np.random.default_rng(5)
    codes = rng.integers(0, 16, (6, 40))          # n % 32 != 0: the 8-code path
    packed = G.gptq_pack_int4(torch.from_numpy(codes.astype(np.uint8)).cuda())
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), O.pack_int4(codes))


# ------------------------------------------------------------------ Hessian
@pytest.mark.parametrize("n,ntok,dtype", [
    (256, 2048, torch.float32), (6, 100, torch.bfloat16), (130, 1000, torch.bfloat16),
    (257, 333, torch.bfloat16), (384, 4096, torch.bfloat16), (520, 70, torch.float32),
    (1000, 3000, torch.bfloat16)])
def test_hessian_matches_oracle(n, ntok, dtype):
    _, X = workloads.random_layer(1, n, ntok, seed=n + ntok, dtype=dtype)
    H = torch.zeros(n, n, dtype=torch.float32, device="cuda")
    G.gptq_hessian_accumulate(H, device_x(X))
    Hg = to_np(H).astype(np.float64)
    Ho = O.hessian(to_np(X))
    assert np.array_equal(Hg, Hg.T)
    assert np.linalg.norm(Hg - Ho) / np.linalg.norm(Ho) <= 1e-4


def test_hessian_accumulates_over_batches_and_alpha():
    _, X = workloads.random_layer(1, 192, 1536, seed=3, dtype=torch.bfloat16)
    H = torch.zeros(192, 192, dtype=torch.float32, device="cuda")
    Xd = device_x(X)
    G.gptq_hessian_accumulate(H, Xd[:, :512])
    G.gptq_hessian_accumulate(H, Xd[:, 512:1024])
    G.gptq_hessian_accumulate(H, Xd[:, 1024:], alpha=1.0)
    Xn = to_np(X).astype(np.float64)
    Ho = 2.0 * Xn[:, :1024] @ Xn[:, :1024].T + Xn[:, 1024:] @ Xn[:, 1024:].T
    Hg = to_np(H)
    assert np.linalg.norm(Hg - Ho) / np.linalg.norm(Ho) <= 1e-4


def test_hessian_zero_tokens_is_a_no_op():
    H = torch.full((16, 16), 3.0, device="cuda")
    X = torch.zeros(16, 8, dtype=torch.bfloat16, device="cuda")
    G.gptq_hessian_accumulate(H, X[:, :0])
    assert torch.all(H == 3.0)


# ------------------------------------------------------------------ Cholesky
# widths that are a multiple of 128 with at least 3 panels below 8192 (384,
# 640, 1024, 2048, 8064) take the persistent factorisation; the others launch
# panel by panel
@pytest.mark.parametrize("n,actorder,dead", [(6, False, ()), (130, True, (7,)),
                                             (256, False, ()), (300, True, (0, 299)),
                                             (384, True, ()), (640, True, ()),
                                             (1024, False, (3, 1000)), (2048, True, ()),
                                             (8064, True, (5,))])
def test_cholesky_inverse_matches_oracle(n, actorder, dead):
    _, X = workloads.random_layer(1, n, 3 * n + 50, seed=n, dead=dead, correlated=0.3)
    Ho32 = O.hessian(to_np(X)).astype(np.float32)          # the oracle's own H, as fp32
    H = torch.from_numpy(Ho32).cuda()
    U, perm, dead_d, info = G.gptq_cholesky_inverse(H, 0.01, actorder)
    torch.cuda.synchronize()
    assert int(info.item()) == 0
    W = np.zeros((1, n))
    prep = O.prepare(Ho32.astype(np.float64), W, 0.01, actorder,
                     forced_perm=perm.cpu().numpy() if actorder else None)
    Uo = O.upper_cholesky_of_inverse(prep["Hp"])
    Ug = to_np(U).astype(np.float64)
    assert np.all(np.tril(Ug, -1) == 0)
    assert np.linalg.norm(Ug - Uo) / np.linalg.norm(Uo) <= 1e-4
    assert np.array_equal(dead_d.cpu().numpy().astype(bool), prep["dead"])
    if not actorder:
        assert np.array_equal(perm.cpu().numpy(), np.arange(n))


@pytest.mark.parametrize("n", [200, 512])
def test_cholesky_reports_failures_in_info(n):
    H = -torch.eye(n, device="cuda")
    _, _, _, info = G.gptq_cholesky_inverse(H, 0.0, False)
    assert int(info.item()) > 0            # not positive definite
    H = torch.eye(n, device="cuda")
    H[5, 5] = float("nan")
    _, _, _, info = G.gptq_cholesky_inverse(H, 0.01, True)
    assert int(info.item()) == -1
    # a negative pivot at column j of a diagonal H: the factorisation runs from
    # the last column to the first, so it is found at step n - 1 - j and
    # reported as j + 1 (a later panel than the first on both paths)
    j = 100
    H = torch.eye(n, device="cuda") * 2.0
    H[j, j] = -1.0
    _, _, _, info = G.gptq_cholesky_inverse(H, 0.0, False)
    assert int(info.item()) == j + 1
    H = torch.eye(n, device="cuda") * 2.0
    _, _, _, info = G.gptq_cholesky_inverse(H, 0.01, True)
    assert int(info.item()) == 0           # the context is still usable


def test_scale_equivariance_on_gpu():
    _, X = workloads.random_layer(1, 256, 900, seed=17, correlated=0.4)
    Ho32 = O.hessian(to_np(X)).astype(np.float32)
    W = workloads.random_layer(40, 256, 1, seed=18)[0].cuda()
    cfg = G.make_config(4, 128, 0.01, True)
    outs = []
    for s in (1.0, 4.0):
        H = torch.from_numpy(Ho32 * np.float32(s)).cuda()
        U, perm, dead, info = G.gptq_cholesky_inverse(H, 0.01, True)
        q = G.gptq_quantize_layer(W, U, perm, dead, cfg)
        outs.append((U.clone(), q["codes"].clone(), perm.clone()))
    assert torch.equal(outs[0][2], outs[1][2])
    assert torch.equal(outs[0][0] * 0.5, outs[1][0])
    assert torch.equal(outs[0][1], outs[1][1])


# ------------------------------------------------------------------ whole layer
LAYERS = [
    # rows, n, ntok, bits, group, actorder, dtype, dead
    (256, 256, 2048, 4, -1, False, torch.float32, ()),     # the 256x256 fp32 layer, full size
    (200, 300, 1000, 4, 128, True, torch.bfloat16, (17,)),
    (64, 384, 1500, 3, 128, False, torch.bfloat16, ()),
    (48, 256, 800, 4, 32, True, torch.bfloat16, ()),
    (48, 256, 800, 4, 64, False, torch.float32, (3,)),
    (33, 512, 1200, 4, 256, True, torch.bfloat16, ()),
    (4, 6, 64, 2, -1, False, torch.float32, ()),
    (1, 130, 300, 4, -1, True, torch.bfloat16, ()),
    (130, 257, 700, 8, 128, True, torch.bfloat16, ()),
    # the widest layer the persistent factorisation and sweep take (63 panels)
    (48, 8064, 9000, 4, 128, True, torch.bfloat16, (5,)),
]


@pytest.mark.parametrize("rows,n,ntok,bits,g,act,dtype,dead", LAYERS)
def test_layer_matches_oracle(rows, n, ntok, bits, g, act, dtype, dead):
    if (rows, n) == (256, 256):
        wl = workloads.WORKLOADS["layer256"]
        W, X = workloads.make_inputs(wl)
    else:
        W, X = workloads.random_layer(rows, n, ntok, seed=rows * 7 + n, dtype=dtype, dead=dead,
                                      correlated=0.3)
    gpu = gpu_layer(W, X, bits, g, 0.01, act)
    compare_layer(gpu, W, X, bits, g, 0.01, act)


@pytest.mark.parametrize("rows,n,ntok,bits,g,act,dtype", [
    (64, 384, 1500, 4, 128, True, torch.bfloat16), (48, 256, 800, 3, -1, False, torch.float32),
    (40, 200, 700, 4, 32, True, torch.bfloat16)])
def test_symmetric_ruler_matches_oracle(rows, n, ntok, bits, g, act, dtype):
    """The opt-in symmetric ruler: zero point on the middle tick, same sweep."""
    W, X = workloads.random_layer(rows, n, ntok, seed=rows + 3 * n, dtype=dtype, correlated=0.3)
    gpu = gpu_layer(W, X, bits, g, 0.01, act, sym=True)
    assert np.all(gpu["zeros"] == 2 ** (bits - 1))
    compare_layer(gpu, W, X, bits, g, 0.01, act, sym=True)


@pytest.mark.parametrize("g,act", [(-1, False), (128, False), (128, True), (32, True)])
def test_identity_hessian_gives_rtn_on_gpu(g, act):
    n, rows = 256, 24
    gains = np.linspace(0.5, 3.0, n)[np.random.default_rng(1).permutation(n)]
    X = workloads.identity_calibration(n, 4, gains, dtype=torch.bfloat16)
    W = workloads.random_layer(rows, n, 1, seed=2)[0]
    gpu = gpu_layer(W, X, 4, g, 0.01, act)
    Ho = O.hessian(to_np(X))
    prep = O.prepare(Ho, to_np(W).astype(np.float64), 0.01, act)
    assert np.array_equal(gpu["perm"], prep["perm"])
    base = O.rtn(prep["Wp"], 4, g)
    assert np.array_equal(gpu["codes"][:, prep["perm"]], base["codes"])
    assert np.array_equal(gpu["zeros"], base["zeros"])
    assert np.array_equal(gpu["scales"], base["scales"])


def test_empty_rows_is_a_no_op():
    cfg = G.make_config(4, 128, 0.01, False)
    W = torch.zeros(0, 128, dtype=torch.bfloat16, device="cuda")
    U = torch.eye(128, device="cuda")
    perm = torch.arange(128, dtype=torch.int32, device="cuda")
    dead = torch.zeros(128, dtype=torch.uint8, device="cuda")
    q = G.gptq_quantize_layer(W, U, perm, dead, cfg)
    assert q["codes"].shape == (0, 128)


def test_quantize_linear_end_to_end():
    W, X = workloads.random_layer(64, 256, 1024, seed=99, dtype=torch.bfloat16, correlated=0.3)
    ql = G.quantize_linear(W.cuda(), device_x(X), bits=4, group_size=128, actorder=True,
                           want_wq=True)
    torch.cuda.synchronize()
    assert int(ql.info.item()) == 0
    w = G.gptq_dequant(ql.packed, 4, 256, ql.scales, ql.zeros, 128, ql.g_idx)
    assert torch.equal(w, ql.Wq)


@pytest.mark.parametrize("g,actorder", [(256, True), (512, False), (256, False)])
def test_groups_wider_than_a_block_with_lookahead(g, actorder):
    """A group of 256 or 512 columns is fitted, when the sweep reaches its
    first column, on all of its current columns -- several blocks.  With the
    look-ahead stream the update that reaches those columns must land before
    the fit: the result equals the one-stream result bit for bit and the
    oracle's up to rounding ties."""
    W, X = workloads.random_layer(192, 1024, 4096, seed=g + actorder, dtype=torch.bfloat16,
                                  correlated=0.4)
    Wd, Xd = W.cuda(), device_x(X)
    H = torch.zeros(1024, 1024, device="cuda")
    G.gptq_hessian_accumulate(H, Xd)
    cfg = G.make_config(4, g, 0.01, actorder)
    outs = []
    for side in (torch.cuda.Stream(), None):
        U, perm, dead, info = G.gptq_cholesky_inverse(H, 0.01, actorder, side_stream=side)
        q = G.gptq_quantize_layer(Wd, U, perm, dead, cfg, want_wq=True, side_stream=side)
        torch.cuda.synchronize()
        assert int(info.item()) == 0
        outs.append(q)
    for k in ("codes", "scales", "zeros", "Wq"):
        assert torch.equal(outs[0][k], outs[1][k]), k
    gpu = gpu_layer(W, X, 4, g, 0.01, actorder, H=H)
    compare_layer(gpu, W, X, 4, g, 0.01, actorder)
