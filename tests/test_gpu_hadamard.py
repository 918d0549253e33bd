"""GPU parity of the Hadamard rotation kernels against the fp64 oracle.

Bound (first order): a block's fast transform has log2(b) butterfly stages,
each adding two partial sums whose magnitudes are at most the block's sum of
|s x|, so the fp32 error of an output is below log2(b) 2^-24 sum|x| / sqrt(b)
before the final scale (exact for b = 4^k, one more rounding otherwise).
The test doubles (log2 b + 1) of that.  A bf16 output adds half a bf16 ulp
of the value (its one rounding)."""
import math

import numpy as np
import pytest
import torch

import post_weight_quantization_25_b200 as G
from oracle import hadamard_oracle as HO

pytestmark = pytest.mark.gpu


def _signs(n, seed):
    g = torch.Generator().manual_seed(seed)
    return (torch.randint(0, 2, (n,), generator=g) * 2 - 1).float()


def _half_ulp_bf16(v):
    a = np.maximum(np.abs(v), 1e-38)
    return np.exp2(np.floor(np.log2(a)) - 8)


def _bound(x_rows, b, out_bf16, y_ref, y_got):
    """x_rows: inputs as (..., n) fp64 with the rotated axis last."""
    n = x_rows.shape[-1]
    S = np.abs(x_rows).reshape(x_rows.shape[:-1] + (n // b, b)).sum(-1)
    fp = 2 * (math.log2(b) + 1) * 2.0 ** -24 * S / math.sqrt(b)
    fp = np.repeat(fp, b, axis=-1)
    if out_bf16:
        fp = fp + np.maximum(_half_ulp_bf16(y_ref), _half_ulp_bf16(y_got))
    return fp + 1e-30


@pytest.mark.parametrize("rows,n,b,it,ot", [
    (3, 1024, 1024, torch.bfloat16, torch.bfloat16), (5, 2048, 1024, torch.float32, torch.float32),
    (7, 96, 32, torch.float32, torch.float32), (2, 512, 64, torch.bfloat16, torch.float32),
    (9, 1536, 512, torch.float32, torch.bfloat16), (1, 256, 128, torch.bfloat16, torch.bfloat16),
    (4, 768, 256, torch.float32, torch.float32)])
def test_rows_match_oracle(rows, n, b, it, ot):
    g = torch.Generator().manual_seed(rows * n + b)
    W = (torch.randn(rows, n, generator=g) * 0.02).to(it)
    W[0, 5] = 3.0  # an outlier, spread over its block
    s = _signs(n, b)
    y = G.gptq_hadamard_rows(W.cuda(), s.cuda(), b, out_dtype=ot).float().cpu().numpy()
    x = W.float().numpy().astype(np.float64)
    ref = HO.rotate_weight(x, s.numpy(), b)
    err = np.abs(y - ref)
    bound = _bound(x, b, ot == torch.bfloat16, ref, y)
    assert np.all(err <= bound), float(np.max(err / bound))


@pytest.mark.parametrize("n,ntok,b,it,ot", [
    (1024, 37, 1024, torch.bfloat16, torch.bfloat16), (2048, 16, 1024, torch.float32, torch.float32),
    (96, 1, 32, torch.float32, torch.float32), (512, 100, 256, torch.bfloat16, torch.float32),
    (3072, 33, 512, torch.float32, torch.bfloat16), (128, 64, 64, torch.bfloat16, torch.bfloat16),
    # bf16 blocks of 1024: whole 64-token tiles on the bf16-tile kernel, then a ragged tail
    (2048, 150, 1024, torch.bfloat16, torch.bfloat16), (1024, 128, 1024, torch.bfloat16, torch.bfloat16)])
def test_cols_match_oracle(n, ntok, b, it, ot):
    g = torch.Generator().manual_seed(n + ntok + b)
    X = torch.randn(n, ntok, generator=g).to(it)
    X[3, :] *= 50  # an outlier channel
    s = _signs(n, ntok)
    y = G.gptq_hadamard_cols(X.cuda(), s.cuda(), b, out_dtype=ot).float().cpu().numpy()
    x = X.float().numpy().astype(np.float64)
    ref = HO.rotate_features(x, s.numpy(), b)
    err = np.abs(y - ref)
    bound = _bound(x.T, b, ot == torch.bfloat16, ref.T, y.T).T
    assert np.all(err <= bound), float(np.max(err / bound))


@pytest.mark.parametrize("ntok", [40, 200])
def test_strided_and_in_place(ntok):
    """Row strides wider than a row (views into a larger buffer) and in-place
    rotation give the same values as the contiguous out-of-place call (200
    tokens: three whole 64-token tiles and a tail)."""
    g = torch.Generator().manual_seed(5)
    n, b = 2048, 1024
    s = _signs(n, 9).cuda()
    big = torch.randn(n, ntok + 24, generator=g).to(torch.bfloat16).cuda()
    X = big[:, 8:8 + ntok]
    left, right = big[:, :8].clone(), big[:, 8 + ntok:].clone()
    want = G.gptq_hadamard_cols(X.contiguous(), s, b)
    got = G.gptq_hadamard_cols(X, s, b)
    assert torch.equal(got, want)
    G.gptq_hadamard_cols(X, s, b, out=X)  # in place, strided
    assert torch.equal(X, want)
    assert torch.equal(big[:, :8], left) and torch.equal(big[:, 8 + ntok:], right)
    Wbig = torch.randn(6, n + 512, generator=g).cuda()
    W = Wbig[:, 256:256 + n]
    want = G.gptq_hadamard_rows(W.contiguous(), s, b)
    G.gptq_hadamard_rows(W, s, b, out=W)
    assert torch.equal(W, want)


def test_rotation_then_its_inverse_is_the_identity_and_the_product_is_kept():
    """R^T R = I: rotating X, then applying H (self-inverse up to 1/b) and the
    signs again, returns X to fp32 rounding; and W' X' = W X."""
    g = torch.Generator().manual_seed(2)
    n, ntok, rows, b = 2048, 64, 32, 1024
    s = _signs(n, 4).cuda()
    X = torch.randn(n, ntok, generator=g).cuda()
    W = torch.randn(rows, n, generator=g).cuda()
    Xr = G.gptq_hadamard_cols(X, s, b)
    Wr = G.gptq_hadamard_rows(W, s, b)
    ones = torch.ones(n, device="cuda")
    back = G.gptq_hadamard_cols(Xr, ones, b) * s[:, None]  # D (H/sqrt b)(H/sqrt b) D X = X
    torch.testing.assert_close(back, X, rtol=0, atol=2e-5 * float(X.abs().max()))
    ref = (W.double() @ X.double())
    got = (Wr.double() @ Xr.double())
    torch.testing.assert_close(got, ref, rtol=0, atol=1e-4 * float(ref.abs().max()))


def test_full_size_70b_down_proj_rotation_sampled():
    """The 70B down-proj workload's rotation at full size (X 28672 x 65536 bf16
    in place, W 8192 x 28672 bf16), checked against the oracle on sampled
    token columns and weight rows."""
    n, ntok, rows, b = 28672, 65536, 8192, 1024
    dev = torch.device("cuda")
    g = torch.Generator(device=dev).manual_seed(72)
    X = torch.randn(n, ntok, generator=g, device=dev).to(torch.bfloat16)
    W = (torch.randn(rows, n, generator=g, device=dev) * 0.01).to(torch.bfloat16)
    s = _signs(n, 3).to(dev)
    rng = np.random.default_rng(0)
    cols = np.sort(rng.choice(ntok, 24, replace=False))
    rws = np.sort(rng.choice(rows, 24, replace=False))
    x_in = X[:, torch.from_numpy(cols).to(dev)].float().cpu().numpy().astype(np.float64)
    w_in = W[torch.from_numpy(rws).to(dev)].float().cpu().numpy().astype(np.float64)
    G.gptq_hadamard_cols(X, s, b, out=X)
    G.gptq_hadamard_rows(W, s, b, out=W)
    torch.cuda.synchronize()
    sn = s.cpu().numpy()
    yx = X[:, torch.from_numpy(cols).to(dev)].float().cpu().numpy()
    rx = HO.rotate_features(x_in, sn, b)
    bx = _bound(x_in.T, b, True, rx.T, yx.T).T
    assert np.all(np.abs(yx - rx) <= bx)
    yw = W[torch.from_numpy(rws).to(dev)].float().cpu().numpy()
    rw = HO.rotate_weight(w_in, sn, b)
    bw = _bound(w_in, b, True, rw, yw)
    assert np.all(np.abs(yw - rw) <= bw)
