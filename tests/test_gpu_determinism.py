"""Repeatability of the kernels whose design claims it.

- gptq_hessian_accumulate: the token chunks of each output tile are added in
  chunk order (a turnstile), not by atomics, so H repeats bit for bit.
- gptq_cholesky_inverse: the look-ahead splits each panel's trailing update
  into a near part (caller's stream) and a far part (side stream), but every
  element still receives the panels' updates in panel order, each once per
  launch.  So the same H gives the same U, bit for bit, however the two
  streams interleave.
- gptq_dequant_matvec (tensor cores): the two column halves of every output
  meet by two atomic adds onto zero; fp32 addition of two terms commutes, so y
  is the same whichever half lands first.  The g_idx (original order) kernel
  sums each output's partial sums over its warps in a fixed order.
"""
import numpy as np
import pytest
import torch

import post_weight_quantization_25_b200 as G

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n,actorder", [(1024, True), (1000, False), (4096, True)])
def test_cholesky_inverse_is_repeatable(n, actorder):
    g = torch.Generator(device="cuda").manual_seed(n)
    X = torch.randn(n, 3 * n, generator=g, device="cuda").to(torch.bfloat16)
    H = torch.zeros(n, n, device="cuda")
    G.gptq_hessian_accumulate(H, X)
    outs = []
    side = torch.cuda.Stream()
    for k in range(4):
        # three runs with the look-ahead on a side stream, one without
        U, perm, dead, info = G.gptq_cholesky_inverse(H, 0.01, actorder,
                                                      side_stream=side if k < 3 else None)
        torch.cuda.synchronize()
        assert int(info.item()) == 0
        outs.append((U.clone(), perm.clone()))
    for U, perm in outs[1:]:
        assert torch.equal(perm, outs[0][1])
        assert torch.equal(U, outs[0][0])


@pytest.mark.parametrize("bits,rows,n,g,batch", [(4, 8192, 4096, 128, 1), (4, 1000, 2048, 32, 8),
                                                 (3, 4096, 4096, 128, 3)])
def test_dequant_matvec_is_repeatable(bits, rows, n, g, batch):
    rng = np.random.default_rng(rows + n)
    codes = torch.from_numpy(rng.integers(0, 2 ** bits, (rows, n)).astype(np.uint8)).cuda()
    packed = G.gptq_pack_int4(codes) if bits == 4 else G.gptq_pack_int3(codes)
    scales = torch.rand(rows, n // g, device="cuda") * 0.01 + 1e-4
    zeros = torch.randint(0, 2 ** bits, (rows, n // g), device="cuda", dtype=torch.uint8)
    perm = torch.randperm(n, device="cuda").to(torch.int32)
    x = torch.randn(batch, n, device="cuda").to(torch.bfloat16)
    ys = [G.gptq_dequant_matvec(packed, bits, n, scales, zeros, x, g, perm=perm)
          for _ in range(4)]
    # the same codes in original order with a g_idx (row-per-lane kernel)
    gidx = torch.randint(0, n // g, (n,), device="cuda", dtype=torch.int32)
    ys += [G.gptq_dequant_matvec(packed, bits, n, scales, zeros, x, g, g_idx=gidx)
           for _ in range(3)]
    torch.cuda.synchronize()
    for y in ys[5:]:
        assert torch.equal(y, ys[4])
    ys = ys[:4]
    torch.cuda.synchronize()
    for y in ys[1:]:
        assert torch.equal(y, ys[0])


@pytest.mark.parametrize("n,ntok", [(512, 65536), (200, 20000), (2048, 32768)])
def test_hessian_is_repeatable_with_split_tokens(n, ntok):
    """The tokens are cut into chunks (several units per output tile); the
    chunks of a tile are added into H in chunk order, so H repeats bit for
    bit.  fp32 X (three products per launch) as well."""
    g = torch.Generator(device="cuda").manual_seed(n + ntok)
    X = torch.randn(n, ntok, generator=g, device="cuda").to(torch.bfloat16)
    Hs = []
    for _ in range(3):
        H = torch.zeros(n, n, device="cuda")
        G.gptq_hessian_accumulate(H, X)
        Hs.append(H)
    Xf = torch.randn(n, 4096, generator=g, device="cuda")
    for _ in range(2):
        H = torch.zeros(n, n, device="cuda")
        G.gptq_hessian_accumulate(H, Xf)
        Hs.append(H)
    torch.cuda.synchronize()
    assert torch.equal(Hs[1], Hs[0]) and torch.equal(Hs[2], Hs[0])
    assert torch.equal(Hs[4], Hs[3])


def test_whole_layer_is_repeatable():
    """LayerQuantizer.run three times on the bench layer's shape (smaller
    token count): H, U, codes, rulers and the packed words are identical,
    with and without the look-ahead streams."""
    rows, n, ntok = 4096, 4096, 32768
    g = torch.Generator(device="cuda").manual_seed(11)
    X = torch.randn(n, ntok, generator=g, device="cuda").to(torch.bfloat16)
    W = (torch.randn(rows, n, generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    outs = []
    for look in (True, True, True, False):
        lq = G.LayerQuantizer(rows, n, ntok, 4, 128, 0.01, True, lookahead=look)
        lq.run(W, X)
        torch.cuda.synchronize()
        lq.check_info()
        outs.append({k: getattr(lq, k).clone() for k in
                     ("H", "U", "perm", "codes", "scales", "zeros", "packed")})
        del lq
    for o in outs[1:]:
        for k, v in o.items():
            assert torch.equal(v, outs[0][k]), k
