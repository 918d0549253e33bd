"""The bounded device waits give up and report instead of hanging.

Every wait inside the library's tensor-core kernels has a time limit; when
it runs out the kernel stops its pipeline, records the timeout in the call's
``info`` word, lets its own copies and MMAs finish, frees its tensor memory
and returns, so the CUDA context stays usable.  The test hook
``gptq_set_wait_gate`` makes every such kernel first wait for a device flag
that nothing sets, with a short limit and nothing in flight; each call must
then report its timeout, and the same calls made afterwards without the gate
must give exactly the results they give on a fresh context.
"""
import pytest
import torch

import post_weight_quantization_25_b200 as G

pytestmark = pytest.mark.gpu

LIMIT_NS = 2_000_000      # 2 ms


def _inputs(n, ntok, rows, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    X = torch.randn(n, ntok, generator=g, device="cuda").to(torch.bfloat16)
    W = (torch.randn(rows, n, generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    return W, X


def _layer(W, X, gate=None):
    """H, U and the sweep, each with its own info word; the gate (if any) is
    set only around these calls."""
    n = X.shape[0]
    side = torch.cuda.Stream()
    info_h = torch.zeros(1, dtype=torch.int32, device="cuda")
    info_q = torch.zeros(1, dtype=torch.int32, device="cuda")
    H = torch.zeros(n, n, device="cuda")
    if gate is not None:
        G.gptq_set_wait_gate(gate, LIMIT_NS)
    try:
        G.gptq_hessian_accumulate(H, X, info=info_h)
        U, perm, dead, info_c = G.gptq_cholesky_inverse(H, 0.01, True, side_stream=side)
        cfg = G.make_config(4, 128, 0.01, True)
        q = G.gptq_quantize_layer(W, U, perm, dead, cfg, info=info_q, side_stream=side)
    finally:
        G.gptq_set_wait_gate(None)
    torch.cuda.synchronize()
    return H, U, q, int(info_h.item()), int(info_c.item()), int(info_q.item())


@pytest.mark.parametrize("n", [128, 512])
def test_waits_time_out_report_and_leave_the_context_usable(n):
    W, X = _inputs(n, 4096, 256, seed=n)
    H0, U0, q0, ih, ic, iq = _layer(W, X)
    assert (ih, ic, iq) == (0, 0, 0)
    gate = torch.zeros(1, dtype=torch.int32, device="cuda")      # never set
    _, _, _, ih, ic, iq = _layer(W, X, gate)
    assert ih == G._lib.GPTQ_ERR_TIMEOUT                         # the Hessian's kernel
    if n > 128:                                                  # panels past the first
        assert ic == -2                                          # the factorisation's update
        assert iq == -2                                          # the sweep's lazy update
    # the context still works, and gives what it gave before the timeouts
    H1, U1, q1, ih, ic, iq = _layer(W, X)
    assert (ih, ic, iq) == (0, 0, 0)
    assert torch.equal(H1, H0)
    assert torch.equal(U1, U0)
    assert torch.equal(q1["codes"], q0["codes"])
    assert torch.equal(q1["scales"], q0["scales"])


def test_an_open_gate_changes_nothing():
    """A gate that is already open: every kernel passes it at once and the
    results are those of a run without the hook."""
    W, X = _inputs(512, 2048, 128, seed=3)
    H0, U0, q0, *_ = _layer(W, X)
    gate = torch.ones(1, dtype=torch.int32, device="cuda")
    H1, U1, q1, ih, ic, iq = _layer(W, X, gate)
    assert (ih, ic, iq) == (0, 0, 0)
    assert torch.equal(H1, H0) and torch.equal(U1, U0)
    assert torch.equal(q1["codes"], q0["codes"])
