"""The layer pipeline: the Hessian of linear l + 1 overlapping the rest of
linear l on a second stream gives every linear the same results as the
oracle (and as the one-stream order) -- the overlap only reorders
independent work."""
import numpy as np
import pytest
import torch

import post_weight_quantization_25_b200 as G
import workloads
from gpu_util import compare_layer, device_x, to_np

pytestmark = pytest.mark.gpu

SHAPES = [(40, 256), (33, 384), (64, 256), (17, 128)]


def _outputs(q):
    torch.cuda.synchronize()
    return {"perm": q.perm.cpu().numpy().astype(np.int64),
            "dead": q.dead.cpu().numpy().astype(bool), "info": int(q.info.item()),
            "codes": q.codes.cpu().numpy().astype(np.int64), "scales": q.scales.cpu().numpy(),
            "zeros": q.zeros.cpu().numpy().astype(np.int64),
            "g_idx": q.g_idx.cpu().numpy().astype(np.int64), "Wq": q.Wq.cpu().numpy(),
            "row_loss": q.row_loss.cpu().numpy().astype(np.float64)}


@pytest.mark.parametrize("overlap", [True, False])
@pytest.mark.parametrize("actorder", [False, True])
def test_pipelined_layers_match_the_oracle(overlap, actorder):
    ntok = 600
    layers = [workloads.random_layer(r, n, ntok, seed=50 + i, dtype=torch.bfloat16,
                                     correlated=0.3)
              for i, (r, n) in enumerate(SHAPES)]
    Ws = [W.cuda() for W, _ in layers]
    Xs = [device_x(X) for _, X in layers]
    pipe = G.LayerPipeline(SHAPES, ntok, bits=4, group_size=64, actorder=actorder,
                           w_dtype=torch.bfloat16, want_wq=True, want_loss=True)
    pipe.run(Ws, Xs, overlap=overlap)
    torch.cuda.synchronize()
    pipe.check_info()
    for q, (W, X) in zip(pipe.layers, layers):
        compare_layer(_outputs(q), W, X, 4, 64, 0.01, actorder)
        # the packed and dequantized outputs belong to the same codes
        deq = to_np(q.deq)
        sc = q.scales.cpu().numpy()[:, q.g_idx.cpu().numpy()]
        zz = q.zeros.cpu().numpy()[:, q.g_idx.cpu().numpy()].astype(np.float64)
        wq = (sc.astype(np.float64) * (q.codes.cpu().numpy() - zz)).astype(np.float32)
        assert np.array_equal(deq, torch.from_numpy(wq).to(torch.bfloat16).float().numpy())


def test_pipeline_runs_again_with_new_inputs():
    """Buffers are reused across runs: a second run on other inputs matches
    a fresh one-layer quantizer on those inputs."""
    ntok = 300
    shapes = SHAPES[:2]
    pipe = G.LayerPipeline(shapes, ntok, group_size=128, want_wq=True, want_loss=True)
    for seed in (1, 2):
        layers = [workloads.random_layer(r, n, ntok, seed=seed * 10 + i, dtype=torch.bfloat16)
                  for i, (r, n) in enumerate(shapes)]
        pipe.run([W.cuda() for W, _ in layers], [device_x(X) for _, X in layers])
        torch.cuda.synchronize()
        for q, (W, X) in zip(pipe.layers, layers):
            compare_layer(_outputs(q), W, X, 4, 128, 0.01, False)


def test_stack_run_stores_each_linear_and_resumes(tmp_path):
    """quantize_linears with LayerQuantizer: each stored file holds exactly the
    device outputs of its linear, and a second call quantizes nothing."""
    ntok = 512
    shapes = {"l0": (40, 256), "l1": (33, 384)}
    inputs = {name: workloads.random_layer(r, n, ntok, seed=70 + i, dtype=torch.bfloat16)
              for i, (name, (r, n)) in enumerate(shapes.items())}
    kept = {}

    def quantize(name):
        r, n = shapes[name]
        q = G.LayerQuantizer(r, n, ntok, bits=4, group_size=128, actorder=True)
        W, X = inputs[name]
        q.run(W.cuda(), device_x(X))
        torch.cuda.synchronize()
        kept[name] = q
        return G.layer_quantizer_outputs(q)

    assert G.quantize_linears(list(shapes), quantize, str(tmp_path)) == list(shapes)
    for name, q in kept.items():
        blob = G.load_quantized(str(tmp_path / f"{name}.pt"))
        for k in ("packed", "scales", "zeros", "g_idx", "perm"):
            assert torch.equal(blob[k], getattr(q, k).cpu())
        assert blob["meta"]["rows"] == shapes[name][0] and blob["meta"]["actorder"]
    assert G.quantize_linears(list(shapes), quantize, str(tmp_path)) == []


def test_streamed_host_batches_match_the_oracle():
    """LayerQuantizer.run_streamed: W and the calibration batches come from
    pinned host memory, the copies overlap the batch-by-batch Hessian; the
    layer matches the oracle on the concatenated X.  Then two calls back to
    back with no synchronisation between them (the second call's copies
    overlap the first call's factorisation and sweep; staging buffers
    reused, more batches than buffers): the last call's results match the
    oracle on its own inputs."""
    r, n = 40, 256

    def inputs(seed, sizes):
        W, X = workloads.random_layer(r, n, sum(sizes), seed=seed, dtype=torch.bfloat16,
                                      correlated=0.3)
        cut = np.cumsum([0] + sizes)
        batches = [X[:, a:b].contiguous().pin_memory() for a, b in zip(cut[:-1], cut[1:])]
        return W, X, W.pin_memory(), batches

    Wa, Xa, Wah, Ba = inputs(91, [512, 512, 304])
    Wb, Xb, Wbh, Bb = inputs(92, [256, 128, 384, 64])
    q = G.LayerQuantizer(r, n, 1328, bits=4, group_size=64, actorder=True, want_wq=True,
                         want_loss=True)
    q.run_streamed(Wah, Ba)
    torch.cuda.synchronize()
    q.check_info()
    compare_layer(_outputs(q), Wa, Xa, 4, 64, 0.01, True)
    q.run_streamed(Wbh, Bb)
    q.run_streamed(Wah, Ba)
    q.run_streamed(Wbh, Bb)
    torch.cuda.synchronize()
    q.check_info()
    compare_layer(_outputs(q), Wb, Xb, 4, 64, 0.01, True)
