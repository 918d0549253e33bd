"""Parity at the workloads' full sizes, in the launch sequence bench.py times.

Every case runs ``LayerQuantizer.run`` (the exact sequence of library calls
that bench.py times: H = 0, Hessian, preparation + U, sweep, packing, bf16
dequant) on the workload's own seeded inputs, then checks outputs the fp64
oracle can compute one piece at a time:

* H: every 256-channel diagonal block, plus one block on sampled channels
  (outlier channels included), recomputed from X in fp64; relative
  Frobenius <= 1e-4 per block.
* Preparation: dead inputs exactly; the act-order permutation must be a
  near-tie reordering of diag(H); lambda from the diagonal.
* U: the oracle's own U (the pages' route: Cholesky, inverse, Cholesky)
  from the GPU's H, relative Frobenius <= 1e-4 over the whole factor.  At
  n = 28672 the route runs as the in-place LAPACK steps (about 3e13 fp64
  flops); the sampled rows there are swept with that oracle U, not the
  GPU's.
* The sweep on sampled rows (rows are independent once U is fixed), replayed
  at rounding ties: no code may differ off a tie, and every tie lies within
  1e-5 tick of a half-integer; raw agreement >= 99.9 % on the rows without a
  tie; zero points exact, rulers within
  1e-4, and the layer-output objective ||W0 X - Wq X||^2 of those rows
  within 1e-3 of the oracle's, from X itself.
* Packing and bf16 dequant of those rows: bit exact.
* q_proj_7b: additionally every one of its 4096 rows is swept by the oracle
  (worker processes, one chunk of rows each): raw agreement of the codes
  over the whole layer >= 99.9 %, and the tie replay over the whole layer.
"""
from __future__ import annotations

import json
import os

import numpy as np
import pytest
import torch

import post_weight_quantization_25_b200 as G
import workloads
import oracle_pool
from oracle import gptq_oracle as O

pytestmark = pytest.mark.gpu

REPORT = os.environ.get("GPTQ_FULLSIZE_REPORT")


def _report(name, d):
    if REPORT:
        with open(REPORT, "a") as f:
            f.write(json.dumps({"case": name, **d}) + "\n")


def _rel(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def _f64_rows(Xc: torch.Tensor, idx) -> np.ndarray:
    return Xc[torch.as_tensor(np.asarray(idx), dtype=torch.long)].float().numpy().astype(np.float64)


def _matvec(M32: np.ndarray, v: np.ndarray, transpose=False, chunk=2048) -> np.ndarray:
    """M v (or M^T v) in fp64 for an fp32 matrix, a row chunk at a time."""
    n = M32.shape[0]
    out = np.zeros(M32.shape[1] if transpose else n)
    for r0 in range(0, n, chunk):
        blk = M32[r0:r0 + chunk].astype(np.float64)
        if transpose:
            out += blk.T @ v[r0:r0 + chunk]
        else:
            out[r0:r0 + chunk] = blk @ v
    return out


def _objective_rows(D: np.ndarray, Xc: torch.Tensor, tok_chunk=8192) -> float:
    """||D X||_F^2 in fp64 for a few rows D, X taken a token chunk at a time."""
    acc = 0.0
    for t0 in range(0, Xc.shape[1], tok_chunk):
        xb = Xc[:, t0:t0 + tok_chunk].float().numpy().astype(np.float64)
        R = D @ xb
        acc += float(np.sum(R * R))
    return acc


def _sample_rows(rows, k, seed):
    rng = np.random.default_rng(seed)
    fixed = {r for r in (0, 1, 127, 128, rows // 2, rows - 1) if r < rows}
    extra = set(rng.choice(rows, size=k, replace=False).tolist())
    return np.array(sorted(fixed | extra))


def _run(wl):
    torch.cuda.empty_cache()
    W, X = workloads.make_inputs(wl, device="cuda")
    lq = G.LayerQuantizer(wl.rows, wl.n, wl.ntok, wl.bits, wl.group_size, wl.percdamp,
                          wl.actorder, x_dtype=X.dtype, w_dtype=W.dtype,
                          out_dtype=torch.bfloat16)
    lq.run(W, X)
    lq.run(W, X)      # a second pass, as in the timed loop: nothing may carry over
    torch.cuda.synchronize()
    lq.check_info()
    out = {
        "H": lq.H.cpu().numpy(), "U": lq.U.cpu().numpy(),
        "perm": lq.perm.cpu().numpy().astype(np.int64),
        "dead": lq.dead.cpu().numpy().astype(bool),
        "codes": lq.codes.cpu().numpy(), "scales": lq.scales.cpu().numpy(),
        "zeros": lq.zeros.cpu().numpy().astype(np.int64),
        "g_idx": lq.g_idx.cpu().numpy().astype(np.int64),
        "packed": lq.packed.cpu().numpy().view(np.uint32),
        "deq": lq.deq.view(torch.int16).cpu().numpy().view(np.uint16),
    }
    Wc, Xc = W.cpu(), X.cpu()
    del lq, W, X
    torch.cuda.empty_cache()
    return Wc, Xc, out


def _check_hessian(wl, Xc, Hg, stats):
    n = wl.n
    worst = 0.0
    for c0 in range(0, n, 256):
        idx = np.arange(c0, min(c0 + 256, n))
        Ho = O.hessian(_f64_rows(Xc, idx))
        worst = max(worst, _rel(Hg[np.ix_(idx, idx)].astype(np.float64), Ho))
    rng = np.random.default_rng(wl.index)
    C = set(rng.choice(n, size=96, replace=False).tolist())
    if wl.outliers and not wl.hadamard_block:
        C |= set(workloads.outlier_channels(wl).tolist())
    C = np.array(sorted(C))
    Ho = O.hessian(_f64_rows(Xc, C))
    off = _rel(Hg[np.ix_(C, C)].astype(np.float64), Ho)
    stats.update(h_diag_blocks_rel=worst, h_sampled_rel=off)
    assert worst <= 1e-4, worst
    assert off <= 1e-4, off


def _check_rows(wl, Wc, Xc, out, U_rows_source, stats, k=18):
    """The sweep on sampled rows with the oracle, given a U (fp64 or fp32)."""
    rows, n, bits, g = wl.rows, wl.n, wl.bits, wl.group_size
    R = _sample_rows(rows, k, seed=wl.index)
    diag = out["diagH"] if "diagH" in out else np.diag(out["H"])
    prep = O.prepare_from_diagonal(diag, wl.percdamp, wl.actorder,
                                   forced_perm=out["perm"] if wl.actorder else None)
    assert np.array_equal(out["dead"], prep["dead"])
    if not wl.actorder:
        assert np.array_equal(out["perm"], np.arange(n))
    perm = prep["perm"]
    W0 = Wc[torch.as_tensor(R)].float().numpy().astype(np.float64)
    W0[:, prep["dead"]] = 0.0
    Wp = W0[:, perm]
    U = U_rows_source
    codes_sw = out["codes"][R][:, perm].astype(np.int64)
    own = O.sweep(Wp, U, bits, g)
    adoptions = []
    rep = O.sweep(Wp, U, bits, g, forced_codes=codes_sw, forced_zeros=out["zeros"][R],
                  adoptions=adoptions)
    agree = float(np.mean(own["codes"] == codes_sw))
    differ = (own["codes"] != codes_sw)
    stats.update(rows_checked=int(len(R)), raw_agreement=agree, ties_replayed=rep["adopted"],
                 mismatched=rep["mismatched"],
                 tie_distances=sorted(a[3] for a in adoptions)[-8:],
                 first_tie_columns=[a[1] for a in adoptions][:8],
                 rows_differing=int(np.count_nonzero(differ.any(axis=1))),
                 codes_differing=int(np.count_nonzero(differ)))
    _report(wl.name + ".rows", stats)
    assert rep["mismatched"] == 0, rep["mismatched"]
    assert np.array_equal(rep["codes"], codes_sw)
    # every divergence starts at a value within 1e-5 tick of a half-integer
    # (fp32 resolves t = w / scale to ~1e-6 tick), far inside the replay's tau
    assert all(a[3] <= 1e-5 for a in adoptions), adoptions
    # One such tie in a row changes that row's later codes (the repair of a
    # code one tick apart moves every later weight), so raw agreement is
    # asserted over the rows without a tie; it is reported in every case.
    tie_rows = {a[0] for a in adoptions}
    clean = np.array([i not in tie_rows for i in range(len(R))])
    agree_clean = float(np.mean(own["codes"][clean] == codes_sw[clean])) if clean.any() else 1.0
    stats["raw_agreement_rows_without_tie"] = agree_clean
    _report(wl.name + ".rows", stats)
    assert agree_clean >= 0.999, agree_clean
    assert np.array_equal(out["zeros"][R], rep["zeros"])
    np.testing.assert_allclose(out["scales"][R], rep["scales"], rtol=1e-6 if g <= 0 else 1e-4)
    gi = np.empty(n, dtype=np.int64)
    gi[perm] = np.arange(n) // (g if g > 0 else n)
    assert np.array_equal(out["g_idx"], gi)
    # w_hat of the GPU (one fp32 product of its own ruler) and the objective
    sc = out["scales"][R][:, out["g_idx"]].astype(np.float64)
    zz = out["zeros"][R][:, out["g_idx"]]
    Wq_gpu = (sc * (out["codes"][R].astype(np.int64) - zz)).astype(np.float32).astype(np.float64)
    Wq_orc = np.empty_like(rep["Wq"])
    Wq_orc[:, perm] = rep["Wq"]
    e_gpu = _objective_rows(W0 - Wq_gpu, Xc)
    e_orc = _objective_rows(W0 - Wq_orc, Xc)
    stats.update(objective_gpu=e_gpu, objective_oracle=e_orc,
                 objective_rel=abs(e_gpu - e_orc) / e_orc)
    assert abs(e_gpu - e_orc) <= 1e-3 * e_orc, (e_gpu, e_orc)
    # storage of the same rows
    packer = O.pack_int4 if bits == 4 else O.pack_int3
    ref_packed = packer(out["codes"][R].astype(np.int64))
    assert np.array_equal(out["packed"][R], ref_packed)
    ref16 = O.dequant(ref_packed, bits, n, out["scales"][R], out["zeros"][R], g, out["g_idx"],
                      out="bf16")
    assert np.array_equal(out["deq"][R], ref16)
    return prep


def _check_all_rows(wl, Wc, out, Uo, stats):
    """Every row of the layer through the oracle's sweep: the raw agreement
    north of 99.9 % over all entries, and the tie replay over all rows."""
    n, bits, g = wl.n, wl.bits, wl.group_size
    prep = O.prepare_from_diagonal(np.diag(out["H"]), wl.percdamp, wl.actorder,
                                   forced_perm=out["perm"] if wl.actorder else None)
    perm = prep["perm"]
    W0 = Wc.float().numpy().astype(np.float64)
    W0[:, prep["dead"]] = 0.0
    Wp = np.ascontiguousarray(W0[:, perm])
    codes_sw = np.ascontiguousarray(out["codes"][:, perm])
    r = oracle_pool.sweep_all_rows(Wp, np.ascontiguousarray(Uo), bits, g, codes_sw,
                                   out["zeros"])
    raw = float(np.mean(r["own"] == codes_sw))
    tie_rows = sorted({a[0] for a in r["adoptions"]})
    stats.update(all_rows=int(wl.rows), all_rows_raw_agreement=raw,
                 all_rows_ties_replayed=r["adopted"], all_rows_mismatched=r["mismatched"],
                 all_rows_tie_rows=len(tie_rows),
                 all_rows_tie_distances_max=max([a[3] for a in r["adoptions"]], default=0.0),
                 all_rows_codes_differing=int(np.count_nonzero(r["own"] != codes_sw)))
    _report(wl.name + ".all_rows", stats)
    assert r["mismatched"] == 0, r["mismatched"]
    assert np.array_equal(r["rep"], codes_sw)
    assert all(a[3] <= 1e-5 for a in r["adoptions"]), r["adoptions"][:8]
    assert raw >= 0.999, raw


@pytest.mark.parametrize("name", ["q_proj_7b", "down_proj_7b"])
def test_full_size_layer(name):
    """The bench workload (Llama-7B q_proj shape, 4-bit g128 act-order) and
    the 7B down-proj (n = 11008, 3-bit g128): U from the oracle in full."""
    wl = workloads.WORKLOADS[name]
    Wc, Xc, out = _run(wl)
    stats = {}
    _check_hessian(wl, Xc, out["H"], stats)
    prep = O.prepare(out["H"], np.zeros((1, wl.n)), wl.percdamp, wl.actorder,
                     forced_perm=out["perm"] if wl.actorder else None)
    Uo = O.upper_cholesky_of_inverse(prep["Hp"])
    Ug = out["U"]
    assert np.all(np.tril(Ug, -1) == 0)
    stats["u_rel"] = _rel(Ug.astype(np.float64), Uo)
    assert stats["u_rel"] <= 1e-4, stats["u_rel"]
    del prep
    _check_rows(wl, Wc, Xc, out, Uo, stats)
    if name == "q_proj_7b":
        _check_all_rows(wl, Wc, out, Uo, stats)
    _report(name, stats)


@pytest.mark.parametrize("block,linear", [(0, 4), (31, 6)])
def test_full_size_stack_linears(block, linear):
    """Two linears of the 7B-shaped stack at 65536 tokens: gate (11008 rows
    of 4096 inputs, more rows than any other case) and down (n = 11008)."""
    wl = workloads.stack_7b_workload(block, linear)
    Wc, Xc, out = _run(wl)
    stats = {}
    _check_hessian(wl, Xc, out["H"], stats)
    prep = O.prepare(out["H"], np.zeros((1, wl.n)), wl.percdamp, wl.actorder)
    Uo = O.upper_cholesky_of_inverse(prep["Hp"])
    stats["u_rel"] = _rel(out["U"].astype(np.float64), Uo)
    assert stats["u_rel"] <= 1e-4, stats["u_rel"]
    del prep
    _check_rows(wl, Wc, Xc, out, Uo, stats, k=10)
    _report(wl.name, stats)


def test_full_size_70b_down_proj():
    """W 8192 x 28672, X 28672 x 65536 with outliers x50 and the random-sign
    Hadamard rotation; 4-bit g128 act-order."""
    wl = workloads.WORKLOADS["down_proj_70b"]
    Wc, Xc, out = _run(wl)
    n = wl.n
    stats = {}
    _check_hessian(wl, Xc, out["H"], stats)
    Hg, Ug = out["H"], out["U"]
    prep = O.prepare_from_diagonal(np.diag(Hg), wl.percdamp, wl.actorder,
                                   forced_perm=out["perm"])
    out["diagH"] = np.diag(Hg).copy()
    # the oracle's own U by the pages' route (in-place LAPACK steps, fp64)
    Uo = O.upper_cholesky_of_inverse_inplace(O.damped_block(Hg, prep, 0, n, row_chunk=1024))
    del Hg, out["H"]
    assert not np.any(np.tril(Ug, -1))
    num = den = 0.0
    for r0 in range(0, n, 2048):
        d = Ug[r0:r0 + 2048].astype(np.float64) - Uo[r0:r0 + 2048]
        num += float(np.sum(d * d))
        den += float(np.sum(Uo[r0:r0 + 2048] * Uo[r0:r0 + 2048]))
    stats["u_rel"] = (num / den) ** 0.5
    assert stats["u_rel"] <= 1e-4, stats["u_rel"]
    del Ug, out["U"]
    _check_rows(wl, Wc, Xc, out, Uo, stats, k=6)
    _report(wl.name, stats)
