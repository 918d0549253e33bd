"""Helpers shared by the GPU parity tests: run the CUDA path through the
binding, run the oracle on the same bytes, compare."""
from __future__ import annotations

import numpy as np
import torch

import post_weight_quantization_25_b200 as G
from oracle import gptq_oracle as O


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def device_x(X: torch.Tensor) -> torch.Tensor:
    """Copy X to the GPU with a row stride that is a multiple of 16 bytes."""
    n, ntok = X.shape
    per16 = 16 // X.element_size()
    ld = max(per16, (ntok + per16 - 1) // per16 * per16)
    buf = torch.zeros(n, ld, dtype=X.dtype, device="cuda")
    buf[:, :ntok] = X.cuda()
    return buf[:, :ntok]


def gpu_layer(W, X, bits, g, percdamp, actorder, H=None, sym=False):
    """The CUDA path for one layer; returns numpy results (original order)."""
    Wd = W.cuda()
    rows, n = W.shape
    if H is None:
        H = torch.zeros(n, n, dtype=torch.float32, device="cuda")
        G.gptq_hessian_accumulate(H, device_x(X))
    cfg = G.make_config(bits, g, percdamp, actorder, sym=sym)
    U, perm, dead, info = G.gptq_cholesky_inverse(H, percdamp, actorder)
    q = G.gptq_quantize_layer(Wd, U, perm, dead, cfg, want_wq=True, want_loss=True)
    torch.cuda.synchronize()
    return {"H": H, "U": to_np(U), "perm": perm.cpu().numpy().astype(np.int64),
            "dead": dead.cpu().numpy().astype(bool), "info": int(info.item()),
            "codes": q["codes"].cpu().numpy().astype(np.int64),
            "scales": q["scales"].cpu().numpy(), "zeros": q["zeros"].cpu().numpy().astype(np.int64),
            "g_idx": q["g_idx"].cpu().numpy().astype(np.int64), "Wq": q["Wq"].cpu().numpy(),
            "row_loss": q["row_loss"].cpu().numpy().astype(np.float64)}


def compare_layer(gpu, W, X, bits, g, percdamp, actorder, H_oracle=None, min_agree=0.999,
                  sym=False):
    """Oracle on the same bytes; the GPU's act-order and codes are replayed
    where they sit on ties.  Asserts the agreed tolerances; returns stats."""
    Wn = to_np(W).astype(np.float64)
    Xn = to_np(X).astype(np.float64)
    Ho = O.hessian(Xn) if H_oracle is None else H_oracle
    fperm = gpu["perm"] if actorder else None
    own = O.gptq_layer(Wn, Ho, bits, g, percdamp, actorder, forced_perm=fperm, sym=sym)
    perm = own["perm"]
    codes_sw = gpu["codes"][:, perm]
    prep = O.prepare(Ho, Wn, percdamp, actorder, forced_perm=fperm)
    adoptions = []
    sw = O.sweep(prep["Wp"], own["U"], bits, g, forced_codes=codes_sw,
                 forced_zeros=gpu["zeros"], adoptions=adoptions, sym=sym)
    rep = O.gptq_layer(Wn, Ho, bits, g, percdamp, actorder, forced_codes=codes_sw,
                       forced_zeros=gpu["zeros"], forced_perm=fperm, sym=sym)
    assert gpu["info"] == 0
    assert np.array_equal(gpu["dead"], own["dead"])
    assert rep["mismatched"] == 0, rep["mismatched"]
    assert np.array_equal(rep["codes_orig"], gpu["codes"])
    assert sw["adopted"] == rep["adopted"]
    # every difference starts at a value within 1e-5 tick of a half-integer
    assert all(a[3] <= 1e-5 for a in adoptions), adoptions
    # raw agreement, over the rows without a replayed tie (a tie decided the
    # other way changes the rest of its row; see the full-size tests)
    agree = float(np.mean(own["codes_orig"] == gpu["codes"]))
    tie_rows = sorted({a[0] for a in adoptions})
    clean = np.ones(gpu["codes"].shape[0], dtype=bool)
    clean[tie_rows] = False
    agree_clean = float(np.mean(own["codes_orig"][clean] == gpu["codes"][clean])) if clean.any() \
        else 1.0
    assert agree_clean >= min_agree, (agree_clean, agree, tie_rows)
    # rulers
    stol = 1e-6 if g <= 0 else 1e-4
    np.testing.assert_allclose(gpu["scales"], rep["scales"], rtol=stol)
    assert np.array_equal(gpu["zeros"], rep["zeros"])
    assert np.array_equal(gpu["g_idx"], rep["g_idx"])
    # the dequantized weights are one fp32 multiply of the GPU's own ruler
    sc = gpu["scales"][:, gpu["g_idx"]]
    zz = gpu["zeros"][:, gpu["g_idx"]]
    exact = (sc.astype(np.float64) * (gpu["codes"] - zz)).astype(np.float32)
    assert np.array_equal(gpu["Wq"], exact)
    # objective ||W0 X - Wq X||^2
    e_gpu = O.objective_direct(own["W0"], gpu["Wq"], Xn)
    e_orc = O.objective_direct(own["W0"], rep["Wq_orig"], Xn)
    assert abs(e_gpu - e_orc) <= 1e-3 * e_orc, (e_gpu, e_orc)
    np.testing.assert_allclose(gpu["row_loss"].sum(), rep["loss"].sum(), rtol=1e-3)
    return {"agree": agree, "agree_without_tie_rows": agree_clean, "adopted": rep["adopted"],
            "tie_rows": tie_rows, "E_gpu": e_gpu, "E_oracle": e_orc}
