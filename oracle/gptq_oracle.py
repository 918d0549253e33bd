"""Plain, slow, fp64 CPU oracle of the GPTQ layer-wise quantizer.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import or call this module.  The CUDA
library never reaches it, and it imports nothing from the CUDA package:
the two share no code.

Source of every formula: the web page "GPTQ, with the code open"
(modelfoundations.com/notes/gptq), cited below by section title:

* § "What quantization is, and why anyone bothers" -- the ruler (grid):
  ``scale = (max - min) / (2^b - 1)``, the zero point rounded to a whole tick
  so that 0.0 is exactly representable, ``w_hat = scale * (q - zero)``.
* § "Measuring damage where it matters" -- ``H = 2 X X^T``.
* § "The repair rule" -- the Optimal Brain Surgeon update
  ``delta_F = -e / [H_F^-1]_qq * (H_F^-1)_{:,q}``.
* § "From one repair to a whole model" -- fixed left-to-right column order
  shared by all rows, the Cholesky factor whose rows hold every
  ``[H_F^-1]`` entry, the per-weight loss ``(w - q)^2 / (2 d^2)``, the lazy
  block of 128 columns, the per-row ruler fitted before any repair and the
  clamping of weights that drift off it.
* § "Paper vs. code" -- dead inputs zeroed, 1 % mean-diagonal damping,
  TF32 off (full fp32), asymmetric min-max ruler stretched to include zero,
  act-order (loudest columns first), a new ruler every 128 columns.

The page "What is GPTQ" (queryfeedz.com glossary), table "Key settings",
lists the bit widths, group sizes and act-order setting exercised here.

Readings where the pages are silent:

* Rounding is IEEE round-half-to-even, for the code and for the zero point;
  the code is ``clamp(rint(w / scale) + zero, 0, 2^b - 1)`` with true division.
* The integer decisions (zero point, code) are taken in binary32, the
  precision the page says the reference runs in (TF32 off, full 32-bit), the
  same precision the CUDA path uses; every other quantity here is fp64.
* An all-zero row or group (scale would be 0) uses the range [-1, +1].
* Order of the preparation steps: dead inputs, then act-order, then damping.
  Act-order is a stable sort on the descending diagonal.
* Group rulers are fitted when the sweep reaches the group's first column,
  from the current (already repaired) weights; under act-order a group is g
  consecutive columns of the sweep order.

Parity pins (tests/test_oracle_pins.py) tie every function below to values
the pages print or to mathematics fixed independently of this module.  The
one choice no pin can fix is the bit layout of the packed codes, which the
pages never give: ``pack_int4`` / ``pack_int3`` are pinned only as a
bijection (round trip) and against a bit-by-bit restatement of the layout --
parity unpinned as to the layout itself.
"""
from __future__ import annotations

import numpy as np

F32 = np.float32


# --------------------------------------------------------------------------
# Hessian  (page "GPTQ, with the code open", § "Measuring damage where it
# matters": H = 2 X X^T;  § "Paper vs. code": built over calibration batches)
# --------------------------------------------------------------------------
def hessian(X: np.ndarray, alpha: float = 2.0, token_chunk: int = 8192) -> np.ndarray:
    """H = alpha * X X^T in fp64, X given as features x tokens.

    The tokens are taken one calibration batch (``token_chunk`` columns) at a
    time and the batch products are summed, as the page describes H being
    built up over calibration batches.
    """
    X = np.asarray(X)
    n, ntok = X.shape
    H = np.zeros((n, n), dtype=np.float64)
    syrk = _blas_syrk()
    for t0 in range(0, ntok, token_chunk):
        Xc = X[:, t0:t0 + token_chunk].astype(np.float64)
        if syrk is not None and n >= 512:
            # the same product through BLAS's symmetric rank-k routine (upper half)
            Hu = syrk(1.0, np.asfortranarray(Xc))
            H += np.triu(Hu) + np.triu(Hu, 1).T
        else:
            H += Xc @ Xc.T
    return alpha * H


def _blas_syrk():
    try:
        from scipy.linalg.blas import dsyrk
    except Exception:  # pragma: no cover - scipy is optional
        return None
    return dsyrk


def hessian_entry(X: np.ndarray, i: int, j: int, alpha: float = 2.0) -> float:
    """One entry alpha * sum_t X[i,t] X[j,t] in fp64 (for sampled checks)."""
    return float(alpha * np.dot(X[i].astype(np.float64), X[j].astype(np.float64)))


# --------------------------------------------------------------------------
# The ruler  (§ "What quantization is, and why anyone bothers"; § "Paper vs.
# code": asymmetric min-max, range stretched to include zero)
# --------------------------------------------------------------------------
def fit_grid(wmin, wmax, bits: int, sym: bool = False):
    """Ruler for values spanning [wmin, wmax]; arrays broadcast.

    Returns ``(scale, zero)``: scale as binary32, zero as int64.  The range is
    first stretched to include 0.  The decisions are binary32 (module notes).

    ``sym``: the opt-in symmetric ruler (page "GPTQ, with the code open",
    § "Paper vs. code").  The pages give no formula; the reading taken is the
    plainest one: the range becomes [-m, m] with m = max(|min|, |max|), the
    same scale formula applies, and the zero point is the middle tick
    (2^b - 1 + 1) / 2, a whole tick, so 0.0 stays exactly representable.
    """
    maxq = F32(2 ** bits - 1)
    xmin = np.minimum(np.asarray(wmin, dtype=np.float64), 0.0).astype(F32)
    xmax = np.maximum(np.asarray(wmax, dtype=np.float64), 0.0).astype(F32)
    if sym:
        m = np.maximum(-xmin, xmax).astype(F32)
        xmin, xmax = (-m).astype(F32), m
    flat = (xmin == 0) & (xmax == 0)
    xmin = np.where(flat, F32(-1), xmin).astype(F32)
    xmax = np.where(flat, F32(1), xmax).astype(F32)
    scale = ((xmax - xmin).astype(F32) / maxq).astype(F32)
    if sym:
        zero = np.full(np.shape(scale), (2 ** bits) // 2, dtype=np.int64)
        return scale, zero
    zero_pre = ((-xmin).astype(F32) / scale).astype(F32)
    zero = np.rint(zero_pre).astype(np.int64)
    return scale, zero


def zero_prevalue(wmin, bits: int, scale) -> np.ndarray:
    """-xmin / scale before rounding (used to recognise rounding ties)."""
    xmin = np.minimum(np.asarray(wmin, dtype=np.float64), 0.0)
    return -xmin / np.asarray(scale, dtype=np.float64)


def quantize(w, scale, zero, bits: int) -> np.ndarray:
    """Tick index of w: clamp(rint(w / scale) + zero, 0, 2^b - 1), binary32 division."""
    maxq = 2 ** bits - 1
    t = (np.asarray(w, dtype=np.float64).astype(F32) / np.asarray(scale, dtype=F32)).astype(F32)
    return np.clip(np.rint(t).astype(np.int64) + np.asarray(zero, dtype=np.int64), 0, maxq)


def dequantize(q, scale, zero) -> np.ndarray:
    """w_hat = scale * (q - zero), exact in fp64 (a 24-bit by 9-bit product)."""
    return np.asarray(scale, dtype=np.float64) * (np.asarray(q, dtype=np.int64)
                                                   - np.asarray(zero, dtype=np.int64))


# --------------------------------------------------------------------------
# Preparation  (§ "Paper vs. code": dead inputs, damping, act-order)
# --------------------------------------------------------------------------
def is_near_tie_order(d: np.ndarray, order, rtol: float) -> bool:
    """True if ``order`` is a permutation that sorts ``d`` descending except
    between entries within a relative ``rtol`` of each other."""
    order = np.asarray(order, dtype=np.int64)
    n = d.shape[0]
    if order.shape != (n,) or not np.array_equal(np.sort(order), np.arange(n)):
        return False
    a, b = d[order[:-1]], d[order[1:]]
    return bool(np.all(a >= b - rtol * np.maximum(np.abs(a), np.abs(b))))


def prepare_from_diagonal(d: np.ndarray, percdamp: float = 0.01, actorder: bool = False,
                          forced_perm=None, perm_rtol: float = 1e-5):
    """The part of the preparation that diag(H) alone fixes.

    Dead inputs are the zero diagonal entries (their diagonal becomes 1);
    with act-order the sweep order is a stable sort by descending diagonal;
    the damping is ``lam = percdamp * mean`` of the (fixed, reordered)
    diagonal.  Returns dict ``dead``, ``perm``, ``lam`` and ``d`` (the fixed
    diagonal, original order).  ``forced_perm`` as in ``prepare``.
    """
    d = np.array(d, dtype=np.float64, copy=True)
    n = d.shape[0]
    dead = d == 0.0
    d[dead] = 1.0
    if actorder:
        perm = np.argsort(-d, kind="stable")
        if forced_perm is not None:
            if not is_near_tie_order(d, forced_perm, perm_rtol):
                raise ValueError("forced act-order is not a near-tie reordering of diag(H)")
            perm = np.asarray(forced_perm, dtype=np.int64)
    else:
        perm = np.arange(n)
    lam = percdamp * float(np.mean(d[perm]))
    return {"dead": dead, "perm": perm, "lam": lam, "d": d}


def damped_block(H: np.ndarray, prep: dict, k0: int, k1: int,
                 row_chunk: int | None = None) -> np.ndarray:
    """Rows and columns [k0, k1) (sweep order) of the prepared matrix
    H' = H[perm][:, perm] + lam I, dead diagonal entries set to 1 first.

    ``row_chunk``: gather that many rows at a time into the fp64 result, so
    no full-size temporary of H's own dtype is made (for n in the tens of
    thousands); the values are the same."""
    idx = np.asarray(prep["perm"])[k0:k1]
    m = k1 - k0
    if row_chunk is None:
        B = np.array(H[np.ix_(idx, idx)], dtype=np.float64)
    else:
        B = np.empty((m, m), dtype=np.float64)
        for r0 in range(0, m, row_chunk):
            B[r0:r0 + row_chunk] = H[idx[r0:r0 + row_chunk]][:, idx]
    dd = np.asarray(prep["dead"])[idx]
    B[np.arange(m)[dd], np.arange(m)[dd]] = 1.0
    B[np.arange(m), np.arange(m)] += prep["lam"]
    return B


def prepare(H: np.ndarray, W: np.ndarray, percdamp: float = 0.01, actorder: bool = False,
            forced_perm=None, perm_rtol: float = 1e-5):
    """Dead inputs -> act-order -> damping.

    Returns dict with ``dead`` (bool[n]), ``perm`` (int64[n], perm[k] = the
    original column quantized k-th), ``Hp`` (damped H in sweep order),
    ``W0`` (dead-zeroed W, original order), ``Wp`` (W0 in sweep order) and
    ``lam`` (the damping added to every diagonal entry).

    ``forced_perm`` replays another run's act-order: it is adopted when it
    orders diag(H) descending up to ties within ``perm_rtol`` (two Hessians
    summed in different precisions may order such near-equal columns either
    way); otherwise ValueError.
    """
    H = np.asarray(H, dtype=np.float64)
    W0 = np.array(W, dtype=np.float64, copy=True)
    n = H.shape[0]
    prep = prepare_from_diagonal(np.diag(H), percdamp, actorder, forced_perm, perm_rtol)
    W0[:, prep["dead"]] = 0.0
    Hp = damped_block(H, prep, 0, n)
    perm = prep["perm"]
    return {"dead": prep["dead"], "perm": perm, "Hp": Hp, "W0": W0, "Wp": W0[:, perm],
            "lam": prep["lam"]}


def upper_cholesky_of_inverse(Hp: np.ndarray) -> np.ndarray:
    """U upper triangular with Hp^-1 = U^T U.

    The page's route (§ "From one repair to a whole model"): Cholesky of H,
    the inverse from that factor, then the upper Cholesky factor of the
    inverse.  Raises numpy.linalg.LinAlgError if Hp is not positive definite.
    """
    L = np.linalg.cholesky(Hp)                 # Hp = L L^T
    Linv = np.linalg.inv(L)
    Hinv = Linv.T @ Linv                       # Hp^-1
    Hinv = 0.5 * (Hinv + Hinv.T)
    return np.linalg.cholesky(Hinv).T          # Hinv = U^T U


def upper_cholesky_of_inverse_inplace(Hp: np.ndarray) -> np.ndarray:
    """The same U as ``upper_cholesky_of_inverse``, by the same route, for
    orders where a general inverse and a full product are too slow (n in the
    tens of thousands): every step is the LAPACK routine for it, on one fp64
    buffer that is overwritten (``Hp`` must be C-contiguous fp64; it becomes
    U).  Steps, in the page's order (§ "From one repair to a whole model"):
      Cholesky           Hp = L L^T                     (dpotrf)
      inverse of L       Linv = L^-1, triangular        (dtrtri)
      the inverse        Hp^-1 = Linv^T Linv            (dlauum)
      Cholesky again     Hp^-1 = L2 L2^T, and U = L2^T  (dpotrf)
    U is upper with Hp^-1 = U^T U; that factor is unique, so this equals the
    general-inverse form.  Raises numpy.linalg.LinAlgError if a step fails.

    The buffer is handed to LAPACK as its transpose (a Fortran-ordered view
    of the same memory), so no copy is made: the lower triangle of that view
    is the upper triangle of ``Hp``.
    """
    from scipy.linalg import lapack

    if Hp.dtype != np.float64 or not Hp.flags.c_contiguous:
        raise ValueError("Hp must be a C-contiguous float64 array")
    F = Hp.T                                   # Fortran view; F == Hp (symmetric)
    for name, fn, kw in (("dpotrf", lapack.dpotrf, {"lower": 1, "overwrite_a": 1, "clean": 0}),
                         ("dtrtri", lapack.dtrtri, {"lower": 1, "overwrite_c": 1}),
                         ("dlauum", lapack.dlauum, {"lower": 1, "overwrite_c": 1}),
                         ("dpotrf", lapack.dpotrf, {"lower": 1, "overwrite_a": 1, "clean": 0})):
        out, info = fn(F, **kw)
        if info != 0:
            raise np.linalg.LinAlgError(f"{name} failed, info={info}")
        if not np.shares_memory(out, Hp):
            raise RuntimeError(f"{name} did not work in place")
    # U = L2^T: the lower triangle of F is the upper triangle of Hp; clear the rest
    n = Hp.shape[0]
    for r0 in range(0, n, 1024):
        r1 = min(n, r0 + 1024)
        blk = Hp[r0:r1]
        rr = np.arange(r0, r1)[:, None]
        blk[np.arange(n)[None, :] < rr] = 0.0
    return Hp


# --------------------------------------------------------------------------
# The column sweep  (§ "The repair rule"; § "From one repair to a whole model")
# --------------------------------------------------------------------------
def _near_half(t, tau: float) -> np.ndarray:
    t = np.asarray(t, dtype=np.float64)
    return np.abs((t - np.floor(t)) - 0.5) < tau


def _half_distance(t) -> float:
    t = float(t)
    return abs((t - np.floor(t)) - 0.5)


def sweep(Wp: np.ndarray, U: np.ndarray, bits: int, group_size: int = -1,
          forced_codes=None, forced_zeros=None, tau: float = 1e-3, trace=None,
          adoptions=None, sym: bool = False):
    """Unblocked GPTQ sweep over the columns of Wp (already in sweep order).

    For each column j, left to right, for every row at once:
      * at the first column of a group, fit the group's ruler on the current
        weights (per-row rulers, group_size <= 0, are fitted before the loop
        on the unrepaired weights);
      * q = quantize(w_j); e = w_j - w_hat; loss += e^2 / (2 U_jj^2);
      * err = e / U_jj;  W[:, j+1:] -= err (outer) U[j, j+1:].

    ``forced_codes`` / ``forced_zeros`` (sweep order) replay another run's
    choices: where this run's code or zero point differs from the forced one
    and its pre-rounding value lies within ``tau`` ticks of a half-integer
    (a rounding tie that two correct implementations may break either way),
    the forced value is adopted; any other difference is counted as a
    mismatch and this run's own value is kept.  ``trace(j, W)`` is called
    after column j's repair with the working matrix.  ``adoptions``, if a
    list, receives ``(row, column, "code" | "zero", distance of the
    pre-rounding value from the half-integer, in ticks)`` for each adoption.

    Returns a dict: codes (int64 rows x n), scales (float32 rows x G), zeros
    (int64 rows x G), Wq (fp64 rows x n), err (fp64 rows x n, the e/U_jj
    terms), loss (fp64 rows), adopted (int), mismatched (int).
    """
    W = np.array(Wp, dtype=np.float64, copy=True)
    rows, n = W.shape
    maxq = 2 ** bits - 1
    g = group_size if group_size > 0 else n
    G = (n + g - 1) // g
    codes = np.zeros((rows, n), dtype=np.int64)
    scales = np.zeros((rows, G), dtype=F32)
    zeros = np.zeros((rows, G), dtype=np.int64)
    Wq = np.zeros((rows, n), dtype=np.float64)
    Err = np.zeros((rows, n), dtype=np.float64)
    loss = np.zeros(rows, dtype=np.float64)
    adopted = 0
    mismatched = 0

    scale = zero = None
    for j in range(n):
        if j % g == 0:
            blk = W[:, j:j + g]
            scale, zero = fit_grid(blk.min(axis=1), blk.max(axis=1), bits, sym)
            if forced_zeros is not None and not sym:
                fz = np.asarray(forced_zeros)[:, j // g].astype(np.int64)
                diff = fz != zero
                zp = zero_prevalue(blk.min(axis=1), bits, scale)
                tie = _near_half(zp, tau)
                adopted += int(np.count_nonzero(diff & tie))
                if adoptions is not None:
                    for r in np.nonzero(diff & tie)[0]:
                        adoptions.append((int(r), j, "zero", _half_distance(zp[r])))
                mismatched += int(np.count_nonzero(diff & ~tie))
                zero = np.where(diff & tie, fz, zero)
            scales[:, j // g] = scale
            zeros[:, j // g] = zero
        w = W[:, j]
        q = quantize(w, scale, zero, bits)
        if forced_codes is not None:
            fq = np.asarray(forced_codes)[:, j].astype(np.int64)
            diff = fq != q
            t = w / scale.astype(np.float64)
            tie = _near_half(t, tau)
            adopted += int(np.count_nonzero(diff & tie))
            if adoptions is not None:
                for r in np.nonzero(diff & tie)[0]:
                    adoptions.append((int(r), j, "code", _half_distance(t[r])))
            mismatched += int(np.count_nonzero(diff & ~tie))
            q = np.where(diff & tie, fq, q)
        codes[:, j] = q
        what = dequantize(q, scale, zero)
        Wq[:, j] = what
        e = w - what
        d = U[j, j]
        loss += e * e / (2.0 * d * d)
        err = e / d
        Err[:, j] = err
        W[:, j + 1:] -= np.outer(err, U[j, j + 1:])
        if trace is not None:
            trace(j, W)
    del maxq
    return {"codes": codes, "scales": scales, "zeros": zeros, "Wq": Wq, "err": Err,
            "loss": loss, "adopted": adopted, "mismatched": mismatched}


def sweep_blocked(Wp: np.ndarray, U: np.ndarray, bits: int, group_size: int, block: int,
                  sym: bool = False):
    """The lazy-batch form (§ "From one repair to a whole model"): repairs
    inside the current block of ``block`` columns at once, the repair of every
    later column deferred to one product per block.  Used only to show that
    it equals ``sweep``; requires block % g == 0 or g % block == 0.
    """
    W = np.array(Wp, dtype=np.float64, copy=True)
    rows, n = W.shape
    g = group_size if group_size > 0 else n
    if group_size > 0 and not (block % g == 0 or g % block == 0):
        raise ValueError("group size and block must divide one another")
    G = (n + g - 1) // g
    codes = np.zeros((rows, n), dtype=np.int64)
    scales = np.zeros((rows, G), dtype=F32)
    zeros = np.zeros((rows, G), dtype=np.int64)
    Wq = np.zeros((rows, n), dtype=np.float64)
    loss = np.zeros(rows, dtype=np.float64)
    scale = zero = None
    for i1 in range(0, n, block):
        i2 = min(i1 + block, n)
        Wb = W[:, i1:i2].copy()
        Errb = np.zeros((rows, i2 - i1))
        for jj in range(i2 - i1):
            j = i1 + jj
            if j % g == 0:
                # a group longer than the block starts on a block boundary
                # (jj == 0): no repair of this block has run yet, and the
                # columns past the block hold every earlier block's repair
                grp = np.concatenate([Wb[:, jj:], W[:, i2:j + g]], axis=1)[:, :g]
                scale, zero = fit_grid(grp.min(axis=1), grp.max(axis=1), bits, sym)
                scales[:, j // g] = scale
                zeros[:, j // g] = zero
            w = Wb[:, jj]
            q = quantize(w, scale, zero, bits)
            codes[:, j] = q
            what = dequantize(q, scale, zero)
            Wq[:, j] = what
            e = w - what
            d = U[j, j]
            loss += e * e / (2.0 * d * d)
            err = e / d
            Errb[:, jj] = err
            Wb[:, jj + 1:] -= np.outer(err, U[j, j + 1:i2])
        W[:, i1:i2] = Wb
        W[:, i2:] -= Errb @ U[i1:i2, i2:]
    return {"codes": codes, "scales": scales, "zeros": zeros, "Wq": Wq, "loss": loss}


def rtn(Wp: np.ndarray, bits: int, group_size: int = -1, sym: bool = False):
    """Round-to-nearest on the same ruler, no repair (§ "The obvious approach,
    and how it fails").  Groups are consecutive columns of Wp's order."""
    W = np.asarray(Wp, dtype=np.float64)
    rows, n = W.shape
    g = group_size if group_size > 0 else n
    G = (n + g - 1) // g
    codes = np.zeros((rows, n), dtype=np.int64)
    scales = np.zeros((rows, G), dtype=F32)
    zeros = np.zeros((rows, G), dtype=np.int64)
    for k in range(G):
        blk = W[:, k * g:(k + 1) * g]
        s, z = fit_grid(blk.min(axis=1), blk.max(axis=1), bits, sym)
        scales[:, k], zeros[:, k] = s, z
        codes[:, k * g:(k + 1) * g] = quantize(blk, s[:, None], z[:, None], bits)
    return {"codes": codes, "scales": scales, "zeros": zeros}


# --------------------------------------------------------------------------
# Whole layer
# --------------------------------------------------------------------------
def gptq_layer(W: np.ndarray, H: np.ndarray, bits: int = 4, group_size: int = -1,
               percdamp: float = 0.01, actorder: bool = False,
               forced_codes=None, forced_zeros=None, tau: float = 1e-3,
               forced_perm=None, perm_rtol: float = 1e-5, sym: bool = False):
    """GPTQ on one linear layer, given its Hessian H (n x n) and weights W.

    Returns the sweep's dict plus, in ORIGINAL column order: ``codes_orig``,
    ``Wq_orig`` and ``g_idx`` (group of each original column), and the
    preparation's ``dead``, ``perm``, ``lam``, ``U``, ``W0``.  Forced
    codes/zeros are given in sweep order (see ``sweep``); ``forced_perm`` as
    in ``prepare``; ``sym`` selects the symmetric ruler (``fit_grid``).
    """
    prep = prepare(H, W, percdamp, actorder, forced_perm, perm_rtol)
    U = upper_cholesky_of_inverse(prep["Hp"])
    res = sweep(prep["Wp"], U, bits, group_size, forced_codes, forced_zeros, tau, sym=sym)
    perm = prep["perm"]
    n = perm.shape[0]
    g = group_size if group_size > 0 else n
    codes_orig = np.empty_like(res["codes"])
    codes_orig[:, perm] = res["codes"]
    Wq_orig = np.empty_like(res["Wq"])
    Wq_orig[:, perm] = res["Wq"]
    g_idx = np.empty(n, dtype=np.int64)
    g_idx[perm] = np.arange(n) // g
    res.update(codes_orig=codes_orig, Wq_orig=Wq_orig, g_idx=g_idx, U=U, **prep)
    return res


def objective_direct(W0: np.ndarray, Wq: np.ndarray, X: np.ndarray) -> float:
    """||W0 X - Wq X||_F^2 (page "What is GPTQ"-style objective, the layer
    output error on the calibration inputs), fp64."""
    D = np.asarray(W0, dtype=np.float64) - np.asarray(Wq, dtype=np.float64)
    R = D @ np.asarray(X, dtype=np.float64)
    return float(np.sum(R * R))


def objective_from_hessian(W0: np.ndarray, Wq: np.ndarray, H: np.ndarray) -> float:
    """The same objective through H = 2 X X^T:  1/2 * sum_r d_r H d_r^T."""
    D = np.asarray(W0, dtype=np.float64) - np.asarray(Wq, dtype=np.float64)
    return float(0.5 * np.sum((D @ np.asarray(H, dtype=np.float64)) * D))


# --------------------------------------------------------------------------
# Storage: packed codes and dequantization  (§ "What quantization is, and why
# anyone bothers": store the tick index plus the ruler; one multiply back)
# Layout (not on the pages): int4 -- column 8i+k of a row in bits [4k, 4k+4)
# of 32-bit word i; int3 -- column 32i+k in bits [3k, 3k+3) of the 96-bit
# little-endian word formed by 32-bit words 3i, 3i+1, 3i+2.
# --------------------------------------------------------------------------
def pack_int4(codes: np.ndarray) -> np.ndarray:
    c = np.asarray(codes, dtype=np.uint64)
    rows, n = c.shape
    if n % 8:
        raise ValueError("n must be a multiple of 8")
    c = c.reshape(rows, n // 8, 8)
    word = np.zeros((rows, n // 8), dtype=np.uint64)
    for k in range(8):
        word |= (c[:, :, k] & 0xF) << np.uint64(4 * k)
    return word.astype(np.uint32)


def unpack_int4(packed: np.ndarray, n: int) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint64)
    rows = p.shape[0]
    out = np.zeros((rows, n // 8, 8), dtype=np.int64)
    for k in range(8):
        out[:, :, k] = ((p >> np.uint64(4 * k)) & np.uint64(0xF)).astype(np.int64)
    return out.reshape(rows, n)


def pack_int3(codes: np.ndarray) -> np.ndarray:
    c = np.asarray(codes, dtype=np.int64)
    rows, n = c.shape
    if n % 32:
        raise ValueError("n must be a multiple of 32")
    c = c.reshape(rows, n // 32, 32)
    big = np.zeros((rows, n // 32), dtype=object)   # exact 96-bit integers
    for k in range(32):
        big = big + ((c[:, :, k] & 7).astype(object) << (3 * k))
    out = np.zeros((rows, n // 32, 3), dtype=np.uint64)
    for w in range(3):
        out[:, :, w] = np.vectorize(lambda v, w=w: (v >> (32 * w)) & 0xFFFFFFFF,
                                    otypes=[np.uint64])(big)
    return out.reshape(rows, 3 * n // 32).astype(np.uint32)


def unpack_int3(packed: np.ndarray, n: int) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint64).reshape(-1, n // 32, 3)
    rows = p.shape[0]
    big = (p[:, :, 0].astype(object) | (p[:, :, 1].astype(object) << 32)
           | (p[:, :, 2].astype(object) << 64))
    out = np.zeros((rows, n // 32, 32), dtype=np.int64)
    for k in range(32):
        out[:, :, k] = np.vectorize(lambda v, k=k: (v >> (3 * k)) & 7, otypes=[np.int64])(big)
    return out.reshape(rows, n)


def bf16_round(x32: np.ndarray) -> np.ndarray:
    """binary32 -> bfloat16 with round-half-to-even, returned as uint16 bits."""
    u = np.asarray(x32, dtype=F32).view(np.uint32).astype(np.uint64)
    bias = np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))
    return ((u + bias) >> np.uint64(16)).astype(np.uint16)


def dequant(packed: np.ndarray, bits: int, n: int, scales: np.ndarray, zeros: np.ndarray,
            group_size: int = -1, g_idx=None, out: str = "f32") -> np.ndarray:
    """w_hat[r, c] = scale[r, G(c)] * (code[r, c] - zero[r, G(c)]) in binary32
    (one rounding of the exact product); ``out='bf16'`` then rounds that to
    bfloat16 (round-half-to-even) and returns the uint16 bit patterns.
    G(c) = g_idx[c] if given, else c // group_size (0 for per-row rulers)."""
    if bits == 4:
        q = unpack_int4(packed, n)
    elif bits == 3:
        q = unpack_int3(packed, n)
    else:
        raise ValueError("bits must be 3 or 4")
    if g_idx is not None:
        G = np.asarray(g_idx, dtype=np.int64)
    elif group_size > 0:
        G = np.arange(n) // group_size
    else:
        G = np.zeros(n, dtype=np.int64)
    s = np.asarray(scales, dtype=F32)[:, G]
    z = np.asarray(zeros, dtype=np.int64)[:, G]
    w = dequantize(q, s, z).astype(F32)
    if out == "bf16":
        return bf16_round(w)
    return w


# --------------------------------------------------------------------------
# Consumer of the packed codes (page "GPTQ, with the code open", section
# "Claims & evidence": generation at batch size 1 reads the packed weights)
# --------------------------------------------------------------------------
def dequant_matvec(packed: np.ndarray, bits: int, n: int, scales: np.ndarray,
                   zeros: np.ndarray, x, group_size: int = -1, g_idx=None, perm=None):
    """y = x w_hat^T in fp64 for activations x (batch x n, or n), with w_hat
    the binary32 dequantized weights of ``dequant``.  With ``perm`` the
    packed columns are in sweep order: column k pairs with x[:, perm[k]].
    Returns ``(y, mag)`` where ``mag = |x| |w_hat|^T`` (the sum of |terms|,
    for error bounds)."""
    W = dequant(packed, bits, n, scales, zeros, group_size, g_idx).astype(np.float64)
    X = np.atleast_2d(np.asarray(x, dtype=np.float64))
    if perm is not None:
        X = X[:, np.asarray(perm, dtype=np.int64)]
    return X @ W.T, np.abs(X) @ np.abs(W).T
