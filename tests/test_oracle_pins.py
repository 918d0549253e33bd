"""Pins of the fp64 oracle against what the pages and the mathematics fix.

Every test here is CPU-only.  Each one is chosen so that a plausible mistake
in the oracle (a dropped term, a flipped sign, a wrong index, a transposed
operand) makes at least one of them fail; ``test_planted_mistakes_are_caught``
plants such mistakes and checks that they are caught.
"""
import json
import os

import numpy as np
import pytest
import torch

from oracle import gptq_oracle as O
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rand_spd(n, seed, ntok=None):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((n, ntok or 3 * n))
    return 2.0 * X @ X.T, X


# ---------------------------------------------------------------- the ruler
def test_worked_grid_from_page():
    g = _golden("worked_grid.json")
    row = np.array([g["row_min"], -0.3, 0.05, g["row_max"]])
    scale, zero = O.fit_grid(row.min(), row.max(), g["bits"])
    assert abs(float(scale) - g["scale"]) <= float(np.spacing(np.float32(g["scale"])))
    assert int(zero) == g["zero"]
    ticks = O.dequantize(np.arange(16), scale, zero)
    assert ticks[g["zero"]] == 0.0                       # zero exactly representable
    np.testing.assert_allclose(ticks, g["ticks"], atol=1e-6)
    # every weight of the row lands on its nearest tick
    q = O.quantize(row, scale, zero, g["bits"])
    assert np.all(np.abs(O.dequantize(q, scale, zero) - row) <= float(scale) / 2 + 1e-7)


def test_grid_range_includes_zero_and_edges():
    s, z = O.fit_grid(0.1, 0.7, 4)             # all positive: stretched down to 0
    assert int(z) == 0 and abs(float(s) - 0.7 / 15) < 1e-8
    s, z = O.fit_grid(-0.9, -0.2, 3)           # all negative: stretched up to 0
    assert int(z) == 7 and abs(float(s) - 0.9 / 7) < 1e-8
    s, z = O.fit_grid(0.0, 0.0, 4)             # flat row: range [-1, 1]
    assert float(s) > 0 and O.dequantize(O.quantize(0.0, s, z, 4), s, z) == 0.0
    # drifted weights clamp to the end ticks
    s, z = O.fit_grid(-0.8, 0.4, 4)
    assert int(O.quantize(5.0, s, z, 4)) == 15 and int(O.quantize(-5.0, s, z, 4)) == 0


def test_symmetric_ruler_closed_form():
    """The opt-in symmetric ruler (page 'GPTQ, with the code open', section
    'Paper vs. code'): range [-m, m] with m = max(|min|, |max|), the same
    step formula, zero point on the middle tick, so 0.0 is exact."""
    s, z = O.fit_grid(-0.8, 0.4, 4, sym=True)
    assert int(z) == 8
    assert float(s) == float(np.float32(np.float32(1.6) / np.float32(15)))
    ticks = O.dequantize(np.arange(16), s, z)
    assert ticks[8] == 0.0 and ticks[0] == -8 * float(s) and ticks[15] == 7 * float(s)
    assert int(O.quantize(0.4, s, z, 4)) == 12            # rint(3.75) + 8
    assert int(O.quantize(-0.8, s, z, 4)) == 0            # rint(-7.5) = -8 (to even)
    # all-positive range: stretched to [0, 0.5], then mirrored to [-0.5, 0.5]
    s2, z2 = O.fit_grid(0.1, 0.5, 4, sym=True)
    assert int(z2) == 8 and float(s2) == float(np.float32(np.float32(1.0) / np.float32(15)))
    # 3 bits: middle tick 4; flat range -> [-1, 1]
    s3, z3 = O.fit_grid(0.0, 0.0, 3, sym=True)
    assert int(z3) == 4 and float(s3) == float(np.float32(np.float32(2.0) / np.float32(7)))
    # only |min| and |max| matter: mirrored ranges give the same ruler
    for a, b in ((0.3, 0.7), (0.7, 0.3), (0.0, 0.2)):
        assert O.fit_grid(-a, b, 4, sym=True) == O.fit_grid(-b, a, 4, sym=True)
    # the asymmetric ruler of the same range differs (zero 10, step 0.08)
    sa, za = O.fit_grid(-0.8, 0.4, 4)
    assert int(za) == 10 and float(sa) != float(s)


def test_symmetric_ruler_in_the_sweep():
    """Blocked and unblocked sweeps agree with the symmetric ruler, and with
    H proportional to I the sweep is round-to-nearest on the same ruler."""
    W, X = _layer(5, 24, 96, seed=808)
    prep = O.prepare(O.hessian(X), W, 0.01, True)
    U = O.upper_cholesky_of_inverse(prep["Hp"])
    for g in (-1, 8):
        ref = O.sweep(prep["Wp"], U, 4, g, sym=True)
        assert np.all(ref["zeros"] == 8)
        for B in (4, 8, 24):
            if g > 0 and not (B % g == 0 or g % B == 0):
                continue
            b = O.sweep_blocked(prep["Wp"], U, 4, g, B, sym=True)
            assert np.array_equal(b["codes"], ref["codes"])
            np.testing.assert_allclose(b["Wq"], ref["Wq"], rtol=0, atol=1e-12)
    n = 16
    Xi = np.concatenate([np.eye(n)] * 3, axis=1) * 1.5
    Wn = np.random.default_rng(9).normal(0, 0.02, (4, n))
    r = O.gptq_layer(Wn, O.hessian(Xi), 3, 8, 0.01, False, sym=True)
    base = O.rtn(r["W0"], 3, 8, sym=True)
    assert np.array_equal(r["codes_orig"], base["codes"])
    assert np.all(r["zeros"] == 4)


def test_rounding_is_half_to_even():
    s, z = np.float32(1.0), 0
    assert list(O.quantize(np.array([0.5, 1.5, 2.5, 3.5]), s, z, 4)) == [0, 2, 2, 4]


def test_rtn_error_bound_and_group_layout():
    rng = np.random.default_rng(3)
    W = rng.normal(0, 0.02, (5, 64))
    r = O.rtn(W, 4, 16)
    assert r["scales"].shape == (5, 4)
    for k in range(4):
        blk = W[:, 16 * k:16 * (k + 1)]
        wq = O.dequantize(r["codes"][:, 16 * k:16 * (k + 1)], r["scales"][:, k:k + 1],
                          r["zeros"][:, k:k + 1])
        assert np.all(np.abs(wq - blk) <= r["scales"][:, k:k + 1] / 2 + 1e-9)


# ---------------------------------------------------------------- Hessian
def test_hessian_closed_form_tiny():
    rng = np.random.default_rng(0)
    X = rng.standard_normal((3, 7)).astype(np.float32)
    H = O.hessian(X, token_chunk=2)
    for i in range(3):
        for j in range(3):
            s = 0.0
            for t in range(7):
                s += float(X[i, t]) * float(X[j, t])
            assert abs(H[i, j] - 2 * s) < 1e-12 * max(1.0, abs(s))
    assert O.hessian_entry(X, 1, 2) == pytest.approx(H[1, 2], rel=1e-14)


def test_hessian_finite_difference():
    """Page 'GPTQ, with the code open', 'Measuring damage where it matters':
    H = 2 X X^T is exactly the Hessian of the layer output error
    (finite-difference check, relative error 1e-7)."""
    rng = np.random.default_rng(1)
    n, N = 5, 40
    X = rng.standard_normal((n, N))
    w0 = rng.standard_normal(n)
    H = O.hessian(X)

    def E(w):
        r = (w - w0) @ X
        return float(r @ r)

    h = 1e-3
    w = rng.standard_normal(n)
    Hfd = np.zeros((n, n))
    for i in range(n):
        for j in range(n):
            ei = np.eye(n)[i] * h
            ej = np.eye(n)[j] * h
            Hfd[i, j] = (E(w + ei + ej) - E(w + ei) - E(w + ej) + E(w)) / h ** 2
    assert np.linalg.norm(Hfd - H) / np.linalg.norm(H) < 1e-7


# ---------------------------------------------------------------- U
def test_upper_cholesky_of_inverse_definition():
    H, _ = _rand_spd(9, 4)
    U = O.upper_cholesky_of_inverse(H)
    assert np.allclose(np.tril(U, -1), 0.0)
    assert np.all(np.diag(U) > 0)
    np.testing.assert_allclose(U.T @ U, np.linalg.inv(H), rtol=1e-9, atol=1e-12)


def test_sub_inverse_relation():
    """Rows of U hold the shrinking inverses: U[j, j:] = inv(H[j:, j:])[0, :] /
    sqrt(inv(H[j:, j:])[0, 0]) (page 'From one repair to a whole model')."""
    for n in (2, 5, 12):
        H, _ = _rand_spd(n, 10 + n)
        U = O.upper_cholesky_of_inverse(H)
        for j in range(n):
            Fi = np.linalg.inv(H[j:, j:])
            np.testing.assert_allclose(U[j, j:], Fi[0] / np.sqrt(Fi[0, 0]), rtol=1e-9, atol=1e-12)
            assert U[j, j] ** 2 == pytest.approx(Fi[0, 0], rel=1e-10)


def test_inplace_lapack_route_matches_definition():
    """The in-place LAPACK form of the route (used at n = 28672) gives the
    factor the definition fixes: upper, positive diagonal, U^T U H = I, rows
    equal to the scaled shrinking inverses; it overwrites its input and
    rejects a matrix that is not positive definite."""
    for n, seed in ((7, 3), (12, 4), (301, 5)):
        H, _ = _rand_spd(n, seed)
        B = np.ascontiguousarray(H.copy())
        U = O.upper_cholesky_of_inverse_inplace(B)
        assert U is B
        assert np.all(np.tril(U, -1) == 0.0)
        assert np.all(np.diag(U) > 0)
        np.testing.assert_allclose(U.T @ U @ H, np.eye(n), atol=1e-8)
        if n <= 12:
            for j in range(n):
                Fi = np.linalg.inv(H[j:, j:])
                np.testing.assert_allclose(U[j, j:], Fi[0] / np.sqrt(Fi[0, 0]), rtol=1e-9,
                                           atol=1e-12)
        ref = O.upper_cholesky_of_inverse(H)
        assert np.linalg.norm(U - ref) / np.linalg.norm(ref) < 1e-11
    bad = np.ascontiguousarray(np.diag([1.0, -1.0, 2.0]))
    with pytest.raises(np.linalg.LinAlgError):
        O.upper_cholesky_of_inverse_inplace(bad)
    with pytest.raises(ValueError):
        O.upper_cholesky_of_inverse_inplace(np.eye(3, dtype=np.float32))


# ---------------------------------------------------------------- the sweep
def _layer(rows, n, ntok, seed, corr=0.5, dead=()):
    W, X = workloads.random_layer(rows, n, ntok, seed, correlated=corr, dead=dead)
    return W.double().numpy(), X.double().numpy()


def test_identity_hessian_gives_rtn_exactly():
    """H proportional to I (any diagonal H): every repair adds err * 0, so GPTQ
    is round-to-nearest exactly (page 'The repair rule': at rho = 0 the
    formula does nothing)."""
    rng = np.random.default_rng(5)
    n, rows = 256, 7
    W = rng.normal(0, 0.02, (rows, n))
    for gains in (None, rng.uniform(0.5, 4.0, n)):
        X = workloads.identity_calibration(n, 3, gains, dtype=torch.float32).double().numpy()
        H = O.hessian(X)
        for g in (-1, 128, 32):
            for act in (False, True):
                r = O.gptq_layer(W, H, 4, g, 0.01, act)
                base = O.rtn(r["Wp"], 4, g)
                assert np.array_equal(r["codes"], base["codes"])
                assert np.array_equal(r["zeros"], base["zeros"])
                assert np.array_equal(r["scales"], base["scales"])
                if gains is not None and act:
                    assert not np.array_equal(r["perm"], np.arange(n))


@pytest.mark.parametrize("rows,n,bits,g,blocks", [
    (4, 6, 2, -1, (1, 2, 3, 6)),
    (3, 8, 2, 4, (4, 2, 8)),
    (5, 20, 3, 4, (4, 8, 12, 20)),
    (3, 24, 4, 8, (4, 8, 16, 24)),
])
def test_blocked_equals_unblocked(rows, n, bits, g, blocks):
    W, X = _layer(rows, n, 4 * n, seed=rows * 100 + n)
    prep = O.prepare(O.hessian(X), W, 0.01, True)
    U = O.upper_cholesky_of_inverse(prep["Hp"])
    ref = O.sweep(prep["Wp"], U, bits, g)
    for B in blocks:
        if g > 0 and not (B % g == 0 or g % B == 0):
            continue
        b = O.sweep_blocked(prep["Wp"], U, bits, g, B)
        assert np.array_equal(b["codes"], ref["codes"])
        assert np.array_equal(b["zeros"], ref["zeros"])
        np.testing.assert_allclose(b["Wq"], ref["Wq"], rtol=0, atol=1e-12)
        np.testing.assert_allclose(b["loss"], ref["loss"], rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("g,act,dead", [(-1, False, ()), (8, True, ()), (16, True, (3, 17)),
                                        (-1, True, (0,))])
def test_objective_identity(g, act, dead):
    """sum of per-weight losses (w - q)^2 / (2 d^2) equals the damped layer
    objective ||(W0 - Wq) X||^2 + (lam/2) ||W0 - Wq||^2 computed directly
    (page 'From one repair to a whole model': the tracked loss matches the
    OBS damage with d^2 = [H_F^-1]_qq)."""
    W, X = _layer(6, 32, 96, seed=7 + g, dead=dead)
    H = O.hessian(X)
    r = O.gptq_layer(W, H, 3, g, 0.01, act)
    D = r["W0"] - r["Wq_orig"]
    direct = O.objective_direct(r["W0"], r["Wq_orig"], X) + 0.5 * r["lam"] * float(np.sum(D * D))
    assert float(np.sum(r["loss"])) == pytest.approx(direct, rel=1e-9)
    # the objective through H agrees with the direct one
    assert O.objective_from_hessian(r["W0"], r["Wq_orig"], H) == pytest.approx(
        O.objective_direct(r["W0"], r["Wq_orig"], X), rel=1e-10)


def test_bruteforce_obs_after_every_column():
    """After column j the free weights equal the exact least-squares minimiser
    of ||(w - w0) X||^2 + (lam/2)||w - w0||^2 with columns <= j fixed
    (page 'The repair rule': the formula agrees with brute force)."""
    rows, n, N = 3, 10, 30
    W, X = _layer(rows, n, N, seed=11)
    H = O.hessian(X)
    prep = O.prepare(H, W, 0.05, False)
    U = O.upper_cholesky_of_inverse(prep["Hp"])
    lam = prep["lam"]
    Xp = X[prep["perm"]]
    states = {}
    res = O.sweep(prep["Wp"], U, 3, -1, trace=lambda j, Wc: states.__setitem__(j, Wc.copy()))
    w0 = prep["Wp"]
    for j in range(n - 1):
        fixed = res["Wq"][:, :j + 1]
        for r in range(rows):
            # minimise ||X_F^T (v - w0_F) + X_C^T (fixed - w0_C)||^2 + lam/2 ||v - w0_F||^2
            A = np.vstack([Xp[j + 1:].T, np.sqrt(lam / 2) * np.eye(n - j - 1)])
            rhs = np.concatenate([-(Xp[:j + 1].T @ (fixed[r] - w0[r, :j + 1])),
                                  np.zeros(n - j - 1)])
            delta, *_ = np.linalg.lstsq(A, rhs, rcond=None)
            np.testing.assert_allclose(states[j][r, j + 1:], w0[r, j + 1:] + delta,
                                       rtol=1e-9, atol=1e-12)


def test_obs_formula_per_step():
    """Each step's repair equals the Optimal Brain Surgeon update
    delta_F = -e / [H_F^-1]_qq * (H_F^-1)_{:,q} taken from a direct inverse of
    the trailing block (page 'GPTQ, with the code open', 'The repair rule');
    its q-th component collapses to -e (the sign the page warns about)."""
    W, X = _layer(4, 12, 40, seed=12)
    prep = O.prepare(O.hessian(X), W, 0.01, False)
    U = O.upper_cholesky_of_inverse(prep["Hp"])
    states = {-1: prep["Wp"].copy()}
    res = O.sweep(prep["Wp"], U, 4, -1, trace=lambda j, Wc: states.__setitem__(j, Wc.copy()))
    for j in range(12):
        Fi = np.linalg.inv(prep["Hp"][j:, j:])
        e = states[j - 1][:, j] - res["Wq"][:, j]
        delta = -np.outer(e / Fi[0, 0], Fi[:, 0])
        np.testing.assert_allclose(delta[:, 0], -e, rtol=1e-12, atol=1e-15)
        np.testing.assert_allclose(states[j][:, j + 1:] - states[j - 1][:, j + 1:], delta[:, 1:],
                                   rtol=1e-8, atol=1e-13)


def test_two_inputs_rho():
    gold = _golden("two_inputs.json")
    for rho in gold["rho_checks"]:
        Hp = np.array([[1.0, rho], [rho, 1.0]])
        U = O.upper_cholesky_of_inverse(Hp)
        W = np.array([[gold["w1"], gold["w2"]]])
        states = {}
        res = O.sweep(W, U, 2, -1, trace=lambda j, Wc: states.__setitem__(j, Wc.copy()))
        e = gold["w1"] - res["Wq"][0, 0]
        # free weight absorbs rho * e; damage is (1 - rho^2) of plain rounding's e^2/2
        assert states[0][0, 1] == pytest.approx(gold["w2"] + rho * e, abs=1e-12)
        loss0 = e * e / (2 * U[0, 0] ** 2)
        assert loss0 == pytest.approx(e * e * (1 - rho ** 2) / 2, rel=1e-12)
    assert 1 - 0.9 ** 2 == pytest.approx(gold["rho_0p9_damage_ratio"])
    # rho -> 1: forcing w1 0.63 -> 0.50 moves w2 -0.41 -> -0.28.  The ruler
    # [-0.5, 1.0] at 2 bits has ticks -0.5, 0, 0.5, 1.0; its end points come
    # from two extra uncorrelated columns.
    rho = 1 - 1e-12
    Hp = np.eye(4)
    Hp[0, 1] = Hp[1, 0] = rho
    Hp[:2, :2] += 1e-9 * np.eye(2)
    U = O.upper_cholesky_of_inverse(Hp)
    W = np.array([[gold["w1"], gold["w2"], 1.0, -0.5]])
    states = {}
    res = O.sweep(W, U, 2, -1, trace=lambda j, Wc: states.__setitem__(j, Wc.copy()))
    assert res["Wq"][0, 0] == pytest.approx(gold["w1_forced"])
    assert states[0][0, 1] == pytest.approx(gold["w2_repaired"], abs=1e-6)


def test_scale_equivariance_exact():
    """Multiplying H by 4 scales U by exactly 1/2 and changes no code."""
    W, X = _layer(5, 48, 120, seed=21)
    H = O.hessian(X)
    a = O.gptq_layer(W, H, 4, 16, 0.01, True)
    b = O.gptq_layer(W, 4.0 * H, 4, 16, 0.01, True)
    assert np.array_equal(a["U"] * 0.5, b["U"])
    assert np.array_equal(a["codes_orig"], b["codes_orig"])
    assert np.array_equal(a["Wq_orig"], b["Wq_orig"])


def test_dead_input_channel():
    W, X = _layer(4, 16, 64, seed=31, dead=(5,))
    H = O.hessian(X)
    assert H[5, 5] == 0 and np.all(H[5] == 0)
    r = O.gptq_layer(W, H, 4, -1, 0.01, True)
    assert r["dead"][5] and r["dead"].sum() == 1
    assert np.all(r["W0"][:, 5] == 0)
    assert np.all(r["Wq_orig"][:, 5] == 0)
    assert np.array_equal(r["codes_orig"][:, 5], r["zeros"][:, 0])
    # the dead diagonal is set to 1 before damping: lam = 0.01 * mean(diag)
    d = np.diag(H).copy()
    d[5] = 1.0
    assert r["lam"] == pytest.approx(0.01 * d.mean(), rel=1e-14)
    # act-order puts the (small) dead channel last
    assert r["perm"][-1] == 5


def test_actorder_is_stable_descending():
    H = np.diag([2.0, 5.0, 2.0, 7.0, 5.0])
    W = np.ones((1, 5)) * 0.1
    p = O.prepare(H, W, 0.0, True)["perm"]
    assert list(p) == [3, 1, 4, 0, 2]


def test_prepared_blocks_come_from_the_diagonal_alone():
    """dead / act-order / damping read only diag(H): any principal block of
    the prepared matrix can be built without forming the whole of it (the
    full-size checks rely on this), and it is the textbook construction
    H[perm][:, perm] + lam I with dead diagonal entries set to 1."""
    H, _ = _rand_spd(40, seed=77)
    for c in (3, 17):
        H[c, :] = 0.0
        H[:, c] = 0.0
    W = np.ones((2, 40))
    for act in (False, True):
        full = O.prepare(H, W, 0.01, act)
        diag_only = O.prepare_from_diagonal(np.diag(H), 0.01, act)
        assert np.array_equal(full["perm"], diag_only["perm"])
        assert np.array_equal(full["dead"], diag_only["dead"])
        d = np.diag(H).copy()
        d[[3, 17]] = 1.0
        assert diag_only["lam"] == pytest.approx(0.01 * d.mean(), rel=1e-14)
        Hd = H.copy()
        Hd[[3, 17], [3, 17]] = 1.0
        p = diag_only["perm"]
        textbook = Hd[p][:, p] + diag_only["lam"] * np.eye(40)
        assert np.array_equal(full["Hp"], textbook)
        for k0, k1 in ((0, 40), (10, 25), (33, 40)):
            assert np.array_equal(O.damped_block(H, diag_only, k0, k1), textbook[k0:k1, k0:k1])
    # dead channels go last under act-order (their diagonal, 1, is the smallest here)
    assert set(O.prepare_from_diagonal(np.diag(H), 0.01, True)["perm"][-2:]) == {3, 17}


def test_gptq_beats_rtn_on_correlated_inputs():
    W, X = _layer(16, 64, 256, seed=41, corr=0.8)
    H = O.hessian(X)
    r = O.gptq_layer(W, H, 3, -1, 0.01, False)
    base = O.rtn(r["W0"], 3, -1)
    Wr = O.dequantize(base["codes"], base["scales"][:, :1], base["zeros"][:, :1])
    assert O.objective_direct(r["W0"], r["Wq_orig"], X) < 0.5 * O.objective_direct(r["W0"], Wr, X)


def test_tie_replay_adopts_only_ties():
    W, X = _layer(3, 16, 64, seed=51)
    prep = O.prepare(O.hessian(X), W, 0.01, False)
    U = O.upper_cholesky_of_inverse(prep["Hp"])
    ref = O.sweep(prep["Wp"], U, 4, -1)
    same = O.sweep(prep["Wp"], U, 4, -1, forced_codes=ref["codes"], forced_zeros=ref["zeros"])
    assert same["adopted"] == 0 and same["mismatched"] == 0
    assert np.array_equal(same["codes"], ref["codes"])
    bad = ref["codes"].copy()
    bad[1, 7] = (bad[1, 7] + 1) % 16          # a flip far from a tie
    r = O.sweep(prep["Wp"], U, 4, -1, forced_codes=bad)
    assert r["mismatched"] >= 1 and r["adopted"] == 0
    # a value exactly on a half tick: the other rounding is adopted, not counted
    U1 = np.eye(3)
    Wt = np.array([[0.5, -1.0, 2.0]])          # ruler [-1, 2] at 2 bits: scale 1, zero 1
    own = O.sweep(Wt, U1, 2, -1)
    assert own["codes"][0, 0] == 1             # rint(0.5) = 0 (half to even), + zero
    other = own["codes"].copy()
    other[0, 0] = 2
    r = O.sweep(Wt, U1, 2, -1, forced_codes=other)
    assert r["adopted"] == 1 and r["mismatched"] == 0 and r["codes"][0, 0] == 2


# ---------------------------------------------------------------- storage
def _scalar_pack(codes, bits):
    """Bit-by-bit statement of the layout: code c of a row, bit i, goes to
    global bit position bits*c + i of the row's little-endian bit string."""
    rows, n = codes.shape
    nwords = n * bits // 32
    out = np.zeros((rows, nwords), dtype=np.uint32)
    for r in range(rows):
        for c in range(n):
            for i in range(bits):
                if (int(codes[r, c]) >> i) & 1:
                    pos = bits * c + i
                    out[r, pos // 32] |= np.uint32(1 << (pos % 32))
    return out


def test_pack_int4_int3_layout_and_roundtrip():
    rng = np.random.default_rng(61)
    c4 = rng.integers(0, 16, (3, 64))
    c3 = rng.integers(0, 8, (3, 96))
    p4, p3 = O.pack_int4(c4), O.pack_int3(c3)
    assert np.array_equal(p4, _scalar_pack(c4, 4))
    assert np.array_equal(p3, _scalar_pack(c3, 3))
    assert np.array_equal(O.unpack_int4(p4, 64), c4)
    assert np.array_equal(O.unpack_int3(p3, 96), c3)
    # codes 10 and 21 of a 32-code group straddle 32-bit words
    c = np.zeros((1, 32), dtype=np.int64)
    c[0, 10] = 7
    assert list(O.pack_int3(c)[0]) == [0xC0000000, 0x1, 0]
    c[0, 10] = 0
    c[0, 21] = 5
    assert list(O.pack_int3(c)[0]) == [0, 0x80000000, 0x2]


def test_dequant_single_rounding_and_bf16():
    rng = np.random.default_rng(71)
    rows, n, g = 4, 64, 16
    codes = rng.integers(0, 16, (rows, n))
    scales = rng.uniform(1e-4, 1e-1, (rows, n // g)).astype(np.float32)
    zeros = rng.integers(0, 16, (rows, n // g))
    w = O.dequant(O.pack_int4(codes), 4, n, scales, zeros, g)
    for r in range(rows):
        for c in range(n):
            exact = float(scales[r, c // g]) * (int(codes[r, c]) - int(zeros[r, c // g]))
            assert w[r, c] == np.float32(exact)
    # bfloat16 rounding agrees with torch's own (round-half-to-even) conversion
    bits = O.dequant(O.pack_int4(codes), 4, n, scales, zeros, g, out="bf16")
    tb = torch.from_numpy(w).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(bits, tb)
    # g_idx overrides the contiguous grouping
    gi = rng.integers(0, n // g, n)
    w2 = O.dequant(O.pack_int4(codes), 4, n, scales, zeros, g, g_idx=gi)
    assert w2[2, 5] == np.float32(float(scales[2, gi[5]]) * (codes[2, 5] - zeros[2, gi[5]]))


# ---------------------------------------------------------------- mutations
def test_dequant_matvec_columns_and_brute_force():
    """A unit activation picks one column of w_hat exactly; a small case
    equals the plain double loop."""
    rng = np.random.default_rng(21)
    for bits, n, g in ((4, 64, 16), (3, 96, 32), (4, 40, -1)):
        rows = 5
        codes = rng.integers(0, 2 ** bits, (rows, n))
        G_ = 1 if g <= 0 else (n + g - 1) // g
        scales = rng.uniform(1e-3, 0.1, (rows, G_)).astype(np.float32)
        zeros = rng.integers(0, 2 ** bits, (rows, G_))
        packed = O.pack_int4(codes) if bits == 4 else O.pack_int3(codes)
        W = O.dequant(packed, bits, n, scales, zeros, g).astype(np.float64)
        for c in (0, n // 2, n - 1):
            e = np.zeros(n)
            e[c] = 1.0
            y, _ = O.dequant_matvec(packed, bits, n, scales, zeros, e, g)
            assert np.array_equal(y[0], W[:, c])
        x = rng.standard_normal((3, n))
        y, mag = O.dequant_matvec(packed, bits, n, scales, zeros, x, g)
        for b in range(3):
            for r in range(rows):
                ref = 0.0
                for c in range(n):
                    gc = (c // g) if g > 0 else 0
                    # w_hat is the binary32 rounding of scale * (code - zero)
                    w = float(np.float32(float(scales[r, gc]) * (codes[r, c] - zeros[r, gc])))
                    ref += w * x[b, c]
                assert abs(y[b, r] - ref) <= 1e-12 * mag[b, r]


def test_planted_mistakes_are_caught():
    """Plant typical mistakes in the oracle's inputs/steps and check the pins
    above would reject them: a transposed U, a flipped repair sign, a dropped
    damping term in the identity."""
    W, X = _layer(5, 24, 80, seed=81)
    H = O.hessian(X)
    prep = O.prepare(H, W, 0.01, False)
    U = O.upper_cholesky_of_inverse(prep["Hp"])

    def identity_gap(Uuse, lam_term=True):
        r = O.sweep(prep["Wp"], Uuse, 3, -1)
        D = prep["Wp"] - r["Wq"]
        Xp = X[prep["perm"]]
        rhs = O.objective_direct(prep["Wp"], r["Wq"], Xp)
        if lam_term:
            rhs += 0.5 * prep["lam"] * float(np.sum(D * D))
        return abs(float(np.sum(r["loss"])) - rhs) / rhs

    assert identity_gap(U) < 1e-9
    assert identity_gap(U.T) > 1e-3                                   # transposed operand
    flipped = 2 * np.diag(np.diag(U)) - U                             # sign of the repair
    assert identity_gap(flipped) > 1e-3
    assert identity_gap(U, lam_term=False) > 1e-6                     # dropped term


def test_forced_actorder_accepts_only_near_ties():
    d = np.array([5.0, 3.0, 3.0 + 1e-7, 1.0])
    H = np.diag(d)
    W = np.full((1, 4), 0.1)
    own = O.prepare(H, W, 0.0, True)["perm"]
    assert list(own) == [0, 2, 1, 3]
    swapped = O.prepare(H, W, 0.0, True, forced_perm=[0, 1, 2, 3])["perm"]
    assert list(swapped) == [0, 1, 2, 3]                 # 3 vs 3+1e-7: a near tie
    with pytest.raises(ValueError):
        O.prepare(H, W, 0.0, True, forced_perm=[1, 0, 2, 3])   # 5 vs 3: not a tie
    with pytest.raises(ValueError):
        O.prepare(H, W, 0.0, True, forced_perm=[0, 0, 2, 3])   # not a permutation


def test_hessian_symmetric_blas_route_equals_plain_product():
    rng = np.random.default_rng(91)
    X = rng.standard_normal((520, 300)).astype(np.float32)
    H = O.hessian(X, token_chunk=128)
    Xd = X.astype(np.float64)
    ref = 2.0 * Xd @ Xd.T
    assert np.array_equal(H, H.T)
    assert np.linalg.norm(H - ref) / np.linalg.norm(ref) < 1e-14


def test_dequant_matvec_sweep_order_equals_original_order():
    """An act-order layer served in sweep order (codes gathered by perm,
    contiguous groups, x gathered by the same perm) gives the same y as the
    original order with g_idx (g_idx[c] = position of c in the sweep / g):
    the same products, summed in another order."""
    rng = np.random.default_rng(33)
    for bits, rows, n, g in ((4, 6, 128, 32), (3, 5, 96, 32), (4, 4, 256, 64)):
        codes = rng.integers(0, 2 ** bits, (rows, n))
        perm = rng.permutation(n)
        G_ = n // g
        scales = rng.uniform(1e-3, 0.1, (rows, G_)).astype(np.float32)
        zeros = rng.integers(0, 2 ** bits, (rows, G_))
        g_idx = np.empty(n, dtype=np.int64)
        g_idx[perm] = np.arange(n) // g
        pack = O.pack_int4 if bits == 4 else O.pack_int3
        x = rng.standard_normal((3, n))
        y_sw, mag = O.dequant_matvec(pack(codes[:, perm]), bits, n, scales, zeros, x, g,
                                     perm=perm)
        y_or, _ = O.dequant_matvec(pack(codes), bits, n, scales, zeros, x, g, g_idx)
        np.testing.assert_allclose(y_sw, y_or, rtol=0, atol=1e-13 * float(np.max(mag)))
        # a planted mistake: x not gathered -- caught
        y_bad, _ = O.dequant_matvec(pack(codes[:, perm]), bits, n, scales, zeros, x, g)
        assert not np.allclose(y_bad, y_or)
