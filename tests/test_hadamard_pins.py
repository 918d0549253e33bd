"""Pins of the Hadamard-rotation oracle (CPU only).

Page "Post-Training Quantization: Calibration, GPTQ and Why Rotations Help",
section "Rotations: making outliers disappear": entries +-1 with mutually
perpendicular rows, a rotation once scaled, the layer's product unchanged
when the activations are rotated and the weights get the inverse, one large
entry spread evenly over the block.  Each pin below would fail for a
plausible mistake in the oracle (a transposed operand, a missing scale, the
signs applied on the wrong side, blocks mixed up), see the planted cases.
"""
import numpy as np
import pytest
import scipy.linalg

from oracle import hadamard_oracle as HO


@pytest.mark.parametrize("b", [1, 2, 4, 8, 32, 256, 1024])
def test_sylvester_matches_the_library_construction(b):
    assert np.array_equal(HO.sylvester(b), scipy.linalg.hadamard(b).astype(np.float64))


def test_sylvester_entries_by_bit_parity():
    b = 16
    H = HO.sylvester(b)
    for i in range(b):
        for j in range(b):
            assert H[i, j] == (-1.0) ** bin(i & j).count("1")


@pytest.mark.parametrize("b", [32, 1024])
def test_rows_are_perpendicular_and_the_scaled_matrix_is_a_rotation(b):
    H = HO.sylvester(b)
    assert np.array_equal(H @ H.T, b * np.eye(b))
    rng = np.random.default_rng(b)
    s = rng.choice([-1.0, 1.0], 3 * b)
    R = HO.rotation_matrix(s, b)
    np.testing.assert_allclose(R @ R.T, np.eye(3 * b), atol=1e-12)
    x = rng.standard_normal(3 * b)
    assert np.linalg.norm(R @ x) == pytest.approx(np.linalg.norm(x), rel=1e-13)


def test_rotated_weights_times_rotated_inputs_is_the_original_product():
    rng = np.random.default_rng(7)
    n, b = 256, 64
    W = rng.standard_normal((5, n))
    X = rng.standard_normal((n, 9))
    s = rng.choice([-1.0, 1.0], n)
    Wr = HO.rotate_weight(W, s, b)
    Xr = HO.rotate_features(X, s, b)
    np.testing.assert_allclose(Wr @ Xr, W @ X, atol=1e-11)
    # ... and not a trivial identity: the operands themselves change
    assert np.max(np.abs(Xr - X)) > 0.5


def test_one_large_entry_is_spread_evenly_over_its_block():
    n, b, k, A = 128, 32, 37, 50.0
    s = np.random.default_rng(1).choice([-1.0, 1.0], n)
    x = np.zeros(n)
    x[k] = A
    y = HO.rotate_features(x, s, b)
    blk = slice((k // b) * b, (k // b + 1) * b)
    np.testing.assert_allclose(np.abs(y[blk]), A / np.sqrt(b), rtol=1e-14)
    y[blk] = 0.0
    assert not np.any(y)  # other blocks untouched


def test_rotation_matches_the_dense_matrix_and_columns_of_H():
    rng = np.random.default_rng(3)
    n, b = 96, 32
    s = rng.choice([-1.0, 1.0], n)
    V = rng.standard_normal((n, 4))
    np.testing.assert_allclose(HO.rotate_features(V, s, b), HO.rotation_matrix(s, b) @ V,
                               atol=1e-13)
    # R e_k = s_k * column k of H_b / sqrt(b) inside block k // b
    k = 45
    e = np.zeros(n)
    e[k] = 1.0
    col = HO.rotate_features(e, s, b)[32:64]
    np.testing.assert_allclose(col, s[k] * HO.sylvester(b)[:, k - 32] / np.sqrt(b), atol=1e-15)


def test_planted_mistakes_are_caught():
    rng = np.random.default_rng(11)
    n, b = 128, 32
    s = rng.choice([-1.0, 1.0], n)
    W = rng.standard_normal((3, n))
    X = rng.standard_normal((n, 5))
    good = HO.rotation_matrix(s, b)

    def invariant(R):
        return np.allclose((W @ R.T) @ (R @ X), W @ X, atol=1e-10)

    assert invariant(good)
    # signs applied after the Hadamard instead of before: R' = H D is not H D
    # on the same vector, and R'^T R must still be I for the invariant, so
    # check the rotation's action on a spike instead
    Hn = np.kron(np.eye(n // b), HO.sylvester(b) / np.sqrt(b))
    wrong_side = np.diag(s) @ Hn
    assert not np.allclose(wrong_side @ X, good @ X)
    # missing 1/sqrt(b): not a rotation, the invariant fails
    assert not invariant(np.kron(np.eye(n // b), HO.sylvester(b)) @ np.diag(s))
    # weights given R instead of R^T: W R R X != W X (R is not symmetric
    # once the signs are in)
    assert not np.allclose((W @ good) @ (good @ X), W @ X, atol=1e-6)
    # blocks of the wrong size
    assert not np.allclose(HO.rotation_matrix(s, 2 * b) @ X, good @ X)
