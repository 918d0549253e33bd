"""Plain fp64 CPU oracle of the random-sign blocked Hadamard rotation.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU legs of ``bench.py`` may import or call this module.  The CUDA library
never reaches it, and it imports nothing from the CUDA package.

Source: the page "Post-Training Quantization: Calibration, GPTQ and Why
Rotations Help" (groundtruth.day), section "Rotations: making outliers
disappear" and its question "Why do Hadamard rotations help quantization?":
a Hadamard matrix has entries +1 and -1 with mutually perpendicular rows;
scaled properly it is a rotation; rotating the activations that enter a layer
and applying the inverse rotation to the layer's weights leaves the product
unchanged, while a single large entry is spread over all entries.

Readings where the page is silent (the rotated 70B workload fixes them):

* The Hadamard matrix of order b (a power of two) is Sylvester's:
  H_1 = [1], H_2k = [[H_k, H_k], [H_k, -H_k]], so H[i][j] = (-1)^popcount(i & j).
* "Scaled properly" is H_b / sqrt(b), which is orthogonal and symmetric.
* The rotation acts on the feature axis in independent blocks of b features
  after a per-feature sign flip s (+1 / -1, drawn by the input generator):
  R = blockdiag(H_b / sqrt(b), ..., H_b / sqrt(b)) diag(s).
* Activations X (features x tokens) become X' = R X and weights W
  (rows x features) become W' = W R^T, so W' X' = W X.
"""
from __future__ import annotations

import numpy as np


def sylvester(b: int) -> np.ndarray:
    """H_b (b a power of two) by Sylvester's doubling, as float64 +-1."""
    if b < 1 or b & (b - 1):
        raise ValueError("b must be a power of two")
    H = np.ones((1, 1))
    while H.shape[0] < b:
        H = np.block([[H, H], [H, -H]])
    return H


def rotation_matrix(signs: np.ndarray, b: int) -> np.ndarray:
    """R = blockdiag(H_b / sqrt(b)) diag(signs), n x n with n = len(signs)."""
    s = np.asarray(signs, dtype=np.float64)
    n = s.shape[0]
    if n % b:
        raise ValueError("n must be a multiple of the block")
    Hn = sylvester(b) / np.sqrt(b)
    R = np.zeros((n, n))
    for k in range(n // b):
        sl = slice(k * b, (k + 1) * b)
        R[sl, sl] = Hn * s[None, sl]
    return R


def rotate_features(V, signs: np.ndarray, b: int) -> np.ndarray:
    """R V for V with the features on axis 0 (X' = R X), in fp64."""
    V = np.asarray(V, dtype=np.float64)
    s = np.asarray(signs, dtype=np.float64)
    Hn = sylvester(b) / np.sqrt(b)
    out = np.empty_like(V)
    for k in range(V.shape[0] // b):
        sl = slice(k * b, (k + 1) * b)
        out[sl] = Hn @ (s[sl].reshape((b,) + (1,) * (V.ndim - 1)) * V[sl])
    return out


def rotate_weight(W, signs: np.ndarray, b: int) -> np.ndarray:
    """W R^T for W with the features on axis 1 (W' = W R^T), in fp64."""
    W = np.asarray(W, dtype=np.float64)
    return rotate_features(W.T, signs, b).T
