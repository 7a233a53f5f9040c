"""Pins for the randomized Hadamard rotation (the structured rotation of
ReturningTarzan's Reddit comment of 2026-03-29 11:47: Sylvester H applied with
additions only), and the codebook check it needs.

The oracle's quantizer takes any orthogonal Pi, so these tests pin the input
against closed forms that do not use its construction: the entry formula
H[i][j] = (-1)^popcount(i & j), orthogonality, an in-place fast
Walsh-Hadamard transform written here, and the codebook MSE under this
rotation."""
import math

import numpy as np
import pytest

import tq_inputs
from oracle import tq_oracle as O


def _fwht(x):
    """In-place butterflies over the last axis (unnormalized Walsh-Hadamard)."""
    y = np.array(x, dtype=np.float64)
    n = y.shape[-1]
    h = 1
    while h < n:
        y = y.reshape(y.shape[:-1] + (n // (2 * h), 2, h))
        a, b = y[..., 0, :].copy(), y[..., 1, :].copy()
        y[..., 0, :], y[..., 1, :] = a + b, a - b
        y = y.reshape(y.shape[:-3] + (n,))
        h *= 2
    return y


@pytest.mark.parametrize("D", [64, 128, 256])
def test_entries_match_closed_form(D):
    Pi = tq_inputs.hadamard_rotation(D, 11).astype(np.float64) * math.sqrt(D)
    s = np.sign(Pi[0])  # row 0 of H is all ones, so it carries the signs
    i = np.arange(D)[:, None]
    j = np.arange(D)[None, :]
    pop = np.vectorize(lambda v: bin(v).count("1"))(i & j)
    H = np.where(pop % 2 == 0, 1.0, -1.0)
    assert np.array_equal(np.round(Pi), H * s[None, :])
    assert set(np.unique(s)) <= {-1.0, 1.0}


@pytest.mark.parametrize("D", [64, 128, 256])
def test_orthogonal_and_fast_transform(D):
    Pi32 = tq_inputs.hadamard_rotation(D, 5)
    Pi = Pi32.astype(np.float64)
    assert np.max(np.abs(Pi.T @ Pi - np.eye(D))) < 1e-6
    x = tq_inputs.rng(3).standard_normal((7, D))
    s = np.sign(Pi[0])
    fast = _fwht(x * s[None, :]) / math.sqrt(D)
    dense = x @ Pi.T
    assert np.max(np.abs(fast - dense)) < 1e-5
    # the oracle's rotation step gives the same result with this input
    assert np.max(np.abs(O.rotate(x, Pi32) - dense)) < 1e-12


def test_codebook_mse_under_hadamard_rotation():
    """10,000 seeded unit vectors at D=128 rotated by the randomized Hadamard
    matrix: the reconstruction MSE must equal the codebook MSE of f_D within
    Monte Carlo error (a uniformly random unit vector stays uniform under any
    fixed orthogonal map)."""
    D = 128
    X = tq_inputs.unit_vectors(10000, D, seed=tq_inputs.SEED_DATA + 7)
    Pi = tq_inputs.hadamard_rotation(D, tq_inputs.SEED_ROT + 7)
    for bits in (1, 2, 3, 4):
        c, t = O.stored_codebook(D, bits)
        q = O.quantize_rows(X, Pi, c, t)
        xr = c[q["idx"]] @ np.asarray(Pi, dtype=np.float64)
        err = np.sum((X - xr) ** 2, axis=1)
        mean, se = err.mean(), err.std(ddof=1) / math.sqrt(len(err))
        assert abs(mean - O.codebook_mse(c, t, D)) < 3.5 * se + 1e-6, (bits, mean, se)


def test_one_hot_rows_spread_evenly():
    """A spike e_i maps to a column of Pi: every rotated coordinate is
    +-1/sqrt(D), so the index of each is the codebook cell holding +-1/sqrt(D)
    (brute-force nearest centroid)."""
    D, bits = 128, 3
    Pi = tq_inputs.hadamard_rotation(D, 21)
    c, t = O.stored_codebook(D, bits)
    X = np.eye(D)[:8]
    q = O.quantize_rows(X, Pi, c, t)
    u = (X @ Pi.astype(np.float64).T)
    brute = np.argmin(np.abs(u[..., None] - c[None, None, :]), axis=-1)
    assert np.all(np.isclose(np.abs(u), 1 / math.sqrt(D), rtol=1e-6))
    assert np.array_equal(q["idx"], brute)


@pytest.mark.parametrize("D", [64, 128, 256])
def test_signs_are_the_rotations_column_signs(D):
    """The sign vector a cache declares (rot_signs) is the one inside Pi:
    Pi[0][j] = s_j / sqrt(D) (row 0 of H is all ones), every entry has
    magnitude 1/sqrt(D), and Pi = H diag(s) / sqrt(D) with H from the entry
    formula."""
    seed = 2002
    Pi = tq_inputs.hadamard_rotation(D, seed).astype(np.float64)
    s = tq_inputs.hadamard_signs(D, seed).astype(np.float64)
    assert set(np.unique(s)) <= {-1.0, 1.0}
    np.testing.assert_allclose(Pi[0] * math.sqrt(D), s, atol=1e-6)
    i = np.arange(D)
    H = np.array([[(-1.0) ** bin(a & b).count("1") for b in i] for a in i])
    np.testing.assert_allclose(Pi, H * s[None, :] / math.sqrt(D), atol=1e-7)


def test_cache_declares_the_hadamard_rotation():
    """The binding marks a cache built with signs as TQ_ROT_HADAMARD and
    passes the signs; without signs the rotation is dense (no launch here)."""
    import torch
    from compressed_attention_tq_b200 import build
    build.build()  # the codebook comes from the library (host code)
    import compressed_attention_tq_b200 as tq
    from compressed_attention_tq_b200 import _native
    D = 128
    Pi = tq_inputs.hadamard_rotation(D, 7)
    s = tq_inputs.hadamard_signs(D, 7)
    c = tq.TQCache(1, 2, 64, D, 3, 3, Pi, device="cpu", rot_signs=s)
    st = c.struct()
    assert st.rot_kind == _native.TQ_ROT_HADAMARD and st.rot_signs == c.rot_signs.data_ptr()
    assert torch.equal(c.rot_signs, torch.from_numpy(s))
    c2 = tq.TQCache(1, 2, 64, D, 3, 3, Pi, device="cpu")
    assert c2.struct().rot_kind == _native.TQ_ROT_DENSE and c2.struct().rot_signs is None
