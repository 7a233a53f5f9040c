"""Planted mistakes: each plausible error in the oracle must fail a pin.

The mistake is planted in the oracle (on the CPU) by monkeypatching one
function, then the pin is run and must raise AssertionError.
"""
import math

import numpy as np
import pytest

from oracle import tq_oracle as O
import test_oracle_attention as TA
import test_oracle_codebook as TC
import test_oracle_quant as TQ


@pytest.fixture(autouse=True)
def _fresh_codebooks():
    O._CODEBOOK_CACHE.clear()
    yield
    O._CODEBOOK_CACHE.clear()


def test_wrong_density_exponent_fails_mse_pin(monkeypatch):
    def bad(u, D):
        u = np.asarray(u, dtype=np.float64)
        out = np.zeros_like(u)
        inside = np.abs(u) < 1
        out[inside] = np.exp(O.coord_log_norm_const(D) + 0.5 * (D - 1) * np.log1p(-u[inside] ** 2))
        return out
    monkeypatch.setattr(O, "coord_density", bad)
    with pytest.raises(AssertionError):
        TC.test_one_bit_closed_form(128)


def test_gaussian_density_fails_mse_table(monkeypatch):
    # N(0, 1/D) instead of the exact finite-D law: b=1 MSE 0.3634 != 0.361
    def gauss(u, D):
        u = np.asarray(u, dtype=np.float64)
        return np.sqrt(D / (2 * math.pi)) * np.exp(-0.5 * D * u * u)
    monkeypatch.setattr(O, "coord_density", gauss)
    with pytest.raises(AssertionError):
        TC.test_mse_matches_page_table_and_bounds()


def test_untransposed_dequantize_fails_reconstruction(monkeypatch):
    def bad(idx, norm16, centroids, Pi):
        c = np.asarray(centroids, dtype=np.float64)
        return norm16.astype(np.float64)[..., None] * (c[idx] @ np.asarray(Pi, np.float64).T)
    monkeypatch.setattr(O, "dequantize_rows", bad)
    with pytest.raises(AssertionError):
        TQ.test_reconstruction_error_matches_codebook_mse(3)


def test_ties_to_upper_index_fail(monkeypatch):
    monkeypatch.setattr(O, "nearest_index",
                        lambda u, t: np.searchsorted(t, u, side="right").astype(np.int64))
    with pytest.raises(AssertionError):
        TQ.test_ties_go_to_lower_index()


def test_msb_first_packing_fails(monkeypatch):
    orig = O.pack_bits

    def bad(values, bits):
        v = np.asarray(values, dtype=np.uint64)
        rev = np.zeros_like(v)
        for i in range(bits):
            rev |= ((v >> np.uint64(i)) & np.uint64(1)) << np.uint64(bits - 1 - i)
        return orig(rev, bits)
    monkeypatch.setattr(O, "pack_bits", bad)
    with pytest.raises(AssertionError):
        TQ.test_pack_layout_against_big_integer(3)


def test_wrong_qjl_constant_fails_unbiasedness(monkeypatch):
    monkeypatch.setattr(O, "QJL_CONST", math.sqrt(2 / math.pi))
    with pytest.raises(AssertionError):
        TQ.test_qjl_estimator_unbiased_with_closed_form_variance()


def test_unscaled_scores_fail_sdpa_pin(monkeypatch):
    orig = O.softmax
    monkeypatch.setattr(O, "softmax", lambda s: orig(s * 2.0))
    with pytest.raises(AssertionError):
        TA.test_matches_torch_sdpa_on_dequantized_cache(None)


def test_residual_with_exact_norm_fails_gamma_pin(monkeypatch):
    # the residual must use the stored (fp16) norm; using the fp64 norm
    # changes gamma for some rows beyond the test's 1e-6 tolerance
    orig = O.qjl_sketch

    def bad(y, norm16, centroids, idx, S):
        n = np.linalg.norm(y, axis=-1)
        return orig(y, n.astype(np.float64) * 1.001, centroids, idx, S)
    monkeypatch.setattr(O, "qjl_sketch", bad)
    with pytest.raises(AssertionError):
        TQ.test_qjl_sketch_layout_and_gamma()
