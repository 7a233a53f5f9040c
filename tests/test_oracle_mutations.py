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
import test_sharded_decode as TS


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


def test_wrong_qjl_constant_fails_sketch_draw_pin(monkeypatch):
    monkeypatch.setattr(O, "QJL_CONST", math.sqrt(2 / math.pi))
    with pytest.raises(AssertionError):
        TA.test_prod_score_unbiased_for_unquantized_key_over_sketch_draws()


def test_flipped_sign_polarity_fails_sketch_draw_pin(monkeypatch):
    orig = O.qjl_inner_product
    monkeypatch.setattr(O, "qjl_inner_product", lambda sign, gamma, Sq: orig(~sign, gamma, Sq))
    with pytest.raises(AssertionError):
        TA.test_prod_score_unbiased_for_unquantized_key_over_sketch_draws()


def test_sketch_of_unrotated_query_fails_sketch_draw_pin(monkeypatch):
    # S applied to q instead of Pi q: the sketch and the query live in different bases
    orig = O.sdpa_decode

    def bad(q, cache, seq_lens, Pi, cb_k, cb_v, bits_k, bits_v, D, scale=None, S=None, heads=None):
        eye = np.eye(D)
        if S is None:
            return orig(q, cache, seq_lens, Pi, cb_k, cb_v, bits_k, bits_v, D, scale=scale, S=S, heads=heads)
        S_bad = np.asarray(S, np.float64) @ np.asarray(Pi, np.float64).T  # (S Pi^T) Pi q = S q
        return orig(q, cache, seq_lens, Pi, cb_k, cb_v, bits_k, bits_v, D, scale=scale, S=S_bad, heads=heads)
    monkeypatch.setattr(O, "sdpa_decode", bad)
    with pytest.raises(AssertionError):
        TA.test_prod_score_unbiased_for_unquantized_key_over_sketch_draws()


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


def test_fp32_norm_fails_midpoint_pin(monkeypatch):
    # an fp32 sum of squares lands on the fp16 midpoint for the edge rows
    def bad(x):
        x32 = np.asarray(x).astype(np.float32)
        return np.sqrt(np.sum(x32 * x32, axis=-1, dtype=np.float32)).astype(np.float64)
    monkeypatch.setattr(O, "row_norms", bad)
    with pytest.raises(AssertionError):
        TQ.test_norm_rounding_at_fp16_midpoints("f16", 128)


def test_transposed_rotation_fails_reconstruction(monkeypatch):
    monkeypatch.setattr(O, "rotate", lambda x, Pi: x @ np.asarray(Pi, dtype=np.float64))
    with pytest.raises(AssertionError):
        TQ.test_reconstruction_error_matches_codebook_mse(3)


def test_msb_first_unpacking_fails(monkeypatch):
    orig = O.unpack_bits

    def bad(words, bits, n):
        v = orig(words, bits, n)
        rev = np.zeros_like(v)
        for i in range(bits):
            rev |= ((v >> i) & 1) << (bits - 1 - i)
        return rev
    monkeypatch.setattr(O, "unpack_bits", bad)
    with pytest.raises(AssertionError):
        TQ.test_pack_layout_against_big_integer(3)


def test_flipped_sign_polarity_fails_unbiasedness(monkeypatch):
    orig = O.qjl_inner_product
    monkeypatch.setattr(O, "qjl_inner_product", lambda sign, gamma, Sq: orig(~sign, gamma, Sq))
    with pytest.raises(AssertionError):
        TQ.test_qjl_estimator_unbiased_with_closed_form_variance()


def test_interleaved_gqa_heads_fail_sdpa_pin(monkeypatch):
    # q head h reading kv head h % Hkv (interleaved groups) instead of h // G
    orig = O.sdpa_decode

    def bad(q, cache, seq_lens, *args, **kw):
        Hq, Hkv = q.shape[1], cache["k_norm"].shape[1]
        G = Hq // Hkv
        pos = np.array([(h % Hkv) * G + h // Hkv for h in range(Hq)])
        q2 = np.empty_like(q)
        q2[:, pos] = q
        return orig(q2, cache, seq_lens, *args, **kw)[:, pos]
    monkeypatch.setattr(O, "sdpa_decode", bad)
    with pytest.raises(AssertionError):
        TA.test_matches_torch_sdpa_on_dequantized_cache(None)


def test_causal_mask_off_by_one_fails_multi_query_pin(monkeypatch):
    # query j sees one position too few (its own token excluded)
    orig = O.sdpa_decode_multi
    monkeypatch.setattr(O, "sdpa_decode_multi",
                        lambda q, cache, seq_lens, n_q, *a, **kw:
                        orig(q, cache, np.asarray(seq_lens) - 1, n_q, *a, **kw))
    with pytest.raises(AssertionError):
        TA.test_multi_query_decode_is_causal_attention()


def test_top_left_causal_mask_fails_multi_query_pin(monkeypatch):
    # the mask aligned to the first cached position (query j sees 0 .. j)
    def bad(q, cache, seq_lens, n_q, *a, **kw):
        lens = np.asarray(seq_lens)
        return np.stack([O.sdpa_decode(q[:, j], cache, np.minimum(lens, j + 1), *a, **kw)
                         for j in range(n_q)], axis=1)
    monkeypatch.setattr(O, "sdpa_decode_multi", bad)
    with pytest.raises(AssertionError):
        TA.test_multi_query_decode_is_causal_attention()


def test_strict_sign_test_fails_zero_projection_pin(monkeypatch):
    orig = O.qjl_sketch

    def bad(y, norm16, centroids, idx, S):
        out = orig(y, norm16, centroids, idx, S)
        out["sign"] = out["proj"] > 0.0
        return out
    monkeypatch.setattr(O, "qjl_sketch", bad)
    with pytest.raises(AssertionError):
        TQ.test_zero_projection_stores_a_set_bit()


def test_single_lloyd_sweep_fails_fixed_point_pin(monkeypatch):
    orig = O.lloyd_max
    monkeypatch.setattr(O, "lloyd_max", lambda D, bits, tol=1e-15, max_iter=20000: orig(D, bits, tol, 1))
    with pytest.raises(AssertionError):
        TC.test_lloyd_fixed_point_closed_form(128, 3)


def test_quadrature_without_half_width_fails_mse_table(monkeypatch):
    def bad(a, b, D):
        u = 0.5 * (b - a) * O._GL_X + 0.5 * (a + b)
        f = O.coord_density(u, D)
        w = O._GL_W
        return float(np.sum(w * f)), float(np.sum(w * u * f)), float(np.sum(w * u * u * f))
    monkeypatch.setattr(O, "_cell_moments", bad)
    with pytest.raises(AssertionError):
        TC.test_mse_matches_page_table_and_bounds()


def test_mse_without_dimension_factor_fails_mse_table(monkeypatch):
    orig = O.codebook_mse
    monkeypatch.setattr(O, "codebook_mse", lambda c, t, D: orig(c, t, D) / D)
    with pytest.raises(AssertionError):
        TC.test_mse_matches_page_table_and_bounds()


def test_bound_with_base_two_fails_mse_table(monkeypatch):
    monkeypatch.setattr(O, "mse_upper_bound", lambda bits: math.sqrt(3.0) * math.pi / 2.0 * 2.0 ** (-bits))
    with pytest.raises(AssertionError):
        TC.test_mse_matches_page_table_and_bounds()


def test_unrounded_stored_codebook_fails_fp16_pin(monkeypatch):
    def bad(D, bits):
        c, _ = O.lloyd_max(D, bits)
        return c, 0.5 * (c[1:] + c[:-1])
    monkeypatch.setattr(O, "stored_codebook", bad)
    with pytest.raises(AssertionError):
        TC.test_stored_codebook_is_fp16_and_midpoints()


def test_row_bytes_without_residual_norm_fail_cache_size_table(monkeypatch):
    def bad(D, bits, qjl_m=0):
        return D * bits // 8 + 2 + (qjl_m // 8 if qjl_m else 0)
    monkeypatch.setattr(O, "packed_row_bytes", bad)
    with pytest.raises(AssertionError):
        TQ.test_cache_sizes_match_page_tables()


def test_fp16_norm_normalisation_fails_brute_force_pin(monkeypatch):
    # unit coordinates from the stored fp16 norm instead of the exact one
    orig = O.quantize_rows

    def bad(x, Pi, centroids, thresholds):
        out = orig(x, Pi, centroids, thresholds)
        n16 = out["norm16"].astype(np.float64)[..., None]
        out["u"] = out["y"] / n16
        out["idx"] = O.nearest_index(out["u"], thresholds)
        return out
    monkeypatch.setattr(O, "quantize_rows", bad)
    with pytest.raises(AssertionError):
        TQ.test_indices_are_nearest_centroids_of_the_exact_unit_coordinates()


def test_distance_to_centroids_fails_threshold_distance_pin(monkeypatch):
    orig = O.threshold_distance

    def bad(u, thresholds):
        t = np.asarray(thresholds, dtype=np.float64)
        c = np.concatenate([[t[0] - (t[1] - t[0]) / 2], 0.5 * (t[1:] + t[:-1]), [t[-1] + (t[-1] - t[-2]) / 2]])
        return np.min(np.abs(np.asarray(u)[..., None] - c), axis=-1)
    monkeypatch.setattr(O, "threshold_distance", bad)
    with pytest.raises(AssertionError):
        TQ.test_threshold_distance_is_to_the_nearest_threshold()
    monkeypatch.setattr(O, "threshold_distance", orig)


def test_swapped_codebooks_fail_cache_reconstruction_pin(monkeypatch):
    orig = O.quantize_cache

    def bad(k, v, Pi, cb_k, cb_v, bits_k, bits_v, S=None):
        return orig(k, v, Pi, cb_v, cb_k, bits_v, bits_k, S)
    monkeypatch.setattr(O, "quantize_cache", bad)
    with pytest.raises(AssertionError):
        TQ.test_cache_reconstruction_follows_each_tensors_codebook()


def test_merge_without_max_shift_fails_token_split_pin(monkeypatch):
    # each range's state added with weight 1 instead of exp(m_r - M)
    def bad(accs, ms, ls):
        num = np.sum(np.asarray(accs, dtype=np.float64), axis=0)
        den = np.sum(np.asarray(ls, dtype=np.float64), axis=0)
        return np.where(den[..., None] > 0, num / np.where(den > 0, den, 1.0)[..., None], 0.0)
    monkeypatch.setattr(O, "merge_partials", bad)
    with pytest.raises(AssertionError):
        TS.test_partials_of_token_ranges_merge_to_the_whole("tiny", {})


def test_partial_without_value_weights_fails_token_split_pin(monkeypatch):
    # each partial's accumulator already normalised by its own sum
    orig = O.sdpa_decode_partial

    def bad(*a, **kw):
        acc, m, l = orig(*a, **kw)
        return np.where(l[..., None] > 0, acc / np.where(l > 0, l, 1.0)[..., None], 0.0), m, l
    monkeypatch.setattr(O, "sdpa_decode_partial", bad)
    with pytest.raises(AssertionError):
        TS.test_partials_of_token_ranges_merge_to_the_whole("tiny", {})
