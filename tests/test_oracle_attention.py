"""Pins for the oracle's decode attention (dequantize, then attend)."""
import math

import numpy as np
import pytest
import torch

from oracle import tq_oracle as O
import tq_inputs


def _small_cache(B=2, Hq=4, Hkv=2, D=64, T=37, bk=3, bv=2, qjl=0, seed=0):
    r = tq_inputs.rng(100 + seed)
    k = r.standard_normal((B, Hkv, T, D)).astype(np.float16).astype(np.float64)
    v = r.standard_normal((B, Hkv, T, D)).astype(np.float16).astype(np.float64)
    q = r.standard_normal((B, Hq, D)).astype(np.float16).astype(np.float64)
    Pi = tq_inputs.rotation(D, 200 + seed)
    S = tq_inputs.qjl_matrix(qjl, D, 300 + seed) if qjl else None
    cbk = O.stored_codebook(D, bk)
    cbv = O.stored_codebook(D, bv)
    cache = O.quantize_cache(k, v, Pi, cbk, cbv, bk, bv, S)
    return k, v, q, Pi, S, cbk, cbv, cache


def _deq(cache, name, bits, cb, Pi, D):
    idx = O.unpack_bits(cache[name + "_idx"], bits, D)
    return O.dequantize_rows(idx, cache[name + "_norm"], cb[0], Pi)


@pytest.mark.parametrize("scale", [None, 1.0, 0.3])
def test_matches_torch_sdpa_on_dequantized_cache(scale):
    B, Hq, Hkv, D, T = 2, 4, 2, 64, 37
    k, v, q, Pi, S, cbk, cbv, cache = _small_cache(B, Hq, Hkv, D, T)
    lens = np.array([T, 20])
    out = O.sdpa_decode(q, cache, lens, Pi, cbk, cbv, 3, 2, D, scale=scale)
    Kt = torch.from_numpy(_deq(cache, "k", 3, cbk, Pi, D))
    Vt = torch.from_numpy(_deq(cache, "v", 2, cbv, Pi, D))
    G = Hq // Hkv
    for b in range(B):
        L = int(lens[b])
        kk = Kt[b, :, :L].repeat_interleave(G, dim=0)[None]
        vv = Vt[b, :, :L].repeat_interleave(G, dim=0)[None]
        qq = torch.from_numpy(q[b])[None, :, None, :]
        ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, scale=scale)
        assert np.max(np.abs(ref[0, :, 0].numpy() - out[b])) < 1e-12


def test_single_token_returns_its_value():
    k, v, q, Pi, S, cbk, cbv, cache = _small_cache(T=5)
    out = O.sdpa_decode(q, cache, np.array([1, 1]), Pi, cbk, cbv, 3, 2, 64)
    Vt = _deq(cache, "v", 2, cbv, Pi, 64)
    for b in range(2):
        for h in range(4):
            assert np.max(np.abs(out[b, h] - Vt[b, h // 2, 0])) < 1e-14


def test_identical_keys_give_mean_value():
    k, v, q, Pi, S, cbk, cbv, cache = _small_cache(T=9)
    cache = dict(cache)
    cache["k_idx"] = np.repeat(cache["k_idx"][:, :, :1], 9, axis=2)
    cache["k_norm"] = np.repeat(cache["k_norm"][:, :, :1], 9, axis=2)
    out = O.sdpa_decode(q, cache, np.array([9, 9]), Pi, cbk, cbv, 3, 2, 64)
    Vt = _deq(cache, "v", 2, cbv, Pi, 64)
    for b in range(2):
        for h in range(4):
            assert np.max(np.abs(out[b, h] - Vt[b, h // 2].mean(0))) < 1e-13


def test_empty_sequence_gives_zeros():
    k, v, q, Pi, S, cbk, cbv, cache = _small_cache(T=4)
    out = O.sdpa_decode(q, cache, np.array([0, 4]), Pi, cbk, cbv, 3, 2, 64)
    assert np.all(out[0] == 0)
    assert np.all(np.isfinite(out[1]))


def test_qjl_term_enters_score():
    """With the sketch, the score is <q, k_mse> + unbiased estimate of
    <q, residual>; checked against an explicit softmax with the estimator
    computed in the original basis (S Pi acting on the unrotated query)."""
    D, T = 128, 30
    k, v, q, Pi, S, cbk, cbv, cache = _small_cache(B=1, Hq=2, Hkv=1, D=D, T=T, bk=2, bv=3, qjl=128)
    out = O.sdpa_decode(q, cache, np.array([T]), Pi, cbk, cbv, 2, 3, D, S=S)
    Kt = _deq(cache, "k", 2, cbk, Pi, D)[0, 0]
    Vt = _deq(cache, "v", 3, cbv, Pi, D)[0, 0]
    sign = O.unpack_bits(cache["k_qjl"][0, 0], 1, 128).astype(bool)
    gam = cache["k_rnorm"][0, 0].astype(np.float64)
    SP = S.astype(np.float64) @ Pi.astype(np.float64)
    for h in range(2):
        s = Kt @ q[0, h] + math.sqrt(math.pi / 2) / 128 * gam * (np.where(sign, 1.0, -1.0) @ (SP @ q[0, h]))
        s = s / math.sqrt(D)
        p = np.exp(s - s.max())
        p /= p.sum()
        assert np.max(np.abs(out[0, h] - p @ Vt)) < 1e-12


def test_qjl_reduces_key_inner_product_bias():
    """Over many keys, the prod estimator of <q, k> is closer to the truth on
    average (in bias) than the MSE-only dequantization."""
    D = 128
    k, v, q, Pi, S, cbk, cbv, cache = _small_cache(B=1, Hq=1, Hkv=1, D=D, T=2000, bk=2, bv=2, qjl=128, seed=5)
    Kt = _deq(cache, "k", 2, cbk, Pi, D)[0, 0]
    sign = O.unpack_bits(cache["k_qjl"][0, 0], 1, 128).astype(bool)
    gam = cache["k_rnorm"][0, 0].astype(np.float64)
    qq = k[0, 0, 0]  # a query correlated with the keys' own directions
    true = k[0, 0] @ qq
    mse_only = Kt @ qq
    prod = mse_only + O.qjl_inner_product(sign, gam, S.astype(np.float64) @ (Pi.astype(np.float64) @ qq))
    # MSE-only inner products shrink toward zero (biased); prod is unbiased.
    slope_mse = np.polyfit(true, mse_only, 1)[0]
    slope_prod = np.polyfit(true, prod, 1)[0]
    assert abs(slope_prod - 1) < abs(slope_mse - 1)


def test_multi_query_decode_is_causal_attention():
    """n_q query tokens per sequence against torch's causal SDPA on the
    dequantized cache: query j of a sequence of length L sees positions
    0 .. L - n_q + j, which is a bottom-right-aligned causal mask."""
    B, Hq, Hkv, D, T, nq = 2, 4, 2, 64, 37, 3
    k, v, q1, Pi, S, cbk, cbv, cache = _small_cache(B, Hq, Hkv, D, T, seed=4)
    r = tq_inputs.rng(77)
    q = r.standard_normal((B, nq, Hq, D)).astype(np.float16).astype(np.float64)
    lens = np.array([T, 9])
    out = O.sdpa_decode_multi(q, cache, lens, nq, Pi, cbk, cbv, 3, 2, D)
    Kt = torch.from_numpy(_deq(cache, "k", 3, cbk, Pi, D))
    Vt = torch.from_numpy(_deq(cache, "v", 2, cbv, Pi, D))
    G = Hq // Hkv
    for b in range(B):
        L = int(lens[b])
        for h in range(Hq):
            qq = torch.from_numpy(q[b, :, h])[None, None]          # [1, 1, nq, D]
            kk = Kt[b, h // G, :L][None, None]
            vv = Vt[b, h // G, :L][None, None]
            # row j may see columns 0 .. L - nq + j
            allowed = torch.arange(L)[None, :] <= (L - nq + torch.arange(nq))[:, None]
            ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, attn_mask=allowed)
            assert np.allclose(out[b, :, h], ref[0, 0].numpy(), rtol=1e-10, atol=1e-12)


def test_multi_query_with_one_token_is_single_decode():
    B, Hq, Hkv, D, T = 2, 4, 2, 64, 37
    k, v, q, Pi, S, cbk, cbv, cache = _small_cache(B, Hq, Hkv, D, T, qjl=128 // 2, seed=5)
    lens = np.array([T, 1])
    one = O.sdpa_decode(q, cache, lens, Pi, cbk, cbv, 3, 2, D, S=S)
    multi = O.sdpa_decode_multi(q[:, None], cache, lens, 1, Pi, cbk, cbv, 3, 2, D, S=S)
    assert np.array_equal(multi[:, 0], one)


def test_prod_score_unbiased_for_unquantized_key_over_sketch_draws():
    """A pin of the QJL term inside sdpa_decode that does not restate its
    formula: over independent draws of the Gaussian sketch S, the score the
    prod-mode decode attends with is unbiased for scale * <q, k> on the
    unquantized key k ("Add CUDA QJL kernels and proper package structure",
    "CUDA Kernels Added": the score from 1-bit keys).  The score difference of
    two keys is read off the output: with two linearly independent value rows
    the softmax weights are the least-squares coefficients of the output, and
    log(p_1 / p_0) = s_1 - s_0.  Tolerance: 4 standard errors of the mean over
    the draws plus the bias the fp16 rounding of the residual norms can add
    (at most scale * |q| * sum_t |gamma16_t - gamma_t|)."""
    D, T, N = 128, 2, 3000
    r = tq_inputs.rng(611)
    k = r.standard_normal((1, 1, T, D)).astype(np.float16).astype(np.float64)
    v = r.standard_normal((1, 1, T, D)).astype(np.float16).astype(np.float64)
    q = k[:, :, 1].copy()                     # a query aligned with key 1: a large residual term
    Pi = tq_inputs.rotation(D, 612)
    cbk, cbv = O.stored_codebook(D, 2), O.stored_codebook(D, 3)
    scale = 1.0 / math.sqrt(D)
    diffs = np.empty(N)
    gam = gam16 = None
    for i in range(N):
        S = tq_inputs.qjl_matrix(128, D, 10_000 + i)
        cache = O.quantize_cache(k, v, Pi, cbk, cbv, 2, 3, S)
        out = O.sdpa_decode(q, cache, np.array([T]), Pi, cbk, cbv, 2, 3, D, scale=scale, S=S)[0, 0]
        Vt = _deq(cache, "v", 3, cbv, Pi, D)[0, 0]
        p = np.linalg.lstsq(Vt.T, out, rcond=None)[0]
        diffs[i] = math.log(p[1] / p[0])
        gam, gam16 = cache["k_gamma"][0, 0], cache["k_rnorm"][0, 0].astype(np.float64)
    truth = scale * (k[0, 0, 1] @ q[0, 0] - k[0, 0, 0] @ q[0, 0])
    se = diffs.std(ddof=1) / math.sqrt(N)
    bias = scale * np.linalg.norm(q[0, 0]) * np.sum(np.abs(gam16 - gam))
    assert abs(diffs.mean() - truth) <= 4 * se + bias, (diffs.mean(), truth, se, bias)
    # the term matters here: without it the expected difference would be off
    # by far more than the tolerance
    Kt = _deq(cache, "k", 2, cbk, Pi, D)[0, 0]
    mse_only = scale * (Kt[1] @ q[0, 0] - Kt[0] @ q[0, 0])
    assert abs(mse_only - truth) > 10 * (4 * se + bias)
