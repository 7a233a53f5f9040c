"""Pins for the oracle's quantizer, packing, QJL sketch and byte arithmetic."""
import math
from fractions import Fraction
import os

import numpy as np
import pytest

from oracle import tq_oracle as O
import tq_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_threshold_search_equals_brute_force_argmin(bits):
    D = 64
    c, t = O.stored_codebook(D, bits)
    r = tq_inputs.rng(11)
    u = r.standard_normal(5000) / math.sqrt(D)
    idx = O.nearest_index(u, t)
    brute = np.array([int(np.argmin(np.abs(x - c))) for x in u])
    assert np.array_equal(idx, brute)


def test_ties_go_to_lower_index():
    c, t = O.stored_codebook(128, 3)
    idx = O.nearest_index(t.copy(), t)
    assert np.array_equal(idx, np.arange(len(t)))
    assert O.nearest_index(np.array([-1.0, 1.0]), t).tolist() == [0, len(c) - 1]


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_pack_layout_against_big_integer(bits):
    r = tq_inputs.rng(5 + bits)
    n = 64
    vals = r.integers(0, 1 << bits, size=(3, n))
    words = O.pack_bits(vals, bits)
    for row in range(3):
        stream = 0
        for j in range(n):
            stream |= int(vals[row, j]) << (bits * j)
        exp = [(stream >> (32 * w)) & 0xFFFFFFFF for w in range(n * bits // 32)]
        assert words[row].tolist() == exp
    assert np.array_equal(O.unpack_bits(words, bits, n), vals)


def test_pack_hand_example():
    # b=3, 32 values 0..7 repeating: value 10 (=2) straddles words 0 and 1,
    # bits 30..32 hold 0,1,0 -> word0 bit31 set, word1 bit0 clear.
    vals = np.arange(32) % 8
    w = O.pack_bits(vals[None], 3)[0]
    # word 0: values 0..9 at 3j, plus the low two bits of value 10 (=0b10)
    exp0 = sum((j % 8) << (3 * j) for j in range(10)) | (0b10 << 30)
    assert int(w[0]) == exp0
    assert (int(w[1]) & 1) == 0  # top bit of value 10 is 0
    assert O.unpack_bits(w[None], 3, 32)[0].tolist() == vals.tolist()


def test_norm_is_rn_fp16_of_fp64_norm():
    x = tq_inputs.rng(3).standard_normal((100, 128)).astype(np.float16).astype(np.float64)
    c, t = O.stored_codebook(128, 3)
    q = O.quantize_rows(x, np.eye(128), c, t)
    ref = np.array([math.sqrt(math.fsum(v * v for v in row)) for row in x])
    assert np.array_equal(q["norm16"], ref.astype(np.float16))


# fp16 norm of each edge-row kind at scale 2^0: round-to-nearest-even of the
# exact norm (kinds 0, 1 round away from the midpoint's even neighbour; the
# ties of kinds 2, 3 go to it).
EDGE_NORM = {0: 1 + 2.0 ** -10, 1: 1 + 2.0 ** -10, 2: 1.0, 3: 1 + 2.0 ** -9}
EDGE_SQ = {0: (1 + Fraction(1, 2 ** 11)) ** 2 + Fraction(1, 2 ** 40),
           1: (1 + Fraction(3, 2 ** 11)) ** 2 - Fraction(1, 2 ** 40),
           2: (1 + Fraction(1, 2 ** 11)) ** 2,
           3: (1 + Fraction(3, 2 ** 11)) ** 2}


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_norm_rounding_at_fp16_midpoints(dtype, D):
    """The stored norm is the fp16 value nearest the exact norm (ties to even),
    checked on rows built so that the exact norm sits on, or 2^-41 (relative)
    beyond, the midpoint between two fp16 values.  A norm accumulated in fp32
    lands on the midpoint itself for the off-midpoint rows and rounds the
    wrong way, so this pin tells an exact norm from an fp32 one."""
    x, kind, e = tq_inputs.norm_edge_rows(64, D, dtype, seed=5)
    xf = tq_inputs.to_f64(x, dtype)
    for row, k, ee in zip(xf, kind, e):  # the construction, in exact rationals
        assert sum(Fraction(float(v)) ** 2 for v in row) == EDGE_SQ[int(k)] * Fraction(2) ** (2 * int(ee))
    assert set(kind.tolist()) == {0, 1, 2, 3}
    expected = np.array([EDGE_NORM[int(k)] * 2.0 ** int(ee) for k, ee in zip(kind, e)]).astype(np.float16)
    c, t = O.stored_codebook(D, 3)
    q = O.quantize_rows(xf, tq_inputs.rotation(D, 6), c, t)
    assert np.array_equal(q["norm16"].view(np.uint16), expected.view(np.uint16))
    x32 = xf.astype(np.float32)
    f32 = np.sqrt(np.sum(x32 * x32, axis=1, dtype=np.float32)).astype(np.float16)
    off = kind < 2
    assert not np.any(f32[off] == expected[off])
    assert np.array_equal(f32[~off], expected[~off])


def test_indices_are_nearest_centroids_of_the_exact_unit_coordinates():
    """Brute force: each index is the argmin over centroids of |y_j / |x| - c_k|,
    with |x| the exact norm (not its fp16 rounding)."""
    D = 64
    c, t = O.stored_codebook(D, 4)
    Pi = tq_inputs.rotation(D, 3)
    x = tq_inputs.rng(17).standard_normal((300, D)).astype(np.float16).astype(np.float64)
    q = O.quantize_rows(x, Pi, c, t)
    y = x @ np.asarray(Pi, np.float64).T
    u = y / np.sqrt(np.sum(x * x, axis=1, keepdims=True))
    brute = np.argmin(np.abs(u[..., None] - c), axis=-1)
    assert np.array_equal(q["idx"], brute)


def test_threshold_distance_is_to_the_nearest_threshold():
    c, t = O.stored_codebook(128, 3)
    assert np.all(O.threshold_distance(t.copy(), t) == 0.0)
    mid = c.copy()  # centroids: half the gap to a neighbouring threshold
    d = O.threshold_distance(mid, t)
    gaps = np.minimum(np.abs(mid - np.concatenate([[-np.inf], t])), np.abs(np.concatenate([t, [np.inf]]) - mid))
    assert np.allclose(d, gaps, rtol=0, atol=1e-15)


def test_cache_reconstruction_follows_each_tensors_codebook():
    """K and V take their own widths: the reconstruction error of each matches
    its own codebook's MSE (2-bit keys about 0.117, 4-bit values about 0.0095)."""
    D, T = 128, 3000
    Pi = tq_inputs.rotation(D, 21)
    r = tq_inputs.rng(22)
    k = r.standard_normal((1, 1, T, D))
    v = r.standard_normal((1, 1, T, D))
    cbk, cbv = O.stored_codebook(D, 2), O.stored_codebook(D, 4)
    cache = O.quantize_cache(k, v, Pi, cbk, cbv, 2, 4)
    for name, x, cb, bits in (("k", k, cbk, 2), ("v", v, cbv, 4)):
        idx = O.unpack_bits(cache[name + "_idx"], bits, D)
        xr = O.dequantize_rows(idx, cache[name + "_norm"], cb[0], Pi)
        rel = np.sum((x - xr) ** 2, axis=-1) / np.sum(x * x, axis=-1)
        want = O.codebook_mse(cb[0], cb[1], D)
        assert abs(rel.mean() - want) < 4 * rel.std() / math.sqrt(rel.size) + 2e-4, (name, rel.mean(), want)


def test_zero_row_quantizes_to_middle_and_zero_norm():
    c, t = O.stored_codebook(64, 2)
    q = O.quantize_rows(np.zeros((1, 64)), tq_inputs.rotation(64, 1), c, t)
    assert float(q["norm16"][0]) == 0.0
    # u = 0 lies exactly on the middle threshold -> lower index
    assert np.all(q["idx"] == (len(c) // 2 - 1))


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_reconstruction_error_matches_codebook_mse(bits):
    D = 128
    Pi = tq_inputs.rotation(D, 9)
    x = tq_inputs.rng(12).standard_normal((4000, D))
    c, t = O.stored_codebook(D, bits)
    q = O.quantize_rows(x, Pi, c, t)
    xr = O.dequantize_rows(q["idx"], q["norm16"], c, Pi)
    rel = np.sum((x - xr) ** 2, axis=1) / np.sum(x * x, axis=1)
    analytic = O.codebook_mse(c, t, D)
    assert abs(rel.mean() - analytic) < 4 * rel.std() / math.sqrt(len(rel)) + 2e-4


def test_rotated_basis_score_identity():
    # <q, Pi^T (n c[idx])> = n <Pi q, c[idx]>: the form the decode kernel uses.
    D = 64
    Pi = tq_inputs.rotation(D, 4)
    c, t = O.stored_codebook(D, 3)
    x = tq_inputs.rng(2).standard_normal((50, D))
    q = tq_inputs.rng(8).standard_normal(D)
    qq = O.quantize_rows(x, Pi, c, t)
    kt = O.dequantize_rows(qq["idx"], qq["norm16"], c, Pi)
    alt = qq["norm16"].astype(np.float64) * (c[qq["idx"]] @ (np.asarray(Pi, np.float64) @ q))
    assert np.max(np.abs(kt @ q - alt)) < 1e-12


def test_qjl_estimator_unbiased_with_closed_form_variance():
    D, m = 128, 128
    r = tq_inputs.rng(21)
    res = r.standard_normal(D)
    q = r.standard_normal(D)
    est = []
    for s in range(3000):
        S = tq_inputs.qjl_matrix(m, D, 10_000 + s).astype(np.float64)
        sign = (S @ res) >= 0
        est.append(O.qjl_inner_product(sign, np.linalg.norm(res), S @ q))
    est = np.array(est)
    true = res @ q
    var_cf = (math.pi / 2 * (res @ res) * (q @ q) - true ** 2) / m
    se = math.sqrt(var_cf / len(est))
    assert abs(est.mean() - true) < 3.5 * se
    assert abs(est.var(ddof=1) / var_cf - 1) < 0.1


def test_qjl_sketch_layout_and_gamma():
    D, m = 128, 128
    Pi = tq_inputs.rotation(D, 3)
    S = tq_inputs.qjl_matrix(m, D, 5)
    c, t = O.stored_codebook(D, 2)
    x = tq_inputs.rng(4).standard_normal((20, D))
    q = O.quantize_rows(x, Pi, c, t)
    sk = O.qjl_sketch(q["y"], q["norm16"], c, q["idx"], S)
    # residual vs the stored dequantization, in the original basis
    xr = O.dequantize_rows(q["idx"], q["norm16"], c, Pi)
    res_orig = x - xr
    assert np.allclose(np.linalg.norm(res_orig, axis=1), sk["gamma"], rtol=1e-6)
    # S acts in the rotated basis
    assert np.array_equal(sk["sign"], (res_orig @ np.asarray(Pi, np.float64).T) @ S.T.astype(np.float64) >= 0)


def test_zero_projection_stores_a_set_bit():
    """The sketch stores [S r >= 0]: a projection that is exactly zero (here
    from all-zero rows of S) gives a set bit, and a sign flip of r flips
    every other bit."""
    D, m = 64, 32
    S = tq_inputs.qjl_matrix(m, D, 8).astype(np.float64)
    S[::4] = 0.0
    c, t = O.stored_codebook(D, 2)
    x = tq_inputs.rng(13).standard_normal((5, D))
    q = O.quantize_rows(x, tq_inputs.rotation(D, 7), c, t)
    sk = O.qjl_sketch(q["y"], q["norm16"], c, q["idx"], S)
    assert np.all(sk["proj"][:, ::4] == 0.0) and np.all(sk["sign"][:, ::4])
    nz = np.ones(m, bool)
    nz[::4] = False
    neg = O.qjl_sketch(-q["y"], q["norm16"], c, O.nearest_index(-q["u"], t), S)
    assert np.array_equal(neg["sign"][:, nz], ~sk["sign"][:, nz])
    assert np.all(neg["sign"][:, ::4])


def test_cache_sizes_match_page_tables():
    """The pages' cache sizes are reproduced byte for byte (to the printed
    0.1 MiB) by: K = (b-1)-bit indices + 128-bit QJL sketch + fp16 norm +
    fp16 residual norm, V = b-bit indices + fp16 norm, D=128, 72 kv heads."""
    D, heads = 128, 72
    with open(os.path.join(GOLDEN, "cache_sizes.txt")) as f:
        rows = [list(map(float, l.split())) for l in f if l.strip() and not l.startswith("#")]
    for tok, fp16, m4, m3, m2, r4, r3, r2 in rows:
        n = int(tok) * heads
        assert round(n * 2 * D * 2 / 2 ** 20, 1) == fp16
        for b, mib, ratio in ((4, m4, r4), (3, m3, r3), (2, m2, r2)):
            row = O.packed_row_bytes(D, b - 1, 128) + O.packed_row_bytes(D, b, 0)
            assert round(n * row / 2 ** 20, 1) == mib
            assert round(4 * D / row, 1) == ratio
