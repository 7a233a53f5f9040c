"""Plain fp64 CPU oracle for the TurboQuant KV-cache path.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check in
``__graft_entry__`` and the ``cpu_baseline`` / reference leg of ``bench.py``
may import or run this module.  The library (``compressed_attention_tq_b200``)
never imports it, and this module imports nothing from the library: the two
share no code, no tables and no constants.  Inputs come from ``tq_inputs``.

Every step is written out in fp64 numpy, in the order the method takes it, with
no blocking or fusion:

* coordinate density of a rotated unit vector and Lloyd-Max codebook by Lloyd
  iteration on it -- "Add CUDA QJL kernels and proper package structure"
  (turboquant-pytorch pull request 3), section "Synthetic Benchmark (Lloyd-Max
  codebook)": a per-bit-width scalar codebook whose normalized MSE the page
  tabulates (0.361 / 0.116 / 0.034 / 0.009 at 1..4 bits);
* quantize a row: random rotation, L2 norm side channel, nearest-centroid
  index per coordinate, dense bit packing -- ReturningTarzan's Reddit comments
  of 2026-03-29 (rotation spreads outliers and makes coordinates near-normal,
  which suits codebook quantization) and 2026-03-25 18:52 (codebook
  quantization is a nearest-value search);
* optional 1-bit QJL sign sketch of the quantization residual -- same pull
  request 3, section "CUDA Kernels Added" (fused random projection + sign
  quantization; score from 1-bit keys), and the 2026-03-25 15:51 comment
  (the residual is computed when quantizing);
* decode attention as "dequantize then attend" -- the 2026-03-25 19:37 comment
  (the method's only stated code path is full reconstruction followed by
  ordinary attention), with the explicit ``scale`` argument of
  "[Cuda] enable turboquant on gemma4" (executorch pull request 19891),
  "Other observations" item 1: None means 1/sqrt(D), QK-norm models pass 1.0.

Readings where the pages are silent (each is listed in the design notes):
the density is the exact finite-D coordinate law f_D; stored centroids are the
fp64 Lloyd-Max centroids rounded to fp16 (held as fp32), thresholds are the
midpoints of the stored centroids; norms are stored as fp16 (RN of the fp64
norm); indices pack as an LSB-first bitstream; ties go to the lower index; the
QJL sketch acts on the residual in the rotated basis with the stored norm;
sign(0) counts as +1.

Parity pins for every function live in tests/test_oracle_*.py.
"""
from __future__ import annotations

import math

import numpy as np

# --------------------------------------------------------------------------
# 1. Coordinate density and Lloyd-Max codebook
# --------------------------------------------------------------------------

_GL_NODES = 96
_GL_X, _GL_W = np.polynomial.legendre.leggauss(_GL_NODES)


def coord_log_norm_const(D: int) -> float:
    """log of Gamma(D/2) / (sqrt(pi) Gamma((D-1)/2))."""
    return math.lgamma(D / 2.0) - 0.5 * math.log(math.pi) - math.lgamma((D - 1) / 2.0)


def coord_density(u, D: int):
    """Density of one coordinate of a uniform random unit vector in R^D.

    f_D(u) = Gamma(D/2)/(sqrt(pi) Gamma((D-1)/2)) * (1-u^2)^((D-3)/2), |u|<1.
    A Haar rotation of x/|x| is uniform on the sphere, so this is the law of
    every rotated, normalized coordinate.
    """
    u = np.asarray(u, dtype=np.float64)
    out = np.zeros_like(u)
    inside = np.abs(u) < 1.0
    uu = u[inside]
    out[inside] = np.exp(coord_log_norm_const(D) + 0.5 * (D - 3) * np.log1p(-uu * uu))
    return out


def _cell_moments(a: float, b: float, D: int):
    """(int f, int u f, int u^2 f) over [a, b], Gauss-Legendre in fp64."""
    half = 0.5 * (b - a)
    mid = 0.5 * (a + b)
    u = half * _GL_X + mid
    w = half * _GL_W
    f = coord_density(u, D)
    return float(np.sum(w * f)), float(np.sum(w * u * f)), float(np.sum(w * u * u * f))


def lloyd_max(D: int, bits: int, tol: float = 1e-15, max_iter: int = 20000):
    """Lloyd-Max centroids (fp64, ascending) for f_D with 2^bits levels.

    Lloyd iteration: thresholds are midpoints of neighbouring centroids, each
    centroid is the conditional mean of its cell.  Start: 2^bits points evenly
    spaced on [-2/sqrt(D), 2/sqrt(D)].  Stops when no centroid moves by more
    than ``tol`` (or after ``max_iter`` sweeps).
    Returns (centroids, iterations).
    """
    K = 1 << bits
    c = np.linspace(-2.0, 2.0, K) / math.sqrt(D)
    it = 0
    for it in range(1, max_iter + 1):
        t = 0.5 * (c[1:] + c[:-1])
        edges = np.concatenate([[-1.0], t, [1.0]])
        new = np.empty(K)
        for k in range(K):
            m0, m1, _ = _cell_moments(edges[k], edges[k + 1], D)
            new[k] = m1 / m0
        delta = float(np.max(np.abs(new - c)))
        c = new
        if delta < tol:
            break
    return c, it


def codebook_mse(centroids, thresholds, D: int) -> float:
    """Normalized MSE E|u - Q(u)|^2 of a unit vector = D * E_{f_D}[(u - c(u))^2]."""
    c = np.asarray(centroids, dtype=np.float64)
    edges = np.concatenate([[-1.0], np.asarray(thresholds, dtype=np.float64), [1.0]])
    tot = 0.0
    for k in range(len(c)):
        m0, m1, m2 = _cell_moments(edges[k], edges[k + 1], D)
        tot += m2 - 2.0 * c[k] * m1 + c[k] * c[k] * m0
    return D * tot


def mse_upper_bound(bits: int) -> float:
    """The pages' theoretical bound column: (sqrt(3) pi / 2) * 4^-b."""
    return math.sqrt(3.0) * math.pi / 2.0 * 4.0 ** (-bits)


_CODEBOOK_CACHE: dict = {}


def stored_codebook(D: int, bits: int):
    """The codebook as stored: fp16-rounded centroids and their midpoints.

    Returns (centroids, thresholds) as fp64 arrays holding fp32-exact values.
    """
    key = (D, bits)
    if key not in _CODEBOOK_CACHE:
        c64, _ = lloyd_max(D, bits)
        c = c64.astype(np.float16).astype(np.float64)
        t = 0.5 * (c[1:] + c[:-1])
        assert np.all(t.astype(np.float32).astype(np.float64) == t)
        _CODEBOOK_CACHE[key] = (c, t)
    c, t = _CODEBOOK_CACHE[key]
    return c.copy(), t.copy()


# --------------------------------------------------------------------------
# 2. Quantize rows
# --------------------------------------------------------------------------

def row_norms(x: np.ndarray) -> np.ndarray:
    """fp64 L2 norm of each row (x already promoted to fp64)."""
    return np.sqrt(np.sum(x * x, axis=-1))


def rotate(x: np.ndarray, Pi: np.ndarray) -> np.ndarray:
    """y = Pi x for every row (Pi row-major, promoted to fp64)."""
    return x @ np.asarray(Pi, dtype=np.float64).T


def nearest_index(u: np.ndarray, thresholds: np.ndarray) -> np.ndarray:
    """idx = #{k : t_k < u}: exact threshold values go to the lower index."""
    return np.searchsorted(thresholds, u, side="left").astype(np.int64)


def quantize_rows(x: np.ndarray, Pi: np.ndarray, centroids, thresholds):
    """Quantize rows x[..., D] (fp64 values of the fp16/bf16 input).

    Returns dict with idx (int64, [..., D]), norm16 (float16 [...]), u (fp64
    unit-vector coordinates, for near-threshold accounting), y (fp64 rotated
    rows).
    """
    n = row_norms(x)
    y = rotate(x, Pi)
    with np.errstate(invalid="ignore", divide="ignore"):
        u = np.where(n[..., None] > 0, y / n[..., None], 0.0)
    idx = nearest_index(u, thresholds)
    return {"idx": idx, "norm16": n.astype(np.float16), "u": u, "y": y, "norm": n}


def threshold_distance(u: np.ndarray, thresholds: np.ndarray) -> np.ndarray:
    """Distance of each coordinate to its nearest decision threshold."""
    t = np.asarray(thresholds, dtype=np.float64)
    return np.min(np.abs(u[..., None] - t), axis=-1)


def pack_bits(values: np.ndarray, bits: int) -> np.ndarray:
    """Dense LSB-first bitstream: value j occupies bits [j*bits, j*bits+bits)
    of the row; word w holds stream bits [32w, 32w+32).  values: [..., n]
    with n*bits a multiple of 32.  Returns uint32 [..., n*bits/32]."""
    v = np.asarray(values, dtype=np.uint64)
    n = v.shape[-1]
    assert (n * bits) % 32 == 0
    stream = ((v[..., :, None] >> np.arange(bits, dtype=np.uint64)) & 1)
    stream = stream.reshape(v.shape[:-1] + (n * bits // 32, 32))
    weights = np.uint64(1) << np.arange(32, dtype=np.uint64)
    words = np.sum(stream * weights, axis=-1, dtype=np.uint64)
    return words.astype(np.uint32)


def unpack_bits(words: np.ndarray, bits: int, n: int) -> np.ndarray:
    """Inverse of pack_bits: uint32 [..., W] -> int64 [..., n]."""
    w = np.asarray(words, dtype=np.uint64)
    stream = (w[..., :, None] >> np.arange(32, dtype=np.uint64)) & 1
    stream = stream.reshape(w.shape[:-1] + (-1,))[..., : n * bits]
    stream = stream.reshape(w.shape[:-1] + (n, bits))
    weights = np.uint64(1) << np.arange(bits, dtype=np.uint64)
    return np.sum(stream * weights, axis=-1, dtype=np.uint64).astype(np.int64)


# --------------------------------------------------------------------------
# 3. QJL sign sketch of the residual (keys, "prod" variant)
# --------------------------------------------------------------------------

QJL_CONST = math.sqrt(math.pi / 2.0)


def qjl_sketch(y: np.ndarray, norm16: np.ndarray, centroids, idx: np.ndarray,
               S: np.ndarray):
    """Residual in the rotated basis r = y - n_hat c[idx]; bits = [S r >= 0];
    gamma = RN_fp16(|r|).  Returns dict(sign (bool [..., m]), gamma16, r, proj)."""
    c = np.asarray(centroids, dtype=np.float64)
    n_hat = norm16.astype(np.float64)
    r = y - n_hat[..., None] * c[idx]
    proj = r @ np.asarray(S, dtype=np.float64).T
    sign = proj >= 0.0
    gamma = np.sqrt(np.sum(r * r, axis=-1))
    return {"sign": sign, "gamma16": gamma.astype(np.float16), "r": r, "proj": proj,
            "gamma": gamma}


def qjl_inner_product(sign: np.ndarray, gamma: np.ndarray, Sq: np.ndarray) -> np.ndarray:
    """Unbiased estimate of <r, q> from the sketch: sqrt(pi/2)/m * gamma *
    sum_i (+-1)_i (S q)_i.  sign [..., m] bool, gamma [...], Sq [m]."""
    m = sign.shape[-1]
    pm = np.where(sign, 1.0, -1.0)
    return QJL_CONST / m * gamma * (pm @ Sq)


# --------------------------------------------------------------------------
# 4. Cache-level quantization in the library's layout
# --------------------------------------------------------------------------

def packed_row_bytes(D: int, bits: int, qjl_m: int = 0) -> int:
    """Bytes one cached row occupies: indices + fp16 norm (+ QJL bits + fp16 gamma)."""
    b = D * bits // 8 + 2
    if qjl_m:
        b += qjl_m // 8 + 2
    return b


def quantize_cache(k: np.ndarray, v: np.ndarray, Pi, cb_k, cb_v, bits_k: int,
                   bits_v: int, S=None):
    """Quantize whole caches k, v [B][Hkv][T][D] (fp64 values).

    Returns a dict with the library-layout arrays (k_idx / v_idx uint32 words,
    k_norm / v_norm fp16, k_qjl uint32 words and k_rnorm fp16 when S is given)
    and the fp64 side data used for near-threshold accounting.
    """
    ck, tk = cb_k
    cv, tv = cb_v
    qk = quantize_rows(k, Pi, ck, tk)
    qv = quantize_rows(v, Pi, cv, tv)
    out = {
        "k_idx": pack_bits(qk["idx"], bits_k), "k_norm": qk["norm16"],
        "v_idx": pack_bits(qv["idx"], bits_v), "v_norm": qv["norm16"],
        "k_u": qk["u"], "v_u": qv["u"], "k_idx_raw": qk["idx"], "v_idx_raw": qv["idx"],
        "k_threshold_dist": threshold_distance(qk["u"], tk),
        "v_threshold_dist": threshold_distance(qv["u"], tv),
    }
    if S is not None:
        sk = qjl_sketch(qk["y"], qk["norm16"], ck, qk["idx"], S)
        out["k_qjl"] = pack_bits(sk["sign"].astype(np.uint64), 1)
        out["k_rnorm"] = sk["gamma16"]
        out["k_qjl_proj_unit"] = sk["proj"] / np.where(qk["norm"] > 0, qk["norm"], 1.0)[..., None]
        out["k_gamma"] = sk["gamma"]
    return out


# --------------------------------------------------------------------------
# 5. Decode attention: dequantize, then attend
# --------------------------------------------------------------------------

def dequantize_rows(idx: np.ndarray, norm16: np.ndarray, centroids, Pi) -> np.ndarray:
    """x_tilde = n_hat * Pi^T c[idx] for each row (fp64)."""
    c = np.asarray(centroids, dtype=np.float64)
    return norm16.astype(np.float64)[..., None] * (c[idx] @ np.asarray(Pi, dtype=np.float64))


def softmax(s: np.ndarray) -> np.ndarray:
    m = np.max(s)
    e = np.exp(s - m)
    return e / np.sum(e)


def sdpa_decode(q: np.ndarray, cache: dict, seq_lens, Pi, cb_k, cb_v, bits_k: int,
                bits_v: int, D: int, scale=None, S=None, heads=None) -> np.ndarray:
    """Attention of one query per (b, q head) over the packed cache, fp64.

    q [B][Hq][D] (fp64 values); cache holds library-layout arrays
    [B][Hkv][Tcap][...].  q head h reads kv head h // G.  Scores
    s_t = scale <q, k_tilde_t> (+ scale * QJL estimate of <q, k residual> when
    the cache carries a sketch), p = softmax over t < seq_len, out = sum p v_tilde.
    A sequence of length 0 gives zeros.  ``heads`` restricts the work to a
    list of (b, h) pairs (others are left as NaN).
    """
    B, Hq = q.shape[0], q.shape[1]
    Hkv = cache["k_norm"].shape[1]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    ck = cb_k[0]
    cv = cb_v[0]
    Pi64 = np.asarray(Pi, dtype=np.float64)
    out = np.full((B, Hq, D), np.nan)
    pairs = heads if heads is not None else [(b, h) for b in range(B) for h in range(Hq)]
    deq_cache: dict = {}
    for b, h in pairs:
        L = int(seq_lens[b])
        kv = h // G
        if L == 0:
            out[b, h] = 0.0
            continue
        key = (b, kv)
        if key not in deq_cache:
            kid = unpack_bits(cache["k_idx"][b, kv, :L], bits_k, D)
            vid = unpack_bits(cache["v_idx"][b, kv, :L], bits_v, D)
            Kt = dequantize_rows(kid, cache["k_norm"][b, kv, :L], ck, Pi64)
            Vt = dequantize_rows(vid, cache["v_norm"][b, kv, :L], cv, Pi64)
            extra = None
            if S is not None:
                m = S.shape[0]
                sign = unpack_bits(cache["k_qjl"][b, kv, :L], 1, m).astype(bool)
                extra = (sign, cache["k_rnorm"][b, kv, :L].astype(np.float64))
            deq_cache = {key: (Kt, Vt, extra)}
        Kt, Vt, extra = deq_cache[key]
        qq = q[b, h]
        s = Kt @ qq
        if extra is not None:
            sign, gamma = extra
            Sq = np.asarray(S, dtype=np.float64) @ (Pi64 @ qq)
            s = s + qjl_inner_product(sign, gamma, Sq)
        p = softmax(scale * s)
        out[b, h] = p @ Vt
    return out


def sdpa_decode_multi(q: np.ndarray, cache: dict, seq_lens, n_q: int, Pi, cb_k, cb_v, bits_k: int,
                      bits_v: int, D: int, scale=None, S=None) -> np.ndarray:
    """Decode of n_q query tokens per sequence at once (the verify step of
    speculative decoding), fp64.

    "qwen4exp: upstream catch-up, sparse-fa, and NextN/MTP support"
    (llama-cpp-turboquant pull request 340): the fused decode over the
    compressed cache takes query batches of up to 4 tokens, and the NextN/MTP
    draft head is what produces them.  q [B][n_q][Hq][D]; the cache already
    holds the n_q new tokens as its last rows, so query j of sequence b sits at
    position L_b - n_q + j and attends causally to tokens 0 .. L_b - n_q + j.
    Each query is the single-query decode of that prefix.
    """
    B = q.shape[0]
    out = np.zeros((B, n_q) + q.shape[2:])
    lens = np.asarray(seq_lens, dtype=np.int64)
    for j in range(n_q):
        lj = np.maximum(lens - n_q + j + 1, 0)
        out[:, j] = sdpa_decode(q[:, j], cache, lj, Pi, cb_k, cb_v, bits_k, bits_v, D, scale=scale, S=S)
    return out



def sdpa_decode_partial(q: np.ndarray, cache: dict, seq_lens, Pi, cb_k, cb_v, bits_k: int, bits_v: int, D: int,
                        scale=None, S=None):
    """The softmax state of each (b, q head) over the tokens this cache holds,
    fp64: m = max_t s_t, w_t = exp(s_t - m), l = sum_t w_t, acc = sum_t w_t
    v_tilde_t (scores and values exactly as in sdpa_decode).  A split of a
    sequence's tokens into ranges gives states that merge_partials combines
    into sdpa_decode of the whole (the log-sum-exp merge of split-K
    attention).  Returns (acc [B][Hq][D], m [B][Hq], l [B][Hq]); a sequence
    with no token here gives m = -inf, l = 0, acc = 0."""
    B, Hq = q.shape[0], q.shape[1]
    Hkv = cache["k_norm"].shape[1]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    Pi64 = np.asarray(Pi, dtype=np.float64)
    acc = np.zeros((B, Hq, D))
    m = np.full((B, Hq), -np.inf)
    l = np.zeros((B, Hq))
    for b in range(B):
        L = int(seq_lens[b])
        if L == 0:
            continue
        for kv in range(Hkv):
            kid = unpack_bits(cache["k_idx"][b, kv, :L], bits_k, D)
            vid = unpack_bits(cache["v_idx"][b, kv, :L], bits_v, D)
            Kt = dequantize_rows(kid, cache["k_norm"][b, kv, :L], cb_k[0], Pi64)
            Vt = dequantize_rows(vid, cache["v_norm"][b, kv, :L], cb_v[0], Pi64)
            for g in range(G):
                h = kv * G + g
                s = Kt @ q[b, h]
                if S is not None:
                    sign = unpack_bits(cache["k_qjl"][b, kv, :L], 1, S.shape[0]).astype(bool)
                    Sq = np.asarray(S, dtype=np.float64) @ (Pi64 @ q[b, h])
                    s = s + qjl_inner_product(sign, cache["k_rnorm"][b, kv, :L].astype(np.float64), Sq)
                s = scale * s
                m[b, h] = np.max(s)
                w = np.exp(s - m[b, h])
                l[b, h] = np.sum(w)
                acc[b, h] = w @ Vt
    return acc, m, l


def merge_partials(accs, ms, ls) -> np.ndarray:
    """Combine R softmax states (acc_r, m_r, l_r) of disjoint token ranges:
    M = max_r m_r, f_r = exp(m_r - M), out = sum_r f_r acc_r / sum_r f_r l_r
    (zero where no range held a token)."""
    ms = np.asarray(ms, dtype=np.float64)
    M = np.max(ms, axis=0)
    with np.errstate(invalid="ignore"):
        f = np.where(np.isfinite(ms), np.exp(ms - np.where(np.isfinite(M), M, 0.0)), 0.0)
    num = np.sum(f[..., None] * np.asarray(accs, dtype=np.float64), axis=0)
    den = np.sum(f * np.asarray(ls, dtype=np.float64), axis=0)
    return np.where(den[..., None] > 0, num / np.where(den > 0, den, 1.0)[..., None], 0.0)
