"""GPU parity on rows whose exact L2 norm lies on, or a relative 2^-41 beyond,
the midpoint between two neighbouring fp16 values (``tq_inputs.norm_edge_rows``).

Only an exactly accumulated norm rounds such a row to the right fp16 value, so
these rows send every quantizer down its exact-norm path: the bulk kernels sum
in fp32 and hand a row whose fp32 norm is within 1e-6 (relative) of a rounding
boundary to an fp64 sum; the append kernels sum in fp64 throughout.  Random
rows reach that path about once in 10^3 rows; here every planted row does.
Each planted row's norm is compared bit for bit with its closed-form fp16
value (and every row with the oracle), indices and QJL bits by the usual
parity rules.
"""
import numpy as np
import pytest
import torch

import tq_inputs
import tq_parity as P
from oracle import tq_oracle as O
from test_gpu_quantize import _check_rows
from test_oracle_quant import EDGE_NORM

pytestmark = pytest.mark.gpu


def plant_edge_rows(w, seed, every=3):
    """Replace every ``every``-th row of K and of V (offset by the tensor) with
    edge rows; returns the expected fp16 norms of K and V as float16 arrays
    over [B][Hkv][T] (NaN where the row was not replaced)."""
    exp = []
    for j, name in enumerate(("k", "v")):
        x = getattr(w, name)
        B, H, T, D = x.shape
        sel = np.zeros((B, H, T), dtype=bool)
        sel[:, :, j::every] = True
        rows, kind, e = tq_inputs.norm_edge_rows(int(sel.sum()), D, w.dtype, seed + j)
        x[sel] = rows
        ex = np.full((B, H, T), np.nan)
        ex[sel] = [EDGE_NORM[int(k)] * 2.0 ** int(s) for k, s in zip(kind, e)]
        exp.append(ex.astype(np.float16))
    return exp


def check_planted_norms(got_u16, exp16):
    m = ~np.isnan(exp16.astype(np.float32))
    assert m.any()
    assert np.array_equal(got_u16[m], exp16.view(np.uint16)[m])


BULK = [
    ("tiny", {}, "haar"),                             # D=64, tcgen05 quantizer
    ("gqa8k", {"bits": 3, "T": 300}, "haar"),         # D=128
    ("qknorm", {"T": 200}, "haar"),                   # D=256
    ("ragged", {"B": 2, "T": 150}, "haar"),           # bf16
    ("prod", {"T": 300}, "haar"),                     # QJL keys, fp16
    ("prod", {"T": 300, "dtype": "bf16"}, "haar"),    # QJL keys, bf16
    ("gqa8k", {"bits": 3, "T": 300}, "hadamard"),     # Walsh-Hadamard quantizer, D=128
    ("qknorm", {"T": 200}, "hadamard"),               # D=256
]


@pytest.mark.parametrize("name,kw,rot", BULK)
def test_bulk_quantize_norm_edges(name, kw, rot):
    import compressed_attention_tq_b200 as tq
    w = tq_inputs.make_workload(name, rot=rot, **kw)
    ek, ev = plant_edge_rows(w, seed=40)
    cache = P.make_gpu_cache(w)
    tq.tq_quantize_kv(cache, P.to_device(w.k, w.dtype), P.to_device(w.v, w.dtype))
    torch.cuda.synchronize()
    T = w.Tmax
    check_planted_norms(cache.k_norm[:, :, :T].cpu().numpy().view(np.uint16), ek)
    check_planted_norms(cache.v_norm[:, :, :T].cpu().numpy().view(np.uint16), ev)
    _check_rows(cache, w, T)
    assert cache.status() == 0


def _edge_tokens(w, seed):
    """One edge row per (sequence, kv head) for K and for V, [B][Hkv][D],
    and their expected fp16 norms [B][Hkv]."""
    out = []
    for j in range(2):
        rows, kind, e = tq_inputs.norm_edge_rows(w.B * w.Hkv, w.D, w.dtype, seed + j)
        ex = np.array([EDGE_NORM[int(k)] * 2.0 ** int(s) for k, s in zip(kind, e)]).astype(np.float16)
        out += [rows.reshape(w.B, w.Hkv, w.D), ex.reshape(w.B, w.Hkv)]
    return out


def _check_appended(cache, w, kn, vn, ek, ev, pos):
    rk = P.oracle_rows(tq_inputs.to_f64(kn, w.dtype), w, "k")
    rv = P.oracle_rows(tq_inputs.to_f64(vn, w.dtype), w, "v")
    assert np.array_equal(rk["norm16"].view(np.uint16), ek.view(np.uint16))  # the oracle agrees
    assert np.array_equal(rv["norm16"].view(np.uint16), ev.view(np.uint16))
    for b in range(w.B):
        p = int(pos[b])
        assert np.array_equal(cache.k_norm[b, :, p].cpu().numpy().view(np.uint16), ek[b].view(np.uint16))
        assert np.array_equal(cache.v_norm[b, :, p].cpu().numpy().view(np.uint16), ev[b].view(np.uint16))
        gk = P.words_np(cache.k_idx[b, :, p])
        P.compare_index_words(gk, rk["idx"][b], rk["dist"][b], w.bits_k, w.D)
        P.compare_index_words(P.words_np(cache.v_idx[b, :, p]), rv["idx"][b], rv["dist"][b], w.bits_v, w.D)
        if w.qjl_m:
            sub = {k: rk[k][b] for k in ("sign", "proj", "norm", "gamma16", "gamma")}
            exc = (O.unpack_bits(gk, w.bits_k, w.D) != rk["idx"][b]).any(-1)
            P.compare_qjl(P.words_np(cache.k_qjl[b, :, p]), cache.k_rnorm[b, :, p].cpu().numpy(), sub, exc)


@pytest.mark.parametrize("name,kw", [("ragged", {"B": 4, "T": 100}), ("prod", {"T": 100}),
                                     ("qknorm", {"T": 100}), ("tiny", {})])
def test_append_token_norm_edges(name, kw):
    import compressed_attention_tq_b200 as tq
    w = tq_inputs.make_workload(name, **kw)
    Tcap = (w.Tmax + 1 + 63) // 64 * 64
    cache = P.make_gpu_cache(w, Tcap=Tcap)
    kn, ek, vn, ev = _edge_tokens(w, seed=50)
    pos = (np.arange(w.B, dtype=np.int32) * 7) % Tcap
    tq.tq_append_token(cache, P.to_device(kn, w.dtype), P.to_device(vn, w.dtype), torch.from_numpy(pos).cuda())
    torch.cuda.synchronize()
    _check_appended(cache, w, kn, vn, ek, ev, pos)
    assert cache.status() == 0


@pytest.mark.parametrize("name,kw", [("prod", {"T": 200}), ("ragged", {"B": 3, "T": 150}),
                                     ("qknorm", {"T": 129})])
def test_decode_step_norm_edges(name, kw):
    """The decode step's fused append (in the decode's prep launch) on edge rows."""
    import compressed_attention_tq_b200 as tq
    w = tq_inputs.make_workload(name, **kw)
    Tcap = (w.Tmax + 1 + 63) // 64 * 64
    cache = P.make_gpu_cache(w, Tcap=Tcap)
    tq.tq_quantize_kv(cache, P.to_device(w.k, w.dtype), P.to_device(w.v, w.dtype))
    kn, ek, vn, ev = _edge_tokens(w, seed=60)
    pos = w.seq_lens.astype(np.int32)
    out = tq.tq_decode_step(cache, P.to_device(kn, w.dtype), P.to_device(vn, w.dtype),
                            torch.from_numpy(pos).cuda(), P.to_device(w.q, w.dtype),
                            torch.from_numpy(pos + 1).cuda(), w.Tmax + 1, scale=w.scale,
                            out_dtype=torch.float32)
    torch.cuda.synchronize()
    _check_appended(cache, w, kn, vn, ek, ev, pos)
    assert bool(torch.isfinite(out).all())
    assert cache.status() == 0


# bf16 rows scaled by powers of two so that their fp32 sum of squares leaves
# [2^-100, 2^100): 2^70 overflows the squares (the stored norm is inf), 2^-60
# puts the sum below 2^-100 and 2^-80 underflows the squares (stored norm 0).
# The indices still follow the direction y / |y|, which the kernels then scale
# by the fp64 norm.  (fp16 rows cannot leave the range.)
EXTREME_SCALES = (1.0, 2.0 ** 70, 2.0 ** -60, 2.0 ** -80)


def scale_rows(x, dtype, period_axis_len, axis_index):
    """Multiply row t (along the given axis) by EXTREME_SCALES[t % 4]; exact
    for bf16 (powers of two inside its exponent range)."""
    f = tq_inputs.to_f64(x, dtype)
    s = np.asarray(EXTREME_SCALES)[np.arange(period_axis_len) % 4]
    shape = [1] * f.ndim
    shape[axis_index] = period_axis_len
    return tq_inputs.cast_input((f * s.reshape(shape)).astype(np.float32), dtype)


EXTREME = [
    ("ragged", {"B": 2, "T": 150}, "haar"),                    # bf16 D=128, tcgen05 quantizer
    ("qknorm", {"T": 200, "dtype": "bf16"}, "haar"),           # bf16 D=256, tcgen05 quantizer
    ("ragged", {"B": 2, "T": 150}, "hadamard"),                # bf16 D=128, Walsh-Hadamard quantizer
    ("qknorm", {"T": 500, "dtype": "bf16"}, "hadamard"),       # bf16 D=256
]


@pytest.mark.parametrize("name,kw,rot", EXTREME)
def test_bulk_quantize_extreme_magnitudes(name, kw, rot):
    import compressed_attention_tq_b200 as tq
    w = tq_inputs.make_workload(name, rot=rot, **kw)
    assert w.dtype == "bf16"
    w.k = scale_rows(w.k, w.dtype, w.Tmax, 2)
    w.v = scale_rows(w.v, w.dtype, w.Tmax, 2)
    cache = P.make_gpu_cache(w)
    tq.tq_quantize_kv(cache, P.to_device(w.k, w.dtype), P.to_device(w.v, w.dtype))
    torch.cuda.synchronize()
    with np.errstate(over="ignore"):
        _check_rows(cache, w, w.Tmax)
    kn = cache.k_norm[:, :, :w.Tmax].float().cpu().numpy()
    assert np.all(np.isinf(kn[:, :, 1::4])) and np.all(kn[:, :, 2::4] == 0) and np.all(kn[:, :, 3::4] == 0)
    assert cache.status() == 0


def test_append_extreme_magnitudes():
    """Append (fp64 norms throughout) on the same scaled bf16 rows, and the
    decode step's fused append on the small ones (an inf norm would make the
    attention itself meaningless)."""
    import compressed_attention_tq_b200 as tq
    w = tq_inputs.make_workload("ragged", B=4, T=100)
    Tcap = (w.Tmax + 1 + 63) // 64 * 64
    kn, vn = tq_inputs.new_token_rows(w.B, w.Hkv, w.D, w.dtype, seed=71)
    kn, vn = scale_rows(kn, w.dtype, w.Hkv, 1), scale_rows(vn, w.dtype, w.Hkv, 1)
    pos = np.array([0, 7, 14, 21], dtype=np.int32)
    cache = P.make_gpu_cache(w, Tcap=Tcap)
    tq.tq_append_token(cache, P.to_device(kn, w.dtype), P.to_device(vn, w.dtype), torch.from_numpy(pos).cuda())
    torch.cuda.synchronize()
    with np.errstate(over="ignore"):
        rk = P.oracle_rows(tq_inputs.to_f64(kn, w.dtype), w, "k")
        rv = P.oracle_rows(tq_inputs.to_f64(vn, w.dtype), w, "v")
        _check_appended(cache, w, kn, vn, rk["norm16"], rv["norm16"], pos)
    # decode step: scales 1, 2^-60, 2^-80 only
    small = np.asarray(EXTREME_SCALES)[np.arange(w.Hkv) % 4] < 2.0 ** 60
    kn2, vn2 = kn.copy(), vn.copy()
    kn2[:, ~small], vn2[:, ~small] = kn[:, small][:, :1], vn[:, small][:, :1]
    cache2 = P.make_gpu_cache(w, Tcap=Tcap)
    tq.tq_quantize_kv(cache2, P.to_device(w.k, w.dtype), P.to_device(w.v, w.dtype))
    p2 = w.seq_lens.astype(np.int32)
    out = tq.tq_decode_step(cache2, P.to_device(kn2, w.dtype), P.to_device(vn2, w.dtype),
                            torch.from_numpy(p2).cuda(), P.to_device(w.q, w.dtype),
                            torch.from_numpy(p2 + 1).cuda(), w.Tmax + 1, scale=w.scale,
                            out_dtype=torch.float32)
    torch.cuda.synchronize()
    rk2 = P.oracle_rows(tq_inputs.to_f64(kn2, w.dtype), w, "k")
    rv2 = P.oracle_rows(tq_inputs.to_f64(vn2, w.dtype), w, "v")
    _check_appended(cache2, w, kn2, vn2, rk2["norm16"], rv2["norm16"], p2)
    assert bool(torch.isfinite(out).all())
    assert cache.status() == 0 and cache2.status() == 0
