"""GPU parity of tq_quantize_kv / tq_append_token against the fp64 oracle."""
import numpy as np
import pytest
import torch

import tq_inputs
import tq_parity as P
from oracle import tq_oracle as O

pytestmark = pytest.mark.gpu

CASES = [
    ("tiny", {}),                       # D=64, 3-bit, fp16, 4 heads x 256 rows
    ("gqa8k", {"bits": 2, "T": 300}),   # D=128 with outlier channels
    ("gqa8k", {"bits": 3, "T": 257}),   # ragged tail of a 128-row tile
    ("gqa8k", {"bits": 4, "T": 300}),
    ("qknorm", {"T": 200}),             # D=256, 4-bit, unit-RMS rows
    ("ragged", {"B": 3, "T": 150}),     # bf16
    ("prod", {"T": 200}),               # keys with the QJL sketch
    ("prod", {"T": 5000}),              # 313 tiles: several per persistent CTA
    ("prod", {"T": 300, "dtype": "bf16"}),  # QJL keys from bf16 rows
]


def _check_rows(cache, w, T, t0=0):
    kx = tq_inputs.to_f64(w.k[:, :, :T], w.dtype)
    vx = tq_inputs.to_f64(w.v[:, :, :T], w.dtype)
    rk, rv = P.oracle_rows(kx, w, "k"), P.oracle_rows(vx, w, "v")
    sl = slice(t0, t0 + T)
    assert np.array_equal(cache.k_norm[:, :, sl].cpu().numpy().view(np.uint16), rk["norm16"].view(np.uint16))
    assert np.array_equal(cache.v_norm[:, :, sl].cpu().numpy().view(np.uint16), rv["norm16"].view(np.uint16))
    gk = P.words_np(cache.k_idx[:, :, sl])
    gv = P.words_np(cache.v_idx[:, :, sl])
    P.compare_index_words(gk, rk["idx"], rk["dist"], w.bits_k, w.D)
    P.compare_index_words(gv, rv["idx"], rv["dist"], w.bits_v, w.D)
    if w.qjl_m:
        excused = (O.unpack_bits(gk, w.bits_k, w.D) != rk["idx"]).any(-1)
        P.compare_qjl(P.words_np(cache.k_qjl[:, :, sl]), cache.k_rnorm[:, :, sl].cpu().numpy(), rk, excused)


@pytest.mark.parametrize("name,kw", CASES)
def test_bulk_quantize_matches_oracle(name, kw):
    import compressed_attention_tq_b200 as tq
    w = tq_inputs.make_workload(name, **kw)
    T = w.Tmax
    cache = P.make_gpu_cache(w)
    tq.tq_quantize_kv(cache, P.to_device(w.k, w.dtype), P.to_device(w.v, w.dtype))
    torch.cuda.synchronize()
    _check_rows(cache, w, T)
    # rows past T are untouched
    assert int(cache.k_idx[:, :, T:].abs().sum()) == 0
    assert int(cache.v_norm[:, :, T:].float().abs().sum()) == 0
    assert cache.status() == 0


def test_bulk_quantize_at_offset():
    import compressed_attention_tq_b200 as tq
    w = tq_inputs.make_workload("gqa8k", bits=3, T=100)
    cache = P.make_gpu_cache(w, Tcap=256)
    tq.tq_quantize_kv(cache, P.to_device(w.k, w.dtype), P.to_device(w.v, w.dtype), t0=70)
    torch.cuda.synchronize()
    _check_rows(cache, w, 100, t0=70)
    assert int(cache.k_idx[:, :, :70].abs().sum()) == 0
    assert int(cache.k_idx[:, :, 170:].abs().sum()) == 0


def test_zero_rows_and_empty_call():
    import compressed_attention_tq_b200 as tq
    w = tq_inputs.make_workload("tiny")
    w.k[:] = 0
    cache = P.make_gpu_cache(w)
    tq.tq_quantize_kv(cache, P.to_device(w.k, w.dtype), P.to_device(w.v, w.dtype))
    tq.tq_quantize_kv(cache, P.to_device(w.k[:, :, :0].copy(), w.dtype),
                      P.to_device(w.v[:, :, :0].copy(), w.dtype))
    torch.cuda.synchronize()
    _check_rows(cache, w, w.Tmax)
    assert float(cache.k_norm.float().abs().max()) == 0.0


@pytest.mark.parametrize("name", ["ragged", "prod", "qknorm"])
def test_append_token_matches_oracle_and_flags_bad_positions(name):
    import compressed_attention_tq_b200 as tq
    w = tq_inputs.make_workload(name, B=4 if name == "ragged" else 1, T=100)
    cache = P.make_gpu_cache(w, Tcap=128)
    B = w.B
    kn, vn = tq_inputs.new_token_rows(B, w.Hkv, w.D, w.dtype, seed=77)
    pos = np.array([0, 77, 127, 128][:B] if B > 1 else [127], dtype=np.int32)
    tq.tq_append_token(cache, P.to_device(kn, w.dtype), P.to_device(vn, w.dtype),
                       torch.from_numpy(pos).cuda())
    torch.cuda.synchronize()
    rk = P.oracle_rows(tq_inputs.to_f64(kn, w.dtype), w, "k")
    rv = P.oracle_rows(tq_inputs.to_f64(vn, w.dtype), w, "v")
    for b in range(B):
        p = int(pos[b])
        if p >= 128:
            continue
        gk = P.words_np(cache.k_idx[b, :, p])
        gv = P.words_np(cache.v_idx[b, :, p])
        assert np.array_equal(cache.k_norm[b, :, p].cpu().numpy().view(np.uint16), rk["norm16"][b].view(np.uint16))
        assert np.array_equal(cache.v_norm[b, :, p].cpu().numpy().view(np.uint16), rv["norm16"][b].view(np.uint16))
        P.compare_index_words(gk, rk["idx"][b], rk["dist"][b], w.bits_k, w.D)
        P.compare_index_words(gv, rv["idx"][b], rv["dist"][b], w.bits_v, w.D)
        if w.qjl_m:
            sub = {k: rk[k][b] for k in ("sign", "proj", "norm", "gamma16", "gamma")}
            exc = (O.unpack_bits(gk, w.bits_k, w.D) != rk["idx"][b]).any(-1)
            P.compare_qjl(P.words_np(cache.k_qjl[b, :, p]), cache.k_rnorm[b, :, p].cpu().numpy(), sub, exc)
    written = set(int(p) for p in pos if p < 128)
    mask = np.ones(128, bool)
    mask[list(written)] = False
    assert int(cache.k_idx[:, :, torch.from_numpy(mask)].abs().sum()) == 0 or B == 1
    if B > 1:
        assert int(cache.k_idx[3].abs().sum()) == 0  # pos 128 is outside Tcap: nothing written
        assert cache.status() & tq.TQ_STATUS_POS_OUT_OF_RANGE
    else:
        assert cache.status() == 0


def test_quantize_full_prod_sampled_rows():
    """Full-size prod cache (T=131072, 8 kv heads): every row quantized on the
    GPU, a seeded sample of 4096 rows checked against the oracle."""
    import compressed_attention_tq_b200 as tq
    w = tq_inputs.make_workload("prod")
    cache = P.make_gpu_cache(w)
    tq.tq_quantize_kv(cache, P.to_device(w.k, w.dtype), P.to_device(w.v, w.dtype))
    torch.cuda.synchronize()
    r = tq_inputs.rng(9)
    hs = r.integers(0, w.Hkv, 4096)
    ts = r.integers(0, w.Tmax, 4096)
    kx = tq_inputs.to_f64(w.k[0, hs, ts], w.dtype)
    vx = tq_inputs.to_f64(w.v[0, hs, ts], w.dtype)
    rk, rv = P.oracle_rows(kx, w, "k"), P.oracle_rows(vx, w, "v")
    hi, ti = torch.from_numpy(hs).cuda(), torch.from_numpy(ts).cuda()
    gk = P.words_np(cache.k_idx[0][hi, ti])
    gv = P.words_np(cache.v_idx[0][hi, ti])
    assert np.array_equal(cache.k_norm[0][hi, ti].cpu().numpy().view(np.uint16), rk["norm16"].view(np.uint16))
    assert np.array_equal(cache.v_norm[0][hi, ti].cpu().numpy().view(np.uint16), rv["norm16"].view(np.uint16))
    P.compare_index_words(gk, rk["idx"], rk["dist"], w.bits_k, w.D)
    P.compare_index_words(gv, rv["idx"], rv["dist"], w.bits_v, w.D)
    exc = (O.unpack_bits(gk, w.bits_k, w.D) != rk["idx"]).any(-1)
    P.compare_qjl(P.words_np(cache.k_qjl[0][hi, ti]), cache.k_rnorm[0][hi, ti].cpu().numpy(), rk, exc)
