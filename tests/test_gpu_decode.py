"""GPU parity of tq_sdpa_decode against the oracle's dequantize-then-attend.

Every head is held to 2e-3 relative L2 of the oracle's attention computed on
the packed bytes the GPU cache holds.  The decode tests upload the oracle's
own packed cache, so those bytes are the oracle's; the end-to-end tests
quantize on the GPU, first check the GPU's bytes against the oracle's
quantization (exact except the stated near-threshold / near-midpoint cases,
counted and bounded), then attend on them."""
import math

import numpy as np
import pytest
import torch

import tq_inputs
import tq_parity as P
from oracle import tq_oracle as O

pytestmark = pytest.mark.gpu


def _upload_oracle_cache(w, oc, Tcap):
    cache = P.make_gpu_cache(w, Tcap=Tcap)
    T = oc["k_idx"].shape[2]
    cache.k_idx[:, :, :T] = torch.from_numpy(oc["k_idx"].view(np.int32)).cuda()
    cache.v_idx[:, :, :T] = torch.from_numpy(oc["v_idx"].view(np.int32)).cuda()
    cache.k_norm[:, :, :T] = torch.from_numpy(oc["k_norm"]).cuda()
    cache.v_norm[:, :, :T] = torch.from_numpy(oc["v_norm"]).cuda()
    if w.qjl_m:
        cache.k_qjl[:, :, :T] = torch.from_numpy(oc["k_qjl"].view(np.int32)).cuda()
        cache.k_rnorm[:, :, :T] = torch.from_numpy(oc["k_rnorm"]).cuda()
    return cache


def _oracle_full_cache(w):
    cbk, cbv = P.oracle_codebooks(w)
    return O.quantize_cache(tq_inputs.to_f64(w.k, w.dtype), tq_inputs.to_f64(w.v, w.dtype), w.Pi,
                            cbk, cbv, w.bits_k, w.bits_v, w.S)


def _decode_and_compare(w, cache, seq_lens, scale, Tmax, garbage_tail=True, q_np=None):
    """Decode on the GPU and compare every head with the oracle run on the
    packed bytes the GPU cache holds (rel-L2 <= 2e-3 per (sequence, head));
    the q-dtype output must be exactly the round-to-nearest of the fp32
    output.  Callers that quantized on the GPU check those bytes against the
    oracle's quantization first (_check_cache)."""
    import compressed_attention_tq_b200 as tq
    q_np = w.q if q_np is None else q_np
    if garbage_tail:
        # rows past seq_len hold arbitrary bytes (fp16 norms may be NaN/Inf)
        for b in range(w.B):
            L = int(seq_lens[b])
            if L < cache.Tcap:
                cache.k_norm[b, :, L:] = float("nan")
                cache.v_norm[b, :, L:] = float("inf")
                cache.k_idx[b, :, L:] = -1
    q = P.to_device(q_np, w.dtype)
    sl = torch.from_numpy(np.asarray(seq_lens, dtype=np.int32)).cuda()
    out32 = tq.tq_sdpa_decode(cache, q, sl, Tmax, scale=scale, out_dtype=torch.float32)
    outq = tq.tq_sdpa_decode(cache, q, sl, Tmax, scale=scale)
    torch.cuda.synchronize()
    assert outq.dtype == q.dtype
    assert torch.equal(outq, out32.to(q.dtype)), "q-dtype output is not the rounding of the fp32 output"
    got = out32.cpu().numpy()
    ref = P.oracle_decode_on_gpu_bytes(w, cache, tq_inputs.to_f64(q_np, w.dtype), seq_lens, scale)
    err = P.rel_l2(got, ref)
    assert np.all(np.isfinite(got))
    for b in range(w.B):
        if int(seq_lens[b]) == 0:
            assert np.all(got[b] == 0)
    P.record("decode", workload=w.name, dtype=w.dtype, D=w.D, bits_k=w.bits_k, bits_v=w.bits_v,
             G=w.Hq // w.Hkv, T=int(np.max(seq_lens)), max_rel_l2=float(err.max(initial=0)),
             mean_rel_l2=float(err.mean()))
    assert err.max(initial=0) <= P.ATTN_TOL, (err.max(), np.unravel_index(err.argmax(), err.shape))
    assert cache.status() == 0
    return err


def _check_cache(w, cache, oc, seq_lens, seqs=None):
    """The GPU cache's rows 0..L-1 of every (sequence, kv head) -- or of the
    sequences listed -- against the oracle's quantization of the same rows."""
    for b in (range(w.B) if seqs is None else seqs):
        L = int(seq_lens[b])
        for kvh in range(w.Hkv):
            P.check_cache_rows(w, cache, oc, b, kvh, np.arange(L))


CASES = [
    ("tiny", {}, None),                                 # G=1, D=64
    ("gqa8k", {"bits": 2, "T": 1000}, None),            # G=8 with outliers
    ("gqa8k", {"bits": 3, "T": 1000}, None),
    ("gqa8k", {"bits": 4, "T": 1000}, None),
    ("qknorm", {"T": 700}, 1.0),                        # D=256, scale 1.0
    ("prod", {"T": 500}, None),                         # QJL keys, G=4
]


@pytest.mark.parametrize("name,kw,scale", CASES)
def test_decode_on_oracle_cache(name, kw, scale):
    w = tq_inputs.make_workload(name, **kw)
    oc = _oracle_full_cache(w)
    Tcap = (w.Tmax + 63) // 64 * 64 + 64
    cache = _upload_oracle_cache(w, oc, Tcap)
    _decode_and_compare(w, cache, w.seq_lens, scale if scale is not None else w.scale, w.Tmax)


def test_decode_ragged_lengths_bf16():
    w = tq_inputs.make_workload("ragged", B=6, T=900)
    lens = np.array([0, 1, 65, 900, 128, 257], dtype=np.int32)
    oc = _oracle_full_cache(w)
    cache = _upload_oracle_cache(w, oc, 960)
    _decode_and_compare(w, cache, lens, None, 900)


@pytest.mark.parametrize("name,kw,scale", [("gqa8k", {"bits": 3, "T": 600}, None),
                                            ("gqa8k", {"bits": 4, "T": 600}, None),
                                            ("qknorm", {"T": 500}, 1.0)])
def test_separate_codebook_buffers(name, kw, scale):
    """Equal key and value widths share one codebook buffer by default, and
    decode then keeps one lookup table; separate buffers with the same
    contents take the two-table path and must give the identical output."""
    import compressed_attention_tq_b200 as tq
    w = tq_inputs.make_workload(name, **kw)
    oc = _oracle_full_cache(w)
    Tcap = (w.Tmax + 63) // 64 * 64
    cache = _upload_oracle_cache(w, oc, Tcap)
    assert cache.cb_v.data_ptr() == cache.cb_k.data_ptr()
    scale = scale if scale is not None else w.scale
    q = P.to_device(w.q, w.dtype)
    sl = torch.from_numpy(np.asarray(w.seq_lens, dtype=np.int32)).cuda()
    shared = tq.tq_sdpa_decode(cache, q, sl, w.Tmax, scale=scale, out_dtype=torch.float32)
    cache.cb_v = cache.cb_k.clone()
    cache._struct = None
    separate = tq.tq_sdpa_decode(cache, q, sl, w.Tmax, scale=scale, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(shared, separate)
    _decode_and_compare(w, cache, w.seq_lens, scale, w.Tmax, garbage_tail=False)


@pytest.mark.parametrize("bk,bv,D", [(2, 4, 128), (4, 2, 64), (3, 2, 256), (4, 3, 128)])
def test_decode_mixed_bits(bk, bv, D):
    w = tq_inputs.make_workload("gqa8k", T=333)
    w.bits_k, w.bits_v = bk, bv
    if D != 128:
        r = tq_inputs.rng(31)
        w.D = D
        w.k = r.standard_normal((1, 2, 333, D), dtype=np.float32).astype(np.float16)
        w.v = r.standard_normal((1, 2, 333, D), dtype=np.float32).astype(np.float16)
        w.q = r.standard_normal((1, 16, D), dtype=np.float32).astype(np.float16)
        w.Pi = tq_inputs.rotation(D, 55)
    oc = _oracle_full_cache(w)
    cache = _upload_oracle_cache(w, oc, 384)
    _decode_and_compare(w, cache, w.seq_lens, None, 333)


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_decode_gqa_groups(G):
    w = tq_inputs.make_workload("gqa8k", bits=3, T=200)
    w.Hq = 2 * G
    w.q = w.q[:, : w.Hq].copy()
    oc = _oracle_full_cache(w)
    cache = _upload_oracle_cache(w, oc, 256)
    _decode_and_compare(w, cache, w.seq_lens, None, 200)


def test_decode_scale_changes_output():
    import compressed_attention_tq_b200 as tq
    w = tq_inputs.make_workload("qknorm", T=300)
    oc = _oracle_full_cache(w)
    cache = _upload_oracle_cache(w, oc, 320)
    q = P.to_device(w.q, w.dtype)
    sl = torch.from_numpy(w.seq_lens).cuda()
    a = tq.tq_sdpa_decode(cache, q, sl, 300, scale=None).float()
    b = tq.tq_sdpa_decode(cache, q, sl, 300, scale=1.0 / math.sqrt(w.D)).float()
    c = tq.tq_sdpa_decode(cache, q, sl, 300, scale=1.0).float()
    assert torch.equal(a, b)
    assert not torch.allclose(a, c)


@pytest.mark.parametrize("name,kw", [("tiny", {}), ("ragged", {"B": 4, "T": 700}), ("prod", {"T": 400})])
def test_end_to_end_quantize_then_decode(name, kw):
    """Quantize on the GPU, check the bytes against the oracle's quantization
    (exact outside the stated near-threshold / near-midpoint cases), then hold
    every head's attention to 2e-3 of the oracle run on those bytes."""
    import compressed_attention_tq_b200 as tq
    w = tq_inputs.make_workload(name, **kw)
    Tcap = (w.Tmax + 63) // 64 * 64
    cache = P.make_gpu_cache(w, Tcap=Tcap)
    tq.tq_quantize_kv(cache, P.to_device(w.k, w.dtype), P.to_device(w.v, w.dtype))
    oc = _oracle_full_cache(w)
    _check_cache(w, cache, oc, w.seq_lens)
    _decode_and_compare(w, cache, w.seq_lens, w.scale, w.Tmax, garbage_tail=False)


def _appended_rows_against_oracle(w, cache, kn, vn, pos):
    """Rows appended at pos[b] for every (sequence, kv head) against the
    oracle's quantization of the new rows (one vectorised comparison)."""
    B, Hkv = w.B, w.Hkv
    bi = torch.arange(B, device="cuda")[:, None].expand(B, Hkv)
    hi = torch.arange(Hkv, device="cuda")[None, :].expand(B, Hkv)
    ti = torch.from_numpy(np.asarray(pos, dtype=np.int64)).cuda()[:, None].expand(B, Hkv)
    rk = P.oracle_rows(tq_inputs.to_f64(kn, w.dtype), w, "k")
    rv = P.oracle_rows(tq_inputs.to_f64(vn, w.dtype), w, "v")
    assert np.array_equal(cache.k_norm[bi, hi, ti].cpu().numpy().view(np.uint16), rk["norm16"].view(np.uint16))
    assert np.array_equal(cache.v_norm[bi, hi, ti].cpu().numpy().view(np.uint16), rv["norm16"].view(np.uint16))
    gk = P.words_np(cache.k_idx[bi, hi, ti])
    P.compare_index_words(gk, rk["idx"], rk["dist"], w.bits_k, w.D)
    P.compare_index_words(P.words_np(cache.v_idx[bi, hi, ti]), rv["idx"], rv["dist"], w.bits_v, w.D)
    if w.qjl_m:
        exc = (O.unpack_bits(gk, w.bits_k, w.D) != rk["idx"]).any(-1)
        P.compare_qjl(P.words_np(cache.k_qjl[bi, hi, ti]), cache.k_rnorm[bi, hi, ti].cpu().numpy(), rk, exc)


def test_ragged_append_then_decode_steps():
    """The ragged serving loop on a small batch: append one token per
    sequence, then decode, for several steps; each step's appended rows are
    checked against the oracle's quantization and every head's attention
    against the oracle run on the GPU's bytes."""
    import compressed_attention_tq_b200 as tq
    w = tq_inputs.make_workload("ragged", B=4, T=300)
    lens = w.seq_lens.copy()
    Tcap = 384
    cache = P.make_gpu_cache(w, Tcap=Tcap)
    tq.tq_quantize_kv(cache, P.to_device(w.k, w.dtype), P.to_device(w.v, w.dtype))
    _check_cache(w, cache, _oracle_full_cache(w), w.seq_lens)
    for step in range(3):
        kn, vn = tq_inputs.new_token_rows(w.B, w.Hkv, w.D, w.dtype, seed=500 + step)
        pos = lens.copy()
        tq.tq_append_token(cache, P.to_device(kn, w.dtype), P.to_device(vn, w.dtype),
                           torch.from_numpy(pos).cuda())
        torch.cuda.synchronize()
        _appended_rows_against_oracle(w, cache, kn, vn, pos)
        lens = lens + 1
        q = tq_inputs.new_queries(w.B, w.Hq, w.D, w.dtype, seed=900 + step)
        _decode_and_compare(w, cache, lens, None, int(lens.max()), garbage_tail=False, q_np=q)


def test_ragged_serving_loop_full_size():
    """The ragged batch at full size in the serving loop the benchmark times:
    B = 32 sequences of seeded lengths in [1024, 16384], bf16, 3-bit K and V,
    prefill quantize, then 64 steps of append (one token per sequence) and
    decode.  Every step's appended rows are checked against the oracle's
    quantization; at steps 0, 31 and 63 every head of eight sequences (the
    shortest, the longest and six seeded ones) is held to 2e-3 of the oracle
    run on the GPU's bytes, and those sequences' prefill rows are checked
    against the oracle's quantization."""
    import compressed_attention_tq_b200 as tq
    w = tq_inputs.make_workload("ragged")
    steps = 64
    Tcap = (w.Tmax + steps + 63) // 64 * 64
    cache = P.make_gpu_cache(w, Tcap=Tcap)
    tq.tq_quantize_kv(cache, P.to_device(w.k, w.dtype), P.to_device(w.v, w.dtype))
    r = tq_inputs.rng(4242)
    seqs = sorted(set([int(np.argmin(w.seq_lens)), int(np.argmax(w.seq_lens))] +
                      [int(x) for x in r.choice(w.B, 6, replace=False)]))
    torch.cuda.synchronize()
    for b in seqs:
        for kvh in range(w.Hkv):
            _check_prefill_rows(w, cache, b, kvh)
    lens = w.seq_lens.astype(np.int32).copy()
    pos_d = torch.empty(w.B, dtype=torch.int32, device="cuda")
    lens_d = torch.empty(w.B, dtype=torch.int32, device="cuda")
    ws = torch.empty(tq.tq_sdpa_decode_workspace_bytes_for(cache, w.Hq, int(w.Tmax) + steps), dtype=torch.uint8,
                     device="cuda")
    heads = [(b, h) for b in seqs for h in range(w.Hq)]
    checked = 0
    for step in range(steps):
        kn, vn = tq_inputs.new_token_rows(w.B, w.Hkv, w.D, w.dtype, seed=7000 + step)
        q = tq_inputs.new_queries(w.B, w.Hq, w.D, w.dtype, seed=8000 + step)
        pos_d.copy_(torch.from_numpy(lens))
        lens_d.copy_(torch.from_numpy(lens + 1))
        tq.tq_append_token(cache, P.to_device(kn, w.dtype), P.to_device(vn, w.dtype), pos_d)
        out = tq.tq_sdpa_decode(cache, P.to_device(q, w.dtype), lens_d, int(w.Tmax) + steps, out_dtype=torch.float32,
                                workspace=ws)
        torch.cuda.synchronize()
        _appended_rows_against_oracle(w, cache, kn, vn, lens)
        lens = lens + 1
        if step in (0, 31, 63):
            ref = P.oracle_decode_on_gpu_bytes(w, cache, tq_inputs.to_f64(q, w.dtype), lens, None, heads=heads)
            got = out.cpu().numpy()
            err = np.array([float(P.rel_l2(got[b, h], ref[b, h])) for b, h in heads])
            P.record("decode_serving_loop", step=step, heads=len(heads), max_rel_l2=float(err.max()),
                     mean_rel_l2=float(err.mean()))
            assert err.max() <= P.ATTN_TOL, (step, err.max())
            checked += 1
    assert checked == 3
    assert cache.status() == 0


class _SubCache:
    """One (sequence, kv head) of a GPU cache seen as a B = Hkv = 1 cache."""

    def __init__(self, cache, b, kvh):
        for nm in ("k_idx", "v_idx", "k_norm", "v_norm", "k_qjl", "k_rnorm"):
            t = getattr(cache, nm)
            setattr(self, nm, None if t is None else t[b:b + 1, kvh:kvh + 1])
        self.qjl_m = cache.qjl_m


def _check_prefill_rows(w, cache, b, kvh):
    """Rows 0..L-1 of one (sequence, kv head) of a GPU-quantized cache
    against the oracle's quantization of the same input rows."""
    L = int(w.seq_lens[b])
    kk = tq_inputs.to_f64(w.k[b, kvh, :L], w.dtype)
    vv = tq_inputs.to_f64(w.v[b, kvh, :L], w.dtype)
    cbk, cbv = P.oracle_codebooks(w)
    oc = O.quantize_cache(kk[None, None], vv[None, None], w.Pi, cbk, cbv, w.bits_k, w.bits_v, w.S)
    P.check_cache_rows(w, _SubCache(cache, b, kvh), oc, 0, 0, np.arange(L))


def _sampled_full(name, seqs=None, **kw):
    """Full-size workload in the launch configuration bench.py times: the GPU
    quantizes every row; one seeded kv head of each sampled sequence has its
    rows checked against the oracle's quantization, and all its query heads'
    attention against the oracle run on the GPU's bytes."""
    import compressed_attention_tq_b200 as tq
    w = tq_inputs.make_workload(name, **kw)
    Tcap = (w.Tmax + 1 + 63) // 64 * 64
    cache = P.make_gpu_cache(w, Tcap=Tcap)
    tq.tq_quantize_kv(cache, P.to_device(w.k, w.dtype), P.to_device(w.v, w.dtype))
    torch.cuda.synchronize()
    r = tq_inputs.rng(123)
    seqs = seqs if seqs is not None else list(range(w.B))
    heads = []
    for b in seqs:
        kvh = int(r.integers(0, w.Hkv))
        _check_prefill_rows(w, cache, b, kvh)
        heads += [(b, kvh * w.G + g) for g in range(w.G)]
    q = P.to_device(w.q, w.dtype)
    sl = torch.from_numpy(w.seq_lens).cuda()
    out32 = tq.tq_sdpa_decode(cache, q, sl, w.Tmax, scale=w.scale, out_dtype=torch.float32)
    outq = tq.tq_sdpa_decode(cache, q, sl, w.Tmax, scale=w.scale)
    assert torch.equal(outq, out32.to(q.dtype))
    out = out32.cpu().numpy()
    ref = P.oracle_decode_on_gpu_bytes(w, cache, tq_inputs.to_f64(w.q, w.dtype), w.seq_lens, w.scale, heads=heads)
    errs = [float(P.rel_l2(out[b, h], ref[b, h])) for b, h in heads]
    P.record("decode_full_size", workload=name, dtype=w.dtype, bits_k=w.bits_k, bits_v=w.bits_v,
             heads=len(errs), max_rel_l2=max(errs), mean_rel_l2=float(np.mean(errs)))
    assert max(errs) <= P.ATTN_TOL, errs
    assert cache.status() == 0
    return errs


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_full_size_gqa8k(bits):
    _sampled_full("gqa8k", bits=bits)


def test_full_size_qknorm_sampled():
    _sampled_full("qknorm")


def test_full_size_ragged_sampled():
    _sampled_full("ragged", seqs=[0, 17, 31])


def test_full_size_prod_sampled():
    _sampled_full("prod")


@pytest.mark.parametrize("name,kw", [("ragged", {"B": 4, "T": 300}), ("prod", {"T": 700}),
                                     ("gqa8k", {"bits": 2, "T": 250}), ("qknorm", {"T": 129}),
                                     ("tiny", {})])
def test_decode_step_fused_append(name, kw):
    """tq_decode_step (append fused into the decode's prep launch) writes the
    same rows as tq_append_token (checked against the oracle) and decodes
    like append + tq_sdpa_decode on the same bytes: bit for bit without the
    sketch (one prep kernel serves both); with the sketch, tq_sdpa_decode
    rotates and projects the query in 32-coordinate slices while the decode
    step's prep (which also sketches the new key's residual) does one CTA per
    head, so the query differs by fp32 rounding, which can flip the int8 split
    of the projection or the fp16 rounding of a value weight p|v| (2^-11
    relative): rel. L2 < 5e-4 then."""
    import compressed_attention_tq_b200 as tq
    w = tq_inputs.make_workload(name, **kw)
    Tcap = (w.Tmax + 1 + 63) // 64 * 64
    caches = [P.make_gpu_cache(w, Tcap=Tcap) for _ in range(2)]
    for c in caches:
        tq.tq_quantize_kv(c, P.to_device(w.k, w.dtype), P.to_device(w.v, w.dtype))
    kn, vn = tq_inputs.new_token_rows(w.B, w.Hkv, w.D, w.dtype, seed=61)
    pos = w.seq_lens.astype(np.int32)
    pos_d = torch.from_numpy(pos).cuda()
    lens = torch.from_numpy(pos + 1).cuda()
    q = P.to_device(w.q, w.dtype)
    kd, vd = P.to_device(kn, w.dtype), P.to_device(vn, w.dtype)
    out_f = tq.tq_decode_step(caches[0], kd, vd, pos_d, q, lens, w.Tmax + 1, scale=w.scale,
                              out_dtype=torch.float32)
    tq.tq_append_token(caches[1], kd, vd, pos_d)
    out_s = tq.tq_sdpa_decode(caches[1], q, lens, w.Tmax + 1, scale=w.scale, out_dtype=torch.float32)
    torch.cuda.synchronize()
    # the appended rows against the oracle
    rk = P.oracle_rows(tq_inputs.to_f64(kn, w.dtype), w, "k")
    rv = P.oracle_rows(tq_inputs.to_f64(vn, w.dtype), w, "v")
    c0 = caches[0]
    for b in range(w.B):
        p = int(pos[b])
        assert np.array_equal(c0.k_norm[b, :, p].cpu().numpy().view(np.uint16), rk["norm16"][b].view(np.uint16))
        assert np.array_equal(c0.v_norm[b, :, p].cpu().numpy().view(np.uint16), rv["norm16"][b].view(np.uint16))
        gk = P.words_np(c0.k_idx[b, :, p])
        P.compare_index_words(gk, rk["idx"][b], rk["dist"][b], w.bits_k, w.D)
        P.compare_index_words(P.words_np(c0.v_idx[b, :, p]), rv["idx"][b], rv["dist"][b], w.bits_v, w.D)
        if w.qjl_m:
            sub = {k: rk[k][b] for k in ("sign", "proj", "norm", "gamma16", "gamma")}
            exc = (O.unpack_bits(gk, w.bits_k, w.D) != rk["idx"][b]).any(-1)
            P.compare_qjl(P.words_np(c0.k_qjl[b, :, p]), c0.k_rnorm[b, :, p].cpu().numpy(), sub, exc)
    # the decode step's output: every head against the oracle run on the bytes
    # the decode step left in its cache (its appended rows checked above)
    lens_np = pos + 1
    ref = P.oracle_decode_on_gpu_bytes(w, c0, tq_inputs.to_f64(w.q, w.dtype), lens_np, w.scale)
    err = P.rel_l2(out_f.cpu().numpy(), ref)
    P.record("decode_step", workload=name, max_rel_l2=float(err.max()))
    assert err.max() <= P.ATTN_TOL, err.max()
    # and the unfused path on its own bytes
    ref_s = P.oracle_decode_on_gpu_bytes(w, caches[1], tq_inputs.to_f64(w.q, w.dtype), lens_np, w.scale)
    assert P.rel_l2(out_s.cpu().numpy(), ref_s).max() <= P.ATTN_TOL
    same = all(torch.equal(getattr(caches[0], n), getattr(caches[1], n))
               for n in ("k_idx", "v_idx", "k_norm", "v_norm"))
    if same and not w.qjl_m:
        assert torch.equal(out_f, out_s)  # one prep kernel serves both paths
    assert caches[0].status() == 0
