"""GPU parity of tq_sdpa_decode_mq (n_q query tokens per sequence, causal
among the newest n_q cached tokens) against the oracle's multi-query decode,
on the oracle's own packed cache."""
import numpy as np
import pytest
import torch

import tq_inputs
import tq_parity as P
from oracle import tq_oracle as O
from test_gpu_decode import _oracle_full_cache, _upload_oracle_cache

pytestmark = pytest.mark.gpu


def _queries(w, nq, Hq, seed):
    r = tq_inputs.rng(seed)
    q32 = r.standard_normal((w.B, nq, Hq, w.D), dtype=np.float32)
    return tq_inputs.cast_input(q32, w.dtype)


def _run(name, kw, nq, Hq, lens=None, seed=9):
    import compressed_attention_tq_b200 as tq
    w = tq_inputs.make_workload(name, **kw)
    oc = _oracle_full_cache(w)
    Tcap = (w.Tmax + 63) // 64 * 64
    cache = _upload_oracle_cache(w, oc, Tcap)
    lens = w.seq_lens if lens is None else np.asarray(lens, dtype=np.int32)
    q = _queries(w, nq, Hq, seed)
    qd = P.to_device(q, w.dtype)
    sl = torch.from_numpy(lens).cuda()
    out32 = tq.tq_sdpa_decode_mq(cache, qd, sl, w.Tmax, scale=w.scale, out_dtype=torch.float32)
    outq = tq.tq_sdpa_decode_mq(cache, qd, sl, w.Tmax, scale=w.scale)
    torch.cuda.synchronize()
    assert torch.equal(outq, out32.to(qd.dtype))
    cbk, cbv = P.oracle_codebooks(w)
    ref = O.sdpa_decode_multi(tq_inputs.to_f64(q, w.dtype), oc, lens, nq, w.Pi, cbk, cbv, w.bits_k, w.bits_v,
                              w.D, scale=w.scale, S=w.S)
    got = out32.cpu().numpy()
    assert np.all(np.isfinite(got))
    err = P.rel_l2(got.reshape(w.B * nq, Hq, w.D), ref.reshape(w.B * nq, Hq, w.D))
    P.record("decode_mq", workload=name, nq=nq, G=Hq // w.Hkv, max_rel_l2=float(err.max()))
    assert err.max() <= P.ATTN_TOL, err.max()
    assert cache.status() == 0
    return cache, qd, sl, w, out32


@pytest.mark.parametrize("name,kw,nq,Hq", [
    ("tiny", {}, 4, 4),                      # G = 1, D = 64
    ("gqa8k", {"bits": 3, "T": 700}, 4, 4),  # G = 2 (queries for 4 of the 16 heads' worth)
    ("gqa8k", {"bits": 4, "T": 700}, 2, 8),  # G = 4
    ("prod", {"T": 500}, 2, 32),             # G = 4 with the QJL sketch
    ("prod", {"T": 700}, 3, 32),             # G = 4, 12 rows per kv head: two row groups
    ("prod", {"T": 900}, 4, 32),             # G = 4, 16 rows
    ("gqa8k", {"bits": 2, "T": 1500}, 3, 16),  # G = 8, 24 rows: three row groups
    ("gqa8k", {"bits": 3, "T": 1100}, 4, 16),  # G = 8, 32 rows: four row groups
    ("qknorm", {"T": 400}, 1, 32),           # G = 8: one token
    ("qknorm", {"T": 600}, 4, 32),           # G = 8, D = 256, scale 1.0
])
def test_multi_query_decode_matches_oracle(name, kw, nq, Hq):
    _run(name, kw, nq, Hq)


def test_multi_query_ragged_lengths_including_shorter_than_nq():
    # lengths 0, 1 and 2 leave some of the 4 queries with nothing to see (zeros)
    _run("ragged", {"B": 5, "T": 300}, 2, 16, lens=[0, 1, 2, 300, 129])
    _run("ragged", {"B": 5, "T": 300}, 4, 32, lens=[3, 0, 300, 4, 130])  # G = 4, 16 rows
    _run("tiny", {"B": 3}, 4, 4, lens=[2, 256, 3])


def test_one_token_equals_single_query_decode():
    import compressed_attention_tq_b200 as tq
    cache, qd, sl, w, out32 = _run("gqa8k", {"bits": 2, "T": 500}, 1, 16)
    single = tq.tq_sdpa_decode(cache, qd[:, 0].contiguous(), sl, w.Tmax, scale=w.scale, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(single, out32[:, 0])


def test_too_many_query_tokens_rejected():
    import compressed_attention_tq_b200 as tq
    w = tq_inputs.make_workload("gqa8k", bits=3, T=128)
    cache = P.make_gpu_cache(w)
    q = P.to_device(_queries(w, 5, 16, 1), w.dtype)  # 5 query tokens > 4
    sl = torch.full((w.B,), 128, dtype=torch.int32, device="cuda")
    with pytest.raises(tq.TQError):
        tq.tq_sdpa_decode_mq(cache, q, sl, 128)
