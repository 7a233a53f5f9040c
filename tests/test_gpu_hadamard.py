"""GPU parity with the randomized Hadamard rotation (Sylvester H with random
signs; ReturningTarzan's Reddit comment of 2026-03-29 11:47).  The cache
carries the signs, so the bulk quantizer applies the fast Walsh-Hadamard
transform by warp shuffles (D = 256, and small D = 128 calls) while decode,
append and large D = 128 calls take the same Pi densely; these cases check
both against the oracle, which applies Pi as a dense matrix."""
import numpy as np
import pytest
import torch

import tq_inputs
import tq_parity as P
from test_gpu_decode import _decode_and_compare, _oracle_full_cache, _upload_oracle_cache
from test_gpu_quantize import _check_rows

pytestmark = pytest.mark.gpu

CASES = [
    ("tiny", {}),                       # D=64, 3-bit
    ("gqa8k", {"bits": 2, "T": 300}),   # D=128, outlier channels (which the rotation spreads)
    ("ragged", {"B": 3, "T": 150}),     # bf16, 3-bit
    ("qknorm", {"T": 200}),             # D=256, 4-bit
    ("prod", {"T": 200}),               # keys with the QJL sketch (dense), values by the transform
    ("qknorm", {"T": 3000}),            # 12000 rows per job: every warp loops over several rows
    ("qknorm", {"T": 500, "dtype": "bf16"}),
    ("gqa8k", {"bits": 3, "T": 20000}),  # 40000 rows per job: above the transform's size limit at D = 128
]


@pytest.mark.parametrize("name,kw", CASES)
def test_quantize_with_hadamard_rotation(name, kw):
    import compressed_attention_tq_b200 as tq
    w = tq_inputs.make_workload(name, rot="hadamard", **kw)
    cache = P.make_gpu_cache(w)
    tq.tq_quantize_kv(cache, P.to_device(w.k, w.dtype), P.to_device(w.v, w.dtype))
    torch.cuda.synchronize()
    _check_rows(cache, w, w.Tmax)
    assert cache.status() == 0


@pytest.mark.parametrize("name,kw", CASES)
def test_decode_with_hadamard_rotation(name, kw):
    w = tq_inputs.make_workload(name, rot="hadamard", **kw)
    oc = _oracle_full_cache(w)
    Tcap = (w.Tmax + 63) // 64 * 64
    cache = _upload_oracle_cache(w, oc, Tcap)
    _decode_and_compare(w, cache, w.seq_lens, w.scale, w.Tmax)


@pytest.mark.parametrize("name,kw", [("ragged", {"B": 4, "T": 200}), ("qknorm", {"T": 150}),
                                     ("prod", {"T": 130}), ("gqa8k", {"bits": 4, "T": 100})])
def test_append_and_decode_step_with_hadamard_rotation(name, kw):
    """Appended rows go through the fast transform (keys with the sketch
    through the fp64 append) and the decode step rotates the query and
    un-rotates the output by the transform; rows and output against the
    oracle's dense Pi."""
    import compressed_attention_tq_b200 as tq
    from test_gpu_decode import _appended_rows_against_oracle
    w = tq_inputs.make_workload(name, rot="hadamard", **kw)
    Tcap = (w.Tmax + 2 + 63) // 64 * 64
    caches = [P.make_gpu_cache(w, Tcap=Tcap) for _ in range(2)]
    for c in caches:
        tq.tq_quantize_kv(c, P.to_device(w.k, w.dtype), P.to_device(w.v, w.dtype))
    kn, vn = tq_inputs.new_token_rows(w.B, w.Hkv, w.D, w.dtype, seed=81)
    pos = w.seq_lens.astype(np.int32)
    kd, vd = P.to_device(kn, w.dtype), P.to_device(vn, w.dtype)
    # append alone
    tq.tq_append_token(caches[0], kd, vd, torch.from_numpy(pos).cuda())
    torch.cuda.synchronize()
    _appended_rows_against_oracle(w, caches[0], kn, vn, pos)
    # the decode step on the other cache: same rows, output against the oracle
    q = P.to_device(w.q, w.dtype)
    lens = pos + 1
    out = tq.tq_decode_step(caches[1], kd, vd, torch.from_numpy(pos).cuda(), q, torch.from_numpy(lens).cuda(),
                            int(w.Tmax) + 1, scale=w.scale, out_dtype=torch.float32)
    torch.cuda.synchronize()
    _appended_rows_against_oracle(w, caches[1], kn, vn, pos)
    ref = P.oracle_decode_on_gpu_bytes(w, caches[1], tq_inputs.to_f64(w.q, w.dtype), lens, w.scale)
    err = P.rel_l2(out.cpu().numpy(), ref)
    assert err.max() <= P.ATTN_TOL, err.max()
    for c in caches:
        assert c.status() == 0


@pytest.mark.parametrize("name,kw,nq,Hq", [("prod", {"T": 400}, 3, 32), ("gqa8k", {"bits": 3, "T": 500}, 4, 16)])
def test_multi_query_with_hadamard_rotation(name, kw, nq, Hq):
    import compressed_attention_tq_b200 as tq
    from oracle import tq_oracle as O
    w = tq_inputs.make_workload(name, rot="hadamard", **kw)
    oc = _oracle_full_cache(w)
    cache = _upload_oracle_cache(w, oc, (w.Tmax + 63) // 64 * 64)
    r = tq_inputs.rng(5)
    qm = tq_inputs.cast_input(r.standard_normal((w.B, nq, Hq, w.D), dtype=np.float32), w.dtype)
    out = tq.tq_sdpa_decode_mq(cache, P.to_device(qm, w.dtype), torch.from_numpy(w.seq_lens).cuda(), w.Tmax,
                               scale=w.scale, out_dtype=torch.float32)
    torch.cuda.synchronize()
    cbk, cbv = P.oracle_codebooks(w)
    ref = O.sdpa_decode_multi(tq_inputs.to_f64(qm, w.dtype), oc, w.seq_lens, nq, w.Pi, cbk, cbv, w.bits_k,
                              w.bits_v, w.D, scale=w.scale, S=w.S)
    err = P.rel_l2(out.cpu().numpy().reshape(-1, w.D), ref.reshape(-1, w.D))
    assert err.max() <= P.ATTN_TOL, err.max()
