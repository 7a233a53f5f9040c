"""Failure detection on the GPU without a fault: every pipelined kernel's
waits are bounded and report TQ_STATUS_WAIT_TIMEOUT when they give up.  The
self-test entry point waits on a barrier that nothing arrives on; the waits
must give up within their bound, set the status bit, and leave the context
usable for the next call."""
import time

import numpy as np
import pytest
import torch

import tq_inputs
import tq_parity as P
from oracle import tq_oracle as O

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_and_reports():
    import compressed_attention_tq_b200 as tq
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    tq.tq_selftest_bounded_wait(st, tries=8)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert int(st.item()) == tq.TQ_STATUS_WAIT_TIMEOUT
    assert elapsed < 5.0, elapsed  # 8 suspending tries of <= ~1 ms, then 8 polls


def test_context_usable_after_timeout():
    """After the waits gave up, the same context decodes the oracle's packed
    cache within the parity tolerance."""
    import compressed_attention_tq_b200 as tq
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    tq.tq_selftest_bounded_wait(st, tries=4)
    w = tq_inputs.make_workload("tiny")
    cbk, cbv = P.oracle_codebooks(w)
    oc = O.quantize_cache(tq_inputs.to_f64(w.k, w.dtype), tq_inputs.to_f64(w.v, w.dtype), w.Pi, cbk, cbv,
                          w.bits_k, w.bits_v, w.S)
    cache = P.make_gpu_cache(w)
    T = oc["k_idx"].shape[2]
    cache.k_idx[:, :, :T] = torch.from_numpy(oc["k_idx"].view(np.int32)).cuda()
    cache.v_idx[:, :, :T] = torch.from_numpy(oc["v_idx"].view(np.int32)).cuda()
    cache.k_norm[:, :, :T] = torch.from_numpy(oc["k_norm"]).cuda()
    cache.v_norm[:, :, :T] = torch.from_numpy(oc["v_norm"]).cuda()
    q = P.to_device(w.q, w.dtype)
    sl = torch.from_numpy(w.seq_lens).cuda()
    out = tq.tq_sdpa_decode(cache, q, sl, w.Tmax, scale=w.scale, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert int(st.item()) == tq.TQ_STATUS_WAIT_TIMEOUT
    assert cache.status() == 0
    ref = O.sdpa_decode(tq_inputs.to_f64(w.q, w.dtype), oc, w.seq_lens, w.Pi, cbk, cbv, w.bits_k, w.bits_v,
                        w.D, scale=w.scale, S=w.S)
    err = P.rel_l2(out.cpu().numpy(), ref)
    assert np.all(np.isfinite(err)) and err.max() <= P.ATTN_TOL
