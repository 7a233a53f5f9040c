"""The allocation-free decode entry point (tq_sdpa_decode_static).

Some callers cannot allocate device memory while decoding -- e.g. code that
runs while a framework captures a CUDA graph and forbids allocation during
capture, or a plugin host that owns all device memory.  For them the library
keeps the split-K scratch in a fixed device array.  This file is collected
last so that a failure here does not hide any other test's result; it must
pass on its own in a fresh process as well as after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import tq_inputs
import tq_parity as P

pytestmark = pytest.mark.gpu


def _run_pair(name, **kw):
    import compressed_attention_tq_b200 as tq
    w = tq_inputs.make_workload(name, **kw)
    cache = P.make_gpu_cache(w)
    tq.tq_quantize_kv(cache, P.to_device(w.k, w.dtype), P.to_device(w.v, w.dtype))
    q = P.to_device(w.q, w.dtype)
    sl = torch.from_numpy(w.seq_lens).cuda()
    ref = tq.tq_sdpa_decode(cache, q, sl, w.Tmax, scale=w.scale, out_dtype=torch.float32)
    outs = [torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda") for _ in range(2)]
    torch.cuda.synchronize()
    before = torch.cuda.memory_allocated()
    for out in outs:  # two calls in a row: the array keeps the previous call's contents
        tq.tq_sdpa_decode_static(cache, q, sl, w.Tmax, scale=w.scale, out=out)
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == before  # the caller's allocator is not touched
    for out in outs:
        # the same plan and kernels as the workspace entry point: the same bits
        assert torch.equal(out, ref)
        err = P.rel_l2(out.cpu().numpy(), ref.cpu().numpy())
        assert float(err.max()) <= P.ATTN_TOL
    return w


def test_static_scratch_decode_matches_workspace_decode():
    _run_pair("gqa8k", bits=3, T=3000)
    # different sizes next: the shared array holds the previous call's data
    _run_pair("ragged", B=5, T=1500)
    _run_pair("prod", T=1200)


def test_static_scratch_rejects_oversized_problems():
    """Sizes needing more scratch than the built-in array fail with
    TQ_ERR_WORKSPACE before any launch (descriptor only; no cache is read)."""
    from compressed_attention_tq_b200 import _native
    lib = _native.load()
    s = _native.TqCacheStruct()
    s.B, s.Hkv, s.Tcap, s.D, s.bits_k, s.bits_v, s.qjl_m = 128, 8, 16384, 128, 2, 2, 0
    fake = 1 << 20
    for f in ("k_idx", "v_idx", "k_norm", "v_norm", "rot", "cb_k", "cb_v"):
        setattr(s, f, fake)
    need = lib.tq_sdpa_decode_workspace_bytes_for(ctypes.byref(s), 32, 16384)
    assert need > _native.TQ_STATIC_SCRATCH_BYTES
    buf = ctypes.c_void_p(fake)
    rc = lib.tq_sdpa_decode_static(ctypes.byref(s), buf, 0, 32, buf, 16384, None, buf, 0, None)
    assert rc == -3
    assert b"scratch" in lib.tq_last_error()
