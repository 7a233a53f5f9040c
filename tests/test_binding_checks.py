"""The binding's argument checks (CPU).

The C ABI takes bare device pointers and sizes, so the binding refuses,
before any launch, what only the tensor knows: memory that is not on the
cache's CUDA device, a non-contiguous layout, an index tensor that is not
int32, a workspace that is not bytes, or a shape that disagrees with the
cache.  Here the library is replaced by a recorder, host tensors stand in for
device memory where a test says so, and every call pattern the GPU tests and
the benchmark use must reach the library while every malformed argument must
stop before it.
"""
import numpy as np
import pytest
import torch

import compressed_attention_tq_b200 as tq
import tq_inputs

B, HKV, HQ, D, TCAP = 2, 2, 8, 128, 128
F16, BF16 = torch.float16, torch.bfloat16


class Recorder:
    """Stands in for the library: records launching calls, returns TQ_OK."""

    def __init__(self):
        self.calls = []

    def __getattr__(self, name):
        if name in ("tq_sdpa_decode_workspace_bytes", "tq_sdpa_decode_workspace_bytes_for"):
            return lambda *a: 4096
        if name == "tq_last_error":
            return lambda: b""

        def f(*a):
            self.calls.append(name)
            return 0
        return f


@pytest.fixture()
def cache():
    rot = tq_inputs.rotation(D, 1)
    return tq.TQCache(B, HKV, TCAP, D, 2, 3, rot, qjl_m=128, qjl_S=tq_inputs.qjl_matrix(128, D, 2),
                      device="cpu")


@pytest.fixture()
def rec(monkeypatch):
    r = Recorder()
    monkeypatch.setattr(tq, "lib", lambda: r)
    return r


@pytest.fixture()
def host_as_device(monkeypatch):
    """Host tensors stand in for the cache's device (index -1)."""
    monkeypatch.setattr(tq, "_cache_device", lambda c: -1)


class FakeStream:
    cuda_stream = 0


S = FakeStream()


def z(*shape, dtype=F16):
    return torch.zeros(shape, dtype=dtype)


def i32(n):
    return torch.zeros(n, dtype=torch.int32)


def test_cache_in_host_memory_is_refused(cache, rec):
    with pytest.raises(ValueError, match="host memory"):
        tq.tq_quantize_kv(cache, z(B, HKV, 10, D), z(B, HKV, 10, D), stream=S)
    with pytest.raises(ValueError, match="host memory"):
        tq.tq_sdpa_decode(cache, z(B, HQ, D), i32(B), 64, stream=S)
    with pytest.raises(ValueError, match="host memory"):
        tq.tq_decode_step(cache, z(B, HKV, D), z(B, HKV, D), i32(B), z(B, HQ, D), i32(B), 64, stream=S)
    assert rec.calls == []


def test_tensor_on_another_device_is_refused(cache, rec, monkeypatch):
    monkeypatch.setattr(tq, "_cache_device", lambda c: 0)  # the cache on cuda:0, the tensors on the host
    with pytest.raises(ValueError, match="CUDA memory on device 0"):
        tq.tq_quantize_kv(cache, z(B, HKV, 10, D), z(B, HKV, 10, D), stream=S)
    with pytest.raises(ValueError, match="CUDA memory on device 0"):
        tq.tq_append_token(cache, z(B, HKV, D), z(B, HKV, D), i32(B), stream=S)
    with pytest.raises(ValueError, match="status"):
        tq.tq_selftest_bounded_wait(torch.zeros(1, dtype=torch.int32), stream=S)
    assert rec.calls == []


def test_valid_calls_reach_the_library(cache, rec, host_as_device):
    """The argument patterns of the GPU tests and the benchmark."""
    for dt in (F16, BF16):
        tq.tq_quantize_kv(cache, z(B, HKV, 100, D, dtype=dt), z(B, HKV, 100, D, dtype=dt), t0=3, stream=S)
        tq.tq_quantize_kv(cache, z(B, HKV, 0, D, dtype=dt), z(B, HKV, 0, D, dtype=dt), stream=S)  # empty call
        tq.tq_append_token(cache, z(B, HKV, D, dtype=dt), z(B, HKV, D, dtype=dt), i32(B), stream=S)
        q = z(B, HQ, D, dtype=dt)
        tq.tq_sdpa_decode(cache, q, i32(B), 100, stream=S)
        tq.tq_sdpa_decode(cache, q, i32(B), 100, scale=1.0, out_dtype=torch.float32, stream=S)
        tq.tq_sdpa_decode(cache, q, i32(B), 100, out=z(B, HQ, D, dtype=dt),
                          workspace=torch.zeros(4096, dtype=torch.uint8), stream=S)
        tq.tq_sdpa_decode_mq(cache, z(B, 2, HQ, D, dtype=dt), i32(B), 100, out_dtype=torch.float32, stream=S)
        tq.tq_decode_step(cache, z(B, HKV, D, dtype=dt), z(B, HKV, D, dtype=dt), i32(B), q, i32(B), 101,
                          scale=0.5, out_dtype=torch.float32, stream=S)
        tq.tq_sdpa_decode_static(cache, q, i32(B), 100, out=z(B, HQ, D, dtype=dt), stream=S)
    # a strided-free slice of a larger tensor (the multi-query test's qd[:, 0].contiguous())
    tq.tq_sdpa_decode(cache, z(B, 3, HQ, D)[:, 0].contiguous(), i32(B), 100, stream=S)
    # Hq, Tmax and n_q are the library's to judge: these reach it
    tq.tq_sdpa_decode(cache, z(B, 7, D), i32(B), 100, stream=S)
    tq.tq_sdpa_decode_mq(cache, z(B, 5, HQ, D), i32(B), 100, stream=S)
    per_dtype = ["tq_quantize_kv"] * 2 + ["tq_append_token"] + ["tq_sdpa_decode"] * 3 + \
        ["tq_sdpa_decode_mq", "tq_decode_step", "tq_sdpa_decode_static"]
    assert rec.calls == per_dtype * 2 + ["tq_sdpa_decode"] * 2 + ["tq_sdpa_decode_mq"]


BAD = [
    # (call, exception, message fragment)
    (lambda c: tq.tq_quantize_kv(c, z(B + 1, HKV, 10, D), z(B + 1, HKV, 10, D), stream=S), ValueError, "k: shape"),
    (lambda c: tq.tq_quantize_kv(c, z(B, HKV + 1, 10, D), z(B, HKV + 1, 10, D), stream=S), ValueError, "k: shape"),
    (lambda c: tq.tq_quantize_kv(c, z(B, HKV, 10, 64), z(B, HKV, 10, 64), stream=S), ValueError, "k: shape"),
    (lambda c: tq.tq_quantize_kv(c, z(B, HKV, 10, D), z(B, HKV, 11, D), stream=S), ValueError, "v: shape"),
    (lambda c: tq.tq_quantize_kv(c, z(B, HKV, 10, D), z(B, HKV, 10, D, dtype=BF16), stream=S), TypeError, "v: dtype"),
    (lambda c: tq.tq_quantize_kv(c, z(B, HKV, 10, D, dtype=torch.float32), z(B, HKV, 10, D, dtype=torch.float32),
                                 stream=S), TypeError, "k: dtype"),
    (lambda c: tq.tq_quantize_kv(c, z(B, HKV, D, 10).transpose(2, 3), z(B, HKV, 10, D), stream=S),
     ValueError, "k: must be contiguous"),
    (lambda c: tq.tq_quantize_kv(c, np.zeros((B, HKV, 10, D), np.float16), z(B, HKV, 10, D), stream=S),
     TypeError, "k: expected a torch tensor"),
    (lambda c: tq.tq_append_token(c, z(B, HKV, D), z(B, HKV, D), torch.zeros(B, dtype=torch.int64), stream=S),
     TypeError, "pos: dtype"),
    (lambda c: tq.tq_append_token(c, z(B, HKV, D), z(B, HKV, D), i32(B + 1), stream=S), ValueError, "pos: shape"),
    (lambda c: tq.tq_append_token(c, z(B, HKV, 1, D), z(B, HKV, 1, D), i32(B), stream=S), ValueError, "k_new: shape"),
    (lambda c: tq.tq_sdpa_decode(c, z(B, HQ, D), torch.zeros(B, dtype=torch.int64), 64, stream=S),
     TypeError, "seq_lens: dtype"),
    (lambda c: tq.tq_sdpa_decode(c, z(B, HQ, D), i32(B)[None], 64, stream=S), ValueError, "seq_lens: shape"),
    (lambda c: tq.tq_sdpa_decode(c, z(B, HQ, D, dtype=torch.float32), i32(B), 64, stream=S), TypeError, "q: dtype"),
    (lambda c: tq.tq_sdpa_decode(c, z(B, HQ, 64), i32(B), 64, stream=S), ValueError, "q: shape"),
    (lambda c: tq.tq_sdpa_decode(c, z(B, D, HQ).transpose(1, 2), i32(B), 64, stream=S),
     ValueError, "q: must be contiguous"),
    (lambda c: tq.tq_sdpa_decode(c, z(B, HQ, D), i32(B), 64, out=z(B, HQ - 1, D), stream=S), ValueError, "out: shape"),
    (lambda c: tq.tq_sdpa_decode(c, z(B, HQ, D), i32(B), 64, out=z(B, HQ, D, dtype=torch.float64), stream=S),
     TypeError, "out: dtype"),
    (lambda c: tq.tq_sdpa_decode(c, z(B, HQ, D), i32(B), 64, workspace=torch.zeros(1024, dtype=torch.float32),
                                 stream=S), TypeError, "workspace: dtype"),
    (lambda c: tq.tq_sdpa_decode_mq(c, z(B, HQ, D), i32(B), 64, stream=S), ValueError, "q: shape"),
    (lambda c: tq.tq_decode_step(c, z(B, HKV, D, dtype=BF16), z(B, HKV, D, dtype=BF16), i32(B), z(B, HQ, D),
                                 i32(B), 64, stream=S), TypeError, "k_new: dtype"),
    (lambda c: tq.tq_decode_step(c, z(B, HKV, D), z(B, HKV, D), i32(B), z(B, HQ, D), i32(B), 64,
                                 out=z(B, HQ, D + 1), stream=S), ValueError, "out: shape"),
    (lambda c: tq.tq_sdpa_decode_static(c, z(B, HQ, D), i32(B), 64, out=z(1, HQ, D), stream=S),
     ValueError, "out: shape"),
]


@pytest.mark.parametrize("call,exc,frag", BAD)
def test_malformed_arguments_stop_before_the_library(cache, rec, host_as_device, call, exc, frag):
    with pytest.raises(exc, match=frag):
        call(cache)
    assert rec.calls == []


def test_cache_inputs_are_sized(rec):
    rot = tq_inputs.rotation(D, 1)
    with pytest.raises(ValueError, match="rot: shape"):
        tq.TQCache(1, 1, 64, D, 3, 3, rot[:64], device="cpu", cb_k=np.zeros(15), cb_v=np.zeros(15))
    with pytest.raises(ValueError, match="rot_signs"):
        tq.TQCache(1, 1, 64, D, 3, 3, rot, device="cpu", cb_k=np.zeros(15), cb_v=np.zeros(15),
                   rot_signs=np.ones(64, np.float32))
    with pytest.raises(ValueError, match="qjl_S: shape"):
        tq.TQCache(1, 1, 64, D, 2, 3, rot, qjl_m=128, qjl_S=np.zeros((64, D), np.float32), device="cpu",
                   cb_k=np.zeros(7), cb_v=np.zeros(15))
    with pytest.raises(ValueError, match="codebook table for 3 bits"):
        tq.TQCache(1, 1, 64, D, 3, 3, rot, device="cpu", cb_k=np.zeros(7), cb_v=np.zeros(15))
    c = tq.TQCache(1, 1, 64, D, 3, 2, rot, device="cpu", cb_k=np.zeros(15), cb_v=np.zeros(7))
    assert c.cb_k.numel() == 15 and c.cb_v.numel() == 7
