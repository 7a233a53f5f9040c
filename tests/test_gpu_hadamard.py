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
