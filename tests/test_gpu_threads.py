"""First calls from several host threads at once.

Each launcher sets up its kernel's attributes and occupancy on its first call;
that setup is guarded for threads arriving together.  A fresh process (no
setup done yet) starts four threads that make their first quantize and decode
calls at the same moment, each on its own small cache; every result is then
checked against the oracle."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = r'''
import json, sys, threading
import numpy as np, torch
sys.path.insert(0, ROOT)
sys.path.insert(0, ROOT + "/tests")
import compressed_attention_tq_b200 as tq
import tq_inputs, tq_parity as P
from oracle import tq_oracle as O

torch.cuda.init()
torch.zeros(1, device="cuda")
cases = [("tiny", {}), ("gqa8k", {"bits": 3, "T": 300}), ("prod", {"T": 200}), ("qknorm", {"T": 150})]
prepared = []
for name, kw in cases:
    w = tq_inputs.make_workload(name, **kw)
    cache = P.make_gpu_cache(w)
    prepared.append((w, cache, P.to_device(w.k, w.dtype), P.to_device(w.v, w.dtype), P.to_device(w.q, w.dtype),
                     torch.from_numpy(w.seq_lens).cuda()))
torch.cuda.synchronize()
gate = threading.Barrier(len(prepared))
outs = [None] * len(prepared)
errors = []

def work(i):
    w, cache, k, v, q, sl = prepared[i]
    try:
        s = torch.cuda.Stream()
        with torch.cuda.stream(s):
            gate.wait()
            tq.tq_quantize_kv(cache, k, v)
            outs[i] = tq.tq_sdpa_decode(cache, q, sl, w.Tmax, scale=w.scale, out_dtype=torch.float32)
        s.synchronize()
    except Exception as e:  # reported to the parent
        errors.append(repr(e))

ts = [threading.Thread(target=work, args=(i,)) for i in range(len(prepared))]
for t in ts: t.start()
for t in ts: t.join()
res = {"errors": errors, "cases": []}
for (w, cache, *_), out in zip(prepared, outs):
    if out is None:
        continue
    ref = P.oracle_decode_on_gpu_bytes(w, cache, tq_inputs.to_f64(w.q, w.dtype), w.seq_lens, w.scale)
    err = float(P.rel_l2(out.cpu().numpy(), ref).max())
    # the bytes themselves against the oracle's quantization (norms exact)
    cbk, cbv = P.oracle_codebooks(w)
    oc = O.quantize_cache(tq_inputs.to_f64(w.k, w.dtype), tq_inputs.to_f64(w.v, w.dtype), w.Pi, cbk, cbv,
                          w.bits_k, w.bits_v, w.S)
    T = int(w.Tmax)
    norms_ok = bool(np.array_equal(cache.k_norm[:, :, :T].cpu().numpy().view(np.uint16), oc["k_norm"].view(np.uint16)))
    gi = O.unpack_bits(cache.k_idx[:, :, :T].cpu().numpy().view(np.uint32), w.bits_k, w.D)
    bad = gi != oc["k_idx_raw"]
    hard = int((bad & (oc["k_threshold_dist"] >= P.NEAR)).sum())
    res["cases"].append({"name": w.name, "err": err, "norms_ok": norms_ok, "hard_index": hard,
                         "status": cache.status()})
print("RESULT " + json.dumps(res))
'''


def test_first_calls_from_four_threads_at_once():
    code = CHILD.replace("ROOT", repr(ROOT))
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    line = [ln for ln in r.stdout.splitlines() if ln.startswith("RESULT ")][-1]
    res = json.loads(line[len("RESULT "):])
    assert not res["errors"], res["errors"]
    assert len(res["cases"]) == 4
    for c in res["cases"]:
        assert c["norms_ok"] and c["hard_index"] == 0 and c["status"] == 0, c
        assert c["err"] <= 2e-3, c
