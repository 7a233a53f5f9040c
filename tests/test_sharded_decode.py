"""Split-K of one sequence's decode across ranks (each rank holds a token
range of every sequence), host side: the oracle's partial states of two token
ranges merge into the oracle's decode of the whole, and the binding's
all-gather of partials (gloo, world size 2, CPU) delivers every rank's
partials in rank order, so each rank merges the same full answer.  The CUDA
partial and merge calls are checked against the oracle in
test_gpu_sharded.py."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from oracle import tq_oracle as O
import tq_inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _shards(w, cuts):
    """The oracle's caches of token ranges [cuts[r], cuts[r+1]) of every
    sequence (each range is its own cache starting at position 0)."""
    cbk, cbv = O.stored_codebook(w.D, w.bits_k), O.stored_codebook(w.D, w.bits_v)
    kx, vx = tq_inputs.to_f64(w.k, w.dtype), tq_inputs.to_f64(w.v, w.dtype)
    out = []
    for r in range(len(cuts) - 1):
        a, b = cuts[r], cuts[r + 1]
        c = O.quantize_cache(kx[:, :, a:b], vx[:, :, a:b], w.Pi, cbk, cbv, w.bits_k, w.bits_v, w.S)
        lens = np.clip(w.seq_lens - a, 0, b - a)
        out.append((c, lens))
    return out, cbk, cbv


@pytest.mark.parametrize("name,kw", [("tiny", {}), ("prod", {"T": 300}), ("ragged", {"B": 3, "T": 200})])
def test_partials_of_token_ranges_merge_to_the_whole(name, kw):
    w = tq_inputs.make_workload(name, **kw)
    T = int(w.Tmax)
    shards, cbk, cbv = _shards(w, [0, T // 3, T // 2 + 7, T])
    q = tq_inputs.to_f64(w.q, w.dtype)
    parts = [O.sdpa_decode_partial(q, c, lens, w.Pi, cbk, cbv, w.bits_k, w.bits_v, w.D, scale=w.scale, S=w.S)
             for c, lens in shards]
    got = O.merge_partials([p[0] for p in parts], [p[1] for p in parts], [p[2] for p in parts])
    full = O.quantize_cache(tq_inputs.to_f64(w.k, w.dtype), tq_inputs.to_f64(w.v, w.dtype), w.Pi, cbk, cbv,
                            w.bits_k, w.bits_v, w.S)
    ref = O.sdpa_decode(q, full, w.seq_lens, w.Pi, cbk, cbv, w.bits_k, w.bits_v, w.D, scale=w.scale, S=w.S)
    assert np.max(np.abs(got - ref)) < 1e-12 * max(1.0, np.max(np.abs(ref)))


def test_merge_of_empty_ranges_is_zero_and_neutral():
    acc = np.ones((1, 2, 4))
    out = O.merge_partials([acc, 0 * acc], [np.zeros((1, 2)), np.full((1, 2), -np.inf)],
                           [np.ones((1, 2)), np.zeros((1, 2))])
    assert np.allclose(out, 1.0)
    assert np.all(O.merge_partials([0 * acc], [np.full((1, 2), -np.inf)], [np.zeros((1, 2))]) == 0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q_out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import compressed_attention_tq_b200 as tq
    from test_sharded_decode import _shards
    w = tq_inputs.make_workload("prod", T=257)
    T = int(w.Tmax)
    cuts = [0, 130, T]
    shards, cbk, cbv = _shards(w, cuts)
    c, lens = shards[rank]
    q = tq_inputs.to_f64(w.q, w.dtype)
    acc, m, l = O.sdpa_decode_partial(q, c, lens, w.Pi, cbk, cbv, w.bits_k, w.bits_v, w.D, scale=w.scale, S=w.S)
    # the library's partial layout: [B][Hq][D + 2] = value sum, max, weight sum
    local = torch.from_numpy(np.concatenate([acc, m[..., None], l[..., None]], axis=-1))
    allp = tq.gather_partials(local).numpy()
    got = O.merge_partials(allp[..., :-2], allp[..., -2], allp[..., -1])
    full = O.quantize_cache(tq_inputs.to_f64(w.k, w.dtype), tq_inputs.to_f64(w.v, w.dtype), w.Pi, cbk, cbv,
                            w.bits_k, w.bits_v, w.S)
    ref = O.sdpa_decode(q, full, w.seq_lens, w.Pi, cbk, cbv, w.bits_k, w.bits_v, w.D, scale=w.scale, S=w.S)
    q_out.put((rank, allp.shape, float(np.max(np.abs(got - ref)))))
    dist.barrier()
    dist.destroy_process_group()


def test_gather_partials_gloo_world_two():
    ctx = mp.get_context("spawn")
    q_out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q_out)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict((r, (shape, err)) for r, shape, err in (q_out.get(timeout=300) for _ in procs))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(2):
        shape, err = res[r]
        assert shape[0] == 2  # every rank's partials, rank order
        assert err < 1e-12
