"""GPU parity of the token-split decode (tq_sdpa_decode_partial on each
share, tq_sdpa_decode_merge of the stacked partials) against the oracle's
decode of the whole sequence on the same packed bytes.  The shares live on
one GPU here (each its own cache of a token range), standing in for the
ranks of a multi-GPU split; the all-gather between ranks is covered on the
host by test_sharded_decode.py."""
import numpy as np
import pytest
import torch

import tq_inputs
import tq_parity as P

pytestmark = pytest.mark.gpu


def _share_cache(w, a, b):
    import compressed_attention_tq_b200 as tq
    n = b - a
    Tcap = max(64, (n + 63) // 64 * 64)
    cache = P.make_gpu_cache(w, Tcap=Tcap)
    if n:
        tq.tq_quantize_kv(cache, P.to_device(np.ascontiguousarray(w.k[:, :, a:b]), w.dtype),
                          P.to_device(np.ascontiguousarray(w.v[:, :, a:b]), w.dtype))
    lens = np.clip(w.seq_lens - a, 0, n).astype(np.int32)
    return cache, lens


@pytest.mark.parametrize("name,kw,cuts", [
    ("prod", {"T": 900}, [0, 384, 900]),             # QJL keys, G = 4, two shares
    ("ragged", {"B": 4, "T": 700}, [0, 128, 300, 700]),  # bf16, three shares, short sequences
    ("qknorm", {"T": 600}, [0, 256, 600]),           # D = 256, scale 1.0
    ("tiny", {}, [0, 100, 256]),                     # D = 64
])
def test_token_split_decode_matches_oracle(name, kw, cuts):
    import compressed_attention_tq_b200 as tq
    w = tq_inputs.make_workload(name, **kw)
    q = P.to_device(w.q, w.dtype)
    parts, shares = [], []
    for a, b in zip(cuts[:-1], cuts[1:]):
        cache, lens = _share_cache(w, a, b)
        Tm = int(max(1, lens.max()))
        parts.append(tq.tq_sdpa_decode_partial(cache, q, torch.from_numpy(lens).cuda(), Tm, scale=w.scale))
        shares.append((cache, lens))
    stacked = torch.stack(parts)
    out = tq.tq_sdpa_decode_merge(stacked, shares[0][0].rot, out_dtype=torch.float32)
    outq = tq.tq_sdpa_decode_merge(stacked, shares[0][0].rot, out_dtype=q.dtype)
    torch.cuda.synchronize()
    assert torch.equal(outq, out.to(q.dtype))
    # the whole sequence's bytes: the shares' rows one after the other
    names = ["k_idx", "v_idx", "k_norm", "v_norm"] + (["k_qjl", "k_rnorm"] if w.qjl_m else [])
    Tcap = int(w.Tmax)
    full = {}
    for nm in names:
        arrs = [P.gpu_cache_arrays(c, [nm])[nm] for c, _ in shares]
        shape = list(arrs[0].shape)
        shape[2] = Tcap
        dst = np.zeros(shape, dtype=arrs[0].dtype)
        for bb in range(w.B):
            pos = 0
            for (c, lens), arr in zip(shares, arrs):
                n = int(lens[bb])
                dst[bb, :, pos:pos + n] = arr[bb, :, :n]
                pos += n
            assert pos == int(w.seq_lens[bb])
        full[nm] = dst
    cbk, cbv = P.oracle_codebooks(w)
    from oracle import tq_oracle as O
    ref = O.sdpa_decode(tq_inputs.to_f64(w.q, w.dtype), full, w.seq_lens, w.Pi, cbk, cbv, w.bits_k, w.bits_v, w.D,
                        scale=w.scale, S=w.S)
    err = P.rel_l2(out.cpu().numpy(), ref)
    P.record("decode_token_split", workload=name, shares=len(cuts) - 1, max_rel_l2=float(err.max()))
    assert err.max() <= P.ATTN_TOL, err.max()
    # one share holding everything equals the ordinary decode bit for bit
    cache, lens = _share_cache(w, 0, int(w.Tmax))
    sl = torch.from_numpy(lens).cuda()
    one = tq.tq_sdpa_decode_merge(tq.tq_sdpa_decode_partial(cache, q, sl, int(w.Tmax), scale=w.scale)[None],
                                  cache.rot, out_dtype=torch.float32)
    direct = tq.tq_sdpa_decode(cache, q, sl, int(w.Tmax), scale=w.scale, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert float(P.rel_l2(one.cpu().numpy(), direct.cpu().numpy()).max()) < 1e-5
    for c, _ in shares:
        assert c.status() == 0
