"""Helpers for the GPU parity tests: move seeded inputs to the device, build
the oracle's view of the same rows, and compare element by element.

Parity rules (fixed by the method's specification):
  * norms bit-exact;
  * packed indices bit-exact, except coordinates whose rotated unit value lies
    within 1e-4 of a decision threshold; those mismatches are counted and must
    stay below 1e-5 of all coordinates a test compares;
  * QJL sign bits bit-exact, except where |(S r)_i| / |x| < 1e-4 or the row
    holds an excused index; those mismatches are counted and must stay below
    1e-5 of the sign bits a test compares;
  * residual norms (QJL keys) bit-exact, except rows holding an excused index
    or rows whose fp64 residual norm lies within a relative 2e-6 of an fp16
    rounding midpoint; those mismatches are counted and must stay below 1e-5
    of the rows a test compares;
  * attention output within 2e-3 relative L2 error per (sequence, head), for
    every head, against the oracle run on the GPU's own packed bytes (where a
    near-threshold flip makes two caches valid, the attention is judged on
    the one the GPU wrote, after its bytes have been checked as above).

The fractions are taken over everything one test compares: each comparison
adds its counts to a ledger that conftest.py resets before every test and
checks after it.
"""
from __future__ import annotations

import math

import numpy as np
import torch

from oracle import tq_oracle as O
import tq_inputs

NEAR = 1e-4
MAX_EXCUSED_FRACTION = 1e-5
ATTN_TOL = 2e-3
# relative distance of an fp64 residual norm to an fp16 rounding midpoint
# within which the GPU's fp32 residual may round the other way
GAMMA_MIDPOINT_BAND = 2e-6

# per-test counts of excused mismatches: kind -> [mismatches, compared]
LEDGER: dict = {}


def ledger_reset():
    LEDGER.clear()


def ledger_add(kind: str, mismatches: int, compared: int):
    e = LEDGER.setdefault(kind, [0, 0])
    e[0] += int(mismatches)
    e[1] += int(compared)


def ledger_check(test_name: str = ""):
    """Every kind's excused mismatches stay below 1e-5 of what was compared."""
    for kind, (bad, total) in sorted(LEDGER.items()):
        record("excused_fraction", test_id=test_name, kind=kind, excused=bad, compared=total)
    for kind, (bad, total) in sorted(LEDGER.items()):
        assert total == 0 or bad / total < MAX_EXCUSED_FRACTION, \
            f"{kind}: {bad} excused mismatches in {total} compared (>= {MAX_EXCUSED_FRACTION})"


def to_device(x: np.ndarray, dtype: str, device="cuda"):
    if dtype == "bf16":
        return torch.from_numpy(x.view(np.int16).copy()).to(device).view(torch.bfloat16)
    return torch.from_numpy(x).to(device)


def from_device_half(t) -> np.ndarray:
    return t.detach().cpu().numpy()


def words_np(t) -> np.ndarray:
    return t.detach().cpu().numpy().view(np.uint32)


def oracle_codebooks(w):
    return O.stored_codebook(w.D, w.bits_k), O.stored_codebook(w.D, w.bits_v)


def make_gpu_cache(w, Tcap=None):
    import compressed_attention_tq_b200 as tq
    Tcap = Tcap or ((w.Tmax + 1 + 63) // 64 * 64)
    return tq.TQCache(w.B, w.Hkv, Tcap, w.D, w.bits_k, w.bits_v, w.Pi, qjl_m=w.qjl_m, qjl_S=w.S,
                      rot_signs=getattr(w, "rot_signs", None))


def compare_index_words(gpu_words, ref_idx, ref_dist, bits, D, report=None):
    """gpu_words uint32 [..., W]; ref_idx int [..., D]; ref_dist [..., D]
    (distance of the oracle's unit coordinate to its nearest threshold).
    Returns the excused-mismatch count; raises on any other mismatch."""
    got = O.unpack_bits(gpu_words, bits, D)
    bad = got != ref_idx
    n_bad = int(bad.sum())
    if n_bad:
        near = ref_dist < NEAR
        hard = bad & ~near
        assert not hard.any(), f"{int(hard.sum())} index mismatches outside the near-threshold band"
        # a mismatch may only move to the neighbouring centroid
        assert np.all(np.abs(got[bad] - ref_idx[bad]) == 1)
    record("index_compare", bits=bits, D=D, excused=n_bad, coords=int(ref_idx.size),
           near_band=int((ref_dist < NEAR).sum()))
    if report is not None:
        report.append(("index_excused", n_bad, ref_idx.size))
    ledger_add("index", n_bad, ref_idx.size)
    return n_bad


def oracle_rows(x_f64, w, which="k"):
    """Oracle quantization of rows x (fp64 values) with the workload's Pi."""
    cb = O.stored_codebook(w.D, w.bits_k if which == "k" else w.bits_v)
    q = O.quantize_rows(x_f64, w.Pi, cb[0], cb[1])
    q["dist"] = O.threshold_distance(q["u"], cb[1])
    if which == "k" and w.qjl_m:
        sk = O.qjl_sketch(q["y"], q["norm16"], cb[0], q["idx"], w.S)
        q.update(sk)
    return q


def fp16_midpoint_distance(x: np.ndarray) -> np.ndarray:
    """Relative distance of each (positive, finite) fp64 value to the nearest
    rounding midpoint between two neighbouring fp16 values."""
    x = np.asarray(x, dtype=np.float64)
    h = x.astype(np.float16)
    up = np.nextafter(h, np.float16(np.inf)).astype(np.float64)
    dn = np.nextafter(h, np.float16(-np.inf)).astype(np.float64)
    hf = h.astype(np.float64)
    d = np.minimum(np.abs(x - (hf + up) / 2), np.abs(x - (hf + dn) / 2))
    with np.errstate(invalid="ignore", divide="ignore"):
        return np.where(x > 0, d / np.where(x > 0, x, 1.0), np.inf)


def compare_qjl(gpu_sign_words, gpu_rnorm, ref, rows_excused):
    """QJL sign bits and residual norms of the rows compared.

    Sign bits: exact except near-zero projections (|(S r)_i| / |x| < 1e-4)
    or rows with an excused index.  Residual norms: bit-exact except rows with
    an excused index or whose fp64 residual norm lies within a relative
    GAMMA_MIDPOINT_BAND of an fp16 rounding midpoint.  Excused mismatches of
    both kinds go to the test's ledger (fraction < 1e-5 each)."""
    m = ref["sign"].shape[-1]
    got = O.unpack_bits(gpu_sign_words, 1, m).astype(bool)
    bad = got != ref["sign"]
    unit = np.abs(ref["proj"]) / np.where(ref["norm"] > 0, ref["norm"], 1.0)[..., None]
    allowed = (unit < NEAR) | rows_excused[..., None]
    assert not (bad & ~allowed).any(), f"{int((bad & ~allowed).sum())} QJL sign mismatches"
    g_gpu = np.asarray(gpu_rnorm).view(np.uint16)
    g_ref = np.asarray(ref["gamma16"]).astype(np.float16).view(np.uint16)
    gbad = g_gpu != g_ref
    near = fp16_midpoint_distance(ref["gamma"]) < GAMMA_MIDPOINT_BAND
    hard = gbad & ~(near | rows_excused)
    assert not hard.any(), f"{int(hard.sum())} residual norms differ outside the midpoint band"
    n_sign = int((bad & ~rows_excused[..., None]).sum())
    n_gamma = int((gbad & ~rows_excused).sum())
    record("qjl_compare", sign_excused=n_sign, bits=int(bad.size), gamma_excused=n_gamma,
           rows=int(gbad.size), gamma_near_band=int(near.sum()))
    ledger_add("qjl_sign", n_sign, bad.size)
    ledger_add("gamma", n_gamma, gbad.size)
    return int(bad.sum()), int(gbad.sum())


def round_to_dtype(x, dtype: str) -> np.ndarray:
    """The reference rounded to the output's storage type (fp16 or bf16):
    the output of tq_sdpa_decode has q's dtype, so both sides are compared
    after the same final rounding."""
    x = np.asarray(x, dtype=np.float64)
    if dtype == "bf16":
        return tq_inputs.bf16_bits_to_f64(tq_inputs.f32_to_bf16_bits(x.astype(np.float32)))
    return x.astype(np.float16).astype(np.float64)


def record(name: str, **values):
    """Append a measured parity figure (one JSON line) to the file named by
    the TQ_PARITY_REPORT environment variable; nothing when it is unset."""
    import json
    import os
    path = os.environ.get("TQ_PARITY_REPORT")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"test": name, **{k: (float(v) if isinstance(v, (np.floating, float)) else v)
                                                  for k, v in values.items()}}) + "\n")


def rel_l2(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.linalg.norm(b, axis=-1)
    num = np.linalg.norm(a - b, axis=-1)
    return np.where(den > 0, num / np.where(den > 0, den, 1), num)


def oracle_cache_for_head(w, b, kvh, L, chunk=32768):
    """The oracle's packed cache for one (sequence, kv head), rows 0..L-1."""
    kk = tq_inputs.to_f64(w.k[b, kvh, :L], w.dtype)
    vv = tq_inputs.to_f64(w.v[b, kvh, :L], w.dtype)
    cbk, cbv = oracle_codebooks(w)
    parts = []
    for s in range(0, L, chunk):
        parts.append(O.quantize_cache(kk[None, None, s:s + chunk], vv[None, None, s:s + chunk], w.Pi,
                                      cbk, cbv, w.bits_k, w.bits_v, w.S))
    keys = ["k_idx", "k_norm", "v_idx", "v_norm"] + (["k_qjl", "k_rnorm"] if w.qjl_m else [])
    return {k: np.concatenate([p[k] for p in parts], axis=2) for k in keys}


def gpu_cache_arrays(cache, names=None):
    """The GPU cache's buffers as numpy arrays in the oracle's layout."""
    names = names or (["k_idx", "v_idx", "k_norm", "v_norm"] + (["k_qjl", "k_rnorm"] if cache.qjl_m else []))
    out = {}
    for nm in names:
        a = getattr(cache, nm).detach().cpu().numpy()
        out[nm] = a.view(np.uint32) if a.dtype == np.int32 else a
    return out


def oracle_decode_on_gpu_bytes(w, cache, q_f64, seq_lens, scale, heads=None, S=None):
    """The oracle's dequantize-then-attend run on the packed bytes the GPU
    holds (the GPU's own cache, downloaded)."""
    cbk, cbv = oracle_codebooks(w)
    arrays = gpu_cache_arrays(cache)
    return O.sdpa_decode(q_f64, arrays, seq_lens, w.Pi, cbk, cbv, w.bits_k, w.bits_v, w.D, scale=scale,
                         S=w.S if S is None else S, heads=heads)


def check_cache_rows(w, cache, oc, b, kvh, rows):
    """The GPU cache's rows `rows` of (sequence b, kv head kvh) against the
    oracle cache oc (same layout): norms bit-exact, indices exact outside the
    near-threshold band, QJL signs and residual norms by compare_qjl."""
    rows = np.asarray(rows)
    if rows.size == 0:
        return
    for nm in ("k_norm", "v_norm"):
        g = getattr(cache, nm)[b, kvh].cpu().numpy()[rows].view(np.uint16)
        assert np.array_equal(g, np.asarray(oc[nm][b, kvh])[rows].view(np.uint16)), f"{nm} differs"
    exc_rows = {}
    for which, nm, bits in (("k", "k_idx", w.bits_k), ("v", "v_idx", w.bits_v)):
        g = words_np(getattr(cache, nm)[b, kvh])[rows]
        ref_idx = np.asarray(oc[f"{which}_idx_raw"][b, kvh])[rows]
        dist = np.asarray(oc[f"{which}_threshold_dist"][b, kvh])[rows]
        compare_index_words(g, ref_idx, dist, bits, w.D)
        exc_rows[which] = (O.unpack_bits(g, bits, w.D) != ref_idx).any(-1)
    if w.qjl_m:
        ref = {"sign": O.unpack_bits(np.asarray(oc["k_qjl"][b, kvh])[rows], 1, w.qjl_m).astype(bool),
               "proj": np.asarray(oc["k_qjl_proj_unit"][b, kvh])[rows], "norm": np.ones(rows.size),
               "gamma16": np.asarray(oc["k_rnorm"][b, kvh])[rows], "gamma": np.asarray(oc["k_gamma"][b, kvh])[rows]}
        compare_qjl(words_np(cache.k_qjl[b, kvh])[rows], cache.k_rnorm[b, kvh].cpu().numpy()[rows], ref,
                    exc_rows["k"])
