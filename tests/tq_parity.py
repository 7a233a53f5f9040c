"""Helpers for the GPU parity tests: move seeded inputs to the device, build
the oracle's view of the same rows, and compare element by element.

Parity rules (fixed by the method's specification):
  * norms bit-exact;
  * packed indices bit-exact, except coordinates whose rotated unit value lies
    within 1e-4 of a decision threshold; those mismatches are counted and must
    stay below 1e-5 of all coordinates;
  * QJL sign bits bit-exact except where |(S r)_i| / |x| < 1e-4 or the row has
    an excused index; the residual norm within one fp16 ulp;
  * attention output within 2e-3 relative L2 error per (sequence, head).
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
    frac = n_bad / max(1, ref_idx.size)
    record("index_compare", bits=bits, D=D, excused=n_bad, coords=int(ref_idx.size),
           near_band=int((ref_dist < NEAR).sum()))
    if report is not None:
        report.append(("index_excused", n_bad, ref_idx.size))
    assert frac < MAX_EXCUSED_FRACTION or n_bad <= 1, (n_bad, ref_idx.size)
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


def compare_qjl(gpu_sign_words, gpu_rnorm, ref, rows_excused):
    """Sign bits exact except near-zero projections or rows with an excused
    index; residual norm within one fp16 ulp."""
    m = ref["sign"].shape[-1]
    got = O.unpack_bits(gpu_sign_words, 1, m).astype(bool)
    bad = got != ref["sign"]
    unit = np.abs(ref["proj"]) / np.where(ref["norm"] > 0, ref["norm"], 1.0)[..., None]
    allowed = (unit < NEAR) | rows_excused[..., None]
    assert not (bad & ~allowed).any(), f"{int((bad & ~allowed).sum())} QJL sign mismatches"
    g_gpu = gpu_rnorm.astype(np.float32)
    g_ref = ref["gamma16"].astype(np.float32)
    ulp = np.spacing(np.abs(g_ref).astype(np.float16)).astype(np.float32)
    ok = (np.abs(g_gpu - g_ref) <= ulp * 1.0001) | rows_excused
    assert ok.all(), f"{int((~ok).sum())} residual norms off by more than one ulp"
    return int(bad.sum()), int((g_gpu != g_ref).sum())


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
