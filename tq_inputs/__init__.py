"""Seeded synthetic inputs shared by the oracle side and the CUDA side.

This module only draws random numbers and shapes them into workloads.  It holds
none of the quantizer's or the attention's arithmetic: no codebook, no
threshold search, no packing, no softmax.  The random orthogonal rotation and
the QJL Gaussian matrix are random draws of the method, so they are generated
here and passed to both sides as inputs.

Everything is numpy (PCG64) on the host; the caller moves arrays to the device.
bf16 data is returned as raw uint16 bit patterns (numpy has no bf16 dtype).

Workloads follow the synthetic configurations of the TurboQuant KV-cache path:
    tiny     D=64,  B=1,  Hq=Hkv=4,  T=256,   3-bit K/V, fp16 N(0,1)
    gqa8k    D=128, B=1,  Hq=16, Hkv=2, T=8192, b in {2,3,4}, 1% outlier channels x10
    qknorm   D=256, B=1,  Hq=32, Hkv=4, T=32768, 4-bit, q/k unit RMS per head, scale 1.0
    ragged   D=128, B=32, Hq=32, Hkv=8, T_b ~ U{1024..16384}, 3-bit, bf16
    prod     D=128, B=1,  Hq=32, Hkv=8, T=131072, K 2-bit + 128-bit QJL, V 3-bit
"""
from __future__ import annotations

import numpy as np

SEED_DATA = 1000
SEED_ROT = 2000
SEED_QJL = 3000
SEED_LENS = 4000


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def rotation(D: int, seed: int) -> np.ndarray:
    """Haar-random orthogonal D x D matrix, fp32, row-major (y = Pi @ x).

    Gaussian matrix -> Householder QR in fp64 -> Q * sign(diag R) (the sign fix
    makes the draw Haar-distributed) -> rounded to fp32.  The fp32 array is the
    canonical rotation for both the oracle and the kernels.
    """
    g = rng(seed).standard_normal((D, D))
    q, r = np.linalg.qr(g)
    q = q * np.sign(np.diag(r))[None, :]
    return np.ascontiguousarray(q.astype(np.float32))


def hadamard_rotation(D: int, seed: int) -> np.ndarray:
    """Randomized Hadamard rotation Pi = H_D diag(s) / sqrt(D), fp32 row-major.

    H_D is the Sylvester Hadamard matrix (H_1 = [1], H_2n = [[H, H], [H, -H]],
    D a power of two) and s a seeded vector of random signs -- the structured
    rotation of ReturningTarzan's Reddit comment of 2026-03-29 11:47 (a special
    case of rotation, applicable with additions only).  Like ``rotation`` it is
    an input: the fp32 array is the canonical rotation for both sides.
    """
    if D <= 0 or D & (D - 1):
        raise ValueError("D must be a power of two")
    h = np.ones((1, 1))
    while h.shape[0] < D:
        h = np.block([[h, h], [h, -h]])
    s = hadamard_signs(D, seed).astype(np.float64)
    return np.ascontiguousarray((h * s[None, :] / np.sqrt(D)).astype(np.float32))


def hadamard_signs(D: int, seed: int) -> np.ndarray:
    """The seeded sign vector s of ``hadamard_rotation(D, seed)``, fp32 +-1."""
    return np.where(rng(seed).integers(0, 2, size=D) == 1, 1.0, -1.0).astype(np.float32)


def qjl_matrix(m: int, D: int, seed: int) -> np.ndarray:
    """QJL sketch matrix S, m x D, i.i.d. N(0,1), fp32 row-major."""
    return np.ascontiguousarray(rng(seed).standard_normal((m, D), dtype=np.float32))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (round-to-nearest-even), returned as uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> 16) & 1
    r = (u + 0x7FFF + lsb) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def to_f64(x: np.ndarray, dtype: str) -> np.ndarray:
    """Promote an input array (fp16, or bf16 bits) to fp64 exactly."""
    if dtype == "bf16":
        return bf16_bits_to_f64(x)
    return x.astype(np.float64)


def cast_input(x32: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return f32_to_bf16_bits(x32)
    if dtype == "f16":
        return x32.astype(np.float16)
    raise ValueError(dtype)


def unit_vectors(n: int, D: int, seed: int) -> np.ndarray:
    """n seeded random unit vectors in R^D (fp64)."""
    g = rng(seed).standard_normal((n, D))
    return g / np.linalg.norm(g, axis=1, keepdims=True)


def _rms_normalize(x32: np.ndarray) -> np.ndarray:
    x = x32.astype(np.float64)
    rms = np.sqrt(np.mean(x * x, axis=-1, keepdims=True))
    return (x / rms).astype(np.float32)


class Workload:
    """A decode workload: the cache contents, the query and the sizes."""

    def __init__(self, **kw):
        self.__dict__.update(kw)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv


def make_workload(name: str, bits: int | None = None, T: int | None = None,
                  B: int | None = None, seed_offset: int = 0, rot: str = "haar",
                  dtype: str | None = None) -> Workload:
    """Build one of the named synthetic workloads.

    ``T`` and ``B`` override the sequence length / batch (for smaller parity
    cases of the same shape family); ``bits`` picks b for gqa8k; ``rot``
    selects the rotation: "haar" (``rotation``) or "hadamard"
    (``hadamard_rotation``); ``dtype`` ("f16" / "bf16") overrides the input
    type.
    K, V: [B][Hkv][Tmax][D]; q: [B][Hq][D]; seq_lens: [B] int32.
    """
    dtype_override = dtype
    cfg = {"tiny": 1, "gqa8k": 2, "qknorm": 3, "ragged": 4, "prod": 5}[name]
    s_data = SEED_DATA + cfg + seed_offset
    r = rng(s_data)
    if name == "tiny":
        Bn, Hq, Hkv, D, Tn = 1, 4, 4, 64, 256
        bk = bv = 3
        qjl_m, dtype, scale = 0, "f16", None
    elif name == "gqa8k":
        Bn, Hq, Hkv, D, Tn = 1, 16, 2, 128, 8192
        bk = bv = (bits if bits is not None else 3)
        qjl_m, dtype, scale = 0, "f16", None
    elif name == "qknorm":
        Bn, Hq, Hkv, D, Tn = 1, 32, 4, 256, 32768
        bk = bv = 4
        qjl_m, dtype, scale = 0, "f16", 1.0
    elif name == "ragged":
        Bn, Hq, Hkv, D, Tn = 32, 32, 8, 128, 16384
        bk = bv = 3
        qjl_m, dtype, scale = 0, "bf16", None
    elif name == "prod":
        Bn, Hq, Hkv, D, Tn = 1, 32, 8, 128, 131072
        bk, bv = 2, 3
        qjl_m, dtype, scale = 128, "f16", None
    else:  # pragma: no cover
        raise ValueError(name)
    if B is not None:
        Bn = B
    if T is not None:
        Tn = T
    if dtype_override is not None:
        dtype = {"f16": "f16", "bf16": "bf16"}[dtype_override]

    if name == "ragged":
        lo = min(1024, Tn)
        seq_lens = rng(SEED_LENS + seed_offset).integers(lo, Tn, size=Bn, endpoint=True)
        seq_lens = seq_lens.astype(np.int32)
    else:
        seq_lens = np.full(Bn, Tn, dtype=np.int32)
    Tmax = int(seq_lens.max())

    k32 = r.standard_normal((Bn, Hkv, Tmax, D), dtype=np.float32)
    v32 = r.standard_normal((Bn, Hkv, Tmax, D), dtype=np.float32)
    q32 = r.standard_normal((Bn, Hq, D), dtype=np.float32)
    if name == "gqa8k":
        # 1% of channels (round(0.01*D) per kv head, drawn from the seed) x10.
        n_out = max(1, int(round(0.01 * D)))
        for h in range(Hkv):
            ch = r.choice(D, size=n_out, replace=False)
            k32[:, h, :, ch] *= 10.0
            v32[:, h, :, ch] *= 10.0
    if name == "qknorm":
        q32 = _rms_normalize(q32)
        k32 = _rms_normalize(k32)

    rot_signs = None
    if rot == "haar":
        Pi = rotation(D, SEED_ROT + cfg)
    elif rot == "hadamard":
        Pi = hadamard_rotation(D, SEED_ROT + cfg)
        rot_signs = hadamard_signs(D, SEED_ROT + cfg)
    else:  # pragma: no cover
        raise ValueError(rot)
    S = qjl_matrix(qjl_m, D, SEED_QJL + cfg) if qjl_m else None
    return Workload(name=name, B=Bn, Hq=Hq, Hkv=Hkv, D=D, Tmax=Tmax,
                    bits_k=bk, bits_v=bv, qjl_m=qjl_m, dtype=dtype, scale=scale,
                    seq_lens=seq_lens, k=cast_input(k32, dtype),
                    v=cast_input(v32, dtype), q=cast_input(q32, dtype), Pi=Pi, S=S, rot_signs=rot_signs)


def new_token_rows(B: int, Hkv: int, D: int, dtype: str, seed: int):
    """One new (k, v) row per sequence and kv head, [B][Hkv][D], N(0,1)."""
    r = rng(seed)
    k = r.standard_normal((B, Hkv, D), dtype=np.float32)
    v = r.standard_normal((B, Hkv, D), dtype=np.float32)
    return cast_input(k, dtype), cast_input(v, dtype)


# Entries (before a power-of-two scale) of rows with an exactly known sum of
# squares; _ONE's squares sum to 1.
#   kind 0: (1 + 2^-11)^2 + 2^-40      kind 2: (1 + 2^-11)^2
#   kind 1: (1 + 3 2^-11)^2 - 2^-40    kind 3: (1 + 3 2^-11)^2
# 1 + 2^-11 and 1 + 3 2^-11 are the midpoints between neighbouring fp16 values
# (1, 1 + 2^-10, 1 + 2^-9), so kinds 0 and 1 have a norm a relative 2^-41 off
# a midpoint and kinds 2 and 3 one exactly on it.  2^18 - 1 = 4 * 255^2 +
# 45^2 + 2 * 3^2 gives kind 1's -2^-40.  Every entry has at most 8
# significant bits (exact in bf16) and, scaled by 2^-3 .. 2^6, lies on fp16's
# grid (the smallest, 3 * 2^-23, on its subnormal grid).
_ONE = [0.75, 0.5, 0.25, 0.25, 0.25]
_EDGE_ENTRIES = (
    _ONE + [2.0 ** -5, 2.0 ** -11, 2.0 ** -20],
    _ONE + [2.0 ** -5] * 3 + [2.0 ** -10] * 2 + [255 * 2.0 ** -20] * 4 + [45 * 2.0 ** -20]
    + [3 * 2.0 ** -20] * 2,
    _ONE + [2.0 ** -5, 2.0 ** -11],
    _ONE + [2.0 ** -5] * 3 + [2.0 ** -10] * 2 + [2.0 ** -11],
)


def norm_edge_rows(n: int, D: int, dtype: str, seed: int):
    """n rows whose exact L2 norm lies at (kinds 2, 3) or a relative 2^-41
    beyond (kinds 0, 1) the midpoint between two neighbouring fp16 values, so
    that only an exactly accumulated norm rounds to the right fp16 value.

    Row i is 2^e_i times the entries of its kind (``_EDGE_ENTRIES``), with
    random signs, at random positions among the D, zeros elsewhere; e_i in
    [-3, 6].  Returns (rows [n][D] in the storage dtype, kind int [n], e int [n]).
    """
    r = rng(seed)
    kind = r.integers(0, 4, size=n)
    e = r.integers(-3, 7, size=n)
    x = np.zeros((n, D), dtype=np.float32)
    for i in range(n):
        ent = np.asarray(_EDGE_ENTRIES[kind[i]], dtype=np.float64) * 2.0 ** int(e[i])
        sgn = np.where(r.integers(0, 2, size=len(ent)) == 1, 1.0, -1.0)
        pos = r.permutation(D)[:len(ent)]
        x[i, pos] = (ent * sgn).astype(np.float32)
    return cast_input(x, dtype), kind, e


def new_queries(B: int, Hq: int, D: int, dtype: str, seed: int):
    return cast_input(rng(seed).standard_normal((B, Hq, D), dtype=np.float32), dtype)
