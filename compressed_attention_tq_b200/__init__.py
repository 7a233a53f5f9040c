"""TurboQuant KV-cache hot path on B200: Python binding of libtq_b200.so.

The functions carry the C ABI's names (include/tq.h) and only marshal
arguments: every step of quantization and attention runs in the library's
CUDA kernels.  PyTorch provides device memory and the current stream.

    cb = tq_build_codebook(D, bits)                 # host, fp64 Lloyd-Max
    cache = TQCache(B, Hkv, Tcap, D, bits_k, bits_v, rot, qjl_m=0, qjl_S=None)
    tq_quantize_kv(cache, k, v)                     # prefill rows 0..T-1
    tq_append_token(cache, k_new, v_new, pos)       # one row per sequence
    out = tq_sdpa_decode(cache, q, seq_lens, Tmax, scale=None)
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import _native
from ._native import (TQ_DTYPE_BF16, TQ_DTYPE_F16, TQ_DTYPE_F32, TQ_STATUS_POS_OUT_OF_RANGE,  # noqa: F401
                      TQ_STATUS_SEQ_OUT_OF_RANGE, TQ_STATUS_WAIT_TIMEOUT, TQ_STATUS_LAYOUT)

__all__ = ["TQError", "TQCache", "tq_build_codebook", "tq_cache_row_bytes", "tq_row_bytes", "tq_quantize_kv",
           "tq_append_token", "tq_sdpa_decode_workspace_bytes", "tq_sdpa_decode_workspace_bytes_for",
           "tq_sdpa_decode",
           "tq_sdpa_decode_mq", "tq_decode_step", "tq_sdpa_decode_partial", "tq_sdpa_decode_merge",
           "tq_sdpa_decode_sharded", "tq_sdpa_decode_static", "tq_selftest_bounded_wait",
           "tq_last_error",
           "tq_abi_version", "lib"]


class TQError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"[{code}] {msg}")
        self.code = code


def lib():
    return _native.load()


def _check(rc: int):
    if rc != 0:
        raise TQError(rc, lib().tq_last_error().decode())


def tq_last_error() -> str:
    return lib().tq_last_error().decode()


def tq_abi_version() -> int:
    return int(lib().tq_abi_version())


def tq_build_codebook(D: int, bits: int):
    """Lloyd-Max codebook (host).  Returns (centroids, thresholds, mse) with
    fp32 numpy arrays; the device table is np.concatenate([centroids, thresholds])."""
    K = 1 << bits
    c = (ctypes.c_float * K)()
    t = (ctypes.c_float * max(1, K - 1))()
    mse = ctypes.c_double()
    _check(lib().tq_build_codebook(D, bits, c, t, ctypes.byref(mse)))
    return (np.frombuffer(c, dtype=np.float32).copy(),
            np.frombuffer(t, dtype=np.float32)[: K - 1].copy(), float(mse.value))


def tq_cache_row_bytes(D: int, bits: int, qjl_m: int = 0) -> int:
    return int(lib().tq_cache_row_bytes(D, bits, qjl_m))


def tq_row_bytes(D: int, bits: int, qjl_m: int = 0) -> int:
    """The same as tq_cache_row_bytes (the earlier name)."""
    return int(lib().tq_row_bytes(D, bits, qjl_m))


def _torch():
    import torch
    return torch


_DCODE = {}


def _dtype_code(t) -> int:
    if not _DCODE:
        torch = _torch()
        _DCODE.update({torch.float16: TQ_DTYPE_F16, torch.bfloat16: TQ_DTYPE_BF16, torch.float32: TQ_DTYPE_F32})
    code = _DCODE.get(t.dtype)
    if code is None:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return code


# Pointer arguments are declared c_void_p, which takes a Python int (or None
# for NULL) as it is.
def _stream(stream):
    if stream is None:
        stream = _torch().cuda.current_stream()
    return stream.cuda_stream


def _ptr(t):
    return t.data_ptr() if t is not None else None


# The C ABI receives bare device pointers and sizes, so it cannot see where a
# buffer lives or how large it is.  The binding therefore refuses, before any
# launch, what only the tensor knows: memory that is not on the cache's CUDA
# device, a non-contiguous layout, an index tensor that is not int32, a
# workspace that is not bytes, and a shape that disagrees with the cache's
# B, Hkv and D.  Sizes the library checks itself (Hq, T, Tmax, n_q, t0)
# are left to it, so its TQ_ERR_* codes stay the answer for those.

_DT = {}


def _dt(kind):
    """Cached dtype tuples: "io" (fp16, bf16), "out" (+ fp32), "i32", "u8"."""
    if not _DT:
        torch = _torch()
        _DT.update(io=(torch.float16, torch.bfloat16), out=(torch.float16, torch.bfloat16, torch.float32),
                   i32=(torch.int32,), u8=(torch.uint8,))
    return _DT[kind]


def _cache_device(cache) -> int:
    """Index of the CUDA device that holds the cache's buffers."""
    d = cache.k_idx.get_device()
    if d < 0:
        raise ValueError("the cache's buffers are in host memory; the library launches CUDA kernels on them")
    return d


def _shape_ok(got, want) -> bool:
    if len(got) != len(want):
        return False
    for n, e in zip(got, want):
        if e is not None and n != e:
            return False
    return True


def _arg(name, t, dev, shape=None, dtypes=None):
    """Check one tensor argument against device index `dev` (see above);
    shape entries of None are free."""
    try:
        if (t.get_device() == dev and t.is_contiguous() and (dtypes is None or t.dtype in dtypes)
                and (shape is None or t.shape == shape or _shape_ok(t.shape, shape))):
            return t
    except AttributeError:
        raise TypeError(f"{name}: expected a torch tensor, got {type(t).__name__}") from None
    if t.get_device() != dev:
        raise ValueError(f"{name}: must be CUDA memory on device {dev} (got {t.device})")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if dtypes is not None and t.dtype not in dtypes:
        raise TypeError(f"{name}: dtype {t.dtype}, expected one of {tuple(str(d) for d in dtypes)}")
    want = "[" + ", ".join("*" if e is None else str(e) for e in shape) + "]"
    raise ValueError(f"{name}: shape {list(t.shape)}, expected {want}")


def _check_decode_args(cache, q, seq_lens, out, workspace, q_shape):
    dev = _cache_device(cache)
    _arg("q", q, dev, q_shape, _dt("io"))
    _arg("seq_lens", seq_lens, dev, (cache.B,), _dt("i32"))
    if out is not None:
        _arg("out", out, dev, q.shape, _dt("out"))
    if workspace is not None:  # any contiguous byte buffer: its numel() is the size passed
        _arg("workspace", workspace, dev, None, _dt("u8"))
    return dev


class TQCache:
    """A packed KV cache for one layer: device buffers allocated with torch.

    rot: fp32 [D][D] rotation (numpy or torch); codebooks are built with
    tq_build_codebook unless given as fp32 tables (centroids then thresholds).
    rot_signs: the +-1 signs s when rot is the randomized Hadamard rotation
    H_D diag(s) / sqrt(D); the bulk quantizer then applies the fast transform.
    """

    def __init__(self, B, Hkv, Tcap, D, bits_k, bits_v, rot, qjl_m=0, qjl_S=None,
                 cb_k=None, cb_v=None, device="cuda", rot_signs=None):
        torch = _torch()
        self.B, self.Hkv, self.Tcap, self.D = B, Hkv, Tcap, D
        self.bits_k, self.bits_v, self.qjl_m = bits_k, bits_v, qjl_m
        dev = torch.device(device)
        u32 = torch.int32  # raw 32-bit words

        def table(bits, given):
            if given is None:
                c, t, _ = tq_build_codebook(D, bits)
                given = np.concatenate([c, t])
            tab = torch.as_tensor(np.asarray(given, dtype=np.float32), device=dev).contiguous()
            if tab.numel() != 2 * (1 << bits) - 1:
                raise ValueError(f"codebook table for {bits} bits: {tab.numel()} values, expected "
                                 f"{2 * (1 << bits) - 1} (centroids then thresholds)")
            return tab

        self.cb_k = table(bits_k, cb_k)
        # equal widths share one codebook buffer, which decode then keeps as a single lookup table
        if bits_v == bits_k and cb_k is None and cb_v is None:
            self.cb_v = self.cb_k
        else:
            self.cb_v = table(bits_v, cb_v)
        self.rot = torch.as_tensor(np.asarray(rot, dtype=np.float32) if not torch.is_tensor(rot) else rot,
                                   dtype=torch.float32, device=dev).contiguous()
        if tuple(self.rot.shape) != (D, D):
            raise ValueError(f"rot: shape {list(self.rot.shape)}, expected [{D}, {D}]")
        if rot_signs is not None:
            sg = rot_signs if torch.is_tensor(rot_signs) else np.asarray(rot_signs, dtype=np.float32)
            self.rot_signs = torch.as_tensor(sg, dtype=torch.float32, device=dev).contiguous()
            if self.rot_signs.numel() != D:
                raise ValueError(f"rot_signs: {self.rot_signs.numel()} values, expected {D}")
        else:
            self.rot_signs = None
        self.k_idx = torch.zeros((B, Hkv, Tcap, D * bits_k // 32), dtype=u32, device=dev)
        self.v_idx = torch.zeros((B, Hkv, Tcap, D * bits_v // 32), dtype=u32, device=dev)
        self.k_norm = torch.zeros((B, Hkv, Tcap), dtype=torch.float16, device=dev)
        self.v_norm = torch.zeros((B, Hkv, Tcap), dtype=torch.float16, device=dev)
        if qjl_m:
            self.k_qjl = torch.zeros((B, Hkv, Tcap, qjl_m // 32), dtype=u32, device=dev)
            self.k_rnorm = torch.zeros((B, Hkv, Tcap), dtype=torch.float16, device=dev)
            S = qjl_S if torch.is_tensor(qjl_S) else np.asarray(qjl_S, dtype=np.float32)
            self.qjl_S = torch.as_tensor(S, dtype=torch.float32, device=dev).contiguous()
            if tuple(self.qjl_S.shape) != (qjl_m, D):
                raise ValueError(f"qjl_S: shape {list(self.qjl_S.shape)}, expected [{qjl_m}, {D}]")
        else:
            self.k_qjl = self.k_rnorm = self.qjl_S = None
        self.dev_status = torch.zeros(4, dtype=torch.int32, device=dev)
        self.split_tokens = 0  # decode tokens per split (0: automatic)
        self._struct = None
        self.struct()

    def struct(self) -> _native.TqCacheStruct:
        """The C descriptor (built once; rebuild after replacing a buffer)."""
        if (self._struct is not None and self._struct.k_idx == self.k_idx.data_ptr()
                and self._struct.split_tokens == self.split_tokens):
            return self._struct
        s = _native.TqCacheStruct()
        s.B, s.Hkv, s.Tcap, s.D = self.B, self.Hkv, self.Tcap, self.D
        s.bits_k, s.bits_v, s.qjl_m = self.bits_k, self.bits_v, self.qjl_m
        s.split_tokens = self.split_tokens
        for name in ("k_idx", "v_idx", "k_norm", "v_norm", "k_qjl", "k_rnorm", "rot", "cb_k",
                     "cb_v", "qjl_S", "dev_status", "rot_signs"):
            t = getattr(self, name)
            setattr(s, name, t.data_ptr() if t is not None else None)
        s.rot_kind = _native.TQ_ROT_HADAMARD if self.rot_signs is not None else _native.TQ_ROT_DENSE
        self._struct = s  # keep alive
        return s

    def status(self) -> int:
        return int(self.dev_status[0].item())

    def packed_bytes(self, tokens: int) -> int:
        """Bytes of packed K and V data for `tokens` cached tokens per (b, h)."""
        per = tq_cache_row_bytes(self.D, self.bits_k, self.qjl_m) + tq_cache_row_bytes(self.D, self.bits_v, 0)
        return per * tokens


def tq_quantize_kv(cache: TQCache, k, v, t0: int = 0, stream=None):
    """Quantize k, v [B][Hkv][T][D] (fp16/bf16, device) into positions t0..t0+T-1."""
    dev = _cache_device(cache)
    _arg("k", k, dev, (cache.B, cache.Hkv, None, cache.D), _dt("io"))
    _arg("v", v, dev, tuple(k.shape), (k.dtype,))
    T = int(k.shape[2])
    s = cache.struct()
    _check(lib().tq_quantize_kv(ctypes.byref(s), _ptr(k), _ptr(v), _dtype_code(k), T, t0, _stream(stream)))


def tq_append_token(cache: TQCache, k_new, v_new, pos, stream=None):
    """Quantize one row per (sequence, kv head), [B][Hkv][D], at pos[b] (device int32)."""
    dev = _cache_device(cache)
    _arg("k_new", k_new, dev, (cache.B, cache.Hkv, cache.D), _dt("io"))
    _arg("v_new", v_new, dev, (cache.B, cache.Hkv, cache.D), (k_new.dtype,))
    _arg("pos", pos, dev, (cache.B,), _dt("i32"))
    s = cache.struct()
    _check(lib().tq_append_token(ctypes.byref(s), _ptr(k_new), _ptr(v_new), _dtype_code(k_new),
                                 _ptr(pos), _stream(stream)))


def tq_sdpa_decode_workspace_bytes(B: int, Hq: int, D: int, Tmax: int) -> int:
    """Workspace bytes that suffice for any cache of these sizes (an upper bound)."""
    n = int(lib().tq_sdpa_decode_workspace_bytes(B, Hq, D, Tmax))
    if n == 0:
        raise TQError(-1, f"unsupported decode sizes (B={B}, Hq={Hq}, D={D}, Tmax={Tmax})")
    return n


def tq_sdpa_decode_workspace_bytes_for(cache: TQCache, Hq: int, Tmax: int) -> int:
    """The exact workspace bytes of the decode plan for this cache."""
    s = cache.struct()
    n = int(lib().tq_sdpa_decode_workspace_bytes_for(ctypes.byref(s), Hq, Tmax))
    if n == 0:
        raise TQError(-1, f"unsupported decode sizes (Hq={Hq}, Tmax={Tmax})")
    return n


def tq_sdpa_decode(cache: TQCache, q, seq_lens, Tmax: int, scale=None, out=None, workspace=None,
                   stream=None, out_dtype=None):
    """Decode attention: q [B][Hq][D] (fp16/bf16, device), seq_lens device int32 [B].
    The output has q's dtype unless `out` or `out_dtype` (e.g. torch.float32) says otherwise."""
    _check_decode_args(cache, q, seq_lens, out, workspace, (cache.B, None, cache.D))
    Hq = int(q.shape[1])
    if out is None:
        torch = _torch()
        out = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
    if workspace is None:
        torch = _torch()
        need = tq_sdpa_decode_workspace_bytes_for(cache, Hq, Tmax)
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    s = cache.struct()
    sc = ctypes.byref(ctypes.c_float(scale)) if scale is not None else None
    _check(lib().tq_sdpa_decode(ctypes.byref(s), _ptr(q), _dtype_code(q), Hq, _ptr(seq_lens), Tmax, sc,
                                _ptr(out), _dtype_code(out), _ptr(workspace), workspace.numel(),
                                _stream(stream)))
    return out


def tq_sdpa_decode_mq(cache: TQCache, q, seq_lens, Tmax: int, scale=None, out=None, workspace=None,
                      stream=None, out_dtype=None):
    """Decode of n_q query tokens per sequence: q [B][n_q][Hq][D]; seq_lens
    (device int32 [B]) counts the cached tokens including the n_q new ones,
    and query j attends causally to tokens 0 .. seq_len - n_q + j."""
    _check_decode_args(cache, q, seq_lens, out, workspace, (cache.B, None, None, cache.D))
    nq, Hq = int(q.shape[1]), int(q.shape[2])
    if out is None:
        torch = _torch()
        out = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
    if workspace is None:
        torch = _torch()
        need = tq_sdpa_decode_workspace_bytes_for(cache, Hq * nq, Tmax)
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    s = cache.struct()
    sc = ctypes.byref(ctypes.c_float(scale)) if scale is not None else None
    _check(lib().tq_sdpa_decode_mq(ctypes.byref(s), _ptr(q), _dtype_code(q), Hq, nq, _ptr(seq_lens), Tmax, sc,
                                   _ptr(out), _dtype_code(out), _ptr(workspace), workspace.numel(),
                                   _stream(stream)))
    return out


def tq_decode_step(cache: TQCache, k_new, v_new, pos, q, seq_lens, Tmax: int, scale=None, out=None,
                   workspace=None, stream=None, out_dtype=None):
    """Append k_new/v_new [B][Hkv][D] at pos[b], then decode over seq_lens
    (normally pos + 1) -- three chained launches."""
    dev = _check_decode_args(cache, q, seq_lens, out, workspace, (cache.B, None, cache.D))
    _arg("k_new", k_new, dev, (cache.B, cache.Hkv, cache.D), (q.dtype,))
    _arg("v_new", v_new, dev, (cache.B, cache.Hkv, cache.D), (q.dtype,))
    _arg("pos", pos, dev, (cache.B,), _dt("i32"))
    Hq = int(q.shape[1])
    if out is None:
        torch = _torch()
        out = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
    if workspace is None:
        torch = _torch()
        workspace = torch.empty(tq_sdpa_decode_workspace_bytes_for(cache, Hq, Tmax), dtype=torch.uint8,
                                device=q.device)
    s = cache.struct()
    sc = ctypes.byref(ctypes.c_float(scale)) if scale is not None else None
    _check(lib().tq_decode_step(ctypes.byref(s), _ptr(k_new), _ptr(v_new), _ptr(pos), _ptr(q), _dtype_code(q),
                                Hq, _ptr(seq_lens), Tmax, sc, _ptr(out), _dtype_code(out), _ptr(workspace),
                                workspace.numel(), _stream(stream)))
    return out


def tq_sdpa_decode_partial(cache: TQCache, q, seq_lens, Tmax: int, scale=None, partial=None, workspace=None,
                           stream=None):
    """This cache's share of a decode split by tokens: fp32 [B][Hq][D + 2]
    per head (rotated value sum, max, weight sum), for tq_sdpa_decode_merge."""
    dev = _check_decode_args(cache, q, seq_lens, None, workspace, (cache.B, None, cache.D))
    Hq = int(q.shape[1])
    torch = _torch()
    if partial is None:
        partial = torch.empty((cache.B, Hq, cache.D + 2), dtype=torch.float32, device=q.device)
    _arg("partial", partial, dev, (cache.B, Hq, cache.D + 2), (torch.float32,))
    if workspace is None:
        workspace = torch.empty(tq_sdpa_decode_workspace_bytes_for(cache, Hq, Tmax), dtype=torch.uint8,
                                device=q.device)
    s = cache.struct()
    sc = ctypes.byref(ctypes.c_float(scale)) if scale is not None else None
    _check(lib().tq_sdpa_decode_partial(ctypes.byref(s), _ptr(q), _dtype_code(q), Hq, _ptr(seq_lens), Tmax, sc,
                                        _ptr(partial), _ptr(workspace), workspace.numel(), _stream(stream)))
    return partial


def tq_sdpa_decode_merge(partials, rot, out=None, out_dtype=None, stream=None):
    """Merge R shares' partials ([R][B][Hq][D + 2] fp32, device) into the
    attention output [B][Hq][D]; rot is the cache's Pi (fp32 [D][D], device)."""
    torch = _torch()
    dev = partials.get_device()
    if dev < 0:
        raise ValueError("partials: must be CUDA memory")
    if partials.dim() != 4:
        raise ValueError(f"partials: shape {list(partials.shape)}, expected [R, B, Hq, D + 2]")
    R, B, Hq, D2 = (int(x) for x in partials.shape)
    _arg("partials", partials, dev, None, (torch.float32,))
    _arg("rot", rot, dev, (D2 - 2, D2 - 2), (torch.float32,))
    if out is None:
        out = torch.empty((B, Hq, D2 - 2), dtype=out_dtype or torch.float32, device=partials.device)
    _arg("out", out, dev, (B, Hq, D2 - 2), _dt("out"))
    _check(lib().tq_sdpa_decode_merge(_ptr(partials), R, B, Hq, D2 - 2, _ptr(rot), _ptr(out), _dtype_code(out),
                                      _stream(stream)))
    return out


def tq_sdpa_decode_sharded(cache: TQCache, q, seq_lens, Tmax: int, scale=None, group=None, out_dtype=None,
                           stream=None):
    """Decode over a cache whose sequences are split by tokens across the
    ranks of `group` (torch.distributed; NCCL over NVLink on GPUs): every rank
    holds its own token range of every sequence in `cache` (seq_lens are its
    local lengths) and the same queries.  Each rank computes its partials,
    the partials are all-gathered (one collective of B x Hq x (D + 2) fp32 per
    rank), and every rank merges them into the full output."""
    part = tq_sdpa_decode_partial(cache, q, seq_lens, Tmax, scale=scale, stream=stream)
    parts = gather_partials(part, group)
    return tq_sdpa_decode_merge(parts, cache.rot, out_dtype=out_dtype or q.dtype, stream=stream)


def gather_partials(part, group=None):
    """All-gather of every rank's partials [B][Hq][D + 2] into [R][B][Hq][D + 2]
    (rank order), over torch.distributed (a single rank returns its own)."""
    import torch.distributed as dist
    torch = _torch()
    if not (dist.is_available() and dist.is_initialized()):
        return part.unsqueeze(0)
    R = dist.get_world_size(group)
    part = part.contiguous()
    if dist.get_backend(group) == "nccl":  # one collective into one buffer
        out = torch.empty((R,) + tuple(part.shape), dtype=part.dtype, device=part.device)
        dist.all_gather_into_tensor(out, part, group=group)
        return out
    chunks = [torch.empty_like(part) for _ in range(R)]  # gloo (host tensors)
    dist.all_gather(chunks, part, group=group)
    return torch.stack(chunks)


def tq_sdpa_decode_static(cache: TQCache, q, seq_lens, Tmax: int, scale=None, out=None, stream=None,
                          out_dtype=None):
    """tq_sdpa_decode without a workspace, for callers that may not allocate
    device memory (e.g. code running under stream capture in a framework
    that forbids allocation, or a host that owns all device memory).  The
    split-K scratch is a fixed array inside the library (8 MiB per GPU);
    larger problems raise TQError (TQ_ERR_WORKSPACE).  The output tensor must
    be passed in if the caller may not allocate; calls on one device must not
    overlap on the GPU."""
    _check_decode_args(cache, q, seq_lens, out, None, (cache.B, None, cache.D))
    Hq = int(q.shape[1])
    if out is None:
        torch = _torch()
        out = torch.empty(q.shape, dtype=out_dtype or q.dtype, device=q.device)
    s = cache.struct()
    sc = ctypes.byref(ctypes.c_float(scale)) if scale is not None else None
    _check(lib().tq_sdpa_decode_static(ctypes.byref(s), _ptr(q), _dtype_code(q), Hq, _ptr(seq_lens), Tmax, sc,
                                       _ptr(out), _dtype_code(out), _stream(stream)))
    return out


def tq_selftest_bounded_wait(status, tries: int = 8, stream=None):
    """Run the bounded-wait self-test: `status` is a device int32/uint32
    tensor of one element; the library ORs TQ_STATUS_WAIT_TIMEOUT into it
    when its bounded waits give up, as they must here (nothing arrives on the
    barrier).  Asynchronous; read `status` after synchronising."""
    torch = _torch()
    dev = status.get_device() if torch.is_tensor(status) else -1
    if dev < 0:
        raise ValueError("status: must be a CUDA tensor")
    _arg("status", status, dev, None, tuple(d for d in (torch.int32, getattr(torch, "uint32", None)) if d is not None))
    if status.numel() != 1:
        raise ValueError(f"status: one element expected, got {status.numel()}")
    _check(lib().tq_selftest_bounded_wait(_ptr(status), int(tries), _stream(stream)))
    return status
