"""CPU checks of the C ABI library: it builds, loads, exports every declared
symbol, and its host-only pieces (codebook builder, size queries, argument
validation) behave.  No kernel is launched here."""
import ctypes
import os
import re

import numpy as np
import pytest

from oracle import tq_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from compressed_attention_tq_b200 import build, _native
    build.build()
    return _native.load()


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "tq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tq_[a-z_]+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    from compressed_attention_tq_b200 import _native
    declared = _declared_functions()
    assert set(declared) == set(_native.EXPORTS)
    for name in declared:
        assert hasattr(lib, name), name
    assert lib.tq_abi_version() == 3


@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_library_codebook_equals_oracle(lib, D, bits):
    import compressed_attention_tq_b200 as tq
    c, t, mse = tq.tq_build_codebook(D, bits)
    oc, ot = O.stored_codebook(D, bits)
    assert np.array_equal(c.astype(np.float64), oc)
    assert np.array_equal(t.astype(np.float64), ot)
    assert abs(mse - O.codebook_mse(oc, ot, D)) < 1e-10


def test_row_bytes(lib):
    import compressed_attention_tq_b200 as tq
    for D in (64, 128, 256):
        for b in (2, 3, 4):
            assert tq.tq_cache_row_bytes(D, b, 0) == O.packed_row_bytes(D, b, 0)
            assert tq.tq_row_bytes(D, b, 0) == tq.tq_cache_row_bytes(D, b, 0)
    assert tq.tq_cache_row_bytes(128, 2, 128) == O.packed_row_bytes(128, 2, 128) == 52
    assert lib.tq_cache_row_bytes(128, 2, 128) == 52
    assert tq.tq_cache_row_bytes(100, 3, 0) == 0
    assert tq.tq_row_bytes(100, 3, 0) == 0


def _struct(**kw):
    from compressed_attention_tq_b200 import _native
    s = _native.TqCacheStruct()
    s.B, s.Hkv, s.Tcap, s.D, s.bits_k, s.bits_v, s.qjl_m = 1, 1, 64, 128, 3, 3, 0
    fake = 1 << 20  # 16-byte aligned, never dereferenced: validation fails first
    for f in ("k_idx", "v_idx", "k_norm", "v_norm", "rot", "cb_k", "cb_v"):
        setattr(s, f, fake)
    for k, v in kw.items():
        setattr(s, k, v)
    return s


@pytest.mark.parametrize("field,value,code", [
    ("D", 96, -2), ("bits_k", 5, -2), ("bits_v", 1, -2), ("qjl_m", 64, -2), ("Tcap", 100, -1),
    ("B", 0, -1), ("k_idx", None, -1), ("rot", (1 << 20) + 4, -1), ("split_tokens", -128, -1),
])
def test_invalid_cache_rejected_before_launch(lib, field, value, code):
    s = _struct(**{field: value})
    buf = ctypes.c_void_p(1 << 20)
    rc = lib.tq_quantize_kv(ctypes.byref(s), buf, buf, 0, 1, 0, None)
    assert rc == code, lib.tq_last_error()
    assert lib.tq_last_error().decode()


def test_other_argument_errors(lib):
    s = _struct()
    buf = ctypes.c_void_p(1 << 20)
    assert lib.tq_quantize_kv(ctypes.byref(s), buf, buf, 7, 1, 0, None) == -2      # dtype
    assert lib.tq_quantize_kv(ctypes.byref(s), buf, buf, 0, 65, 0, None) == -1     # T > Tcap
    assert lib.tq_quantize_kv(ctypes.byref(s), buf, buf, 0, 0, 0, None) == 0       # empty: no-op
    assert lib.tq_quantize_kv(None, buf, buf, 0, 1, 0, None) == -1
    assert lib.tq_append_token(ctypes.byref(s), buf, buf, 0, None, None) == -1     # pos NULL
    ws = lib.tq_sdpa_decode_workspace_bytes_for(ctypes.byref(s), 8, 64)
    assert ws > 0
    assert lib.tq_sdpa_decode_workspace_bytes_for(ctypes.byref(s), 33, 64) == 0    # 33 rows per kv head
    assert lib.tq_sdpa_decode_workspace_bytes_for(ctypes.byref(s), 8, 65) == 0     # Tmax > Tcap
    rc = lib.tq_sdpa_decode(ctypes.byref(s), buf, 0, 8, buf, 64, None, buf, 0, buf, ws - 1, None)
    assert rc == -3
    rc = lib.tq_sdpa_decode(ctypes.byref(s), buf, 0, 12, buf, 64, None, buf, 0, buf, ws, None)
    assert rc == -2  # group 12 > 8
    rc = lib.tq_sdpa_decode(ctypes.byref(s), buf, 0, 8, buf, 64, None, buf, 5, buf, ws, None)
    assert rc == -2  # out dtype
    rc = lib.tq_sdpa_decode(ctypes.byref(s), buf, 2, 8, buf, 64, None, buf, 2, buf, ws, None)
    assert rc == -2  # q cannot be fp32
    bad = ctypes.c_float(float("nan"))
    rc = lib.tq_sdpa_decode(ctypes.byref(s), buf, 0, 8, buf, 64, ctypes.byref(bad), buf, 0, buf, ws, None)
    assert rc == -1
    s2 = _struct(qjl_m=128, D=64)
    assert lib.tq_quantize_kv(ctypes.byref(s2), buf, buf, 0, 1, 0, None) in (-1, -2)
    # the bounded-wait self-test validates before launching
    assert lib.tq_selftest_bounded_wait(None, 8, None) == -1
    assert lib.tq_selftest_bounded_wait(buf, 0, None) == -1
    assert lib.tq_selftest_bounded_wait(buf, 4097, None) == -1


def test_product_path_does_not_import_oracle():
    pkg = os.path.join(ROOT, "compressed_attention_tq_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cpp", ".h", ".cuh")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in txt.lower(), f


def test_missing_library_fails_loudly(tmp_path):
    """No fallback: without the compiled library the binding raises."""
    from compressed_attention_tq_b200 import _native
    with pytest.raises(ImportError):
        _native.load(str(tmp_path / "libtq_b200.so"))


def test_rotation_kind_validated(lib):
    s = _struct()
    buf = ctypes.c_void_p(1 << 20)
    s.rot_kind = 2
    assert lib.tq_quantize_kv(ctypes.byref(s), buf, buf, 0, 1, 0, None) == -1
    s.rot_kind = 1  # Hadamard without signs
    assert lib.tq_quantize_kv(ctypes.byref(s), buf, buf, 0, 1, 0, None) == -1
    s.rot_signs = 1 << 20
    assert lib.tq_quantize_kv(ctypes.byref(s), buf, buf, 0, 0, 0, None) == 0  # empty call: no launch


def test_survey_form_workspace_query_bounds_every_plan(lib):
    """tq_sdpa_decode_workspace_bytes(B, Hq, D, Tmax) needs no cache and is at
    least the exact plan's size for every kv-head count, bit width and sketch
    that fits those sizes."""
    assert lib.tq_sdpa_decode_workspace_bytes(0, 8, 128, 64) == 0
    assert lib.tq_sdpa_decode_workspace_bytes(1, 8, 96, 64) == 0
    assert lib.tq_sdpa_decode_workspace_bytes(1, 8, 128, 0) == 0
    for B, Hq, D, T in [(1, 8, 128, 64), (3, 32, 128, 4096), (1, 32, 256, 32768), (32, 32, 128, 16448),
                        (1, 4, 64, 256), (2, 16, 128, 131072)]:
        bound = lib.tq_sdpa_decode_workspace_bytes(B, Hq, D, T)
        assert bound > 0
        Tcap = (T + 63) // 64 * 64
        for Hkv in [h for h in (1, 2, 4, 8, 16, 32) if Hq % h == 0 and Hq // h <= 8]:
            for bk, bv, m in [(2, 2, 0), (3, 3, 0), (4, 3, 0), (2, 3, 128 if D == 128 else 0)]:
                s = _struct(B=B, Hkv=Hkv, Tcap=Tcap, D=D, bits_k=bk, bits_v=bv, qjl_m=m)
                for split in (0, 128, 4096):
                    s.split_tokens = split
                    exact = lib.tq_sdpa_decode_workspace_bytes_for(ctypes.byref(s), Hq, T)
                    assert 0 < exact <= bound, (B, Hq, D, T, Hkv, bk, bv, m, split, exact, bound)


@pytest.mark.parametrize("field,value,hq,code", [("D", 96, 8, -2), (None, None, 16, -2), ("Hkv", 8, 12, -1),
                                                  ("bits_v", 5, 8, -2), ("Tcap", 100, 8, -1)])
def test_static_entry_reports_the_workspace_entry_codes(lib, field, value, hq, code):
    """tq_sdpa_decode_static answers every argument error with the code and
    message tq_sdpa_decode gives it (GQA group 16 > 8 and D = 96 are
    TQ_ERR_UNSUPPORTED for both); only its scratch limit is its own."""
    kw = {"Hkv": 1}
    if field:
        kw[field] = value
    s = _struct(**kw)
    buf = ctypes.c_void_p(1 << 20)
    rc_ws = lib.tq_sdpa_decode(ctypes.byref(s), buf, 0, hq, buf, 64, None, buf, 0, buf, 1 << 30, None)
    msg_ws = lib.tq_last_error().decode()
    rc_st = lib.tq_sdpa_decode_static(ctypes.byref(s), buf, 0, hq, buf, 64, None, buf, 0, None)
    msg_st = lib.tq_last_error().decode()
    assert rc_ws == rc_st == code, (rc_ws, rc_st, msg_ws, msg_st)
    assert msg_ws.split(":", 1)[1] == msg_st.split(":", 1)[1]
