"""Host-side checks of the C ABI: the library loads, exports every declared
entry point, and rejects bad arguments before enqueuing anything (these
calls return before any CUDA call, so they run without a GPU)."""
import ctypes
import os
import re

import pytest

from mla_latent_kv_43_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mla.h")

FAKE = 0x10000          # a non-null, 256-byte aligned address that is never dereferenced


def declared_symbols():
    src = open(HEADER).read()
    return re.findall(r"MLA_API\s+[\w\s\*]+?\b(mla_\w+)\s*\(", src)


def test_library_exports_every_declared_symbol():
    L = B.lib()
    names = declared_symbols()
    assert len(names) >= 8
    for n in names:
        assert hasattr(L, n), n
    out = os.popen(f"nm -D --defined-only {B.LIB_PATH}").read()
    exported = set(re.findall(r" T (mla_\w+)", out))
    assert set(names) <= exported, set(names) - exported


def v3(dtype="bf16", **kw):
    a = dict(heads=128, d_c=512, d_rope=64, qk_nope=128, v_dim=128, dtype=dtype)
    a.update(kw)
    return B.make_dims(**a)


def decode_raw(dims, batch=2, n_q=1, ptrs=FAKE, capacity=100, max_len=100, ws_bytes=None,
               ws=FAKE, splits=0, status=FAKE, seq=FAKE, out=FAKE):
    L = B.lib()
    if ws_bytes is None:
        ws_bytes = L.mla_decode_workspace_bytes(ctypes.byref(dims), batch, n_q, max_len, splits) if dims else 0
    d = ctypes.byref(dims) if dims is not None else None
    return L.mla_decode(d, batch, n_q, ptrs, ptrs, ptrs, ptrs, ptrs, capacity, seq, max_len, out,
                        ws, ws_bytes, splits, status, None)


@pytest.mark.parametrize("mut,code", [
    (dict(heads=0), "MLA_ERR_ARG"), (dict(d_rope=63), "MLA_ERR_ARG"), (dict(d_c=-4), "MLA_ERR_ARG"),
    (dict(dtype=7), "MLA_ERR_ARG"), (dict(softmax_scale=0.0), "MLA_ERR_ARG"),
    (dict(softmax_scale=float("nan")), "MLA_ERR_ARG"), (dict(rope_base=1.0), "MLA_ERR_ARG"),
    (dict(qk_nope=0), "MLA_ERR_ARG"), (dict(v_dim=-1), "MLA_ERR_ARG"),
])
def test_decode_rejects_bad_dims(mut, code):
    dims = v3(**mut)
    assert decode_raw(dims, ws_bytes=1 << 30) == B.CODES[code]


def test_decode_rejects_null_and_sizes():
    dims = v3()
    assert decode_raw(None) == B.CODES["MLA_ERR_ARG"]
    assert decode_raw(dims, ptrs=None) == B.CODES["MLA_ERR_ARG"]
    assert decode_raw(dims, seq=None) == B.CODES["MLA_ERR_ARG"]
    assert decode_raw(dims, status=None) == B.CODES["MLA_ERR_ARG"]
    assert decode_raw(dims, out=None) == B.CODES["MLA_ERR_ARG"]
    assert decode_raw(dims, max_len=101) == B.CODES["MLA_ERR_ARG"]          # > capacity
    assert decode_raw(dims, n_q=2, max_len=1, capacity=100, ws_bytes=1 << 30) == B.CODES["MLA_ERR_ARG"]
    assert decode_raw(dims, splits=-1, ws_bytes=1 << 30) == B.CODES["MLA_ERR_ARG"]
    assert decode_raw(dims, capacity=0, ws_bytes=1 << 30) == B.CODES["MLA_ERR_ARG"]
    assert decode_raw(dims, batch=-1, ws_bytes=1 << 30) == B.CODES["MLA_ERR_ARG"]


def test_decode_workspace_and_alignment():
    dims = v3()
    need = B.mla_decode_workspace_bytes(dims, 2, 1, 100)
    assert need > 0
    assert decode_raw(dims, ws_bytes=need - 1) == B.CODES["MLA_ERR_WORKSPACE"]
    assert decode_raw(dims, ws=FAKE + 16) == B.CODES["MLA_ERR_ALIGN"]


def test_decode_empty_work_is_a_noop():
    dims = v3()
    assert decode_raw(dims, batch=0, ptrs=None, seq=None, out=None, ws=None, status=None) == 0
    assert decode_raw(dims, n_q=0, ptrs=None, seq=None, out=None, ws=None, status=None) == 0


def test_workspace_layout_regions_are_disjoint_and_aligned():
    for dims, batch, n_q, max_len in ((v3(), 64, 1, 4096), (v3(), 32, 2, 4098), (v3(), 4, 1, 131072),
                                      (v3("fp32", heads=4, d_c=64, d_rope=16, qk_nope=32, v_dim=32), 2, 1, 100)):
        L = B.mla_decode_workspace_layout(dims, batch, n_q, max_len)
        regions = sorted((L[k], L[k + "_bytes"]) for k in ("q_lat", "o_lat", "part_o", "part_lse", "sched")
                         if L[k + "_bytes"])
        end = 0
        for off, n in regions:
            assert off % 256 == 0 and off >= end
            end = off + n
        assert end <= L["total"]
        assert B.mla_decode_workspace_bytes(dims, batch, n_q, max_len) == L["total"]
    assert B.mla_decode_workspace_bytes(v3(d_rope=3), 2, 1, 10) == 0


def test_append_argument_checks():
    L = B.lib()
    dims = v3()
    d = ctypes.byref(dims)
    ok = lambda **k: L.mla_append(d, k.get("batch", 2), k.get("n_new", 1), k.get("hidden", 7168),
                                  k.get("x", FAKE), k.get("W", FAKE), k.get("gamma", None),
                                  k.get("pos", FAKE), k.get("cache", FAKE), k.get("cap", 10),
                                  k.get("status", FAKE), None)
    # a gamma is accepted (latent RMSNorm); argument errors are still reported
    # before anything is launched
    assert ok(gamma=FAKE, cache=None) == B.CODES["MLA_ERR_ARG"]
    assert ok(cache=None) == B.CODES["MLA_ERR_ARG"]
    assert ok(pos=None) == B.CODES["MLA_ERR_ARG"]
    assert ok(status=None) == B.CODES["MLA_ERR_ARG"]
    assert ok(hidden=0) == B.CODES["MLA_ERR_ARG"]
    assert ok(cap=0) == B.CODES["MLA_ERR_ARG"]
    assert ok(batch=0, x=None, W=None, pos=None, cache=None, status=None) == 0
    assert ok(n_new=0, x=None, W=None, pos=None, cache=None, status=None) == 0


def test_rope_argument_checks():
    L = B.lib()
    dims = v3()
    assert L.mla_rope(ctypes.byref(dims), 4, FAKE, 63, FAKE, None) == B.CODES["MLA_ERR_ARG"]
    assert L.mla_rope(ctypes.byref(dims), 4, None, 576, FAKE, None) == B.CODES["MLA_ERR_ARG"]
    assert L.mla_rope(ctypes.byref(dims), 0, None, 576, None, None) == 0


def test_status_strings():
    for code, name in B.STATUS.items():
        assert B.mla_status_string(code) == name
    assert B.mla_status_string(99) == "MLA_ERR_UNKNOWN"
    assert B.lib().mla_get_status(None, None, None) == B.CODES["MLA_ERR_ARG"]


def test_sparse_decode_argument_checks():
    """mla_decode_sparse reports argument errors before anything is launched."""
    L = B.lib()

    def sparse(dims, max_sel=16, max_len=100, sel=FAKE, n_sel=FAKE, ws_bytes=None, capacity=100):
        d = ctypes.byref(dims)
        if ws_bytes is None:
            ws_bytes = L.mla_decode_workspace_bytes(d, 2, 1, max(1, min(max_sel, max_len)), 0)
        return L.mla_decode_sparse(d, 2, 1, FAKE, FAKE, FAKE, FAKE, FAKE, capacity, FAKE, max_len, sel, n_sel,
                                   max_sel, FAKE, FAKE, ws_bytes, 0, FAKE, None)

    assert sparse(v3(), sel=None) == B.CODES["MLA_ERR_ARG"]
    assert sparse(v3(), n_sel=None) == B.CODES["MLA_ERR_ARG"]
    assert sparse(v3(), max_sel=0) == B.CODES["MLA_ERR_ARG"]
    assert sparse(v3(), max_sel=101) == B.CODES["MLA_ERR_ARG"]            # > max_len
    assert sparse(v3(), ws_bytes=0) == B.CODES["MLA_ERR_WORKSPACE"]
    assert sparse(v3(dtype="fp32")) == B.CODES["MLA_ERR_UNSUPPORTED"]     # tensor-core path only
    assert sparse(v3(), capacity=1 << 30, max_len=100) == B.CODES["MLA_ERR_UNSUPPORTED"]   # batch*capacity > 2^31
    assert B.CODES["MLA_ERR_INDEX"] == 9 and B.STATUS[9] == "MLA_ERR_INDEX"


def test_output_projection_argument_checks():
    """mla_output_projection rejects bad sizes and pointers before any launch;
    zero tokens is a no-op that touches nothing."""
    L = B.lib()
    d = ctypes.byref(v3())
    P = FAKE
    assert L.mla_output_projection(d, -1, 7168, P, P, P, P, None) == B.CODES["MLA_ERR_ARG"]
    assert L.mla_output_projection(d, 4, 0, P, P, P, P, None) == B.CODES["MLA_ERR_ARG"]
    assert L.mla_output_projection(d, 0, 7168, None, None, None, None, None) == B.CODES["MLA_OK"]
    assert L.mla_output_projection(d, 4, 7168, None, P, P, P, None) == B.CODES["MLA_ERR_ARG"]
    assert L.mla_output_projection(d, 4, 7168, P, P, P, None, None) == B.CODES["MLA_ERR_ARG"]
    assert L.mla_output_projection(d, 4, 7168, P + 2, P, P, P, None) == B.CODES["MLA_ERR_ALIGN"]


def test_prefill_argument_checks():
    """mla_prefill reports argument errors before anything is launched."""
    L = B.lib()

    def pre(dims, batch=2, n_q=4, capacity=100, max_len=100, ws_bytes=None, ptr=FAKE, out=FAKE):
        d = ctypes.byref(dims)
        if ws_bytes is None:
            ws_bytes = L.mla_prefill_workspace_bytes(d, batch, n_q, max_len)
        return L.mla_prefill(d, batch, n_q, ptr, FAKE, FAKE, FAKE, FAKE, capacity, FAKE, max_len, out, FAKE,
                             ws_bytes, FAKE, None)

    assert pre(v3(), batch=0) == B.CODES["MLA_OK"]
    assert pre(v3(), n_q=0) == B.CODES["MLA_OK"]
    assert pre(v3(), max_len=3) == B.CODES["MLA_ERR_ARG"]           # < n_q
    assert pre(v3(), max_len=101) == B.CODES["MLA_ERR_ARG"]         # > capacity
    assert pre(v3(), ptr=None) == B.CODES["MLA_ERR_ARG"]
    assert pre(v3(dtype="fp32")) == B.CODES["MLA_ERR_UNSUPPORTED"]
    assert pre(v3(), ws_bytes=0) == B.CODES["MLA_ERR_WORKSPACE"]
    assert pre(v3(), out=FAKE + 2) == B.CODES["MLA_ERR_ALIGN"]
    assert pre(v3(), capacity=1 << 30, max_len=100) == B.CODES["MLA_ERR_UNSUPPORTED"]   # batch * capacity
    # the workspace covers the rotated queries and the expanded keys and values
    d = ctypes.byref(v3())
    need = L.mla_prefill_workspace_bytes(d, 2, 4, 100)
    assert need >= 2 * 4 * 128 * 64 * 2 + 2 * (2 * 100 * 128 * 128 * 2)


def test_header_is_c_and_links_from_c(tmp_path):
    """include/mla.h compiles as C99 and libmla.so links and answers from a C
    program (host-checkable calls only: sizes, argument errors, strings)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    lib_dir = os.path.dirname(B.LIB_PATH)
    exe = str(tmp_path / "abi_check")
    cmd = [gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "abi_check.c"), "-L", lib_dir, "-lmla", f"-Wl,-rpath,{lib_dir}", "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "FAIL" not in r.stdout and r.stdout.count("ok ") == 11, r.stdout
