"""ctypes binding of libmla (include/mla.h): argument marshalling only.

Each function carries the name of the C entry point it calls and takes torch
tensors for the buffers (their device pointers are passed through).  Every
step of the computation runs in the library's CUDA kernels; there is no
fallback.  If libmla.so is missing, loading raises immediately.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmla.so")

MLA_BF16, MLA_FP32 = 0, 1
STATUS = {0: "MLA_OK", 1: "MLA_ERR_ARG", 2: "MLA_ERR_ALIGN", 3: "MLA_ERR_WORKSPACE",
          4: "MLA_ERR_UNSUPPORTED", 5: "MLA_ERR_CUDA", 6: "MLA_ERR_LEN", 7: "MLA_ERR_POS",
          8: "MLA_ERR_TIMEOUT", 9: "MLA_ERR_INDEX"}
CODES = {v: k for k, v in STATUS.items()}


class MlaError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {STATUS.get(code, code)}")
        self.code = code


class MlaDims(ctypes.Structure):
    _fields_ = [("heads", ctypes.c_int32), ("d_c", ctypes.c_int32), ("d_rope", ctypes.c_int32),
                ("qk_nope", ctypes.c_int32), ("v_dim", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float), ("rope_base", ctypes.c_float)]


class MlaWsLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in (
        "total", "q_lat", "q_lat_bytes", "o_lat", "o_lat_bytes", "part_o", "part_o_bytes",
        "part_lse", "part_lse_bytes", "sched", "sched_bytes")] + [
        ("compute_dtype", ctypes.c_int32), ("splits", ctypes.c_int32)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libmla.so (built in-tree by mla_latent_kv_43_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libmla.so not built ({LIB_PATH}); run python -m mla_latent_kv_43_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        D = ctypes.POINTER(MlaDims)
        L.mla_decode_workspace_bytes.argtypes = [D, I32, I32, I64, I32]
        L.mla_decode_workspace_bytes.restype = SZ
        L.mla_decode_workspace_layout.argtypes = [D, I32, I32, I64, I32, ctypes.POINTER(MlaWsLayout)]
        L.mla_decode_workspace_layout.restype = ctypes.c_int
        L.mla_rope.argtypes = [D, I64, P, I64, P, P]
        L.mla_rope.restype = ctypes.c_int
        L.mla_append.argtypes = [D, I32, I32, I32, P, P, P, P, P, I64, P, P]
        L.mla_append.restype = ctypes.c_int
        L.mla_decode.argtypes = [D, I32, I32, P, P, P, P, P, I64, P, I64, P, P, SZ, I32, P, P]
        L.mla_decode.restype = ctypes.c_int
        L.mla_decode_sparse.argtypes = [D, I32, I32, P, P, P, P, P, I64, P, I64, P, P, I32, P, P, SZ, I32, P, P]
        L.mla_decode_sparse.restype = ctypes.c_int
        L.mla_prefill_workspace_bytes.argtypes = [D, I32, I32, I64]
        L.mla_prefill_workspace_bytes.restype = ctypes.c_size_t
        L.mla_prefill.argtypes = [D, I32, I32, P, P, P, P, P, I64, P, I64, P, P, ctypes.c_size_t, P, P]
        L.mla_prefill.restype = ctypes.c_int
        L.mla_output_projection.argtypes = [D, I32, I32, P, P, P, P, P]
        L.mla_output_projection.restype = ctypes.c_int
        L.mla_selftest_wait_timeout.argtypes = [P, I64, P]
        L.mla_selftest_wait_timeout.restype = ctypes.c_int
        L.mla_get_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_int32)]
        L.mla_get_status.restype = ctypes.c_int
        L.mla_status_string.argtypes = [ctypes.c_int]
        L.mla_status_string.restype = ctypes.c_char_p
        L.mla_last_launch_count.argtypes = []
        L.mla_last_launch_count.restype = ctypes.c_int32
        L.mla_decode_noalloc.argtypes = [D, I32, I32, P, P, P, P, P, I64, P, I64, P, I32, P, P]
        L.mla_decode_noalloc.restype = ctypes.c_int
        L.mla_profile_enable.argtypes = [ctypes.c_int]
        L.mla_profile_enable.restype = ctypes.c_int
        L.mla_profile_read.argtypes = [ctypes.c_char_p, SZ, ctypes.POINTER(ctypes.c_int32),
                                       ctypes.POINTER(ctypes.c_float), I32]
        L.mla_profile_read.restype = ctypes.c_int
        _lib = L
    return _lib


def make_dims(*, heads, d_c, d_rope, qk_nope, v_dim, dtype, softmax_scale=None,
              rope_base=10000.0) -> MlaDims:
    if softmax_scale is None:
        softmax_scale = (qk_nope + d_rope) ** -0.5
    dt = {"bf16": MLA_BF16, "fp32": MLA_FP32, torch.bfloat16: MLA_BF16, torch.float32: MLA_FP32}.get(dtype, dtype)
    return MlaDims(heads, d_c, d_rope, qk_nope, v_dim, dt, softmax_scale, rope_base)


def dims_of(w) -> MlaDims:
    """MlaDims for a generated workload (mla_latent_kv_43_b200.inputs.Workload)."""
    return make_dims(heads=w.heads, d_c=w.d_c, d_rope=w.d_rope, qk_nope=w.qk_nope, v_dim=w.v_dim,
                     dtype=w.dtype, softmax_scale=w.softmax_scale, rope_base=w.rope_base)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def _check(rc: int, where: str):
    if rc != 0:
        raise MlaError(rc, where)


def mla_decode_workspace_bytes(dims: MlaDims, batch: int, n_q: int, max_len: int, splits: int = 0) -> int:
    return lib().mla_decode_workspace_bytes(ctypes.byref(dims), batch, n_q, max_len, splits)


def mla_decode_workspace_layout(dims: MlaDims, batch: int, n_q: int, max_len: int, splits: int = 0) -> dict:
    L = MlaWsLayout()
    _check(lib().mla_decode_workspace_layout(ctypes.byref(dims), batch, n_q, max_len, splits,
                                             ctypes.byref(L)), "mla_decode_workspace_layout")
    return {n: getattr(L, n) for n, _ in MlaWsLayout._fields_}


def mla_rope(dims: MlaDims, n_rows: int, x: torch.Tensor, row_stride: int,
             positions: torch.Tensor, stream=None, offset_elems: int = 0):
    """Rotate d_rope elements of each row, starting ``offset_elems`` into x."""
    ptr = x.data_ptr() + offset_elems * x.element_size()
    _check(lib().mla_rope(ctypes.byref(dims), n_rows, ptr, row_stride, _ptr(positions),
                          _stream(stream)), "mla_rope")


def mla_append(dims: MlaDims, x: torch.Tensor, W_dkv: torch.Tensor, positions: torch.Tensor,
               cache: torch.Tensor, status: torch.Tensor, *, batch: int, n_new: int,
               rms_gamma: Optional[torch.Tensor] = None, stream=None):
    hidden = x.shape[-1]
    _check(lib().mla_append(ctypes.byref(dims), batch, n_new, hidden, _ptr(x), _ptr(W_dkv),
                            _ptr(rms_gamma), _ptr(positions), _ptr(cache), cache.shape[1],
                            _ptr(status), _stream(stream)), "mla_append")


def mla_decode(dims: MlaDims, q_nope: torch.Tensor, q_rope: torch.Tensor, W_uk: torch.Tensor,
               W_uv: torch.Tensor, cache: torch.Tensor, seq_lens: torch.Tensor, max_len: int,
               out: torch.Tensor, workspace: torch.Tensor, status: torch.Tensor, splits: int = 0,
               stream=None):
    batch, n_q = q_nope.shape[0], q_nope.shape[1]
    _check(lib().mla_decode(ctypes.byref(dims), batch, n_q, _ptr(q_nope), _ptr(q_rope), _ptr(W_uk),
                            _ptr(W_uv), _ptr(cache), cache.shape[1], _ptr(seq_lens), max_len,
                            _ptr(out), _ptr(workspace), workspace.numel() * workspace.element_size(),
                            splits, _ptr(status), _stream(stream)), "mla_decode")


def mla_decode_sparse(dims: MlaDims, q_nope: torch.Tensor, q_rope: torch.Tensor, W_uk: torch.Tensor,
                      W_uv: torch.Tensor, cache: torch.Tensor, seq_lens: torch.Tensor, max_len: int,
                      sel: torch.Tensor, n_sel: torch.Tensor, out: torch.Tensor, workspace: torch.Tensor,
                      status: torch.Tensor, splits: int = 0, stream=None):
    """Decode over the selected cache slots sel[b][j][:n_sel[b][j]] of each query."""
    batch, n_q = q_nope.shape[0], q_nope.shape[1]
    _check(lib().mla_decode_sparse(ctypes.byref(dims), batch, n_q, _ptr(q_nope), _ptr(q_rope), _ptr(W_uk),
                                   _ptr(W_uv), _ptr(cache), cache.shape[1], _ptr(seq_lens), max_len,
                                   _ptr(sel), _ptr(n_sel), sel.shape[-1], _ptr(out), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), splits, _ptr(status),
                                   _stream(stream)), "mla_decode_sparse")


def mla_prefill_workspace_bytes(dims: MlaDims, batch: int, n_q: int, max_len: int) -> int:
    return lib().mla_prefill_workspace_bytes(ctypes.byref(dims), batch, n_q, max_len)


def mla_prefill(dims: MlaDims, q_nope: torch.Tensor, q_rope: torch.Tensor, W_uk: torch.Tensor,
                W_uv: torch.Tensor, cache: torch.Tensor, seq_lens: torch.Tensor, max_len: int,
                out: torch.Tensor, workspace: torch.Tensor, status: torch.Tensor, stream=None):
    """The decode's attention in the materialised factorisation (many query tokens)."""
    batch, n_q = q_nope.shape[0], q_nope.shape[1]
    _check(lib().mla_prefill(ctypes.byref(dims), batch, n_q, _ptr(q_nope), _ptr(q_rope), _ptr(W_uk), _ptr(W_uv),
                             _ptr(cache), cache.shape[1], _ptr(seq_lens), max_len, _ptr(out), _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _ptr(status), _stream(stream)),
           "mla_prefill")


def mla_output_projection(dims: MlaDims, out: torch.Tensor, W_O: torch.Tensor, y: torch.Tensor,
                          status: torch.Tensor, stream=None):
    """y [tokens][hidden] = heads of out [..][H][v_dim] concatenated, times W_O."""
    tokens = out.numel() // (dims.heads * dims.v_dim)
    _check(lib().mla_output_projection(ctypes.byref(dims), tokens, y.shape[-1], _ptr(out), _ptr(W_O), _ptr(y),
                                       _ptr(status), _stream(stream)), "mla_output_projection")


def mla_selftest_wait_timeout(status: torch.Tensor, limit_ns: int, stream=None):
    """Run the library's bounded wait on a barrier nothing arrives on."""
    _check(lib().mla_selftest_wait_timeout(_ptr(status), limit_ns, _stream(stream)), "mla_selftest_wait_timeout")


def mla_decode_noalloc(dims: MlaDims, q_nope: torch.Tensor, q_rope: torch.Tensor, W_uk: torch.Tensor,
                       W_uv: torch.Tensor, cache: torch.Tensor, seq_lens: torch.Tensor, max_len: int,
                       out: torch.Tensor, status: torch.Tensor, splits: int, stream=None):
    """mla_decode with the library's fixed scratch area instead of a workspace."""
    batch, n_q = q_nope.shape[0], q_nope.shape[1]
    _check(lib().mla_decode_noalloc(ctypes.byref(dims), batch, n_q, _ptr(q_nope), _ptr(q_rope), _ptr(W_uk),
                                    _ptr(W_uv), _ptr(cache), cache.shape[1], _ptr(seq_lens), max_len,
                                    _ptr(out), splits, _ptr(status), _stream(stream)), "mla_decode_noalloc")


NOALLOC_SCRATCH_BYTES = 16 << 20


def mla_get_status(status: torch.Tensor, stream=None) -> int:
    v = ctypes.c_int32(-1)
    _check(lib().mla_get_status(_ptr(status), _stream(stream), ctypes.byref(v)), "mla_get_status")
    return v.value


def mla_status_string(code: int) -> str:
    return lib().mla_status_string(code).decode()


def mla_last_launch_count() -> int:
    return lib().mla_last_launch_count()


def mla_profile_enable(on: bool):
    _check(lib().mla_profile_enable(1 if on else 0), "mla_profile_enable")


def mla_profile_read(max_kernels: int = 32) -> dict:
    """{kernel name: (launches, total ms)} since the previous read (waits for the events)."""
    buf = ctypes.create_string_buffer(4096)
    counts = (ctypes.c_int32 * max_kernels)()
    ms = (ctypes.c_float * max_kernels)()
    n = lib().mla_profile_read(buf, len(buf), counts, ms, max_kernels)
    if n < 0:
        raise MlaError(-n, "mla_profile_read")
    names = buf.raw.split(b"\0")[:n]
    return {nm.decode(): (counts[i], ms[i]) for i, nm in enumerate(names)}
