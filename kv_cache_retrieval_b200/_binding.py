"""ctypes binding of libhhr.so: argument marshalling only.

Each function has the name and argument order of its C counterpart in
``include/hhr.h``.  Tensor arguments may be torch tensors (their data pointer
is passed), plain integers (raw device addresses) or None (NULL).  ``stream``
defaults to torch's current CUDA stream.  A non-zero status raises HhrError.
Every computation runs in the CUDA library; nothing here has a fallback.
"""
from __future__ import annotations

import ctypes as C
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libhhr.so")

HHR_OK = 0
HHR_ERR_INVALID_ARG = 1
HHR_ERR_UNSUPPORTED = 2
HHR_ERR_WORKSPACE = 3
HHR_ERR_CUDA = 4
HHR_ERR_TIMEOUT = 5
HHR_MAX_PAGES = 16384
HHR_NOALLOC_SCRATCH_BYTES = 4 << 20


class HhrError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_string(status)} (status {status})")
        self.status = status


HHR_FLAG_META_F32 = 1   # page metadata in float32 (unrounded extrema)
HHR_FLAG_GQA_SUM = 2    # token distance = sum over the group's heads
HHR_FLAG_SIMT_BOUNDS = 4  # Eq. 3 on the CUDA cores (comparison form of the tensor-core tiles)


class hhr_dims(C.Structure):
    _fields_ = [("B", C.c_int32), ("Hq", C.c_int32), ("Hkv", C.c_int32), ("d", C.c_int32),
                ("bits", C.c_int32), ("page", C.c_int32), ("n_cap", C.c_int32),
                ("flags", C.c_int32)]

    def __repr__(self):
        return "hhr_dims(" + ", ".join(f"{n}={getattr(self, n)}" for n, _ in self._fields_) + ")"


def make_dims(B, Hq, Hkv, d, bits, page, n_cap, flags=0) -> hhr_dims:
    return hhr_dims(B, Hq, Hkv, d, bits, page, n_cap, flags)


_lib = None

_P = C.c_void_p
_I32 = C.c_int32
_SIGS = {
    "hhr_version": (_I32, []),
    "hhr_status_string": (C.c_char_p, [_I32]),
    "hhr_encode_keys": (_I32, [C.POINTER(hhr_dims), _P, _P, _P, _I32, _I32, _P, _P, _P]),
    "hhr_workspace_size": (C.c_size_t, [C.POINTER(hhr_dims), _I32, _I32]),
    "hhr_select": (_I32, [C.POINTER(hhr_dims), _P, _P, _P, _P, _P, _I32, _I32, _I32, _P, _P, _P,
                          _P, _P, _P, C.c_size_t, _P]),
    "hhr_sparse_attend": (_I32, [C.POINTER(hhr_dims), _P, _P, _P, _P, _P, _I32, C.c_float, _P, _P,
                                 C.c_size_t, _P]),
    "hhr_dense_attend": (_I32, [C.POINTER(hhr_dims), _P, _P, _P, _I32, C.c_float, _P, _P, C.c_size_t,
                                _P]),
    "hhr_decode_step": (_I32, [C.POINTER(hhr_dims), _P, _P, _P, _P, _P, _P, _P, _I32, _I32, _I32,
                               C.c_float, _P, _P, _P, _P, _P, C.c_size_t, _P]),
    "hhr_decode_step_host": (_I32, [C.POINTER(hhr_dims), _P, _P, _P, _P, _P, _P, _P, _P, _I32, _I32,
                                    _I32, C.c_float, _P, _P, _P, _P, _P, _P, C.c_size_t, _P]),
    "hhr_decode_step_noalloc": (_I32, [C.POINTER(hhr_dims), _P, _P, _P, _P, _P, _P, _P, _I32, _I32,
                                       _I32, C.c_float, _P, _P, _P, _P, _P]),
    "hhr_read_status": (_I32, [_P, _P]),
    "hhr_noalloc_read_status": (_I32, [_P]),
    "hhr_encode_status": (_I32, [_P]),
    "hhr_test_arm_timeout": (_I32, [_I32, C.c_uint64]),
}


def lib() -> C.CDLL:
    """Load libhhr.so from the package directory (no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m kv_cache_retrieval_b200.build`")
        L = C.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def exported_symbols() -> list[str]:
    return list(_SIGS)


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(status: int, where: str) -> None:
    if status != HHR_OK:
        raise HhrError(status, where)


def _nbytes(t):
    return t.numel() * t.element_size()


def status_string(status: int) -> str:
    return lib().hhr_status_string(status).decode()


def hhr_version() -> int:
    return lib().hhr_version()


def hhr_status_string(status: int) -> str:
    return status_string(status)


def hhr_encode_keys(dims, K, R, W, n_begin, n_end, codes, meta, stream=None) -> None:
    _check(lib().hhr_encode_keys(C.byref(dims), _ptr(K), _ptr(R), _ptr(W), n_begin, n_end,
                                 _ptr(codes), _ptr(meta), _stream(stream)), "hhr_encode_keys")


def hhr_workspace_size(dims, P, k) -> int:
    return lib().hhr_workspace_size(C.byref(dims), P, k)


def hhr_select(dims, q, R, W, codes, meta, n_valid, P, k, page_idx, tok_idx, n_sel,
               dbg_U=None, dbg_D=None, workspace=None, ws_bytes=None, stream=None) -> None:
    ws_bytes = _nbytes(workspace) if ws_bytes is None and workspace is not None else (ws_bytes or 0)
    _check(lib().hhr_select(C.byref(dims), _ptr(q), _ptr(R), _ptr(W), _ptr(codes), _ptr(meta),
                            n_valid, P, k, _ptr(page_idx), _ptr(tok_idx), _ptr(n_sel),
                            _ptr(dbg_U), _ptr(dbg_D), _ptr(workspace), ws_bytes, _stream(stream)),
           "hhr_select")


def hhr_sparse_attend(dims, q, K, V, tok_idx, n_sel, k, scale, out, workspace=None,
                      ws_bytes=None, stream=None) -> None:
    ws_bytes = _nbytes(workspace) if ws_bytes is None and workspace is not None else (ws_bytes or 0)
    _check(lib().hhr_sparse_attend(C.byref(dims), _ptr(q), _ptr(K), _ptr(V), _ptr(tok_idx),
                                   _ptr(n_sel), k, scale, _ptr(out), _ptr(workspace), ws_bytes,
                                   _stream(stream)), "hhr_sparse_attend")


def hhr_dense_attend(dims, q, K, V, n_valid, scale, out, workspace=None, ws_bytes=None,
                     stream=None) -> None:
    ws_bytes = _nbytes(workspace) if ws_bytes is None and workspace is not None else (ws_bytes or 0)
    _check(lib().hhr_dense_attend(C.byref(dims), _ptr(q), _ptr(K), _ptr(V), n_valid, scale, _ptr(out),
                                  _ptr(workspace), ws_bytes, _stream(stream)), "hhr_dense_attend")


def hhr_decode_step(dims, q, R, W, codes, meta, K, V, n_valid, P, k, scale, page_idx, tok_idx,
                    n_sel, out, workspace=None, ws_bytes=None, stream=None) -> None:
    ws_bytes = _nbytes(workspace) if ws_bytes is None and workspace is not None else (ws_bytes or 0)
    _check(lib().hhr_decode_step(C.byref(dims), _ptr(q), _ptr(R), _ptr(W), _ptr(codes),
                                 _ptr(meta), _ptr(K), _ptr(V), n_valid, P, k, scale,
                                 _ptr(page_idx), _ptr(tok_idx), _ptr(n_sel), _ptr(out),
                                 _ptr(workspace), ws_bytes, _stream(stream)), "hhr_decode_step")


def hhr_decode_step_host(dims, q_host, q, R, W, codes, meta, K, V, n_valid, P, k, scale, page_idx,
                         tok_idx, n_sel, out, out_host, workspace=None, ws_bytes=None,
                         stream=None) -> None:
    """hhr_decode_step with the query and output in (pinned) host memory; blocks."""
    ws_bytes = _nbytes(workspace) if ws_bytes is None and workspace is not None else (ws_bytes or 0)
    _check(lib().hhr_decode_step_host(C.byref(dims), _ptr(q_host), _ptr(q), _ptr(R), _ptr(W),
                                      _ptr(codes), _ptr(meta), _ptr(K), _ptr(V), n_valid, P, k, scale,
                                      _ptr(page_idx), _ptr(tok_idx), _ptr(n_sel), _ptr(out),
                                      _ptr(out_host), _ptr(workspace), ws_bytes, _stream(stream)),
           "hhr_decode_step_host")


def prepare(name, *args):
    """A call of C function `name` with its arguments marshalled once (tensors
    by data pointer, as above): returns a function that makes the call again
    and raises HhrError on a non-zero status.  For repeated calls on the same
    buffers (a decode loop), where per-call marshalling would dominate."""
    fn = getattr(lib(), name)
    conv = []
    for a, t in zip(args, fn.argtypes):
        if isinstance(a, hhr_dims):
            conv.append(C.byref(a))
        elif t is _P:
            conv.append(C.c_void_p(_ptr(a)))
        else:
            conv.append(t(a))
    conv = tuple(conv)

    def call():
        st = fn(*conv)
        if st != HHR_OK:
            raise HhrError(st, name)
    return call


def hhr_decode_step_noalloc(dims, q, R, W, codes, meta, K, V, n_valid, P, k, scale, page_idx,
                            tok_idx, n_sel, out, stream=None) -> None:
    """hhr_decode_step with the library's built-in scratch (no workspace)."""
    _check(lib().hhr_decode_step_noalloc(C.byref(dims), _ptr(q), _ptr(R), _ptr(W), _ptr(codes),
                                         _ptr(meta), _ptr(K), _ptr(V), n_valid, P, k, scale,
                                         _ptr(page_idx), _ptr(tok_idx), _ptr(n_sel), _ptr(out),
                                         _stream(stream)), "hhr_decode_step_noalloc")


def hhr_read_status(workspace, stream=None) -> int:
    """Device status word of a workspace (HHR_OK or HHR_ERR_TIMEOUT), cleared after reading."""
    st = lib().hhr_read_status(_ptr(workspace), _stream(stream))
    if st == HHR_ERR_CUDA:
        raise HhrError(st, "hhr_read_status")
    return st


def hhr_noalloc_read_status(stream=None) -> int:
    """Status word of hhr_decode_step_noalloc's built-in scratch, cleared after reading."""
    st = lib().hhr_noalloc_read_status(_stream(stream))
    if st == HHR_ERR_CUDA:
        raise HhrError(st, "hhr_noalloc_read_status")
    return st


def hhr_encode_status(stream=None) -> int:
    """Sticky status of the key-encoding kernels (HHR_OK or HHR_ERR_TIMEOUT), cleared after reading."""
    st = lib().hhr_encode_status(_stream(stream))
    if st == HHR_ERR_CUDA:
        raise HhrError(st, "hhr_encode_status")
    return st


def hhr_test_arm_timeout(where, spin_cycles) -> None:
    """Test hook: the next matching call's bounded waits run out (see hhr.h)."""
    _check(lib().hhr_test_arm_timeout(where, spin_cycles), "hhr_test_arm_timeout")
