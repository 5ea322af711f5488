"""CPU checks of the C ABI: the library loads, exports every function the
header declares, and rejects bad arguments on the host before touching CUDA."""
import ctypes as C
import os
import re

import pytest
import torch

import kv_cache_retrieval_b200 as hhr
from kv_cache_retrieval_b200 import _binding as Bnd
from kv_cache_retrieval_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hhr.h")


@pytest.fixture(scope="module", autouse=True)
def built():
    kbuild.build()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^[A-Za-z_][\w \*]*?\b(hhr_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_expected_calls():
    names = declared_functions()
    for want in ["hhr_encode_keys", "hhr_select", "hhr_sparse_attend", "hhr_decode_step",
                 "hhr_workspace_size", "hhr_read_status", "hhr_status_string", "hhr_version"]:
        assert want in names


def test_library_exports_every_declared_function():
    L = C.CDLL(Bnd.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(L, n)]
    assert not missing, missing
    assert set(declared_functions()) == set(Bnd.exported_symbols())


def test_status_strings_and_version():
    assert hhr.hhr_version() >= 100
    assert hhr.hhr_status_string(hhr.HHR_OK) == "ok"
    for st in range(1, 6):
        assert hhr.hhr_status_string(st) not in ("ok", "unknown status")
    assert hhr.hhr_status_string(99) == "unknown status"


def _dims(**kw):
    base = dict(B=1, Hq=32, Hkv=8, d=128, bits=128, page=16, n_cap=4096)
    base.update(kw)
    return hhr.make_dims(**base)


FAKE = 1 << 20  # a 256-byte aligned non-null address; never dereferenced on the host


@pytest.mark.parametrize("kw,status", [
    (dict(d=64), hhr.HHR_ERR_UNSUPPORTED),
    (dict(bits=64), hhr.HHR_ERR_UNSUPPORTED),
    (dict(bits=160), hhr.HHR_ERR_UNSUPPORTED),
    (dict(page=3), hhr.HHR_ERR_UNSUPPORTED),
    (dict(page=128), hhr.HHR_ERR_UNSUPPORTED),
    (dict(Hq=24, Hkv=8), hhr.HHR_ERR_UNSUPPORTED),   # group of 3
    (dict(Hq=30, Hkv=8), hhr.HHR_ERR_INVALID_ARG),   # not a multiple
    (dict(B=0), hhr.HHR_ERR_INVALID_ARG),
    (dict(n_cap=0), hhr.HHR_ERR_INVALID_ARG),
])
def test_bad_dims_are_rejected(kw, status):
    d = _dims(**kw)
    st = hhr.lib().hhr_encode_keys(C.byref(d), FAKE, FAKE, FAKE, 0, 1, FAKE, FAKE, None)
    assert st == status
    assert hhr.hhr_workspace_size(d, 4, 4) == 0


def test_null_dims_rejected():
    assert hhr.lib().hhr_encode_keys(None, FAKE, FAKE, FAKE, 0, 1, FAKE, FAKE, None) == hhr.HHR_ERR_INVALID_ARG


@pytest.mark.parametrize("nb,ne", [(-1, 4), (5, 4), (0, 4097)])
def test_encode_rejects_bad_ranges(nb, ne):
    d = _dims()
    assert hhr.lib().hhr_encode_keys(C.byref(d), FAKE, FAKE, FAKE, nb, ne, FAKE, FAKE, None) == hhr.HHR_ERR_INVALID_ARG


def test_encode_rejects_null_and_misaligned():
    d = _dims()
    L = hhr.lib()
    assert L.hhr_encode_keys(C.byref(d), None, FAKE, FAKE, 0, 1, FAKE, FAKE, None) == hhr.HHR_ERR_INVALID_ARG
    assert L.hhr_encode_keys(C.byref(d), FAKE + 2, FAKE, FAKE, 0, 1, FAKE, FAKE, None) == hhr.HHR_ERR_INVALID_ARG
    # an empty range is a no-op that succeeds without a device
    assert L.hhr_encode_keys(C.byref(d), FAKE, FAKE, FAKE, 7, 7, FAKE, FAKE, None) == hhr.HHR_OK


def test_workspace_size_grows_with_the_problem():
    a = hhr.hhr_workspace_size(_dims(), 32, 128)
    b = hhr.hhr_workspace_size(_dims(n_cap=131072), 32, 128)
    c = hhr.hhr_workspace_size(_dims(B=4, n_cap=131072), 32, 128)
    assert 0 < a < b < c
    assert a % 256 == 0


def _select(d, ws_bytes=1 << 30, ws=FAKE, P=8, k=16, n_valid=100, codes=FAKE):
    return hhr.lib().hhr_select(C.byref(d), FAKE, FAKE, FAKE, codes, FAKE, n_valid, P, k, FAKE, FAKE,
                                FAKE, None, None, ws, ws_bytes, None)


def test_select_validation_happens_on_the_host():
    d = _dims()
    assert _select(d, P=0) == hhr.HHR_ERR_INVALID_ARG
    assert _select(d, k=0) == hhr.HHR_ERR_INVALID_ARG
    assert _select(d, n_valid=-1) == hhr.HHR_ERR_INVALID_ARG
    assert _select(d, n_valid=4097) == hhr.HHR_ERR_INVALID_ARG
    assert _select(d, codes=FAKE + 4) == hhr.HHR_ERR_INVALID_ARG
    assert _select(d, ws=None) == hhr.HHR_ERR_WORKSPACE
    assert _select(d, ws=FAKE + 16) == hhr.HHR_ERR_WORKSPACE
    assert _select(d, ws_bytes=hhr.hhr_workspace_size(d, 8, 16) - 1) == hhr.HHR_ERR_WORKSPACE
    big = _dims(n_cap=16 * (hhr.HHR_MAX_PAGES + 1))
    assert _select(big) == hhr.HHR_ERR_UNSUPPORTED


def test_attend_and_step_validation():
    d = _dims()
    L = hhr.lib()
    assert L.hhr_sparse_attend(C.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, 16, C.c_float(float("nan")),
                               FAKE, FAKE, 1 << 30, None) == hhr.HHR_ERR_INVALID_ARG
    assert L.hhr_sparse_attend(C.byref(d), FAKE, FAKE, FAKE, None, FAKE, 16, 0.1, FAKE, FAKE,
                               1 << 30, None) == hhr.HHR_ERR_INVALID_ARG
    assert L.hhr_decode_step(C.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, 10, 4, 4, 0.1,
                             FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == hhr.HHR_ERR_INVALID_ARG


def test_python_binding_raises_on_error_status():
    d = _dims(d=64)
    with pytest.raises(hhr.HhrError) as e:
        hhr.hhr_encode_keys(d, FAKE, FAKE, FAKE, 0, 1, FAKE, FAKE, stream=0)
    assert e.value.status == hhr.HHR_ERR_UNSUPPORTED


def test_dense_attend_validation():
    d = _dims()
    L = hhr.lib()
    ws = 1 << 30
    assert L.hhr_dense_attend(C.byref(d), FAKE, FAKE, FAKE, 4097, C.c_float(0.1), FAKE, FAKE, ws,
                              None) == hhr.HHR_ERR_INVALID_ARG
    assert L.hhr_dense_attend(C.byref(d), FAKE, FAKE, FAKE, -1, C.c_float(0.1), FAKE, FAKE, ws,
                              None) == hhr.HHR_ERR_INVALID_ARG
    assert L.hhr_dense_attend(C.byref(d), FAKE, FAKE, FAKE, 10, C.c_float(float("inf")), FAKE, FAKE,
                              ws, None) == hhr.HHR_ERR_INVALID_ARG
    assert L.hhr_dense_attend(C.byref(d), FAKE, FAKE, FAKE, 10, C.c_float(0.1), None, FAKE, ws,
                              None) == hhr.HHR_ERR_INVALID_ARG
    assert L.hhr_dense_attend(C.byref(d), FAKE, FAKE, FAKE, 10, C.c_float(0.1), FAKE, None, ws,
                              None) == hhr.HHR_ERR_WORKSPACE


def test_variant_flags_validation():
    assert _select(_dims(flags=8)) == hhr.HHR_ERR_INVALID_ARG
    assert _select(_dims(flags=-1)) == hhr.HHR_ERR_INVALID_ARG
    plain, summed = _dims(), _dims(flags=hhr.HHR_FLAG_GQA_SUM)
    assert hhr.hhr_workspace_size(summed, 64, 256) > hhr.hhr_workspace_size(plain, 64, 256)
    assert hhr.hhr_workspace_size(_dims(flags=16), 64, 256) == 0


def test_cache_buffers_follow_the_flags():
    """HHRCache sizes its buffers from the dims (host-side, no kernel runs)."""
    base = dict(batch=1, q_heads=8, kv_heads=2, capacity=512, P=8, k=32, device="cpu")
    c0 = hhr.HHRCache(**base)
    c1 = hhr.HHRCache(**base, flags=hhr.HHR_FLAG_META_F32 | hhr.HHR_FLAG_GQA_SUM)
    assert c0.meta.dtype == torch.bfloat16 and c1.meta.dtype == torch.float32
    assert c1.meta.shape == c0.meta.shape == (1, 2, 32, 2, 128)
    assert c1.workspace.numel() > c0.workspace.numel()   # wider distance histograms
    assert c1.dims.flags == hhr.HHR_FLAG_META_F32 | hhr.HHR_FLAG_GQA_SUM
