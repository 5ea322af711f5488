"""ctypes wrapper of the CPU oracle (TEST INFRASTRUCTURE ONLY).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference arm may import this module.  The CUDA library and its Python binding
never do.

All arrays are numpy; bf16 data is passed as uint16 bit patterns.  The per-unit
functions follow "HHR: Hierarchical Hash Retrieval for Efficient LLM
Generation" (arXiv 2610.01230) as cited in ``hhr_oracle.cpp``.  The whole-
workload helpers loop over (sequence, KV head) units; units are independent,
so they may run on a thread pool (each oracle call itself is single-threaded,
and ctypes releases the GIL during the call).
"""
from __future__ import annotations

import ctypes as C
import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = os.environ.get("HHR_ORACLE_LIB") or _build.build()
        L = C.CDLL(path)
        p = C.c_void_p
        i32, i64, f64 = C.c_int32, C.c_int64, C.c_double
        sig = {
            "hhro_rotate": (None, [p, i64, i32, p, p]),
            "hhro_project_sign": (i64, [p, i64, i32, i32, p, p, p]),
            "hhro_page_meta": (None, [p, i64, i64, i32, i32, i64, i64, p]),
            "hhro_encode_unit": (i64, [p, i64, i64, i32, i32, i32, p, p, p, p]),
            "hhro_query_prep": (i64, [p, i32, i32, i32, p, p, p, p]),
            "hhro_page_bounds": (None, [p, i32, i32, p, i64, p, p]),
            "hhro_top_largest": (i64, [p, i64, i64, p]),
            "hhro_hamming": (None, [p, i32, i32, p, p, i64, i32, i64, p]),
            "hhro_top_tokens": (i64, [p, p, i64, i32, i64, p]),
            "hhro_attend": (None, [p, i32, i32, p, p, p, i64, f64, p]),
            "hhro_decode_unit": (i64, [p, i32, i32, i32, i32, p, p, p, p, p, p,
                                       i64, i64, i64, f64, p, p, p, p, p, p]),
            "hhro_page_meta_f32": (None, [p, i64, i64, i32, i32, i64, i64, p]),
            "hhro_top_logits": (i64, [p, i32, i32, p, i64, i64, p]),
            "hhro_encode_unit_f32": (i64, [p, i64, i64, i32, i32, i32, p, p, p, p]),
            "hhro_page_bounds_f32": (None, [p, i32, i32, p, i64, p, p]),
            "hhro_hamming_agg": (None, [p, i32, i32, p, p, i64, i32, i64, i32, p]),
            "hhro_decode_unit_v": (i64, [p, i32, i32, i32, i32, p, p, p, p, p, p,
                                         i64, i64, i64, f64, i32, p, p, p, p, p, p]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a


# ---------------------------------------------------------------- primitives

def rotate(x_bits, R):
    """§3.3.1 Eq. 4: float32(x R) with x given as bf16 bits [n][d]."""
    x = _c(x_bits, np.uint16)
    R = _c(R, np.float32)
    n, d = x.shape
    out = np.empty((n, d), np.float32)
    lib().hhro_rotate(_p(x), n, d, _p(R), _p(out))
    return out


def project_sign(x_bits, W, want_z=False):
    """§3.3.2 Eq. 10 + sign: packed codes [n][bits/32], ambiguous count (, z)."""
    x = _c(x_bits, np.uint16)
    W = _c(W, np.float32)
    n, d = x.shape
    bits = W.shape[1]
    codes = np.empty((n, bits // 32), np.uint32)
    z = np.empty((n, bits), np.float64) if want_z else None
    amb = lib().hhro_project_sign(_p(x), n, d, bits, _p(W), _p(codes), _p(z))
    return (codes, amb, z) if want_z else (codes, amb)


def page_meta(kt, n_valid, page, p_begin=0, p_end=None, t0=0, meta=None, f32=False):
    """Extrema of §3.3.1 (Eq. 3): rounded outward to bf16, [np][2][d] uint16;
    with ``f32`` (variant V1) kept as float32, [np][2][d] float32."""
    kt = _c(kt, np.float32)
    d = kt.shape[1]
    if p_end is None:
        p_end = (n_valid + page - 1) // page
    if meta is None:
        meta = np.zeros((p_end, 2, d), np.float32 if f32 else np.uint16)
    fn = lib().hhro_page_meta_f32 if meta.dtype == np.float32 else lib().hhro_page_meta
    fn(_p(kt), t0, n_valid, d, page, p_begin, p_end, _p(meta))
    return meta


def encode_unit(K_unit, n_begin, n_end, page, R_g, W_g, codes_unit, meta_unit):
    """Encode keys [n_begin, n_end) of one unit in place; returns ambiguous count.
    A float32 ``meta_unit`` selects the float32-metadata variant (V1)."""
    assert K_unit.flags.c_contiguous and codes_unit.flags.c_contiguous and meta_unit.flags.c_contiguous
    d = K_unit.shape[1]
    bits = W_g.shape[1]
    fn = lib().hhro_encode_unit_f32 if meta_unit.dtype == np.float32 else lib().hhro_encode_unit
    return fn(_p(K_unit), n_begin, n_end, d, bits, page, _p(_c(R_g, np.float32)),
              _p(_c(W_g, np.float32)), _p(codes_unit), _p(meta_unit))


def query_prep(q_bits, R_g, W_g):
    """q~ = q R (float32 [r][d]), query codes [r][bits/32], ambiguous count."""
    q = _c(q_bits, np.uint16)
    r, d = q.shape
    bits = W_g.shape[1]
    qt = np.empty((r, d), np.float32)
    qc = np.empty((r, bits // 32), np.uint32)
    amb = lib().hhro_query_prep(_p(q), r, d, bits, _p(_c(R_g, np.float32)),
                                _p(_c(W_g, np.float32)), _p(qt), _p(qc))
    return qt, qc, amb


def page_bounds(qt, meta_unit, n_pages, per_head=False):
    """§3.3.1 Eq. 3, max over the group's heads: U [np] float64 (, Uh [r][np]).
    bf16 (uint16) or float32 (variant V1) metadata."""
    qt = _c(qt, np.float32)
    f32 = np.asarray(meta_unit).dtype == np.float32
    meta = _c(meta_unit, np.float32 if f32 else np.uint16)
    r, d = qt.shape
    U = np.empty(n_pages, np.float64)
    Uh = np.empty((r, n_pages), np.float64) if per_head else None
    fn = lib().hhro_page_bounds_f32 if f32 else lib().hhro_page_bounds
    fn(_p(qt), r, d, _p(meta), n_pages, _p(U), _p(Uh))
    return (U, Uh) if per_head else U


def top_largest(s, m):
    s = _c(s, np.float64)
    out = np.empty(min(m, s.shape[0]), np.int32)
    cnt = lib().hhro_top_largest(_p(s), s.shape[0], m, _p(out))
    return out[:cnt]


def hamming(qcode, codes_unit, pages, page, n_valid, gqa_sum=False):
    """§3.1 Eq. 2 over the group's heads: min (reading R4) or sum (variant V2)."""
    qc = _c(qcode, np.uint32)
    codes = _c(codes_unit, np.uint32)
    pages = _c(pages, np.int32)
    r, words = qc.shape
    D = np.empty(pages.shape[0] * page, np.int32)
    lib().hhro_hamming_agg(_p(qc), r, words, _p(codes), _p(pages), pages.shape[0], page, n_valid,
                           1 if gqa_sum else 0, _p(D))
    return D


def top_tokens(D, pages, page, k):
    D = _c(D, np.int32)
    pages = _c(pages, np.int32)
    out = np.empty(k, np.int32)
    cnt = lib().hhro_top_tokens(_p(D), _p(pages), pages.shape[0], page, k, _p(out))
    return out[:cnt]


def top_logits(q_bits, K_unit, n_valid, m):
    """Diagnostic reference: the m keys of [0, n_valid) with the largest exact
    group logit max_h q_h . k_n, ties to the lower index, ascending."""
    q = _c(q_bits, np.uint16)
    r, d = q.shape
    out = np.empty(min(m, n_valid), np.int32)
    cnt = lib().hhro_top_logits(_p(q), r, d, _p(_c(K_unit, np.uint16)), n_valid, m, _p(out))
    return out[:cnt]


def attend(q_bits, K_unit, V_unit, idx, scale):
    q = _c(q_bits, np.uint16)
    r, d = q.shape
    idx = _c(idx, np.int32)
    out = np.empty((r, d), np.float32)
    lib().hhro_attend(_p(q), r, d, _p(_c(K_unit, np.uint16)), _p(_c(V_unit, np.uint16)),
                      _p(idx), idx.shape[0], float(scale), _p(out))
    return out


def decode_unit(q_bits, R_g, W_g, codes_unit, meta_unit, K_unit, V_unit, n_valid, page, P, k,
                scale, attend_too=True, gqa_sum=False):
    """One decode step of one unit; returns a dict of numpy outputs.  A float32
    ``meta_unit`` selects variant V1, ``gqa_sum`` variant V2."""
    q = _c(q_bits, np.uint16)
    r, d = q.shape
    bits = W_g.shape[1]
    np_ = (n_valid + page - 1) // page
    page_idx = np.empty(P, np.int32)
    tok_idx = np.empty(k, np.int32)
    U = np.empty(np_, np.float64)
    D = np.empty(P * page, np.int32)
    out = np.empty((r, d), np.float32) if attend_too else None
    amb = C.c_int64(0)
    f32 = np.asarray(meta_unit).dtype == np.float32
    flags = (1 if f32 else 0) | (2 if gqa_sum else 0)
    n_sel = lib().hhro_decode_unit_v(
        _p(q), r, d, bits, page, _p(_c(R_g, np.float32)), _p(_c(W_g, np.float32)),
        _p(_c(codes_unit, np.uint32)), _p(_c(meta_unit, np.float32 if f32 else np.uint16)),
        _p(_c(K_unit, np.uint16)), _p(_c(V_unit, np.uint16)),
        n_valid, P, k, float(scale), flags, _p(page_idx), _p(tok_idx), _p(U), _p(D), _p(out),
        C.byref(amb))
    return dict(page_idx=page_idx, tok_idx=tok_idx, n_sel=int(n_sel), U=U, D=D, out=out,
                q_ambiguous=int(amb.value))


# ------------------------------------------------------- whole-workload loops

def default_threads() -> int:
    return max(1, min(64, os.cpu_count() or 1))


def _units(w, units):
    return [(b, g) for b in range(w.B) for g in range(w.Hkv)] if units is None else list(units)


def encode_all(inp, n_begin=0, n_end=None, codes=None, meta=None, units=None, threads=None,
               meta_f32=False):
    """Oracle key encoding of ``inp`` (a ``workloads.Inputs``) for [n_begin, n_end).

    Returns (codes [B][Hkv][n_cap][w] uint32, meta [B][Hkv][NPcap][2][d] uint16
    -- float32 with ``meta_f32`` (variant V1) --, ambiguous count).  ``units``
    restricts the work to some (b, g) pairs.
    """
    w = inp.w
    n_end = w.N if n_end is None else n_end
    if codes is None:
        codes = np.zeros((w.B, w.Hkv, w.n_cap, w.words), np.uint32)
    if meta is None:
        meta = np.zeros((w.B, w.Hkv, w.np_cap, 2, w.d), np.float32 if meta_f32 else np.uint16)
    us = _units(w, units)

    def one(bg):
        b, g = bg
        return encode_unit(inp.K[b, g], n_begin, n_end, w.page, inp.R[g], inp.W[g],
                           codes[b, g], meta[b, g])

    with ThreadPoolExecutor(threads or default_threads()) as ex:
        amb = sum(ex.map(one, us))
    return codes, meta, amb


def decode_all(inp, codes, meta, step=0, P=None, k=None, scale=None, attend_too=True,
               units=None, threads=None, gqa_sum=False):
    """Oracle decode step ``step`` over all (or the listed) units.

    Returns dict with page_idx [B][Hkv][P], tok_idx [B][Hkv][k], n_sel [B][Hkv],
    out [B][Hq][d] (float32; zero for units not computed), U (list per unit),
    D [B][Hkv][P*S], q_ambiguous [B][Hkv].
    """
    w = inp.w
    P = w.P if P is None else P
    k = w.k if k is None else k
    scale = 1.0 / math.sqrt(w.d) if scale is None else scale
    n_valid = inp.n_valid(step)
    us = _units(w, units)
    res = dict(page_idx=np.full((w.B, w.Hkv, P), -1, np.int32),
               tok_idx=np.full((w.B, w.Hkv, k), -1, np.int32),
               n_sel=np.zeros((w.B, w.Hkv), np.int32),
               out=np.zeros((w.B, w.Hq, w.d), np.float32),
               D=np.full((w.B, w.Hkv, P * w.page), -1, np.int32),
               q_ambiguous=np.zeros((w.B, w.Hkv), np.int64),
               U={})
    r = w.r

    def one(bg):
        b, g = bg
        return bg, decode_unit(inp.q[step, b, g * r:(g + 1) * r], inp.R[g], inp.W[g],
                               codes[b, g], meta[b, g], inp.K[b, g], inp.V[b, g],
                               n_valid, w.page, P, k, scale, attend_too, gqa_sum)

    with ThreadPoolExecutor(threads or default_threads()) as ex:
        for (b, g), o in ex.map(one, us):
            res["page_idx"][b, g] = o["page_idx"]
            res["tok_idx"][b, g] = o["tok_idx"]
            res["n_sel"][b, g] = o["n_sel"]
            res["D"][b, g] = o["D"]
            res["q_ambiguous"][b, g] = o["q_ambiguous"]
            res["U"][(b, g)] = o["U"]
            if attend_too:
                res["out"][b, g * r:(g + 1) * r] = o["out"]
    return res
