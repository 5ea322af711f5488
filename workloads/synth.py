"""Seeded synthetic inputs shared by the oracle side and the CUDA side.

This module produces the bytes both sides consume: bf16 keys/values/queries
(stored as raw uint16 bit patterns), the per-KV-head orthogonal matrix R and
the per-KV-head projection W.  It holds none of the retrieval method's
arithmetic: no rotation of keys, no bounds, no codes, no selection.

Recipe (per workload, see ``workloads.configs``):

* Per (sequence, KV head): channel scales s_c = exp(0.5 z), z ~ N(0, 1)
  (LogNormal(0, 0.5)); ``n_outlier`` distinct random channels get s_c equal to
  ``outlier_scale``.  Keys are N(0, 1) * s, rounded to bf16.
* Values ~ N(0, 1), queries ~ N(0, 1), both bf16.
* Planted keys: ``planted`` distinct random positions in [0, N); the j-th is
  3 * q_h / |q_h| * sqrt(d) + N(0, 0.1^2) with h = g*r + (j mod r), q_h the
  (bf16) query of that head at the first decode step, so its logit with q_h
  is about 3 |q_h| sqrt(d).
* R_g: Q factor of a QR decomposition (float64) of a 128x128 Gaussian, columns
  sign-fixed so that the triangular factor has a positive diagonal, stored as
  float32.  W_g: a d x b Gaussian, float32.
* Optional RoPE (rotate-half pairing of channels j and j + d/2, inverse
  frequencies base^(-2i/d)) on keys at their positions 0..n_cap-1 and on the
  query of decode step i at position N + i; planted keys are written after
  RoPE.

Every stream comes from ``numpy.random.Generator(PCG64(SeedSequence(...)))``
keyed by (workload seed, stream id, sequence, KV head), so a unit's inputs do
not depend on how many other units are generated.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from .configs import Workload


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest even.

    Inputs are finite Gaussian draws, so NaN handling is not needed.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    h = np.ascontiguousarray(h, dtype=np.uint16)
    return (h.astype(np.uint32) << np.uint32(16)).view(np.float32)


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key))))


def _rope(x: np.ndarray, pos: np.ndarray, base: float) -> np.ndarray:
    """Rotate-half RoPE of rows ``x`` [n, d] at integer positions ``pos`` [n]."""
    d = x.shape[-1]
    half = d // 2
    inv_freq = base ** (-np.arange(0, half, dtype=np.float64) * 2.0 / d)
    ang = pos.astype(np.float64)[:, None] * inv_freq[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1 = x[:, :half].astype(np.float64)
    x2 = x[:, half:].astype(np.float64)
    out = np.empty(x.shape, dtype=np.float32)
    out[:, :half] = x1 * c - x2 * s
    out[:, half:] = x1 * s + x2 * c
    return out


@dataclass
class Inputs:
    w: Workload
    K: np.ndarray        # uint16 [B][Hkv][n_cap][d]   bf16 bits
    V: np.ndarray        # uint16 [B][Hkv][n_cap][d]   bf16 bits
    q: np.ndarray        # uint16 [steps][B][Hq][d]    bf16 bits
    R: np.ndarray        # float32 [Hkv][d][d]
    W: np.ndarray        # float32 [Hkv][d][bits]
    planted_pos: np.ndarray  # int64 [B][Hkv][planted], ascending

    @property
    def steps(self) -> int:
        return self.q.shape[0]

    def n_valid(self, step: int = 0) -> int:
        """Valid keys at decode step ``step`` (after that step's append)."""
        return self.w.N + (step + 1 if self.w.appends else 0)


def make_rw(w: Workload) -> tuple[np.ndarray, np.ndarray]:
    R = np.empty((w.Hkv, w.d, w.d), dtype=np.float32)
    W = np.empty((w.Hkv, w.d, w.bits), dtype=np.float32)
    for g in range(w.Hkv):
        rng = _rng(w.seed, 0, g)
        A = rng.standard_normal((w.d, w.d))
        Q, T = np.linalg.qr(A)
        Q = Q * np.sign(np.diag(T))[None, :]
        R[g] = Q.astype(np.float32)
        W[g] = rng.standard_normal((w.d, w.bits), dtype=np.float32)
    return R, W


def make_queries(w: Workload) -> np.ndarray:
    steps = max(1, w.appends)
    rng = _rng(w.seed, 2)
    q0 = rng.standard_normal((w.B, w.Hq, w.d), dtype=np.float32)
    out = np.empty((steps, w.B, w.Hq, w.d), dtype=np.uint16)
    for i in range(steps):
        if w.rope_base:
            flat = q0.reshape(-1, w.d)
            pos = np.full(flat.shape[0], w.N + i, dtype=np.int64)
            out[i] = f32_to_bf16_bits(_rope(flat, pos, w.rope_base)).reshape(w.B, w.Hq, w.d)
        else:
            out[i] = f32_to_bf16_bits(q0)
    return out


def make_unit(w: Workload, b: int, g: int, q_step0: np.ndarray):
    """Keys, values and planted positions of one (sequence b, KV head g).

    ``q_step0``: uint16 [Hq][d], the first decode step's queries of sequence b.
    """
    rng = _rng(w.seed, 1, b, g)
    s = np.exp(0.5 * rng.standard_normal(w.d)).astype(np.float32)
    if w.n_outlier:
        ch = rng.choice(w.d, size=w.n_outlier, replace=False)
        s[ch] = np.float32(w.outlier_scale)
    k = rng.standard_normal((w.n_cap, w.d), dtype=np.float32) * s[None, :]
    if w.rope_base:
        k = _rope(k, np.arange(w.n_cap, dtype=np.int64), w.rope_base)
    pos = np.sort(rng.choice(w.N, size=w.planted, replace=False)) if w.planted else np.zeros(0, np.int64)
    qf = bf16_bits_to_f32(q_step0).astype(np.float64)
    for j, p in enumerate(pos):
        h = g * w.r + (j % w.r)
        qh = qf[h]
        k[p] = (3.0 * qh / np.linalg.norm(qh) * np.sqrt(w.d)
                + 0.1 * rng.standard_normal(w.d)).astype(np.float32)
    v = rng.standard_normal((w.n_cap, w.d), dtype=np.float32)
    return f32_to_bf16_bits(k), f32_to_bf16_bits(v), pos.astype(np.int64)


def make_inputs(w: Workload) -> Inputs:
    R, W = make_rw(w)
    q = make_queries(w)
    K = np.empty((w.B, w.Hkv, w.n_cap, w.d), dtype=np.uint16)
    V = np.empty_like(K)
    planted = np.zeros((w.B, w.Hkv, w.planted), dtype=np.int64)
    for b in range(w.B):
        for g in range(w.Hkv):
            K[b, g], V[b, g], planted[b, g] = make_unit(w, b, g, q[0, b])
    return Inputs(w=w, K=K, V=V, q=q, R=R, W=W, planted_pos=planted)
