"""Helpers shared by the GPU parity tests: move seeded inputs to the device,
run the CUDA path through the C ABI, and compare with the oracle under the
parity rules:

* codes and Hamming distances bit-exact, except projections whose oracle
  value has |z| < 1e-4 (counted and reported);
* page and token index sets identical, except candidates whose score lies
  within 1e-3 (relative) of the cutoff score (reported);
* attention outputs within 2e-3 max-abs.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import kv_cache_retrieval_b200 as hhr
from oracle import oracle as O
from workloads import bf16_bits_to_f32

ATTN_TOL = 2e-3
NEAR_CUTOFF = 1e-3


def bf16_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)


def u32_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int32)).cuda()


def bits_host(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def u32_host(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint32)


class Dev:
    """Device copies of a workload's inputs plus output buffers."""

    def __init__(self, inp, P=None, k=None, flags=0):
        w = inp.w
        self.w = w
        self.inp = inp
        self.P = w.P if P is None else P
        self.k = w.k if k is None else k
        self.flags = flags
        self.dims = hhr.make_dims(w.B, w.Hq, w.Hkv, w.d, w.bits, w.page, w.n_cap, flags)
        self.K = bf16_dev(inp.K)
        self.V = bf16_dev(inp.V)
        self.q = bf16_dev(inp.q)                   # [steps][B][Hq][d]
        self.R = torch.from_numpy(inp.R).cuda()
        self.W = torch.from_numpy(inp.W).cuda()
        self.codes = torch.zeros(w.B, w.Hkv, w.n_cap, w.words, dtype=torch.int32, device="cuda")
        meta_dtype = torch.float32 if flags & hhr.HHR_FLAG_META_F32 else torch.bfloat16
        self.meta = torch.zeros(w.B, w.Hkv, w.np_cap, 2, w.d, dtype=meta_dtype, device="cuda")
        self.page_idx = torch.full((w.B, w.Hkv, self.P), -7, dtype=torch.int32, device="cuda")
        self.tok_idx = torch.full((w.B, w.Hkv, self.k), -7, dtype=torch.int32, device="cuda")
        self.n_sel = torch.full((w.B, w.Hkv), -7, dtype=torch.int32, device="cuda")
        self.out = torch.full((w.B, w.Hq, w.d), float("nan"), dtype=torch.float32, device="cuda")
        ws = hhr.hhr_workspace_size(self.dims, self.P, self.k)
        self.ws = torch.zeros(ws, dtype=torch.uint8, device="cuda")
        self.scale = 1.0 / math.sqrt(w.d)

    def encode(self, n_begin=0, n_end=None):
        n_end = self.w.N if n_end is None else n_end
        hhr.hhr_encode_keys(self.dims, self.K, self.R, self.W, n_begin, n_end, self.codes, self.meta)

    def load_state(self, codes: np.ndarray, meta: np.ndarray):
        """Use oracle-encoded codes / metadata (identical bytes) as the state."""
        self.codes.copy_(u32_dev(codes))
        if meta.dtype == np.float32:
            self.meta.copy_(torch.from_numpy(np.ascontiguousarray(meta)).cuda())
        else:
            self.meta.copy_(bf16_dev(meta))

    def meta_host(self) -> np.ndarray:
        """The metadata as the oracle stores it: bf16 bits, or float32."""
        return self.meta.cpu().numpy() if self.meta.dtype == torch.float32 else bits_host(self.meta)

    def select(self, step=0, n_valid=None, dbg=True):
        w = self.w
        n_valid = self.inp.n_valid(step) if n_valid is None else n_valid
        NP = (n_valid + w.page - 1) // w.page
        self.dbg_U = torch.full((w.B, w.Hkv, max(NP, 1)), float("nan"), device="cuda") if dbg else None
        self.dbg_D = torch.full((w.B, w.Hkv, self.P * w.page), -7, dtype=torch.int32, device="cuda") if dbg else None
        hhr.hhr_select(self.dims, self.q[step], self.R, self.W, self.codes, self.meta, n_valid, self.P,
                       self.k, self.page_idx, self.tok_idx, self.n_sel, self.dbg_U, self.dbg_D, self.ws)

    def attend(self, step, tok_idx, n_sel):
        hhr.hhr_sparse_attend(self.dims, self.q[step], self.K, self.V, tok_idx, n_sel, self.k,
                              self.scale, self.out, self.ws)

    def decode(self, step=0, n_valid=None):
        n_valid = self.inp.n_valid(step) if n_valid is None else n_valid
        hhr.hhr_decode_step(self.dims, self.q[step], self.R, self.W, self.codes, self.meta, self.K,
                            self.V, n_valid, self.P, self.k, self.scale, self.page_idx, self.tok_idx,
                            self.n_sel, self.out, self.ws)

    def status(self):
        return hhr.hhr_read_status(self.ws)


# ----------------------------------------------------------------- comparisons

def compare_encode(inp, codes_g, meta_g, units, n_end, n_begin=0):
    """Codes bit-exact except oracle |z| < 1e-4; metadata equal (a differing
    bound may only be one bf16 step further out or in, reported).  float32
    metadata (meta_g float32): equal up to the float32 rotation error."""
    w = inp.w
    f32 = meta_g.dtype == np.float32
    report = dict(code_bits=0, ambiguous=0, meta_vals=0, meta_diff=0)
    codes_o, meta_o, _ = O.encode_all(inp, n_begin=0, n_end=n_end, units=units, meta_f32=f32)
    for (b, g) in units:
        c_o, _, z = O.project_sign(inp.K[b, g, n_begin:n_end], inp.W[g], want_z=True)
        c_g = codes_g[b, g, n_begin:n_end]
        bits_o = np.unpackbits(c_o.view(np.uint8), bitorder="little").reshape(z.shape)
        bits_g = np.unpackbits(np.ascontiguousarray(c_g).view(np.uint8), bitorder="little").reshape(z.shape)
        amb = np.abs(z) < 1e-4
        bad = (bits_o != bits_g) & ~amb
        assert not bad.any(), f"unit {(b, g)}: {int(bad.sum())} code bits differ with |z| >= 1e-4"
        report["code_bits"] += bits_o.size
        report["ambiguous"] += int(amb.sum())
        p0, p1 = n_begin // w.page, (n_end + w.page - 1) // w.page
        mo = meta_o[b, g, p0:p1] if f32 else meta_o[b, g, p0:p1].astype(np.int32)
        mg = meta_g[b, g, p0:p1] if f32 else meta_g[b, g, p0:p1].astype(np.int32)
        diff = mo != mg
        report["meta_vals"] += mo.size
        report["meta_diff"] += int(diff.sum())
        if diff.any():
            # The GPU rotates in float32, the oracle in double.  A stored
            # bound may differ by the float32 dot-product error bound
            # (gamma_128 * sum_i |k_i R_ij| <= 1e-5 * sum_i |k_i R_ij|) plus
            # one bf16 step at the larger of the two values.
            t0 = p0 * w.page
            kf = np.abs(bf16_bits_to_f32(inp.K[b, g, t0:n_end]).astype(np.float64))
            mag = kf @ np.abs(inp.R[g].astype(np.float64))              # [n][d]
            pad = (p1 - p0) * w.page - mag.shape[0]
            mag = np.pad(mag, ((0, pad), (0, 0))).reshape(p1 - p0, w.page, w.d).max(1)
            eps = np.broadcast_to((1e-5 * mag)[:, None, :], mo.shape)
            if f32:
                fo, fg = mo.astype(np.float64), mg.astype(np.float64)
                step = 0.0
            else:
                fo = bf16_bits_to_f32(meta_o[b, g, p0:p1]).astype(np.float64)
                fg = bf16_bits_to_f32(meta_g[b, g, p0:p1]).astype(np.float64)
                step = np.maximum(np.abs(fo), np.abs(fg)) * 2.0 ** -7
            ok = np.abs(fo - fg) <= eps + step + 1e-30
            assert np.all(ok[diff]), "metadata differs by more than the float32 rotation error"
    return report


# Every comparison adds its counts here; tests/conftest.py prints the totals
# in the pytest terminal summary, so they are visible under -q.
REPORTS = []

MAX_PAGE_SWAPS = 2      # near-cutoff page swaps tolerated per unit

# Selection-quality diagnostics (tests/test_selection_quality.py), printed in
# the terminal summary.
QUALITY = []


def compare_select(w, ores, page_idx, tok_idx, n_sel, units, dbg_U=None, dbg_D=None, P=None,
                   k=None, inp=None, step=0, out_g=None, name=""):
    """Compare one decode step's selection (and, when out_g is given, its
    attention output) unit by unit.

    Pages: the sets must be equal except for pages whose oracle bound lies
    within 1e-3 (relative) of the cutoff bound, at most MAX_PAGE_SWAPS per
    unit.  Tokens: with equal page sets and no ambiguous query bit the
    distances must be bit-exact and the token lists identical.  Otherwise
    every token in the symmetric difference must be explained: it lies in a
    swapped page, or its oracle distance is within q_ambiguous of the oracle's
    cutoff distance (a flipped query bit moves a distance by at most one per
    bit); distances of tokens in shared pages may differ by at most
    q_ambiguous.  Attention: units whose token lists match are compared with
    the oracle's output; the others with the oracle's attention over the
    GPU's own selection (needs inp).  Nothing is skipped silently: the counts
    are returned and recorded in REPORTS."""
    P = w.P if P is None else P
    k = w.k if k is None else k
    rep = dict(name=name, units=0, units_exact=0, units_explained=0, near_cutoff_pages=0,
               tok_set_diff=0, q_ambiguous=0, attn_vs_oracle=0, attn_vs_oracle_on_gpu_idx=0,
               attn_max_err=0.0)
    r = w.r
    for (b, g) in units:
        rep["units"] += 1
        U_o = ores["U"][(b, g)]
        NP = U_o.shape[0]
        po = ores["page_idx"][b, g]
        pg = page_idx[b, g]
        if dbg_U is not None and NP:
            ug = dbg_U[b, g, :NP].astype(np.float64)
            tol = 2e-5 * (np.abs(U_o) + np.abs(U_o).mean() + 1.0)
            assert np.all(np.abs(ug - U_o) <= tol), f"unit {(b, g)}: page bounds differ"
        so, sg = set(po[po >= 0].tolist()), set(pg[pg >= 0].tolist())
        assert len(sg) == len(so) == min(P, NP), f"unit {(b, g)}: page counts differ"
        assert np.all(pg[len(sg):] == -1) and np.all(np.diff(pg[:len(sg)]) > 0), f"unit {(b, g)}: page_idx layout"
        swapped = so ^ sg
        if swapped:
            cut = np.sort(U_o)[::-1][min(P, NP) - 1]
            for p in swapped:
                assert abs(U_o[p] - cut) <= NEAR_CUTOFF * max(abs(cut), 1e-30), \
                    f"unit {(b, g)}: page {p} differs but is not near the cutoff"
            assert len(so - sg) <= MAX_PAGE_SWAPS, f"unit {(b, g)}: {len(so - sg)} near-cutoff page swaps"
            rep["near_cutoff_pages"] += len(swapped)
        qa = int(ores["q_ambiguous"][b, g])
        rep["q_ambiguous"] += qa
        to, tg = ores["tok_idx"][b, g], tok_idx[b, g]
        ns_o, ns_g = int(ores["n_sel"][b, g]), int(n_sel[b, g])
        assert ns_g == ns_o, f"unit {(b, g)}: n_sel {ns_g} != {ns_o}"
        assert np.all(tg[ns_g:] == -1) and np.all(np.diff(tg[:ns_g]) > 0), f"unit {(b, g)}: tok_idx layout"
        D_o = ores["D"][b, g]
        if not swapped and qa == 0:
            assert np.array_equal(to, tg), f"unit {(b, g)}: token selection differs"
            if dbg_D is not None:
                assert np.array_equal(D_o, dbg_D[b, g]), f"unit {(b, g)}: distances differ"
            rep["units_exact"] += 1
        else:
            # the oracle's distance of each candidate token, by token index
            slot_o = {int(p): i for i, p in enumerate(po[po >= 0])}
            def dist_o(n):
                p = n // w.page
                return int(D_o[slot_o[p] * w.page + n % w.page]) if p in slot_o else None
            sel_o = to[:ns_o]
            # the cutoff distance of each selection, in oracle distances (a
            # swapped page changes the candidate set and may move the cutoff)
            T = max((dist_o(int(n)) for n in sel_o), default=0)
            T_g = max((dist_o(int(n)) for n in tg[:ns_g] if (int(n) // w.page) not in swapped), default=T)
            lo, hi = min(T, T_g) - qa, max(T, T_g) + qa
            diff = set(sel_o.tolist()) ^ set(tg[:ns_g].tolist())
            for n in diff:
                if (int(n) // w.page) in swapped:
                    continue
                dn = dist_o(int(n))
                assert dn is not None and lo <= dn <= hi, \
                    f"unit {(b, g)}: token {n} (distance {dn}, cutoffs {T}/{T_g}) differs without a cause"
            if dbg_D is not None:
                shared = [(i, p) for i, p in enumerate(pg[pg >= 0]) if p in slot_o]
                for i, p in shared:
                    dg = dbg_D[b, g, i * w.page:(i + 1) * w.page]
                    do = D_o[slot_o[p] * w.page:(slot_o[p] + 1) * w.page]
                    assert np.all(np.abs(dg.astype(np.int64) - do) <= qa), f"unit {(b, g)}: distances differ"
            rep["tok_set_diff"] += len(diff)
            rep["units_explained"] += 1
        if out_g is not None:
            og = out_g[b, g * r:(g + 1) * r]
            if np.array_equal(to, tg):
                e = float(np.abs(ores["out"][b, g * r:(g + 1) * r] - og).max())
                rep["attn_vs_oracle"] += 1
            else:
                assert inp is not None, "attention of a differing selection needs the inputs"
                ref = O.attend(inp.q[step, b, g * r:(g + 1) * r], inp.K[b, g], inp.V[b, g],
                               tg[:ns_g], 1.0 / math.sqrt(w.d))
                e = float(np.abs(ref - og).max())
                rep["attn_vs_oracle_on_gpu_idx"] += 1
            assert e <= ATTN_TOL, f"unit {(b, g)}: attention max-abs error {e}"
            rep["attn_max_err"] = max(rep["attn_max_err"], e)
    assert rep["units"] > 0
    REPORTS.append(rep)
    return rep


def compare_out(w, out_o, out_g, units):
    r = w.r
    err = 0.0
    for (b, g) in units:
        e = float(np.abs(out_o[b, g * r:(g + 1) * r] - out_g[b, g * r:(g + 1) * r]).max())
        err = max(err, e)
    assert err <= ATTN_TOL, f"attention max-abs error {err}"
    return err
