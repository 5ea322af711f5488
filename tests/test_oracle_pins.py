"""Pins of the CPU oracle against things other than itself.

Each test ties one oracle function to a library routine, a closed form, an
invariant, brute force on a tiny input, or the hand-worked example in
``tests/golden/`` -- chosen so that a dropped term, a wrong sign, a wrong
index or a transposed operand in the oracle fails at least one of them.
Passages cited are from "HHR: Hierarchical Hash Retrieval for Efficient LLM
Generation" (arXiv 2610.01230).
"""
import math
import os

import numpy as np
import pytest
import torch

from oracle import oracle as O
from workloads import bf16_bits_to_f32, f32_to_bf16_bits, get, make_inputs, scaled
from workloads.synth import make_rw

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16(x):
    return f32_to_bf16_bits(np.asarray(x, np.float32))


def _f(bits):
    return bf16_bits_to_f32(bits).astype(np.float64)


def _rand_bits(rng, shape, scale=1.0):
    return _bf16(rng.standard_normal(shape).astype(np.float32) * scale)


# ------------------------------------------------------------ rotation, Eq. 4

def test_rotation_is_row_vector_matmul():
    """Eq. 4 writes k~ = k R (row vector times R): compare with numpy matmul."""
    rng = np.random.default_rng(1)
    x = _rand_bits(rng, (40, 128), 3.0)
    R = rng.standard_normal((128, 128)).astype(np.float32)
    got = O.rotate(x, R)
    ref = (_f(x) @ R.astype(np.float64)).astype(np.float32)
    # same double sum in another order: at most one float32 ulp apart
    np.testing.assert_array_max_ulp(got, ref, maxulp=1)
    # a transposed operand would be far off
    assert not np.allclose(got, (_f(x) @ R.T.astype(np.float64)), rtol=1e-3, atol=1e-3)


def test_generated_rotation_is_orthogonal_and_preserves_logits():
    """R R^T = I keeps q.k unchanged (§3.3.1, Eq. 4 and the identity after it)."""
    R, _ = make_rw(get("llama8b_32k"))
    for g in range(R.shape[0]):
        Rg = R[g].astype(np.float64)
        assert np.abs(Rg.T @ Rg - np.eye(128)).max() <= 1e-5
    rng = np.random.default_rng(2)
    q = _rand_bits(rng, (8, 128))
    k = _rand_bits(rng, (64, 128), 4.0)
    qt = O.rotate(q, R[3]).astype(np.float64)
    kt = O.rotate(k, R[3]).astype(np.float64)
    exact = _f(q) @ _f(k).T
    bound = 1e-4 * np.linalg.norm(_f(q), axis=1)[:, None] * np.linalg.norm(_f(k), axis=1)[None, :]
    assert np.all(np.abs(qt @ kt.T - exact) <= bound)


# ------------------------------------------------- projection + sign, Eq. 10

def test_code_bit_layout_closed_form():
    """Bit t of the code lands in word t/32 at position t%32 (LSB first)."""
    d, bits = 128, 128
    W = np.zeros((d, bits), np.float32)
    W[np.arange(d), np.arange(d)] = 1.0            # z = x
    x = np.full((1, d), -1.0, np.float32)
    x[0, [0, 33, 64, 65, 127]] = 2.0
    codes, amb = O.project_sign(_bf16(x), W)
    assert amb == 0
    assert codes.tolist() == [[0x1, 0x2, 0x3, 0x80000000]]


def test_code_signs_match_matmul_and_zero_maps_to_zero():
    rng = np.random.default_rng(3)
    x = _rand_bits(rng, (50, 128), 2.0)
    W = rng.standard_normal((128, 256)).astype(np.float32)
    codes, amb, z = O.project_sign(x, W, want_z=True)
    ref_z = _f(x) @ W.astype(np.float64)
    np.testing.assert_allclose(z, ref_z, rtol=1e-12, atol=1e-9)
    bits = np.unpackbits(codes.view(np.uint8), bitorder="little").reshape(50, 256)
    clear = np.abs(ref_z) >= 1e-4
    assert np.array_equal(bits[clear], (ref_z > 0)[clear])
    # an exactly zero projection is bit 0 and counted as ambiguous
    W0 = np.zeros((128, 32), np.float32)
    W0[0, :16] = 1.0
    c0, a0 = O.project_sign(_bf16(np.ones((1, 128))), W0)
    assert c0.tolist() == [[0x0000FFFF]] and a0 == 16


# --------------------------------------------------------- page metadata

def test_metadata_is_outward_rounded_extrema():
    """Lower/upper per dimension (§3.3.1 under Eq. 3), stored as the nearest
    bf16 at or below / at or above the float32 extremum."""
    rng = np.random.default_rng(4)
    kt = (rng.standard_normal((16 * 9 + 5, 128)) * 7).astype(np.float32)
    n_valid = kt.shape[0]
    meta = O.page_meta(kt, n_valid, 16)
    for p in range(meta.shape[0]):
        rows = kt[p * 16:min((p + 1) * 16, n_valid)]
        mn, mx = rows.min(0), rows.max(0)
        lo, hi = bf16_bits_to_f32(meta[p, 0]), bf16_bits_to_f32(meta[p, 1])
        assert np.all(lo <= mn) and np.all(hi >= mx)
        # no bf16 value strictly between the stored bound and the extremum
        lo_next = bf16_bits_to_f32(_next_toward_zero_or_up(meta[p, 0], up=True))
        hi_prev = bf16_bits_to_f32(_next_toward_zero_or_up(meta[p, 1], up=False))
        assert np.all((lo == mn) | (lo_next > mn))
        assert np.all((hi == mx) | (hi_prev < mx))


def _next_toward_zero_or_up(bits, up):
    """Next bf16 value above (up=True) or below the given ones."""
    out = []
    for b in np.asarray(bits, np.uint16).tolist():
        neg = b & 0x8000
        mag = b & 0x7FFF
        if up:
            nb = (b - 1) if (neg and mag) else (b + 1 if not neg else 0x0001)
        else:
            nb = (b + 1) if neg else (b - 1 if mag else 0x8001)
        out.append(nb & 0xFFFF)
    return np.array(out, np.uint16)


def test_partial_last_page_ignores_tokens_past_n_valid():
    rng = np.random.default_rng(5)
    kt = rng.standard_normal((48, 128)).astype(np.float32)
    m1 = O.page_meta(kt, 37, 16)
    kt2 = kt.copy()
    kt2[37:] = 1e6
    m2 = O.page_meta(kt2, 37, 16)
    assert m1.shape[0] == 3 and np.array_equal(m1, m2)
    last = bf16_bits_to_f32(m1[2, 1])
    assert np.all(last >= kt[32:37].max(0))


def test_identity_rotation_gives_raw_extrema():
    """R = I reduces GKR to QUEST-style raw per-channel min/max (§3.3.1,
    ref. [38]); bf16 keys are then stored exactly."""
    w = scaled(get("tiny_4k"), N=200, planted=0)
    inp = make_inputs(w)
    R = np.eye(128, dtype=np.float32)
    codes = np.zeros((w.n_cap, 4), np.uint32)
    meta = np.zeros((w.np_cap, 2, 128), np.uint16)
    O.encode_unit(inp.K[0, 0], 0, 200, 16, R, inp.W[0], codes, meta)
    k = bf16_bits_to_f32(inp.K[0, 0, :200])
    for p in range(13):
        rows = k[p * 16:(p + 1) * 16]
        assert np.array_equal(bf16_bits_to_f32(meta[p, 0]), rows.min(0))
        assert np.array_equal(bf16_bits_to_f32(meta[p, 1]), rows.max(0))


# ----------------------------------------------------------- bound, Eq. 3

def _read_golden():
    vals = {}
    with open(os.path.join(GOLDEN, "bound_example_d4.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, rest = line.split(":", 1)
            vals[key.strip()] = [float(t) for t in rest.split()]
    return vals


def test_bound_hand_worked_example():
    g = _read_golden()
    keys = np.array([g[f"key {i}"] for i in range(5)], np.float32)
    q = np.array([g["query"]], np.float32)
    R = np.eye(4, dtype=np.float32)
    kt = O.rotate(_bf16(keys), R)
    meta = O.page_meta(kt, 5, 2)
    for p in range(3):
        assert bf16_bits_to_f32(meta[p, 0]).tolist() == g[f"lower {p}"]
        assert bf16_bits_to_f32(meta[p, 1]).tolist() == g[f"upper {p}"]
    qt = O.rotate(_bf16(q), R)
    U = O.page_bounds(qt, meta, 3)
    assert U.tolist() == g["bound"]
    assert O.top_largest(U, 2).tolist() == [int(v) for v in g["keep2"]]
    assert O.top_largest(U, 1).tolist() == [int(v) for v in g["keep1"]]


def test_bound_is_max_over_box_corners():
    """The max of a linear function over the box [l, u] sits at a corner:
    brute force over all 2^d corners for d = 6."""
    rng = np.random.default_rng(6)
    d = 6
    corners = np.array([[(c >> j) & 1 for j in range(d)] for c in range(1 << d)], np.float64)
    for _ in range(20):
        kt = (rng.standard_normal((4, d)) * 3).astype(np.float32)
        meta = O.page_meta(kt, 4, 4)
        qt = rng.standard_normal((1, d)).astype(np.float32)
        lo, hi = _f(meta[0, 0]), _f(meta[0, 1])
        box = lo + corners * (hi - lo)
        brute = (box @ qt[0].astype(np.float64)).max()
        U = O.page_bounds(qt, meta, 1)
        assert U[0] == pytest.approx(brute, rel=1e-12, abs=1e-12)


def test_bound_validity_on_generated_keys():
    """Every page bound is >= the largest exact logit of its page (§3.3.1,
    the sentence after Eq. 3)."""
    w = scaled(get("llama8b_32k"), B=1, Hkv=2, Hq=8, N=3000, planted=8)
    inp = make_inputs(w)
    codes, meta, _ = O.encode_all(inp, threads=2)
    for g in range(w.Hkv):
        q = inp.q[0, 0, g * w.r:(g + 1) * w.r]
        qt, _, _ = O.query_prep(q, inp.R[g], inp.W[g])
        np_ = w.n_pages()
        U, Uh = O.page_bounds(qt, meta[0, g], np_, per_head=True)
        logits = _f(q) @ _f(inp.K[0, g, :w.N]).T                       # [r][N]
        qtd = qt.astype(np.float64)
        lom, him = _f(meta[0, g, :np_, 0]), _f(meta[0, g, :np_, 1])
        eps = 1e-5 * (np.abs(qtd)[:, None, :] * np.maximum(np.abs(lom), np.abs(him))[None]).sum(-1)
        for p in range(np_):
            page_max = logits[:, p * 16:min((p + 1) * 16, w.N)].max(1)
            assert np.all(Uh[:, p] >= page_max - eps[:, p])
        assert np.array_equal(U, Uh.max(0))


def test_bound_equals_logit_for_single_token_pages():
    """With R = I and S = 1 the box is a point, so Eq. 3 is the exact logit."""
    rng = np.random.default_rng(7)
    k = _rand_bits(rng, (64, 128), 2.0)
    q = _rand_bits(rng, (3, 128))
    R = np.eye(128, dtype=np.float32)
    meta = O.page_meta(O.rotate(k, R), 64, 1)
    _, Uh = O.page_bounds(O.rotate(q, R), meta, 64, per_head=True)
    np.testing.assert_allclose(Uh, _f(q) @ _f(k).T, rtol=1e-12, atol=1e-9)


def test_group_scores_reduce_to_single_head():
    """GQA reading: group bound = max over heads, group distance = min."""
    rng = np.random.default_rng(8)
    w = scaled(get("llama8b_32k"), B=1, Hkv=1, Hq=4, N=500, planted=0)
    inp = make_inputs(w)
    codes, meta, _ = O.encode_all(inp, threads=1)
    q = inp.q[0, 0]
    qt, qc, _ = O.query_prep(q, inp.R[0], inp.W[0])
    np_ = w.n_pages()
    U = O.page_bounds(qt, meta[0, 0], np_)
    singles = [O.page_bounds(qt[h:h + 1], meta[0, 0], np_) for h in range(4)]
    assert np.array_equal(U, np.max(singles, axis=0))
    pages = np.sort(rng.choice(np_, 10, replace=False)).astype(np.int32)
    D = O.hamming(qc, codes[0, 0], pages, 16, w.N)
    Ds = [O.hamming(qc[h:h + 1], codes[0, 0], pages, 16, w.N) for h in range(4)]
    assert np.array_equal(D, np.min(Ds, axis=0))


# ---------------------------------------------------------- Hamming, Eq. 2

def test_hamming_matches_bit_loop_and_sign_product_identity():
    rng = np.random.default_rng(9)
    for bits in (128, 256):
        words = bits // 32
        codes = rng.integers(0, 2**32, size=(40, words), dtype=np.uint64).astype(np.uint32)
        qc = rng.integers(0, 2**32, size=(1, words), dtype=np.uint64).astype(np.uint32)
        D = O.hamming(qc, codes, np.array([0, 2], np.int32), 16, 40)
        qb = np.unpackbits(qc.view(np.uint8), bitorder="little").astype(int)
        for slot, p in enumerate([0, 2]):
            for t in range(16):
                n = p * 16 + t
                if n >= 40:
                    assert D[slot * 16 + t] == -1
                    continue
                kb = np.unpackbits(codes[n].view(np.uint8), bitorder="little").astype(int)
                loop = sum(1 for j in range(bits) if qb[j] != kb[j])
                sq, sk = 2 * qb - 1, 2 * kb - 1
                assert D[slot * 16 + t] == loop == (bits - int(sq @ sk)) // 2


# ----------------------------------------------------------- selection

def _rank_select(scores, m, larger=True):
    """Brute force: i is kept iff fewer than m entries beat it."""
    s = np.asarray(scores)
    out = []
    for i in range(len(s)):
        beat = (s > s[i]) if larger else (s < s[i])
        tie_before = (s == s[i]) & (np.arange(len(s)) < i)
        if np.count_nonzero(beat | tie_before) < m:
            out.append(i)
    return out


def test_top_largest_matches_rank_count_with_ties():
    rng = np.random.default_rng(10)
    for n, m in [(50, 7), (64, 64), (30, 45), (200, 13)]:
        s = rng.integers(0, 6, n).astype(np.float64)   # many ties
        assert O.top_largest(s, m).tolist() == _rank_select(s, m, True)


def test_top_tokens_matches_rank_count_with_ties():
    rng = np.random.default_rng(11)
    pages = np.array([1, 4, 5, 9], np.int32)
    D = rng.integers(0, 5, 4 * 8).astype(np.int32)
    D[-3:] = -1                                         # past n_valid
    toks = (pages[:, None] * 8 + np.arange(8)[None]).reshape(-1)
    valid = D >= 0
    for k in (1, 5, 17, 29, 40):
        got = O.top_tokens(D, pages, 8, k).tolist()
        picked = _rank_select(D[valid], k, larger=False)
        assert got == sorted(toks[valid][picked].tolist())


# ----------------------------------------------------------- attention

def test_attention_matches_torch_sdpa_in_float64():
    rng = np.random.default_rng(12)
    K = _rand_bits(rng, (300, 128), 2.0)
    V = _rand_bits(rng, (300, 128))
    q = _rand_bits(rng, (4, 128))
    idx = np.sort(rng.choice(300, 77, replace=False)).astype(np.int32)
    got = O.attend(q, K, V, idx, 1 / math.sqrt(128))
    tq = torch.from_numpy(_f(q))[None, :, None, :]                  # [1, r, 1, d]
    tk = torch.from_numpy(_f(K[idx]))[None, None].expand(1, 4, -1, -1)
    tv = torch.from_numpy(_f(V[idx]))[None, None].expand(1, 4, -1, -1)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)[0, :, 0].numpy()
    np.testing.assert_allclose(got, ref, rtol=0, atol=1e-6)


def test_attention_closed_forms():
    rng = np.random.default_rng(13)
    K = _rand_bits(rng, (20, 128))
    V = _rand_bits(rng, (20, 128))
    q = _rand_bits(rng, (2, 128))
    one = O.attend(q, K, V, np.array([7], np.int32), 0.1)
    assert np.array_equal(one, np.stack([bf16_bits_to_f32(V[7])] * 2))
    zero_q = O.attend(np.zeros((1, 128), np.uint16), K, V, np.arange(20, dtype=np.int32), 1.0)
    np.testing.assert_allclose(zero_q[0], _f(V).mean(0), atol=1e-6)
    none = O.attend(q, K, V, np.zeros(0, np.int32), 0.1)
    assert not none.any()


def test_full_budgets_reduce_to_dense_attention():
    """P >= pages and k >= keys keep everything: dense softmax attention."""
    w = scaled(get("llama8b_32k"), B=1, Hkv=1, Hq=4, N=700, planted=4)
    inp = make_inputs(w)
    codes, meta, _ = O.encode_all(inp, threads=1)
    res = O.decode_all(inp, codes, meta, P=10_000, k=10_000, threads=1)
    assert res["n_sel"][0, 0] == 700
    assert res["tok_idx"][0, 0, :700].tolist() == list(range(700))
    q = _f(inp.q[0, 0])
    tq = torch.from_numpy(q)[None, :, None, :]
    tk = torch.from_numpy(_f(inp.K[0, 0, :700]))[None, None].expand(1, 4, -1, -1)
    tv = torch.from_numpy(_f(inp.V[0, 0, :700]))[None, None].expand(1, 4, -1, -1)
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv)[0, :, 0].numpy()
    np.testing.assert_allclose(res["out"][0], ref, atol=1e-6)


# ----------------------------------------------------------- encode / append

def test_append_encoding_equals_one_shot_encoding():
    """Encoding keys in pieces (appends into a partly filled page) gives the
    same codes and metadata as encoding them at once."""
    w = scaled(get("tiny_4k"), N=300, planted=3)
    inp = make_inputs(w)
    c1 = np.zeros((w.n_cap, 4), np.uint32)
    m1 = np.zeros((w.np_cap, 2, 128), np.uint16)
    O.encode_unit(inp.K[0, 0], 0, 300, 16, inp.R[0], inp.W[0], c1, m1)
    c2 = np.zeros_like(c1)
    m2 = np.zeros_like(m1)
    for a, b in [(0, 37), (37, 38), (38, 64), (64, 65), (65, 299), (299, 300)]:
        O.encode_unit(inp.K[0, 0], a, b, 16, inp.R[0], inp.W[0], c2, m2)
    assert np.array_equal(c1, c2) and np.array_equal(m1, m2)


def test_decode_unit_composes_the_primitives():
    w = scaled(get("llama8b_32k"), B=1, Hkv=1, Hq=4, N=2000, P=20, k=100, planted=4)
    inp = make_inputs(w)
    codes, meta, _ = O.encode_all(inp, threads=1)
    res = O.decode_all(inp, codes, meta, threads=1)
    qt, qc, _ = O.query_prep(inp.q[0, 0], inp.R[0], inp.W[0])
    U = O.page_bounds(qt, meta[0, 0], w.n_pages())
    pages = O.top_largest(U, 20)
    D = O.hamming(qc, codes[0, 0], pages, 16, w.N)
    tok = O.top_tokens(D, pages, 16, 100)
    assert res["page_idx"][0, 0].tolist() == pages.tolist()
    assert res["tok_idx"][0, 0].tolist() == tok.tolist()
    assert np.array_equal(res["U"][(0, 0)], U)
    # the planted keys (logit ~ 3 |q| sqrt(d)) are found
    assert set(inp.planted_pos[0, 0].tolist()) <= set(tok.tolist())


# ------------------------------------------- variants: float32 metadata (V1)

def test_f32_metadata_is_exact_extrema():
    """Variant V1 keeps the per-dimension extrema of §3.3.1 (under Eq. 3) in
    float32 unrounded: numpy's min / max over each page's valid rows."""
    rng = np.random.default_rng(21)
    kt = (rng.standard_normal((16 * 7 + 9, 128)) * 5).astype(np.float32)
    n_valid = kt.shape[0] - 4
    meta = O.page_meta(kt, n_valid, 16, f32=True)
    assert meta.dtype == np.float32 and meta.shape == (8, 2, 128)
    for p in range(8):
        rows = kt[p * 16:min((p + 1) * 16, n_valid)]
        assert np.array_equal(meta[p, 0], rows.min(0))
        assert np.array_equal(meta[p, 1], rows.max(0))


def test_bf16_metadata_is_the_outward_rounding_of_f32_metadata():
    """The default bf16 bounds are the float32 bounds of V1 rounded outward:
    lo_bf16 <= lo_f32 with no bf16 value in between (and the mirror for hi)."""
    rng = np.random.default_rng(22)
    kt = (rng.standard_normal((16 * 5, 128)) * 9).astype(np.float32)
    m16 = O.page_meta(kt, kt.shape[0], 16)
    m32 = O.page_meta(kt, kt.shape[0], 16, f32=True)
    lo16, hi16 = bf16_bits_to_f32(m16[:, 0]), bf16_bits_to_f32(m16[:, 1])
    assert np.all(lo16 <= m32[:, 0]) and np.all(hi16 >= m32[:, 1])
    lo_next = bf16_bits_to_f32(_next_toward_zero_or_up(m16[:, 0].ravel(), up=True)).reshape(lo16.shape)
    hi_prev = bf16_bits_to_f32(_next_toward_zero_or_up(m16[:, 1].ravel(), up=False)).reshape(hi16.shape)
    assert np.all((lo16 == m32[:, 0]) | (lo_next > m32[:, 0]))
    assert np.all((hi16 == m32[:, 1]) | (hi_prev < m32[:, 1]))


def test_f32_bound_is_the_rotated_logit_for_single_token_pages():
    """With one key per page and float32 metadata the box of Eq. 3 is the point
    k~ itself, so U = q~ . k~ (numpy dot in float64 of the float32 values),
    which equals q . k up to the float32 rounding of the rotation (Eq. 4).  The
    bf16 bound (outward rounding) can only be larger."""
    rng = np.random.default_rng(23)
    R, _ = make_rw(get("tiny_4k"))
    k = _rand_bits(rng, (48, 128), 2.0)
    q = _rand_bits(rng, (2, 128))
    kt, qt = O.rotate(k, R[0]), O.rotate(q, R[0])
    meta32 = O.page_meta(kt, 48, 1, f32=True)
    _, Uh = O.page_bounds(qt, meta32, 48, per_head=True)
    np.testing.assert_allclose(Uh, qt.astype(np.float64) @ kt.astype(np.float64).T, rtol=1e-12, atol=1e-12)
    exact = _f(q) @ _f(k).T
    scale = np.linalg.norm(_f(q), axis=1)[:, None] * np.linalg.norm(_f(k), axis=1)[None]
    assert np.all(np.abs(Uh - exact) <= 1e-4 * scale)
    _, Uh16 = O.page_bounds(qt, O.page_meta(kt, 48, 1), 48, per_head=True)
    assert np.all(Uh16 >= Uh)


def test_f32_bound_validity_and_tightness_on_generated_keys():
    """V1 bounds stay >= every logit of their page (§3.3.1) and are never above
    the bf16 bounds of the same keys."""
    w = scaled(get("llama8b_32k"), B=1, Hkv=2, Hq=8, N=2500, planted=8)
    inp = make_inputs(w)
    codes16, meta16, _ = O.encode_all(inp, threads=2)
    codes32, meta32, _ = O.encode_all(inp, threads=2, meta_f32=True)
    assert meta32.dtype == np.float32 and np.array_equal(codes16, codes32)
    np_ = w.n_pages()
    for g in range(w.Hkv):
        q = inp.q[0, 0, g * w.r:(g + 1) * w.r]
        qt, _, _ = O.query_prep(q, inp.R[g], inp.W[g])
        _, Uh = O.page_bounds(qt, meta32[0, g], np_, per_head=True)
        _, Uh16 = O.page_bounds(qt, meta16[0, g], np_, per_head=True)
        logits = _f(q) @ _f(inp.K[0, g, :w.N]).T
        qtd = qt.astype(np.float64)
        mag = np.maximum(np.abs(meta32[0, g, :np_, 0]), np.abs(meta32[0, g, :np_, 1])).astype(np.float64)
        eps = 1e-5 * (np.abs(qtd)[:, None, :] * mag[None]).sum(-1)
        for p in range(np_):
            assert np.all(Uh[:, p] >= logits[:, p * 16:min((p + 1) * 16, w.N)].max(1) - eps[:, p])
        assert np.all(Uh <= Uh16 + 1e-9 * np.abs(Uh16))


def test_f32_append_encoding_equals_one_shot_encoding():
    w = scaled(get("tiny_4k"), N=200, planted=2)
    inp = make_inputs(w)
    c1 = np.zeros((w.n_cap, 4), np.uint32)
    m1 = np.zeros((w.np_cap, 2, 128), np.float32)
    O.encode_unit(inp.K[0, 0], 0, 200, 16, inp.R[0], inp.W[0], c1, m1)
    c2, m2 = np.zeros_like(c1), np.zeros_like(m1)
    for a, b in [(0, 17), (17, 18), (18, 150), (150, 200)]:
        O.encode_unit(inp.K[0, 0], a, b, 16, inp.R[0], inp.W[0], c2, m2)
    assert np.array_equal(c1, c2) and np.array_equal(m1, m2)


# ------------------------------------------------ variants: GQA-sum (V2)

def test_gqa_sum_distance_matches_summed_sign_closed_form():
    """Eq. 2 summed over the r heads of a group: with ±1 signs,
    sum_h popc(c_h xor c) = (r b - (sum_h s_h) . s) / 2 -- one dot product of
    the summed query signs with the key signs (numpy)."""
    rng = np.random.default_rng(24)
    for r, bits in ((4, 128), (2, 256), (8, 128)):
        words = bits // 32
        codes = rng.integers(0, 2**32, size=(64, words), dtype=np.uint64).astype(np.uint32)
        qc = rng.integers(0, 2**32, size=(r, words), dtype=np.uint64).astype(np.uint32)
        pages = np.array([0, 3], np.int32)
        D = O.hamming(qc, codes, pages, 16, 60, gqa_sum=True)
        sq = 2 * np.unpackbits(qc.view(np.uint8), bitorder="little").reshape(r, bits).astype(np.int64) - 1
        sk = 2 * np.unpackbits(codes.view(np.uint8), bitorder="little").reshape(64, bits).astype(np.int64) - 1
        for slot, p in enumerate(pages):
            for t in range(16):
                n = p * 16 + t
                want = -1 if n >= 60 else (r * bits - int(sq.sum(0) @ sk[n])) // 2
                assert D[slot * 16 + t] == want


def test_gqa_sum_and_min_agree_for_one_head_and_differ_for_groups():
    rng = np.random.default_rng(25)
    codes = rng.integers(0, 2**32, size=(32, 4), dtype=np.uint64).astype(np.uint32)
    pages = np.array([0, 1], np.int32)
    q1 = rng.integers(0, 2**32, size=(1, 4), dtype=np.uint64).astype(np.uint32)
    assert np.array_equal(O.hamming(q1, codes, pages, 16, 32, gqa_sum=True),
                          O.hamming(q1, codes, pages, 16, 32))
    q4 = rng.integers(0, 2**32, size=(4, 4), dtype=np.uint64).astype(np.uint32)
    s, m = O.hamming(q4, codes, pages, 16, 32, gqa_sum=True), O.hamming(q4, codes, pages, 16, 32)
    assert np.all(s >= 4 * m) and np.all(s <= 4 * 128) and not np.array_equal(s, m)


def test_decode_unit_variants_compose_the_primitives():
    """The flags of one decode step route to the variant primitives: float32
    bounds (V1) and summed distances (V2), the rest unchanged."""
    w = scaled(get("llama8b_32k"), B=1, Hkv=1, Hq=4, N=1800, P=25, k=90, planted=4)
    inp = make_inputs(w)
    codes, meta32, _ = O.encode_all(inp, threads=1, meta_f32=True)
    for gqa_sum in (False, True):
        res = O.decode_all(inp, codes, meta32, threads=1, gqa_sum=gqa_sum)
        qt, qc, _ = O.query_prep(inp.q[0, 0], inp.R[0], inp.W[0])
        U = O.page_bounds(qt, meta32[0, 0], w.n_pages())
        pages = O.top_largest(U, 25)
        D = O.hamming(qc, codes[0, 0], pages, 16, w.N, gqa_sum=gqa_sum)
        tok = O.top_tokens(D, pages, 16, 90)
        assert res["page_idx"][0, 0].tolist() == pages.tolist()
        assert res["tok_idx"][0, 0].tolist() == tok.tolist()
        assert res["D"][0, 0, :25 * 16].tolist() == D.tolist()
        assert np.array_equal(res["U"][(0, 0)], U)


# ------------------------------------------- selection-quality reference

def test_top_logits_matches_brute_force_ranking():
    """The exact top-m keys by group logit (max over the heads of q_h . k):
    numpy float64 logits and rank counting, ties to the lower index."""
    rng = np.random.default_rng(26)
    q = _rand_bits(rng, (4, 128))
    k = _rand_bits(rng, (300, 128), 2.0)
    k[50] = k[7]                     # an exact tie: the lower index wins
    logits = (_f(q) @ _f(k).T).max(0)
    for m in (1, 7, 40, 300, 500):
        got = O.top_logits(q, k, 280, m)
        assert got.tolist() == _rank_select(logits[:280], m, True)
    assert 7 in O.top_logits(q[:, :], k, 280, 280).tolist()
