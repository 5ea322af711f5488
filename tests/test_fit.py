"""CPU checks of the offline R / W fitting (kv_cache_retrieval_b200.fit):
its Eq. 3 against the oracle's, its relaxed hash distance against the
oracle's Hamming distance, the zero cases of each objective, orthogonality of
the Cayley rotation, and that fitting lowers the objectives ("HHR:
Hierarchical Hash Retrieval for Efficient LLM Generation", §3.3.1 Eqs. 5-9,
§3.3.2 Eqs. 10-15)."""
import numpy as np
import pytest
import torch

from kv_cache_retrieval_b200 import fit
from oracle import oracle as O
from workloads import bf16_bits_to_f32, f32_to_bf16_bits


def _bits(rng, shape, scale=1.0):
    return f32_to_bf16_bits((rng.standard_normal(shape) * scale).astype(np.float32))


def test_cayley_is_orthogonal_and_identity_at_zero():
    g = torch.Generator().manual_seed(0)
    A = torch.randn(128, 128, generator=g, dtype=torch.float64)
    R = fit.cayley(A)
    assert torch.allclose(R.T @ R, torch.eye(128, dtype=torch.float64), atol=1e-10)
    assert torch.linalg.det(R) > 0
    assert torch.equal(fit.cayley(torch.zeros(8, 8, dtype=torch.float64)), torch.eye(8, dtype=torch.float64))


def test_page_bounds_match_the_oracle_eq3():
    """The fitting's Eq. 3 (min / max split) equals the oracle's Eq. 3 on
    float32 metadata, head by head."""
    rng = np.random.default_rng(1)
    k, q = _bits(rng, (64, 128), 2.0), _bits(rng, (3, 128))
    R = np.linalg.qr(rng.standard_normal((128, 128)))[0].astype(np.float32)
    kt, qt = O.rotate(k, R), O.rotate(q, R)
    meta = O.page_meta(kt, 64, 16, f32=True)
    _, Uh = O.page_bounds(qt, meta, 4, per_head=True)
    U = fit.page_bounds(torch.from_numpy(qt).double(), torch.from_numpy(kt).double(), 16)
    np.testing.assert_allclose(U.numpy(), Uh, rtol=1e-12, atol=1e-9)


def test_hash_distance_of_sign_codes_is_the_hamming_distance():
    """For ±1 codes (bit = z > 0, as in the decode path), (b - c_q . c_k)/2 is
    the oracle's Eq. 2; the relaxed codes of Eq. 10 approach those codes as
    the projection grows."""
    rng = np.random.default_rng(2)
    k, q = _bits(rng, (32, 128)), _bits(rng, (1, 128))
    W = rng.standard_normal((128, 128)).astype(np.float32)
    codes, _ = O.project_sign(k, W)
    qc, _ = O.project_sign(q, W)
    D_o = O.hamming(qc, codes, np.array([0, 1], np.int32), 16, 32)
    kx, qx = torch.from_numpy(bf16_bits_to_f32(k)).double(), torch.from_numpy(bf16_bits_to_f32(q)).double()
    Wt = torch.from_numpy(W).double()
    sgn = lambda x: torch.where(x @ Wt > 0, 1.0, -1.0).double()
    D = fit.hash_distance(sgn(qx), sgn(kx))
    assert D.numpy()[0].tolist() == D_o.tolist()
    Dr = fit.hash_distance(fit.relaxed_codes(qx, Wt * 1e4), fit.relaxed_codes(kx, Wt * 1e4))
    assert np.abs(Dr.numpy()[0] - D_o).max() < 0.5


def _head(seed=3, N=1024, B=6):
    g = torch.Generator().manual_seed(seed)
    scales = torch.exp(0.5 * torch.randn(128, generator=g, dtype=torch.float64))
    scales[:4] *= 8.0
    K = torch.randn(N, 128, generator=g, dtype=torch.float64) * scales
    Q = torch.randn(B, 128, generator=g, dtype=torch.float64)
    W = torch.randn(128, 128, generator=g, dtype=torch.float64) / 128 ** 0.5
    return K, Q, W


def test_gkr_loss_zero_cases():
    K, Q, W = _head()
    R = torch.eye(128, dtype=torch.float64)
    NP = K.shape[0] // 16
    # every page kept: nothing is missed, the recall objective is 0
    lr, lp, la = fit.gkr_losses(R, K, Q, W, 16, NP, 20)
    assert float(lr) == 0.0 and float(lp) >= 0.0 and float(la) >= 0.0
    # a bound that never overestimates: one key per page makes U = U*, so s = 0
    lr1, lp1, _ = fit.gkr_losses(R, K, Q, W, 1, 50, 20)
    assert float(lp1) == pytest.approx(0.0, abs=1e-12)


def test_lhp_loss_zero_cases():
    K, Q, W = _head()
    Wo = torch.linalg.qr(W)[0]                      # orthonormal columns
    cand = torch.ones(Q.shape[0], K.shape[0], dtype=torch.bool)
    _, lo, _, _ = fit.lhp_losses(Wo, K, Q, cand, 16)
    assert float(lo) == pytest.approx(0.0, abs=1e-20)
    # keys in +/- pairs: every relaxed bit averages to 0 (Eq. 14)
    Ks = torch.cat([K, -K])
    _, _, _, lb = fit.lhp_losses(Wo, Ks, Q, torch.ones(Q.shape[0], Ks.shape[0], dtype=torch.bool), 16)
    assert float(lb) == pytest.approx(0.0, abs=1e-20)


def test_fitting_lowers_the_objectives_and_keeps_r_orthogonal():
    K, Q, W = _head(N=2048, B=8)
    NP = K.shape[0] // 16
    R, hist_r = fit.fit_rotation(K, Q, W, 16, keep=NP // 5, top_k=30, steps=40)
    assert min(hist_r) < hist_r[0]
    lr_, lp, la = fit.gkr_losses(R, K, Q, W, 16, NP // 5, 30)
    best = float(lr_ + fit.LAMBDA["precision"] * lp + fit.LAMBDA["align"] * la)
    assert best == pytest.approx(min(hist_r), rel=1e-9)   # the returned R is the best iterate
    assert torch.allclose(R.T @ R, torch.eye(128, dtype=torch.float64), atol=1e-8)
    W1, hist_w = fit.fit_projection(K, Q, R, W, 16, keep=NP // 5, top_n=20, steps=40)
    assert min(hist_w) < hist_w[0]
    assert W1.shape == W.shape and torch.isfinite(W1).all()
