"""Offline fitting of the rotation R and the projection W of one KV head.

"HHR: Hierarchical Hash Retrieval for Efficient LLM Generation" trains both
matrices offline:

* GKR (§3.3.1): R = (I + A)^-1 (I - A) with A skew-symmetric (the Cayley
  transform, orthogonal by construction, so logits are unchanged, Eq. 4), fit
  to L_R = L_recall + λ1 L_precision + λ2 L_align (Eqs. 5-9): important pages
  (holding one of the exact top-K keys) missed by the page budget should clear
  the threshold by a margin (Eq. 5); kept pages without an important key are
  penalised by how far their bound overestimates their largest logit (Eq. 6);
  the combined retention score zscore(U) + zscore(H), H the page's
  log-sum-exp hash similarity (Eq. 7), should match the softmax of the
  pages' exact maxima (Eq. 8).
* LHP (§3.3.2): W, fit to L_LHP = L_retrieval + λ3 L_orth + λ4 L_decor +
  λ5 L_bal (Eqs. 11-15) on relaxed codes tanh(0.1 x W) (Eq. 10): the exact
  top-N keys among the candidates GKR keeps should fall inside the N+1
  closest by soft hash distance (Eq. 11); W close to orthonormal columns
  (Eq. 12); bits decorrelated (Eq. 13) and balanced (Eq. 14).

This is the offline tool, not the decode path: plain PyTorch with autograd,
on any device.  The paper gives λ1..λ5 (Appendix A, Table 5: 0.05, 0.25,
0.02, 0.02, 0.02) and leaves the rest open; the readings taken here are the
defaults of the functions below:
* the threshold c_h is the keep-th largest bound of the query (the page
  budget of the decode path), and the margin m is 0.1 standard deviations of
  the pages' exact maxima;
* s_max = 3; temperatures τ_h = τ_page = τ_sel = 1 (distances in bit
  units, bounds and maxima z-scored);
* the hash distance of a key is the relaxed Hamming distance
  (b - ĉ_q · ĉ_k) / 2, which is the Hamming distance for ±1 codes, and W
  applies to the unrotated key and query (as in the decode path);
* R is fit first, with the hash term of Eq. 7 from the W it is given; W is
  then fit on the keys of the pages the fitted R keeps (the paper's
  "keys retained from GKR-selected pages");
* optimiser Adam (learning rate 2e-3 for A, 1e-2 for W), a fixed number of
  full-batch steps, and the iterate with the lowest objective is returned
  (the objective is not monotone along the path: the threshold c_h moves
  with R); R starts at the identity (A = 0), W at the given matrix.
"""
from __future__ import annotations

import torch

LAMBDA = {"precision": 0.05, "align": 0.25, "orth": 0.02, "decor": 0.02, "bal": 0.02}


def cayley(A: torch.Tensor) -> torch.Tensor:
    """R = (I + S)^-1 (I - S) with S = A - A^T skew-symmetric (orthogonal)."""
    S = A - A.T
    eye = torch.eye(A.shape[0], dtype=A.dtype, device=A.device)
    return torch.linalg.solve(eye + S, eye - S)


def page_bounds(qt: torch.Tensor, kt: torch.Tensor, page: int) -> torch.Tensor:
    """Eq. 3 for queries qt [B, d] and rotated keys kt [N, d] (N a multiple of
    the page size): U [B, NP] = sum_j max(q_j l_j, q_j u_j), written as
    min(q, 0) l + max(q, 0) u, which equals it because l <= u."""
    lo = kt.view(-1, page, kt.shape[1]).amin(1)
    hi = kt.view(-1, page, kt.shape[1]).amax(1)
    return qt.clamp(max=0) @ lo.T + qt.clamp(min=0) @ hi.T


def relaxed_codes(x: torch.Tensor, W: torch.Tensor) -> torch.Tensor:
    """Eq. 10: ĉ = tanh(0.1 x W)."""
    return torch.tanh(0.1 * (x @ W))


def hash_distance(cq: torch.Tensor, ck: torch.Tensor) -> torch.Tensor:
    """Relaxed Hamming distance (b - ĉ_q . ĉ_k) / 2, [B, N]."""
    return 0.5 * (cq.shape[1] - cq @ ck.T)


def _zscore(x: torch.Tensor) -> torch.Tensor:
    return (x - x.mean(1, keepdim=True)) / x.std(1, keepdim=True).clamp_min(1e-12)


def _top_mask(scores: torch.Tensor, m: int) -> torch.Tensor:
    """Boolean mask of the m largest entries per row."""
    idx = scores.topk(m, dim=1).indices
    return torch.zeros_like(scores, dtype=torch.bool).scatter_(1, idx, True)


def gkr_losses(R, K, Q, W, page, keep, top_k, margin_sd=0.1, s_max=3.0, tau_h=1.0, tau_page=1.0):
    """The three GKR objectives (Eqs. 5, 6, 8) for keys K [N, d] and queries
    Q [B, d] (float, the bf16 values).  Returns (recall, precision, align)."""
    B = Q.shape[0]
    U = page_bounds(Q @ R, K @ R, page)                            # [B, NP]
    logits = Q @ K.T                                               # exact, R-invariant
    Ustar = logits.view(B, -1, page).amax(2)                       # oracle page bound U*
    imp = torch.zeros_like(logits, dtype=torch.bool).scatter_(1, logits.topk(top_k, dim=1).indices, True)
    imp = imp.view(B, -1, page).any(2)                             # important pages
    kept = _top_mask(U.detach(), keep)
    c = U.detach().topk(keep, dim=1).values[:, -1:]                # threshold c_h
    sd = Ustar.std(1, keepdim=True).clamp_min(1e-12)
    # Eq. 5: missed important pages should clear c_h by the margin
    missed = imp & ~kept
    hinge = torch.relu(c + margin_sd * sd - U) * missed
    l_recall = (hinge.sum(1) / missed.sum(1).clamp_min(1)).mean()
    # Eq. 6: kept pages without an important key, weighted by overestimation
    fp = kept & ~imp
    s = (torch.relu(U - Ustar) / sd).clamp(max=s_max)
    w = (1 + s) * fp
    l_prec = ((w * torch.log1p(s)).sum(1) / w.sum(1).clamp_min(1e-12)).mean()
    # Eqs. 7-8: combined retention score against the pages' exact maxima
    D = hash_distance(relaxed_codes(Q, W), relaxed_codes(K, W))
    H = torch.logsumexp((-D / tau_h).view(B, -1, page), dim=2)
    C = _zscore(U) + _zscore(H)
    Pstar = torch.softmax(_zscore(Ustar) / tau_page, dim=1)
    l_align = (Pstar * (torch.log(Pstar.clamp_min(1e-30)) - torch.log_softmax(C, dim=1))).sum(1).mean()
    return l_recall, l_prec, l_align


def lhp_losses(W, K, Q, cand, top_n, tau_sel=1.0):
    """The LHP objectives (Eqs. 11-14) for keys K [N, d], queries Q [B, d] and
    the candidate mask cand [B, N] (keys of the kept pages).  Returns
    (retrieval, orth, decor, bal)."""
    ck, cq = relaxed_codes(K, W), relaxed_codes(Q, W)
    D = hash_distance(cq, ck)
    inf = torch.tensor(float("inf"), dtype=D.dtype, device=D.device)
    Dc = torch.where(cand, D, inf)
    d_n1 = Dc.sort(dim=1).values[:, top_n: top_n + 1]             # (N+1)-th closest candidate
    m = torch.sigmoid((d_n1 - D) / tau_sel)                        # soft selection
    logits = torch.where(cand, Q @ K.T, -inf)
    star = torch.zeros_like(cand).scatter_(1, logits.topk(top_n, dim=1).indices, True)
    l_ret = -torch.log(((m * star).sum(1) / top_n).clamp_min(1e-12)).mean()     # Eq. 11
    eye = torch.eye(W.shape[1], dtype=W.dtype, device=W.device)
    l_orth = ((W.T @ W - eye) ** 2).sum()                                         # Eq. 12
    mu = ck.mean(0)
    cen = ck - mu
    cov = cen.T @ cen / ck.shape[0]
    l_decor = ((cov - torch.diag(torch.diag(cov))) ** 2).sum()                    # Eq. 13
    l_bal = (mu ** 2).sum()                                                       # Eq. 14
    return l_ret, l_orth, l_decor, l_bal


def fit_rotation(K, Q, W, page, keep, top_k, steps=200, lr=2e-3, lam=LAMBDA, **kw):
    """Fits R (Cayley, from the identity) to Eq. 9; returns (R with the lowest
    objective seen, objective per step)."""
    A = torch.zeros(K.shape[1], K.shape[1], dtype=K.dtype, device=K.device, requires_grad=True)
    opt = torch.optim.Adam([A], lr=lr)
    hist, best, best_R = [], float("inf"), None
    for _ in range(steps):
        R = cayley(A)
        lr_, lp, la = gkr_losses(R, K, Q, W, page, keep, top_k, **kw)
        loss = lr_ + lam["precision"] * lp + lam["align"] * la
        hist.append(float(loss))
        if hist[-1] < best:
            best, best_R = hist[-1], R.detach().clone()
        opt.zero_grad()
        loss.backward()
        opt.step()
    return best_R, hist


def fit_projection(K, Q, R, W0, page, keep, top_n, steps=200, lr=1e-2, lam=LAMBDA, **kw):
    """Fits W (from W0) to Eq. 15 on the keys of the pages R keeps; returns
    (W with the lowest objective seen, objective per step)."""
    with torch.no_grad():
        kept = _top_mask(page_bounds(Q @ R, K @ R, page), keep)
        cand = kept.repeat_interleave(page, dim=1)
    W = W0.clone().requires_grad_(True)
    opt = torch.optim.Adam([W], lr=lr)
    hist, best, best_W = [], float("inf"), None
    for _ in range(steps):
        lret, lo, ld, lb = lhp_losses(W, K, Q, cand, top_n, **kw)
        loss = lret + lam["orth"] * lo + lam["decor"] * ld + lam["bal"] * lb
        hist.append(float(loss))
        if hist[-1] < best:
            best, best_W = hist[-1], W.detach().clone()
        opt.zero_grad()
        loss.backward()
        opt.step()
    return best_W, hist
