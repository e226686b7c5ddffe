"""float64 gradients of the HiLS-Attention forward pass, for a fixed selection.

TEST INFRASTRUCTURE, like the rest of ``oracle/``: only ``tests/`` and the bench's
baseline legs may import it, and the CUDA library never loads it.

The forward is written again here in plain, differentiable PyTorch float64 operations,
following "Hierarchical Sparse Attention Done Right" (summary page): the landmark
summaries of Methodology 1 (Eq. 8), the chunk scores of Eq. 7 for the kept chunks, and
the hierarchical combination of Eq. 10 with one normaliser over the kept chunks and
the sliding window (the readings of the C oracle in ``hils_oracle.c``). The selection
(idx, nsel) is an input: top-K is piecewise constant, so the gradient flows only
through the kept chunks' scores, summaries, and the token logits. Gradients come from
torch autograd over that forward; the pins in ``tests/test_oracle_backward.py`` tie
them to finite differences and tie the forward to the C oracle.

Shapes: Q, Qcal [B,H,N,d]; K, V [B,Hk,N,d] (query head h reads key-value head h // G,
G = H / Hk); LQ [B,H,C,d]; idx [B,Hk,N,Kk] (-1 padding), nsel [B,Hk,N].
"""
from __future__ import annotations

import numpy as np
import torch


def _t(x):
    return (x if isinstance(x, torch.Tensor) else torch.from_numpy(np.ascontiguousarray(x))).to(torch.float64)


def summaries(K, LQ, S: int, scale: float):
    """Eq. 8 for every complete chunk of every query head: k'_c = sum_j p_j k_j and
    b'_c = -sum_j p_j log p_j, p = softmax_j(scale q'_c . k_j)."""
    B, H, C, d = LQ.shape
    G = H // K.shape[1]
    Kh = K.repeat_interleave(G, dim=1)[:, :, : C * S].reshape(B, H, C, S, d)
    logit = scale * torch.einsum("bhcd,bhcsd->bhcs", LQ, Kh)
    p = torch.softmax(logit, dim=-1)
    Ksum = torch.einsum("bhcs,bhcsd->bhcd", p, Kh)
    Bsum = -(p * torch.log_softmax(logit, dim=-1)).sum(-1)
    return Ksum, Bsum


def forward(Q, K, V, Qcal, LQ, idx, nsel, S: int, W: int, scale: float):
    """Eq. 8 -> Eq. 7 (kept chunks) -> Eq. 10. Returns O [B,H,N,d], lse [B,H,N] and the
    kept chunks' scores [B,H,N,Kk] (padding -inf), with Ksum and Bsum."""
    B, H, N, d = Q.shape
    Hk = K.shape[1]
    G = H // Hk
    Ksum, Bsum = summaries(K, LQ, S, scale)
    C = LQ.shape[2]
    idx = torch.as_tensor(np.asarray(idx), dtype=torch.int64).reshape(B, Hk, N, -1)
    nsel = torch.as_tensor(np.asarray(nsel), dtype=torch.int64).reshape(B, Hk, N)
    Kk = idx.shape[-1]
    idx_h = idx.repeat_interleave(G, dim=1)  # [B,H,N,Kk]
    nsel_h = nsel.repeat_interleave(G, dim=1)
    kept = (torch.arange(Kk).view(1, 1, 1, Kk) < nsel_h.unsqueeze(-1)) & (idx_h >= 0)
    cidx = idx_h.clamp(min=0, max=max(C - 1, 0))
    # Eq. 7: s^ = scale q~ . k'_c + b'_c of each kept chunk
    ks = torch.gather(Ksum, 2, cidx.reshape(B, H, N * Kk, 1).expand(B, H, N * Kk, d)).reshape(B, H, N, Kk, d)
    bs = torch.gather(Bsum, 2, cidx.reshape(B, H, N * Kk)).reshape(B, H, N, Kk)
    score = scale * torch.einsum("bhnd,bhnkd->bhnk", Qcal, ks) + bs
    score = torch.where(kept, score, torch.full_like(score, -torch.inf))
    # token logits and the sliding window [max(0, i-W+1), i]
    Kh = K.repeat_interleave(G, dim=1)
    Vh = V.repeat_interleave(G, dim=1)
    L = scale * torch.einsum("bhid,bhjd->bhij", Q, Kh)
    i = torch.arange(N).view(N, 1)
    j = torch.arange(N).view(1, N)
    win = (j <= i) & (j > i - W)
    Lw = torch.where(win, L, torch.full_like(L, -torch.inf))
    # each kept chunk's own softmax output o_c over its S tokens
    tok = cidx.unsqueeze(-1) * S + torch.arange(S).view(1, 1, 1, 1, S)  # [B,H,N,Kk,S]
    Lc = torch.gather(L.unsqueeze(3).expand(B, H, N, Kk, N), 4, tok)
    pc = torch.softmax(Lc, dim=-1)
    Vc = torch.gather(Vh.unsqueeze(2).unsqueeze(2).expand(B, H, N, Kk, N, d), 4,
                      tok.unsqueeze(-1).expand(B, H, N, Kk, S, d))
    oc = torch.einsum("bhnks,bhnksd->bhnkd", pc, Vc)
    # Eq. 10: one normaliser over the kept chunks' masses and the window's tokens
    masses = torch.cat([score, Lw], dim=-1)  # [B,H,N,Kk+N]
    lse = torch.logsumexp(masses, dim=-1)
    finite = torch.isfinite(lse)
    lse_safe = torch.where(finite, lse, torch.zeros_like(lse))
    wc = torch.exp(score - lse_safe.unsqueeze(-1))
    ww = torch.exp(Lw - lse_safe.unsqueeze(-1))
    O = torch.einsum("bhnk,bhnkd->bhnd", wc, oc) + torch.einsum("bhij,bhjd->bhid", ww, Vh)
    O = torch.where(finite.unsqueeze(-1), O, torch.zeros_like(O))
    return O, lse, score, Ksum, Bsum


def grads(Q, K, V, Qcal, LQ, idx, nsel, dO, S: int, W: int, scale: float):
    """Gradients of sum(O * dO) for the given selection: a dict with dQ, dK, dV, dQcal,
    dLQ (the inputs), and the intermediate dscore [B,H,N,Kk] (0 padding), dKsum, dBsum,
    with the forward's O and lse."""
    leaves = [_t(x).clone().requires_grad_(True) for x in (Q, K, V, Qcal, LQ)]
    Qd, Kd, Vd, Qcd, LQd = leaves
    O, lse, score, Ksum, Bsum = forward(Qd, Kd, Vd, Qcd, LQd, idx, nsel, S, W, scale)
    score.retain_grad()
    Ksum.retain_grad()
    Bsum.retain_grad()
    (O * _t(dO)).sum().backward()
    out = {name: leaf.grad.detach() for name, leaf in zip(("dQ", "dK", "dV", "dQcal", "dLQ"), leaves)}
    ds = score.grad.detach() if score.grad is not None else torch.zeros_like(score)
    out["dscore"] = torch.where(torch.isfinite(score.detach()), ds, torch.zeros_like(ds))
    out["dKsum"] = Ksum.grad.detach() if Ksum.grad is not None else torch.zeros_like(Ksum)
    out["dBsum"] = Bsum.grad.detach() if Bsum.grad is not None else torch.zeros_like(Bsum)
    out["O"], out["lse"] = O.detach(), lse.detach()
    return out
