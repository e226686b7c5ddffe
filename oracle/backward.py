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


def forward(Q, K, V, Qcal, LQ, idx, nsel, S: int, W: int, scale: float, rows=None):
    """Eq. 8 -> Eq. 7 (kept chunks) -> Eq. 10. Returns O [B,H,R,d], lse [B,H,R] and the
    kept chunks' scores [B,H,R,Kk] (padding -inf), with Ksum and Bsum, for the query rows
    ``rows`` (a 1-D index array; all N rows when None). Query row i's output depends on
    Q_i, Qcal_i and its own selection only, so a subset of rows gives those rows'
    outputs exactly, and the gradients of a sum over rows add up over disjoint subsets."""
    B, H, N, d = Q.shape
    Hk = K.shape[1]
    G = H // Hk
    Ksum, Bsum = summaries(K, LQ, S, scale)
    C = LQ.shape[2]
    rows = torch.arange(N) if rows is None else torch.as_tensor(np.asarray(rows), dtype=torch.int64).reshape(-1)
    R = rows.numel()
    idx = torch.as_tensor(np.asarray(idx), dtype=torch.int64).reshape(B, Hk, N, -1)[:, :, rows]
    nsel = torch.as_tensor(np.asarray(nsel), dtype=torch.int64).reshape(B, Hk, N)[:, :, rows]
    Qr, Qcr = Q[:, :, rows], Qcal[:, :, rows]
    Kk = idx.shape[-1]
    idx_h = idx.repeat_interleave(G, dim=1)  # [B,H,R,Kk]
    nsel_h = nsel.repeat_interleave(G, dim=1)
    kept = (torch.arange(Kk).view(1, 1, 1, Kk) < nsel_h.unsqueeze(-1)) & (idx_h >= 0)
    cidx = idx_h.clamp(min=0, max=max(C - 1, 0))
    # slots that are not kept still gather (their values are masked below): with no
    # complete chunk (C = 0) nothing can be kept, and one zero row keeps those gathers in
    # range
    Kg = torch.cat([Ksum, Ksum.new_zeros(B, H, 1, d)], dim=2) if C == 0 else Ksum
    Bg = torch.cat([Bsum, Bsum.new_zeros(B, H, 1)], dim=2) if C == 0 else Bsum
    # Eq. 7: s^ = scale q~ . k'_c + b'_c of each kept chunk
    ks = torch.gather(Kg, 2, cidx.reshape(B, H, R * Kk, 1).expand(B, H, R * Kk, d)).reshape(B, H, R, Kk, d)
    bs = torch.gather(Bg, 2, cidx.reshape(B, H, R * Kk)).reshape(B, H, R, Kk)
    score = scale * torch.einsum("bhnd,bhnkd->bhnk", Qcr, ks) + bs
    score = torch.where(kept, score, torch.full_like(score, -torch.inf))
    # token logits and the sliding window [max(0, i-W+1), i]
    Kh = K.repeat_interleave(G, dim=1)
    Vh = V.repeat_interleave(G, dim=1)
    L = scale * torch.einsum("bhid,bhjd->bhij", Qr, Kh)  # [B,H,R,N]
    i = rows.view(R, 1)
    j = torch.arange(N).view(1, N)
    win = (j <= i) & (j > i - W)
    Lw = torch.where(win, L, torch.full_like(L, -torch.inf))
    # each kept chunk's own softmax output o_c over its S tokens
    # [B,H,R,Kk,S]; a kept chunk's tokens are all < C S <= N, the clamp only touches masked slots
    tok = (cidx.unsqueeze(-1) * S + torch.arange(S).view(1, 1, 1, 1, S)).clamp(max=N - 1)
    Lc = torch.gather(L, 3, tok.reshape(B, H, R, Kk * S)).reshape(B, H, R, Kk, S)
    pc = torch.softmax(Lc, dim=-1)
    Vc = Vh[torch.arange(B).view(B, 1, 1, 1, 1), torch.arange(H).view(1, H, 1, 1, 1), tok]  # [B,H,R,Kk,S,d]
    oc = torch.einsum("bhnks,bhnksd->bhnkd", pc, Vc)
    # Eq. 10: one normaliser over the kept chunks' masses and the window's tokens
    masses = torch.cat([score, Lw], dim=-1)  # [B,H,R,Kk+N]
    lse = torch.logsumexp(masses, dim=-1)
    finite = torch.isfinite(lse)
    lse_safe = torch.where(finite, lse, torch.zeros_like(lse))
    wc = torch.exp(score - lse_safe.unsqueeze(-1))
    ww = torch.exp(Lw - lse_safe.unsqueeze(-1))
    O = torch.einsum("bhnk,bhnkd->bhnd", wc, oc) + torch.einsum("bhij,bhjd->bhid", ww, Vh)
    O = torch.where(finite.unsqueeze(-1), O, torch.zeros_like(O))
    return O, lse, score, Ksum, Bsum


def grads(Q, K, V, Qcal, LQ, idx, nsel, dO, S: int, W: int, scale: float, batch=None):
    """Gradients of sum(O * dO) for the given selection: a dict with dQ, dK, dV, dQcal,
    dLQ (the inputs), and the intermediate dscore [B,H,N,Kk] (0 padding), dKsum, dBsum,
    with the forward's O and lse. With ``batch`` set, the forward and backward run over
    consecutive blocks of that many query rows and the gradients are summed over the
    blocks (the loss is a sum over rows), which bounds the memory at long sequences."""
    leaves = [_t(x).clone().requires_grad_(True) for x in (Q, K, V, Qcal, LQ)]
    Qd, Kd, Vd, Qcd, LQd = leaves
    dO = _t(dO)
    B, H, N, d = Q.shape
    Kk = np.asarray(idx).shape[-1]
    C = LQ.shape[2]
    f64 = dict(dtype=torch.float64)
    out = {"dscore": torch.zeros(B, H, N, Kk, **f64), "dKsum": torch.zeros(B, H, C, d, **f64),
           "dBsum": torch.zeros(B, H, C, **f64), "O": torch.zeros(B, H, N, d, **f64),
           "lse": torch.zeros(B, H, N, **f64)}
    step = N if batch is None else int(batch)
    for r0 in range(0, N, step):
        rows = torch.arange(r0, min(N, r0 + step))
        O, lse, score, Ksum, Bsum = forward(Qd, Kd, Vd, Qcd, LQd, idx, nsel, S, W, scale, rows=rows)
        score.retain_grad()
        Ksum.retain_grad()
        Bsum.retain_grad()
        (O * dO[:, :, rows]).sum().backward()
        if score.grad is not None:
            out["dscore"][:, :, rows] = torch.where(torch.isfinite(score.detach()), score.grad, torch.zeros_like(score))
        if Ksum.grad is not None:
            out["dKsum"] += Ksum.grad
        if Bsum.grad is not None:
            out["dBsum"] += Bsum.grad
        out["O"][:, :, rows], out["lse"][:, :, rows] = O.detach(), lse.detach()
    for name, leaf in zip(("dQ", "dK", "dV", "dQcal", "dLQ"), leaves):
        out[name] = leaf.grad.detach() if leaf.grad is not None else torch.zeros_like(leaf.detach())
    return out
