"""Library-based references used to pin the oracle (CPU, float64, torch).

These build gated attention out of torch's own scaled_dot_product_attention
with an additive float mask, and take every gradient from autograd, so the
oracle's hand-derived backward (including dS through the gate softmax) is
checked against an independent derivation. Selection uses ``torch.topk``.
"""
from __future__ import annotations

import math

import numpy as np
import torch
import torch.nn.functional as F


def _selection_mask(S, Nb, mode, topk, tau=None):
    """bool [B,H,Nb,Nb]: key block c attended as history by query block r.

    Threshold mode keeps, of the blocks whose gate over the whole history
    (torch.softmax of the row) reaches tau, the topk with the largest scores."""
    B, H = S.shape[:2]
    r = torch.arange(Nb)[:, None]
    c = torch.arange(Nb)[None, :]
    hist = (c < r).expand(B, H, Nb, Nb).clone()
    if mode == "train":
        return hist, hist
    sel = torch.zeros(B, H, Nb, Nb, dtype=torch.bool)
    for b in range(B):
        for h in range(H):
            for rr in range(1, Nb):
                k = min(topk, rr)
                if mode == "threshold":
                    gates = torch.softmax(S[b, h, rr, :rr].detach(), dim=0)
                    k = min(k, int((gates >= tau).sum()))
                if k:
                    top = torch.topk(S[b, h, rr, :rr].detach(), k).indices
                    sel[b, h, rr, top] = True
    return sel, hist


def sdpa_gated(Q, K, V, S, block, mode="train", topk=None, scale=None, renormalise=True,
               dO=None, gate="log_softmax", tau=None):
    """(O, LSE, dQ, dK, dV, dS) from SDPA + additive mask + autograd, float64."""
    Q = torch.as_tensor(np.asarray(Q, dtype=np.float64)).requires_grad_(True)
    K = torch.as_tensor(np.asarray(K, dtype=np.float64)).requires_grad_(True)
    V = torch.as_tensor(np.asarray(V, dtype=np.float64)).requires_grad_(True)
    S = torch.as_tensor(np.asarray(S, dtype=np.float64)).requires_grad_(True)
    B, Hq, N, d = Q.shape
    G = Hq // K.shape[1]
    Nb = S.shape[2]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    sel, hist = _selection_mask(S, Nb, mode, topk, tau)
    norm_set = sel if renormalise else hist
    ls = torch.log_softmax(S.masked_fill(~norm_set, -1e300), dim=-1)
    if gate == "ones":
        ls = ls * 0.0
    logg = torch.where(sel, ls, torch.zeros_like(ls))
    tb = torch.arange(N) // block
    logg_tok = logg[:, :, tb][:, :, :, tb]
    sel_tok = sel[:, :, tb][:, :, :, tb]
    i = torch.arange(N)[:, None]
    j = torch.arange(N)[None, :]
    diag_tok = (tb[:, None] == tb[None, :]) & (j <= i)
    neg = torch.full_like(logg_tok, -math.inf)
    mask = torch.where(sel_tok, logg_tok, torch.where(diag_tok, torch.zeros_like(neg), neg))
    Kr = K.repeat_interleave(G, dim=1)
    Vr = V.repeat_interleave(G, dim=1)
    O = F.scaled_dot_product_attention(Q, Kr, Vr, attn_mask=mask, scale=scale)
    LSE = torch.logsumexp(scale * (Q @ Kr.transpose(-1, -2)) + mask, dim=-1)
    out = {"O": O.detach().numpy(), "LSE": LSE.detach().numpy()}
    if dO is not None:
        O.backward(torch.as_tensor(np.asarray(dO, dtype=np.float64)))
        out.update(dQ=Q.grad.numpy(), dK=K.grad.numpy(), dV=V.grad.numpy(),
                   dS=torch.where(norm_set, S.grad, torch.zeros_like(S.grad)).numpy())
    return out


def sdpa_dense_causal(Q, K, V, scale=None):
    """Plain causal softmax attention from torch SDPA (is_causal=True), float64."""
    Q = torch.as_tensor(np.asarray(Q, dtype=np.float64))
    K = torch.as_tensor(np.asarray(K, dtype=np.float64))
    V = torch.as_tensor(np.asarray(V, dtype=np.float64))
    G = Q.shape[1] // K.shape[1]
    d = Q.shape[-1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    Kr = K.repeat_interleave(G, dim=1)
    Vr = V.repeat_interleave(G, dim=1)
    O = F.scaled_dot_product_attention(Q, Kr, Vr, is_causal=True, scale=scale)
    N = Q.shape[2]
    causal = torch.ones(N, N, dtype=torch.bool).tril()
    logits = (scale * (Q @ Kr.transpose(-1, -2))).masked_fill(~causal, -math.inf)
    return O.numpy(), torch.logsumexp(logits, dim=-1).numpy()


def rel_err(x, ref):
    """Normwise relative error max|x - ref| / max|ref| (NaN-safe)."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    m = np.isfinite(ref)
    den = np.max(np.abs(ref[m])) if m.any() else 0.0
    num = np.max(np.abs(x[m] - ref[m])) if m.any() else 0.0
    return num / den if den > 0 else num
