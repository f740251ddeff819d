"""Float64 CPU oracle for gated block-sparse causal attention (SAS).

TEST INFRASTRUCTURE. This module is the checker, not the product: only the test
suite, ``__graft_entry__.smoke()`` and the CPU-baseline / reference arm of
``bench.py`` may import it. It shares no code with the CUDA library and imports
nothing from it; both sides only receive the same seeded input arrays.

What it computes (the method as read from the pages; every equation here is our
reading because the pages print none):

* "SAS: Simple Attention Sparsification via End-to-End Optimization of Context
  Ranking" (NeurIPS 2026 poster page), Abstract: a selector scores context units
  (tokens or blocks); its continuous scores enter the attention softmax as a gate
  in log form; in training every context unit stays active; at inference a fixed
  budget of units per query is attended.
* Same title, Hugging Face paper page, Abstract: the gates are normalised
  softmax gates that weigh historical context against the current block, which
  is always retained.
* "SAS Learns Token Importance for Sparse Attention" (ai.viyan.live),
  section "The Logit Injection Mechanism": the selector output is added to the
  query-key logit before the softmax, so the loss gradient reaches the selector.

Equations (notation: block size ``bs``, query block r, key block c, historical
set H_r = {0..r-1}, attended historical set A_r, q-head h uses kv-head h // G):

  A_r  = H_r in training mode; the min(K, r) members of H_r with the largest
         S[r, c] in sparse mode (ties go to the lower index).
  log g[r, c] = S[r, c] - log sum_{c' in A_r} exp S[r, c']        (c in A_r)
  z_ij = scale * q_i . k_j + b_ij, with
         b_ij = log g[r(i), c(j)]  if c(j) in A_r(i)
              = 0                  if c(j) == r(i) and j <= i
              = -inf               otherwise
  O_i  = sum_j softmax_j(z_ij) v_j,       LSE_i = ln sum_j exp z_ij
  Backward (dO given):  P = softmax(z), dP = dO V^T, dZ = P o (dP - rowsum(P o dP)),
         dQ = scale dZ K, dK = scale dZ^T Q, dV = P^T dO (summed over the q-heads
         of a kv group), G[r, c] = sum_{i in r, j in c} dZ_ij,
         dS[r, c'] = G[r, c'] - g[r, c'] sum_{c in A_r} G[r, c]  for c' in A_r,
         0 elsewhere.
  Decode: one query at position L-1 of a cache of length L; its current block
         is floor((L-1)/bs); A is chosen from the score row S[b, h, :].
  Paged decode: sequence b's cache is its pages gathered by a block table and
         cut to its own length L_b, then decoded as above; group-shared
         selection gives every q-head of a kv group that group's score row.

Options that exist only to pin the oracle against textbook results:
``gate="ones"`` replaces every log-gate by 0 (dense causal attention over the
attended set) and ``renormalise=False`` keeps training-mode gates (normalised
over all of H_r) in sparse mode.

Parity pins (see tests/test_oracle_pins.py): dense causal attention through
torch's SDPA; SDPA with an additive mask plus autograd for every gradient
including dS; the training normaliser slse against torch's masked log_softmax
and a constant-row closed form; central finite differences; gate rows summing to one; dS rows
summing to zero; shift invariance in S; Top-K against a brute-force rank count;
full-budget Top-K equal to training mode; a hand-derived closed form; decode
equal to the last row of sparse prefill; GQA equal to repeated KV heads; paged
decode equal to contiguous decode under a random page placement and per-length
truncation; group-shared selection equal to per-head selection on repeated rows.
No function here is parity-unpinned.
"""
from __future__ import annotations

import numpy as np

TRAIN = "train"
SPARSE = "sparse"
THRESHOLD = "threshold"


def _as_f64(x):
    return np.asarray(x, dtype=np.float64)


def _logsumexp(x):
    """ln sum exp over a 1-D float64 array, with the max subtracted first."""
    m = np.max(x)
    return m + np.log(np.sum(np.exp(x - m)))


def threshold_count(s_row, r, tau):
    """Number of blocks c < r whose training-mode gate g[r, c] is at least tau.

    The dynamic threshold of the viyan blog ("Implementation and Efficiency":
    only blocks above a threshold are computed) read on the normalised gate:
    S[r, c] - logsumexp(S[r, :r]) >= ln tau.
    """
    if r == 0:
        return 0
    s = _as_f64(s_row[:r])
    return int(np.sum(s - _logsumexp(s) >= np.log(tau)))


def attended_blocks(s_row, r, mode, topk, tau=None):
    """The historical set A_r of query block r (ascending block indices).

    Training mode keeps every earlier block (poster Abstract: all context units
    stay active during training). Sparse mode keeps a fixed budget of min(K, r)
    earlier blocks with the largest scores (poster Abstract: fixed attention
    budget; HF page Abstract: hard Top-K). Threshold mode keeps the blocks whose
    gate reaches tau, at most K of them (the largest scores first); since the
    passing blocks are exactly the highest-scoring ones, it is Top-K with
    K = min(topk, threshold_count). Ordering is score descending, then block
    index ascending; -0.0 and +0.0 compare equal.
    """
    if mode == TRAIN:
        return np.arange(r, dtype=np.int64)
    if mode not in (SPARSE, THRESHOLD):
        raise ValueError(f"unknown mode {mode!r}")
    if topk is None or topk < 0:
        raise ValueError("sparse and threshold modes need topk >= 0")
    k = min(int(topk), r)
    if mode == THRESHOLD:
        if tau is None or not (0.0 < tau <= 1.0):
            raise ValueError("threshold mode needs 0 < tau <= 1")
        k = min(k, threshold_count(s_row, r, tau))
    if k == 0:
        return np.zeros(0, dtype=np.int64)
    s = _as_f64(s_row[:r])
    cand = np.arange(r, dtype=np.int64)
    # np.lexsort sorts by the last key first: primary -s (descending s), then c.
    order = np.lexsort((cand, -s))
    return np.sort(order[:k])


def log_gates(s_row, A, r, renormalise=True, gate="log_softmax"):
    """log g[r, c] for c in A (aligned with A).

    Normalised softmax gates in log form (HF page Abstract; viyan blog,
    "Differentiable Budget Constraints"). Training mode normalises over H_r;
    sparse mode normalises over A_r unless ``renormalise`` is False, in which
    case the training-mode gates over all of H_r are kept.
    """
    if gate == "ones":
        return np.zeros(len(A), dtype=np.float64)
    if gate != "log_softmax":
        raise ValueError(f"unknown gate {gate!r}")
    if len(A) == 0:
        return np.zeros(0, dtype=np.float64)
    s = _as_f64(s_row)
    norm_set = A if renormalise else np.arange(r, dtype=np.int64)
    return s[A] - _logsumexp(s[norm_set])


def _query_block(Q, K, V, S, b, h, r, bs, N, G, mode, topk, scale, renormalise, gate, tau=None):
    """Keys, values, logits and bookkeeping of one (batch, q-head, query block)."""
    i0, i1 = r * bs, min((r + 1) * bs, N)
    A = attended_blocks(S[b, h, r], r, mode, topk, tau)
    lg = log_gates(S[b, h, r], A, r, renormalise, gate)
    kv = h // G
    cols = [np.arange(c * bs, (c + 1) * bs) for c in A]
    cols.append(np.arange(i0, i1))
    cols = np.concatenate(cols).astype(np.int64)
    bias = np.zeros((i1 - i0, len(cols)), dtype=np.float64)
    for a, c in enumerate(A):
        bias[:, a * bs:(a + 1) * bs] = lg[a]
    # current block: bias 0 with the causal mask j <= i
    nh = len(A) * bs
    qi = np.arange(i0, i1)[:, None]
    kj = cols[None, nh:]
    bias[:, nh:] = np.where(kj <= qi, 0.0, -np.inf)
    q = _as_f64(Q[b, h, i0:i1])
    k = _as_f64(K[b, kv, cols])
    v = _as_f64(V[b, kv, cols])
    z = scale * (q @ k.T) + bias
    return A, lg, cols, q, k, v, z, (i0, i1), kv


def _softmax_rows(z):
    m = np.max(z, axis=1, keepdims=True)
    p = np.exp(z - m)
    l = np.sum(p, axis=1, keepdims=True)
    return p / l, (m + np.log(l))[:, 0]


def _check_shapes(Q, K, V, S, bs):
    B, Hq, N, d = Q.shape
    Bk, Hkv, Nk, dk = K.shape
    if (Bk, Nk, dk) != (B, N, d) or V.shape != K.shape:
        raise ValueError("K and V must be [B, Hkv, N, d] matching Q")
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    Nb = -(-N // bs)
    if S.shape[:3] != (B, Hq, Nb) or S.shape[3] < Nb:
        raise ValueError("S must be [B, Hq, Nb, Nb]")
    return B, Hq, Hkv, N, d, Nb


def gated_attention_forward(Q, K, V, S, block, mode=TRAIN, topk=None, scale=None,
                            renormalise=True, gate="log_softmax", rows=None, tau=None):
    """Forward pass, blockwise: returns (O, LSE) in float64.

    Never forms the N x N matrix; each query block gathers the keys of
    A_r plus its own block (viyan blog, "Implementation and Efficiency": blocks
    are processed one at a time instead of materialising the full matrix).
    ``rows`` optionally restricts the work to a list of (b, h, r) triples;
    unvisited rows stay NaN.
    """
    B, Hq, Hkv, N, d, Nb = _check_shapes(Q, K, V, S, block)
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    O = np.full((B, Hq, N, d), np.nan)
    LSE = np.full((B, Hq, N), np.nan)
    todo = rows if rows is not None else [(b, h, r) for b in range(B) for h in range(Hq) for r in range(Nb)]
    for b, h, r in todo:
        *_, v, z, (i0, i1), _ = _query_block(Q, K, V, S, b, h, r, block, N, G, mode, topk,
                                             scale, renormalise, gate, tau)
        p, lse = _softmax_rows(z)
        O[b, h, i0:i1] = p @ v
        LSE[b, h, i0:i1] = lse
    return O, LSE


def gated_attention_backward(Q, K, V, S, dO, block, mode=TRAIN, topk=None, scale=None,
                             renormalise=True, gate="log_softmax", heads=None, tau=None):
    """Backward pass: returns (dQ, dK, dV, dS, Gsum) in float64.

    The gradient reaches the scores because they sit inside the softmax
    (viyan blog, "The Logit Injection Mechanism"). dS follows the chain rule
    through the gate softmax: dS[r, c'] = G[r, c'] - g[r, c'] * sum_c G[r, c]
    over the attended historical set (the direct form, not a shortcut).
    ``heads`` restricts the work to a list of (b, kv_head) groups; the other
    entries stay NaN. Gsum is the per-(r, c) sum of dZ (c in A_r and c = r).
    """
    B, Hq, Hkv, N, d, Nb = _check_shapes(Q, K, V, S, block)
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    dQ = np.full((B, Hq, N, d), np.nan)
    dK = np.full((B, Hkv, N, d), np.nan)
    dV = np.full((B, Hkv, N, d), np.nan)
    dS = np.full(S.shape, np.nan)
    Gsum = np.full((B, Hq, Nb, Nb), np.nan)
    groups = heads if heads is not None else [(b, g) for b in range(B) for g in range(Hkv)]
    for b, g in groups:
        dK[b, g] = 0.0
        dV[b, g] = 0.0
        for h in range(g * G, (g + 1) * G):
            dS[b, h] = 0.0
            Gsum[b, h] = 0.0
            for r in range(Nb):
                A, lg, cols, q, k, v, z, (i0, i1), kv = _query_block(
                    Q, K, V, S, b, h, r, block, N, G, mode, topk, scale, renormalise, gate, tau)
                p, _ = _softmax_rows(z)
                do = _as_f64(dO[b, h, i0:i1])
                dp = do @ v.T
                dz = p * (dp - np.sum(p * dp, axis=1, keepdims=True))
                dQ[b, h, i0:i1] = scale * (dz @ k)
                # cols holds distinct key positions, so fancy-index += adds once each
                dK[b, kv, cols] += scale * (dz.T @ q)
                dV[b, kv, cols] += p.T @ do
                gs = np.array([dz[:, a * block:(a + 1) * block].sum() for a in range(len(A))])
                Gsum[b, h, r, A] = gs
                Gsum[b, h, r, r] = dz[:, len(A) * block:].sum()
                if gate == "ones" or len(A) == 0:
                    continue
                if renormalise or mode == TRAIN:
                    g_att = np.exp(lg)
                    dS[b, h, r, A] = gs - g_att * gs.sum()
                else:
                    # gates normalised over all of H_r, only A_r attended
                    Hr = np.arange(r)
                    g_full = np.exp(_as_f64(S[b, h, r, :r]) - _logsumexp(_as_f64(S[b, h, r, :r])))
                    dS[b, h, r, A] += gs
                    dS[b, h, r, Hr] -= g_full * gs.sum()
    return dQ, dK, dV, dS, Gsum


def gated_attention_naive(Q, K, V, S, block, mode=TRAIN, topk=None, scale=None,
                          renormalise=True, gate="log_softmax", tau=None):
    """Forward pass with the full N x N logit matrix per head (tiny inputs only).

    Returns (O, LSE, bias) with the token-level bias matrix [B, Hq, N, N].
    """
    B, Hq, Hkv, N, d, Nb = _check_shapes(Q, K, V, S, block)
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    O = np.zeros((B, Hq, N, d))
    LSE = np.zeros((B, Hq, N))
    bias = np.full((B, Hq, N, N), -np.inf)
    for b in range(B):
        for h in range(Hq):
            for i in range(N):
                r = i // block
                A = attended_blocks(S[b, h, r], r, mode, topk, tau)
                lg = log_gates(S[b, h, r], A, r, renormalise, gate)
                for a, c in enumerate(A):
                    bias[b, h, i, c * block:(c + 1) * block] = lg[a]
                for j in range(r * block, i + 1):
                    bias[b, h, i, j] = 0.0
            z = scale * (_as_f64(Q[b, h]) @ _as_f64(K[b, h // G]).T) + bias[b, h]
            p, lse = _softmax_rows(z)
            O[b, h] = p @ _as_f64(V[b, h // G])
            LSE[b, h] = lse
    return O, LSE, bias


def select_blocks(S, block_count, topk, mode=SPARSE, tau=None):
    """Index-list form of A_r for every (b, h, r): (idx, cnt, logg, slse).

    idx [B, H, Nb, K] int32 ascending, padded with -1; cnt [B, H, Nb] int32;
    logg [B, H, Nb, K] float64 (0 in padding); slse [B, H, Nb] the log-sum-exp
    of S over H_r (training-mode normaliser; -inf when r = 0). In training mode
    K is taken as Nb - 1 so the list holds all of H_r.
    """
    S = np.asarray(S)
    B, H, Nb = S.shape[:3]
    assert Nb == block_count
    K = (Nb - 1) if mode == TRAIN else int(topk)
    idx = np.full((B, H, Nb, max(K, 0)), -1, dtype=np.int32)
    cnt = np.zeros((B, H, Nb), dtype=np.int32)
    logg = np.zeros((B, H, Nb, max(K, 0)), dtype=np.float64)
    slse = np.full((B, H, Nb), -np.inf)
    for b in range(B):
        for h in range(H):
            for r in range(Nb):
                A = attended_blocks(S[b, h, r], r, mode, K, tau)
                cnt[b, h, r] = len(A)
                idx[b, h, r, :len(A)] = A
                logg[b, h, r, :len(A)] = log_gates(S[b, h, r], A, r)
                if r > 0:
                    slse[b, h, r] = _logsumexp(_as_f64(S[b, h, r, :r]))
    return idx, cnt, logg, slse


def gated_decode(q, Kc, Vc, S_dec, L, block, topk, scale=None, seqs=None, gate="log_softmax",
                 mode=SPARSE, tau=None):
    """Sparse decode of one query per sequence: returns (O [B,Hq,d], LSE [B,Hq]).

    The query sits at position L-1 (HF page Abstract: the current block is
    always retained; poster Abstract: a fixed budget of context units per query
    at inference). Its current block cur = floor((L-1)/bs) is attended up to
    position L-1 with bias 0; the historical blocks are the Top-K of
    S_dec[b, h, :cur] with gates renormalised over the selection.
    ``seqs`` restricts the work to a list of batch indices (others NaN).
    """
    B, Hq, d = q.shape
    Hkv = Kc.shape[1]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    cur = (L - 1) // block
    O = np.full((B, Hq, d), np.nan)
    LSE = np.full((B, Hq), np.nan)
    for b in (seqs if seqs is not None else range(B)):
        for h in range(Hq):
            A = attended_blocks(S_dec[b, h], cur, mode, topk, tau)
            lg = log_gates(S_dec[b, h], A, cur, True, gate)
            cols = [np.arange(c * block, (c + 1) * block) for c in A]
            cols.append(np.arange(cur * block, L))
            cols = np.concatenate(cols).astype(np.int64)
            bias = np.concatenate([np.repeat(lg, block), np.zeros(L - cur * block)])
            k = _as_f64(Kc[b, h // G, cols])
            v = _as_f64(Vc[b, h // G, cols])
            z = scale * (k @ _as_f64(q[b, h])) + bias
            m = np.max(z)
            p = np.exp(z - m)
            l = np.sum(p)
            O[b, h] = (p / l) @ v
            LSE[b, h] = m + np.log(l)
    return O, LSE


def gated_decode_paged(q, Kpool, Vpool, block_table, seq_lens, S_dec, block, topk, scale=None,
                       group_shared=False, mode=SPARSE, tau=None, seqs=None):
    """Decode over a paged, variable-length KV cache: returns (O [B,Hq,d], LSE [B,Hq]).

    A serving-side layout of the decode above (the pages' long-context
    inference setting; the layout itself is not on the pages): the cache of
    sequence b is the concatenation of pages Kpool[block_table[b, c]] for its
    blocks c = 0 .. ceil(L_b / bs) - 1, truncated to its own length
    L_b = seq_lens[b]; each page holds one context block of every kv head,
    Kpool [num_pages, Hkv, bs, d]. With ``group_shared`` the G q-heads of a kv
    group share one score row and so one selection: S_dec is [B, Hkv, Nb] and
    q-head h reads row h // G. Every sequence is then decoded exactly as
    gated_decode does it at its own length.
    """
    B, Hq, d = q.shape
    Hkv = Kpool.shape[1]
    G = Hq // Hkv
    O = np.full((B, Hq, d), np.nan)
    LSE = np.full((B, Hq), np.nan)
    for b in (seqs if seqs is not None else range(B)):
        L = int(seq_lens[b])
        nb = -(-L // block)
        pages = [int(block_table[b, c]) for c in range(nb)]
        Kc = np.concatenate([_as_f64(Kpool[pg]) for pg in pages], axis=1)[:, :L]
        Vc = np.concatenate([_as_f64(Vpool[pg]) for pg in pages], axis=1)[:, :L]
        rows = _as_f64(S_dec[b])
        if group_shared:
            rows = np.repeat(rows, G, axis=0)
        o, lse = gated_decode(q[b:b + 1], Kc[None], Vc[None], rows[None, :, :nb], L, block, topk,
                              scale=scale, mode=mode, tau=tau)
        O[b], LSE[b] = o[0], lse[0]
    return O, LSE


def attended_pairs(S, N, block, mode=TRAIN, topk=None, tau=None):
    """Number of attended (i, j) pairs per (b, h): the FLOP-count basis.

    A historical block contributes bs*bs pairs; the current block the causal
    triangle of its rows.
    """
    B, H, Nb = S.shape[:3]
    out = np.zeros((B, H), dtype=np.int64)
    for b in range(B):
        for h in range(H):
            tot = 0
            for r in range(Nb):
                rows = min(N, (r + 1) * block) - r * block
                A = attended_blocks(S[b, h, r], r, mode, topk, tau)
                tot += len(A) * block * rows + rows * (rows + 1) // 2
            out[b, h] = tot
    return out
