"""fp64 oracle: exact attention written out from its definition.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``): nothing on the product
path imports this module.

What it computes, for every (b, h) independently, with every intermediate
materialised (this is the "standard attention" the pages contrast with the
fused kernel, [Concept] "How it works", first paragraph):

    S = scale * Q K^T                      (N x N)     [Concept] "How it works"
    S_ij = -inf for j > i   (causal)                    reading: key j visible iff j <= i
    m_i  = max_j S_ij                                   [Librarian] online softmax, eq. 1
    l_i  = sum_j exp(S_ij - m_i)                        [Librarian] online softmax, eq. 1
    P    = exp(S - m) / l                               [Librarian] online softmax, eq. 1
    O    = P V                                          [Concept] "How it works"
    L_i  = m_i + ln l_i                                 [Concept] "How it works" (logsumexp)

The fused kernel reaches the same O and L up to rounding: the pages state that
the online form is exact and that FlashAttention does not change the
mathematics of attention ([Librarian] "Why standard attention was the
bottleneck" and "The trick that made it all possible: online softmax").

The backward pass is not written out on the pages, which only fix that P is
recomputed from L ([Concept] "How it works"; [Lineage] "FA1 (2022)", idea 3).
The oracle therefore uses the textbook gradient of the definition above with
respect to the loss sum(O * dO):

    dV = P^T dO
    dP = dO V^T
    D_i = sum_j P_ij dP_ij          (= sum_d dO_id O_id; both are returned)
    dS = P * (dP - D)
    dQ = scale * dS K
    dK = scale * dS^T Q

Pins (``tests/test_oracle_attention.py``): brute-force scalar loops, torch fp64
SDPA and autograd on CPU, central finite differences, rows of P summing to 1,
N = 1 giving O = V, identical keys giving the mean of V, scale = 0 closed
forms, permutation and shift invariances, and the hand-worked fixture in
``tests/golden/attn_tiny_handworked.txt``.
"""
from __future__ import annotations

from typing import Optional, NamedTuple, Sequence

import numpy as np


def _as_f64(x) -> np.ndarray:
    """Exact conversion of a numpy array or a (CPU) torch tensor to fp64.

    bf16 -> fp64 is exact, so the oracle sees precisely the values the GPU
    path is given.
    """
    if hasattr(x, "detach"):  # torch tensor (bf16 has no numpy dtype)
        import torch

        return x.detach().to(device="cpu", dtype=torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def causal_mask(n_q: int, n_k: int) -> np.ndarray:
    """Boolean mask, True where key j is visible to query i (j <= i).

    The pages name causal masking without defining its alignment ([Librarian]
    "Cases where FlashAttention does not help": FA ships causal, sliding
    window and ALiBi).  Reading: with N_q = N_k, key j is visible to query i
    iff j <= i, so no row is ever fully masked.
    """
    i = np.arange(n_q)[:, None]
    j = np.arange(n_k)[None, :]
    return j <= i


def window_mask(n_q: int, n_k: int, window: int) -> np.ndarray:
    """Causal sliding window: True where i - window <= j <= i.

    The librarian page names sliding-window masks among those FA ships
    ("Cases where FlashAttention does not help") without a formula; the
    reading is the left window of the causal mask, ``window`` keys before the
    query plus the query's own key.
    """
    i = np.arange(n_q)[:, None]
    j = np.arange(n_k)[None, :]
    return (j <= i) & (j >= i - window)


def softmax_ref(x: np.ndarray) -> np.ndarray:
    """Safe (max-subtracted) softmax along the last axis, fp64.

    [Librarian] "The trick that made it all possible: online softmax", eq. 1:
    softmax(x_i) = e^{x_i - m} / sum_j e^{x_j - m},  m = max_j x_j.
    Entries equal to -inf get probability 0.
    """
    x = np.asarray(x, dtype=np.float64)
    m = np.max(x, axis=-1, keepdims=True)
    e = np.exp(x - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def scores_ref(q2: np.ndarray, k2: np.ndarray, scale: float, causal: bool) -> np.ndarray:
    """S = scale * Q K^T for one (b, h), with -inf where the causal mask hides a key."""
    s = float(scale) * (q2 @ k2.T)
    if causal:
        s = np.where(causal_mask(q2.shape[0], k2.shape[0]), s, -np.inf)
    return s


def attn_fwd_ref(q, k, v, scale: float, causal: bool):
    """Exact attention forward.  q, k, v: [B, H, N, d].  Returns (O, L).

    O has shape [B, H, N, d], L (the natural-log logsumexp of the scaled,
    masked scores, [Concept] "How it works") has shape [B, H, N]; both fp64.
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    B, H, N, d = q.shape
    o = np.zeros((B, H, N, v.shape[-1]), dtype=np.float64)
    lse = np.zeros((B, H, N), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            s = scores_ref(q[b, h], k[b, h], scale, causal)
            m = np.max(s, axis=1)                       # row max
            ell = np.sum(np.exp(s - m[:, None]), axis=1)  # row normaliser
            p = np.exp(s - m[:, None]) / ell[:, None]     # eq. 1
            o[b, h] = p @ v[b, h]
            lse[b, h] = m + np.log(ell)
    return o, lse


def attn_fwd_rows_ref(q, k, v, scale: float, causal: bool, rows, window=None):
    """The forward definition for selected query rows of one head.

    q, k, v: [N, d] (one head); ``rows``: query indices.  Row i sees keys
    j <= i when causal (and j >= i - window with a sliding window).  Returns
    (O [len(rows), d], L [len(rows)]), fp64.  Used where a whole head is too
    large to materialise (N up to 16K).
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    rows = np.asarray(rows, dtype=np.int64)
    o = np.zeros((rows.size, v.shape[1]))
    lse = np.zeros(rows.size)
    for n, i in enumerate(rows):
        lo = 0 if window is None else max(0, i - window)
        kk, vv = (k[lo: i + 1], v[lo: i + 1]) if causal else (k, v)
        srow = float(scale) * (kk @ q[i])
        m = np.max(srow)
        e = np.exp(srow - m)
        o[n] = (e / e.sum()) @ vv
        lse[n] = m + np.log(e.sum())
    return o, lse


class BwdResult(NamedTuple):
    dq: np.ndarray
    dk: np.ndarray
    dv: np.ndarray
    delta_from_p: np.ndarray   # D_i = sum_j P_ij dP_ij
    delta_from_o: np.ndarray   # D_i = sum_d dO_id O_id


def attn_bwd_ref(q, k, v, do, scale: float, causal: bool) -> BwdResult:
    """Exact attention backward for the loss sum(O * dO); q, k, v, do: [B, H, N, d].

    P is rebuilt from the logsumexp, P = exp(S - L), as the pages describe for
    the recomputing backward ([Concept] "How it works"); L itself comes from
    the definition in ``attn_fwd_ref``.
    """
    q, k, v, do = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(do)
    B, H, N, d = q.shape
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    d_p = np.zeros((B, H, N))
    d_o = np.zeros((B, H, N))
    o, lse = attn_fwd_ref(q, k, v, scale, causal)
    for b in range(B):
        for h in range(H):
            s = scores_ref(q[b, h], k[b, h], scale, causal)
            p = np.exp(s - lse[b, h][:, None])
            dv[b, h] = p.T @ do[b, h]
            dp = do[b, h] @ v[b, h].T
            delta = np.sum(p * dp, axis=1)
            d_p[b, h] = delta
            d_o[b, h] = np.sum(do[b, h] * o[b, h], axis=1)
            ds = p * (dp - delta[:, None])
            dq[b, h] = float(scale) * (ds @ k[b, h])
            dk[b, h] = float(scale) * (ds.T @ q[b, h])
    return BwdResult(dq, dk, dv, d_p, d_o)


def online_softmax_ref(x, block_sizes: Sequence[int]):
    """The online normaliser recurrence over a 1-D score vector, fp64.

    [Librarian] "The trick that made it all possible: online softmax", eq. 2:
    for each new block with local maximum m_new,
        m^(t+1) = max(m^(t), m_new)
        l^(t+1) = e^{m^(t) - m^(t+1)} l^(t) + sum_{j in block} e^{x_j - m^(t+1)}
    starting from m = -inf, l = 0.  ``block_sizes`` splits x into consecutive
    blocks (they must sum to len(x)).  Returns (m, l, softmax) where softmax is
    e^{x - m} / l with the final (m, l).
    """
    x = np.asarray(x, dtype=np.float64).ravel()
    if sum(block_sizes) != x.size:
        raise ValueError("block sizes must cover x exactly")
    m, ell = -np.inf, 0.0
    start = 0
    for bs in block_sizes:
        blk = x[start:start + bs]
        start += bs
        if blk.size == 0:
            continue
        m_next = max(m, float(np.max(blk)))
        if m_next == -np.inf:          # everything so far masked: state unchanged
            continue
        alpha = 0.0 if m == -np.inf else np.exp(m - m_next)
        ell = alpha * ell + float(np.sum(np.exp(blk - m_next)))
        m = m_next
    return m, ell, np.exp(x - m) / ell


def attn_fwd_online_ref(q, k, v, scale: float, causal: bool, block_sizes: Sequence[int],
                        tau_log2: float = 0.0, stats: Optional[dict] = None):
    """Attention for one head with K/V streamed in blocks, fp64.

    This is the algorithm the pages describe ([Concept] "How it works",
    second paragraph; [Librarian] online softmax section): for each query
    row, stream the K/V blocks, update the running (m, l) with eq. 2, rescale
    the running output o by the same factor e^{m_old - m_new} and add the new
    block's e^{S - m_new} V; after the last block divide by l once (deferred
    normalisation, [Lineage] "FA2 (2023)", refinement 2) and emit L = m + ln l.

    ``tau_log2`` > 0 is the conditional rescale ([Librarian] "FA4", idea 2;
    [Lineage] "FA4 (2026)", change 2), in the reading that the pages leave
    open: the running max moves only when a block's max exceeds it by more
    than tau (log2 units, i.e. by a factor 2^tau); until then the stale max
    is used for p, l, o and L alike, so p <= 2^tau and the result is the
    same up to rounding.  ``stats``, if given, receives the number of
    rescales and the largest p used.

    q: [N_q, d], k and v: [N_k, d].  Returns (O [N_q, d], L [N_q]).
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    if sum(block_sizes) != k.shape[0]:
        raise ValueError("block sizes must cover the keys exactly")
    s_full = scores_ref(q, k, scale, causal)
    n_q = q.shape[0]
    o = np.zeros((n_q, v.shape[1]))
    lse = np.zeros(n_q)
    tau = float(tau_log2) * np.log(2.0)       # the threshold in the natural-log units of S
    rescales, p_max = 0, 0.0
    for i in range(n_q):
        m, ell = -np.inf, 0.0
        acc = np.zeros(v.shape[1])
        start = 0
        for bs in block_sizes:
            s_blk = s_full[i, start:start + bs]
            v_blk = v[start:start + bs]
            start += bs
            if s_blk.size == 0:
                continue
            m_blk = float(np.max(s_blk))
            if m_blk == -np.inf and m == -np.inf:
                continue
            alpha = 1.0
            if m == -np.inf or m_blk > m + tau:   # move the running max
                alpha = 0.0 if m == -np.inf else np.exp(m - m_blk)
                m = m_blk
                rescales += 1
            p_blk = np.exp(s_blk - m)
            p_max = max(p_max, float(np.max(p_blk)))
            ell = alpha * ell + float(np.sum(p_blk))
            acc = alpha * acc + p_blk @ v_blk
        o[i] = acc / ell
        lse[i] = m + np.log(ell)
    if stats is not None:
        stats["rescales"], stats["p_max"] = rescales, p_max
    return o, lse


def alibi_bias(n_q: int, n_k: int, slope: float) -> np.ndarray:
    """ALiBi bias -slope * |i - j| added to the scaled scores.

    The librarian page names ALiBi among the masks FA ships ("Cases where
    FlashAttention does not help") without a formula; the reading is the
    linear distance penalty of the ALiBi method, one non-negative slope per
    query head, in the units of the scaled scores (natural log).  With the
    causal mask |i - j| = i - j on every visible pair.
    """
    i = np.arange(n_q)[:, None]
    j = np.arange(n_k)[None, :]
    return -float(slope) * np.abs(i - j)


def _scores_window(q2, k2, scale, causal, window, slope=None):
    s = scores_ref(q2, k2, scale, causal)
    if window is not None:
        s = np.where(window_mask(q2.shape[0], k2.shape[0], window), s, -np.inf)
    if slope is not None:
        s = s + alibi_bias(q2.shape[0], k2.shape[0], slope)
    return s


def attn_fwd_gqa_ref(q, k, v, scale: float, causal: bool, window=None, alibi=None):
    """Attention with grouped K/V heads, fp64.  q: [B, H, N, d]; k, v: [B, H_kv, N, d].
    ``window`` (causal only): the sliding window of ``window_mask``;
    ``alibi``: H slopes, the bias of ``alibi_bias`` for query head h.

    The librarian page lists GQA/MQA among the variants FlashAttention
    supports ("Cases where FlashAttention does not help") without a formula;
    the reading used: query head h of batch b uses K/V head h // G, G = H / H_kv.
    Each query head is then plain attention (``attn_fwd_ref``'s definition).
    Returns (O [B, H, N, d], L [B, H, N]).
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    B, H, N, d = q.shape
    h_kv = k.shape[1]
    if H % h_kv:
        raise ValueError("H must be a multiple of H_kv")
    g = H // h_kv
    o = np.zeros((B, H, N, v.shape[-1]))
    lse = np.zeros((B, H, N))
    for b in range(B):
        for h in range(H):
            kk, vv = k[b, h // g], v[b, h // g]
            s = _scores_window(q[b, h], kk, scale, causal, window, None if alibi is None else alibi[h])
            m = np.max(s, axis=1)
            e = np.exp(s - m[:, None])
            ell = np.sum(e, axis=1)
            o[b, h] = (e / ell[:, None]) @ vv
            lse[b, h] = m + np.log(ell)
    return o, lse


def attn_bwd_gqa_ref(q, k, v, do, scale: float, causal: bool, window=None, alibi=None):
    """Gradients of sum(O * dO) for grouped K/V heads, fp64.

    dQ of head h is that of plain attention with K/V head h // G; since a
    K/V head feeds G query heads, its dK and dV are the sums of the G heads'
    gradients (the chain rule over the shared input).  Returns (dq, dk, dv)
    with dk, dv of shape [B, H_kv, N, d].
    """
    q, k, v, do = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(do)
    B, H, N, d = q.shape
    h_kv = k.shape[1]
    g = H // h_kv
    _, lse = attn_fwd_gqa_ref(q, k, v, scale, causal, window, alibi)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    for b in range(B):
        for h in range(H):
            kk, vv = k[b, h // g], v[b, h // g]
            p = np.exp(_scores_window(q[b, h], kk, scale, causal, window,
                                      None if alibi is None else alibi[h]) - lse[b, h][:, None])
            dp = do[b, h] @ vv.T
            ds = p * (dp - np.sum(p * dp, axis=1)[:, None])
            dq[b, h] = float(scale) * (ds @ kk)
            dk[b, h // g] += float(scale) * (ds.T @ q[b, h])
            dv[b, h // g] += p.T @ do[b, h]
    return dq, dk, dv
