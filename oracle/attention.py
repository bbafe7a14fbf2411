"""fp64 CPU oracle for exact scaled-dot-product attention, forward and backward.

TEST INFRASTRUCTURE ONLY.  This module is the slow, plainly written reference that the CUDA path is
checked against.  Only the tests, ``__graft_entry__.smoke()`` and the bench's CPU-baseline leg may
import it; the library never does, and it imports nothing from the library.

Sources (web pages on FlashAttention; cited by page title and section):
  [P1] robocikowo.com "Flash Attention" -- algorithm summary (tile loop, running max m and sum l,
       the update O <- rescale(O_prev, m_old, m_new) + exp(S_new - m_new) V_j), the backward
       "recomputes from the saved O and L (logsumexp)", and "exact attention ... modulo causal mask".
  [P2] systems-analysis.info "FlashAttention (PL)" -- section "Problematyka standardowego
       mechanizmu uwagi": Attention(Q,K,V) = softmax(Q K^T / sqrt(d_k)) V; section "Obliczanie
       Softmax w trybie online": two running values (maximum and sum of exponentials).
  [P3] chipfoundryservices.com glossary "Flash Attention" -- the definition, and "Tiling
       Algorithm" steps 1-6; "Online Softmax Trick".
  [P4] dexblog.ro "FlashAttention" -- table row "Softmax online": the blockwise softmax gives an
       identical result.

Readings where the pages are silent (each also listed in the design notes):
  * L is the natural-log logsumexp of the *scaled* scores, one fp32 value per query row.
  * Causal: query i sees keys j <= i (N_q = N_k, so top-left and bottom-right alignment agree).
  * The backward is not spelled out on the pages beyond "recompute P from O and L"; it is taken as
    the exact gradient of the definition: dV = P^T dO, dP = dO V^T, D = rowsum(dO * O),
    dS = P * (dP - D), dQ = s dS K, dK = s dS^T Q, with P recomputed as exp(s Q K^T - L).

Every function works in float64 on whatever values it is given (callers widen the bf16 inputs
exactly).  Arrays are [B, H, N, d]; L and D are [B, H, N].
"""
from __future__ import annotations

import os

import numpy as np


def _scores(q: np.ndarray, k: np.ndarray, scale: float, causal: bool) -> np.ndarray:
    """S = scale * q k^T for one head, with -inf above the diagonal when causal.

    Definition of the scores: [P2] "Problematyka standardowego mechanizmu uwagi", [P3] first
    paragraph; causal mask: [P1] "modulo causal mask".
    """
    s = scale * (q @ k.T)
    if causal:
        nq, nk = s.shape
        s = s.copy()
        s[np.triu_indices(nq, k=1, m=nk)] = -np.inf
    return s


def attention_forward(q, k, v, causal: bool, scale: float):
    """Two-pass (standard) attention: O = softmax(S) V and L = logsumexp(S), per head.

    This is the plain definition ([P2] formula, [P3] "Standard attention computes"): form S,
    subtract the row max, exponentiate, normalise by the row sum, multiply by V.
    Returns (O [B,H,N,d] float64, L [B,H,N] float64).
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    B, H, N, d = q.shape
    O = np.empty((B, H, N, v.shape[-1]))
    L = np.empty((B, H, N))
    for b in range(B):
        for h in range(H):
            s = _scores(q[b, h], k[b, h], scale, causal)
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            l = e.sum(axis=1, keepdims=True)
            O[b, h] = (e / l) @ v[b, h]
            L[b, h] = (m + np.log(l))[:, 0]
    return O, L


def attention_probs(q, k, causal: bool, scale: float):
    """P = softmax(S) for every head, [B,H,N,N] float64 (small inputs only; used by the pins)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    B, H, N, _ = q.shape
    P = np.empty((B, H, N, k.shape[2]))
    for b in range(B):
        for h in range(H):
            s = _scores(q[b, h], k[b, h], scale, causal)
            e = np.exp(s - s.max(axis=1, keepdims=True))
            P[b, h] = e / e.sum(axis=1, keepdims=True)
    return P


def _block_summary(s_blk, v_blk):
    """Softmax statistics of one block of keys for a block of query rows: the row max m, the sum
    of exponentials l = sum_j exp(s_j - m) and the unnormalised output u = sum_j exp(s_j - m) v_j.

    A row whose scores in this block are all -inf (every key masked) has no maximum; it gets
    m = -inf, l = 0 and u = 0, the identity of the combination below.
    """
    m = s_blk.max(axis=1)
    seen = np.isfinite(m)
    e = np.exp(s_blk - np.where(seen, m, 0.0)[:, None])
    return m, e.sum(axis=1), e @ v_blk


def _combine(a, b):
    """Merge the statistics of two disjoint key sets ([P1] rescale(O_prev, m_old, m_new); [P3]
    "Online Softmax Trick"): move both onto the larger maximum and add.  The operation is
    associative and commutative, so any grouping of the key blocks gives the same softmax."""
    (m1, l1, u1), (m2, l2, u2) = a, b
    m = np.maximum(m1, m2)
    ref = np.where(np.isfinite(m), m, 0.0)
    w1 = np.where(np.isfinite(m1), np.exp(m1 - ref), 0.0)
    w2 = np.where(np.isfinite(m2), np.exp(m2 - ref), 0.0)
    return m, w1 * l1 + w2 * l2, w1[:, None] * u1 + w2[:, None] * u2


def attention_forward_online(q, k, v, causal: bool, scale: float, block_r: int, block_c: int,
                             tree: bool = False):
    """The blockwise forward: the softmax of a row is assembled from per-block statistics.

    The keys are cut into blocks of ``block_c`` and the queries into blocks of ``block_r``
    ([P3] "Tiling Algorithm"; [P1]: a Q block against every K, V block).  For each (query block,
    key block) pair the scores exist only for that pair; their summary (row max m, exponential
    sum l, unnormalised output u, see ``_block_summary``) is folded into the running summary by
    ``_combine`` ([P1] rescale rule; [P2] "Obliczanie Softmax w trybie online": the two running
    values).  Left to right (``tree=False``) this is the running recurrence; ``tree=True`` merges
    the block summaries pairwise instead, which associativity says must give the same result.
    Finally O = u / l and L = m + ln l ([P1]: L is kept for the backward).
    Masked entries are -inf and contribute exp(-inf) = 0.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    B, H, N, d = q.shape
    Nk = k.shape[2]
    O = np.empty((B, H, N, v.shape[-1]))
    L = np.empty((B, H, N))
    for b in range(B):
        for h in range(H):
            for r0 in range(0, N, block_r):
                r1 = min(N, r0 + block_r)
                parts = []
                for c0 in range(0, Nk, block_c):
                    c1 = min(Nk, c0 + block_c)
                    s = scale * (q[b, h, r0:r1] @ k[b, h, c0:c1].T)
                    if causal:
                        hidden = np.arange(c0, c1)[None, :] > np.arange(r0, r1)[:, None]
                        s = np.where(hidden, -np.inf, s)
                    parts.append(_block_summary(s, v[b, h, c0:c1]))
                if tree:
                    while len(parts) > 1:
                        nxt = [_combine(parts[i], parts[i + 1])
                               for i in range(0, len(parts) - 1, 2)]
                        if len(parts) % 2:
                            nxt.append(parts[-1])
                        parts = nxt
                    m, l, u = parts[0]
                else:
                    m, l, u = parts[0]
                    for part in parts[1:]:
                        m, l, u = _combine((m, l, u), part)
                O[b, h, r0:r1] = u / l[:, None]
                L[b, h, r0:r1] = m + np.log(l)
    return O, L


def attention_backward(q, k, v, o, lse, do, causal: bool, scale: float):
    """Gradients dQ, dK, dV of the loss whose upstream gradient at O is dO.

    P is recomputed from the saved logsumexp ([P1]: the backward recomputes the attention matrix
    from O and L instead of storing it): P = exp(S - L).  Then, per head,
      dV = P^T dO,  dP = dO V^T,  D_i = sum_c dO_ic O_ic,  dS = P * (dP - D),
      dQ = scale * dS K,  dK = scale * dS^T Q.
    ``o`` and ``lse`` are the forward's outputs (this oracle passes its own fp64 ones).
    Returns (dQ, dK, dV) as float64 arrays shaped like q, k, v.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    o = np.asarray(o, np.float64)
    lse = np.asarray(lse, np.float64)
    do = np.asarray(do, np.float64)
    B, H, N, d = q.shape
    dq = np.empty_like(q)
    dk = np.empty_like(k)
    dv = np.empty_like(v)
    for b in range(B):
        for h in range(H):
            s = _scores(q[b, h], k[b, h], scale, causal)
            p = np.exp(s - lse[b, h][:, None])
            dv[b, h] = p.T @ do[b, h]
            dp = do[b, h] @ v[b, h].T
            D = np.sum(do[b, h] * o[b, h], axis=1)
            ds = p * (dp - D[:, None])
            dq[b, h] = scale * (ds @ k[b, h])
            dk[b, h] = scale * (ds.T @ q[b, h])
    return dq, dk, dv


def attention_rows(q, k, v, rows, causal: bool, scale: float):
    """Forward outputs of selected query rows of ONE head (q, k, v: [N, d] arrays).

    A row of the definition needs only its own scores against all keys ([P2], [P3] formula), so
    sampled rows of very long sequences are computed exactly without the N x N matrix.
    Returns (O_rows [len(rows), d], L_rows [len(rows)]).
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    rows = np.asarray(rows)
    # causal: keys after the last requested row are hidden from every one of them (they would
    # contribute exp(-inf) = 0), so they are left out of the products
    nk = min(k.shape[0], int(rows.max()) + 1) if causal else k.shape[0]
    s = scale * (q[rows] @ k[:nk].T)
    if causal:
        s = np.where(np.arange(nk)[None, :] > rows[:, None], -np.inf, s)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    return (e / l) @ v[:nk], (m + np.log(l))[:, 0]


def attention_dq_rows(q, k, v, do, rows, causal: bool, scale: float):
    """dQ of selected query rows of ONE head: dQ_i = scale * sum_j P_ij (dP_ij - D_i) k_j with
    dP_ij = dO_i . v_j and D_i = dO_i . O_i -- row i needs only its own P row and O row."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    do = np.asarray(do, np.float64)
    rows = np.asarray(rows)
    O, L = attention_rows(q, k, v, rows, causal, scale)
    s = scale * (q[rows] @ k.T)
    if causal:
        s = np.where(np.arange(k.shape[0])[None, :] > rows[:, None], -np.inf, s)
    p = np.exp(s - L[:, None])
    dp = do[rows] @ v.T
    D = np.sum(do[rows] * O, axis=1)
    ds = p * (dp - D[:, None])
    return scale * (ds @ k)


def attention_row_stats(q, k, v, do, causal: bool, scale: float, block: int = 256):
    """L_i and D_i = dO_i . O_i for EVERY query row of ONE head (q, k, v, do: [N, d] arrays).

    Each row needs its own scores against all keys only ([P2], [P3] formula), so the rows are
    taken ``block`` at a time and no N x N array is ever formed.  Returns (L [N], D [N]).
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    do = np.asarray(do, np.float64)
    N = q.shape[0]
    L = np.empty(N)
    D = np.empty(N)

    def one_block(r0):
        rows = np.arange(r0, min(N, r0 + block))
        O, L[rows] = attention_rows(q, k, v, rows, causal, scale)
        D[rows] = np.sum(do[rows] * O, axis=1)

    # the blocks are independent; numpy releases the interpreter lock inside its array
    # operations, so one thread per core (each with a single-threaded BLAS) keeps the host's cores
    # busy on long heads
    from concurrent.futures import ThreadPoolExecutor

    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=1), \
            ThreadPoolExecutor(max_workers=len(os.sched_getaffinity(0))) as ex:
        list(ex.map(one_block, range(0, N, block)))
    return L, D


def attention_dkdv_key_rows(q, k, v, do, keys, causal: bool, scale: float, stats=None):
    """dK and dV of selected KEY rows of ONE head (q, k, v, do: [N, d] arrays).

    Key j's gradients are column sums over the query rows that see it:
      dV_j = sum_i P_ij dO_i,  dK_j = scale * sum_i P_ij (dP_ij - D_i) q_i,
    with P_ij = exp(scale q_i . k_j - L_i) recomputed from the logsumexp ([P1]: the backward
    recomputes P from L), dP_ij = dO_i . v_j and D_i = dO_i . O_i.  L and D of all rows come from
    ``attention_row_stats`` (pass them as ``stats`` to reuse them).  Returns (dK [len(keys), d],
    dV [len(keys), d]).
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    do = np.asarray(do, np.float64)
    keys = np.asarray(keys)
    L, D = attention_row_stats(q, k, v, do, causal, scale) if stats is None else stats
    s = scale * (q @ k[keys].T)                                   # [N, len(keys)]
    p = np.exp(s - L[:, None])
    if causal:
        p = np.where(keys[None, :] > np.arange(q.shape[0])[:, None], 0.0, p)
    dv = p.T @ do
    dp = do @ v[keys].T
    ds = p * (dp - D[:, None])
    return scale * (ds.T @ q), dv


def _group_size(q, k):
    H, Hkv = q.shape[1], k.shape[1]
    if Hkv < 1 or H % Hkv:
        raise ValueError("the key/value head count must divide the query head count")
    return H // Hkv


def attention_forward_gqa(q, k, v, causal: bool, scale: float):
    """Grouped-query attention forward: q [B,H,N,d], k and v [B,H_kv,N,d] with H_kv dividing H.

    [P2] section "FlashAttention-2 (2023)" lists multi-query attention (one key/value head for all
    query heads) among the method's extensions; the grouped form lets query head h read key/value
    head h // (H // H_kv), consecutive groups of query heads sharing one.  Written as the plain
    definition: attention with each key/value head repeated for the query heads of its group.
    Returns (O [B,H,N,d], L [B,H,N]).
    """
    G = _group_size(q, k)
    k_rep = np.repeat(np.asarray(k, np.float64), G, axis=1)
    v_rep = np.repeat(np.asarray(v, np.float64), G, axis=1)
    return attention_forward(q, k_rep, v_rep, causal, scale)


def attention_backward_gqa(q, k, v, o, lse, do, causal: bool, scale: float):
    """Gradients of the grouped-query attention above.

    A shared key/value row enters the loss once per query head of its group, so its gradient is
    the sum of the per-head gradients: dK and dV of the repeated heads, summed over each group.
    Returns (dQ [B,H,N,d], dK [B,H_kv,N,d], dV [B,H_kv,N,d]).
    """
    G = _group_size(q, k)
    B, Hkv, N, d = k.shape
    k_rep = np.repeat(np.asarray(k, np.float64), G, axis=1)
    v_rep = np.repeat(np.asarray(v, np.float64), G, axis=1)
    dq, dk_rep, dv_rep = attention_backward(q, k_rep, v_rep, o, lse, do, causal, scale)
    dk = dk_rep.reshape(B, Hkv, G, N, d).sum(axis=2)
    dv = dv_rep.reshape(B, Hkv, G, N, v.shape[-1]).sum(axis=2)
    return dq, dk, dv


def attention_forward_rect(q, k, v, causal: bool, scale: float):
    """Attention of Nq queries against Nk keys per head: q [B,H,Nq,d], k and v [B,H_kv,Nk,d]
    (H_kv dividing H, query head h reading key/value head h // (H // H_kv)).

    The plain definition ([P2] "Problematyka standardowego mechanizmu uwagi", [P3] first
    paragraph) for rectangular score matrices.  Causal aligns the queries with the end of the
    keys: query i sees keys j <= i + Nk - Nq (a decoding step's last query sees every key); it
    needs Nq <= Nk so that every query sees at least one key.  Returns (O [B,H,Nq,d], L [B,H,Nq]).
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    G = _group_size(q, k)
    B, H, Nq, _ = q.shape
    Nk = k.shape[2]
    if causal and Nq > Nk:
        raise ValueError("causal attention needs Nq <= Nk")
    O = np.empty((B, H, Nq, v.shape[-1]))
    L = np.empty((B, H, Nq))
    for b in range(B):
        for h in range(H):
            s = scale * (q[b, h] @ k[b, h // G].T)
            if causal:
                hidden = np.arange(Nk)[None, :] > (np.arange(Nq)[:, None] + (Nk - Nq))
                s = np.where(hidden, -np.inf, s)
            m = s.max(axis=1, keepdims=True)
            e = np.exp(s - m)
            l = e.sum(axis=1, keepdims=True)
            O[b, h] = (e / l) @ v[b, h // G]
            L[b, h] = (m + np.log(l))[:, 0]
    return O, L
