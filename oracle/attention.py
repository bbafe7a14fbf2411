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


def attention_forward_online(q, k, v, causal: bool, scale: float, block_r: int, block_c: int):
    """The tiled forward with the online-softmax recurrence, in the pages' order.

    [P3] "Tiling Algorithm": (1) split Q into B_r x d blocks and K, V into B_c x d blocks;
    (2) for each Q block iterate over all K, V blocks; (3) S_ij = Q_i K_j^T (scaled);
    (4) track the running row max m and row sum l; (5) update O_i, rescaling the previous partial
    result by exp(m_old - m_new) and adding exp(S_ij - m_new) V_j ([P1] update rule);
    (6) after the last block divide O_i by l.  L_i = m_i + ln l_i is kept for the backward ([P1]).
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
                qi = q[b, h, r0:r1]
                m = np.full(r1 - r0, -np.inf)
                l = np.zeros(r1 - r0)
                acc = np.zeros((r1 - r0, v.shape[-1]))
                for c0 in range(0, Nk, block_c):
                    c1 = min(Nk, c0 + block_c)
                    s = scale * (qi @ k[b, h, c0:c1].T)
                    if causal:
                        rows = np.arange(r0, r1)[:, None]
                        cols = np.arange(c0, c1)[None, :]
                        s = np.where(cols > rows, -np.inf, s)
                    m_new = np.maximum(m, s.max(axis=1))
                    # a row whose keys so far are all masked keeps m = -inf; nothing to add yet
                    safe = np.isfinite(m_new)
                    m_ref = np.where(safe, m_new, 0.0)
                    p = np.exp(s - m_ref[:, None])
                    alpha = np.where(safe, np.exp(m - m_ref), 1.0)
                    acc = alpha[:, None] * acc + p @ v[b, h, c0:c1]
                    l = alpha * l + p.sum(axis=1)
                    m = m_new
                O[b, h, r0:r1] = acc / l[:, None]
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


def attention_head_subset(q, k, v, do, causal: bool, scale: float, heads):
    """Forward + backward on a subset of (b, h) heads only (heads are independent).

    Used where the full workload is too large for the oracle: the returned arrays hold complete
    results for the listed heads.  Returns dict head -> (O, L, dQ, dK, dV), each one head's slice.
    """
    out = {}
    for (b, h) in heads:
        sl = (slice(b, b + 1), slice(h, h + 1))
        O, L = attention_forward(q[sl], k[sl], v[sl], causal, scale)
        res = [O[0, 0], L[0, 0]]
        if do is not None:
            dq, dk, dv = attention_backward(q[sl], k[sl], v[sl], O, L, do[sl], causal, scale)
            res += [dq[0, 0], dk[0, 0], dv[0, 0]]
        out[(b, h)] = tuple(res)
    return out


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
    s = scale * (q[rows] @ k.T)
    if causal:
        s = np.where(np.arange(k.shape[0])[None, :] > rows[:, None], -np.inf, s)
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    return (e / l) @ v, (m + np.log(l))[:, 0]


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
