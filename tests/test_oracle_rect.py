"""Pins for the rectangular (Nq != Nk) oracle used by the split-key forward's parity tests.

It is checked against a brute-force loop over single query rows that applies the end-aligned
causal rule (query i sees keys j <= i + Nk - Nq) by hand, and against the square oracle (pinned in
test_oracle.py): the last Nq rows of a square causal attention over all Nk positions are exactly
the rectangular result for those Nq queries, and without a mask each query row does not depend
on the others.  Planted mistakes (top-left alignment, an off-by-one offset, the key/value head
mapping h % H_kv) must fail a pin.
"""
import math

import numpy as np
import pytest

from oracle import attention_forward, attention_forward_rect


def rand(shape, seed, sigma=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * sigma


def _row(q, k, v, b, h, i, G, causal, scale):
    Nq, Nk = q.shape[2], k.shape[2]
    hk = h // G
    sc = [(j, scale * sum(q[b, h, i, c] * k[b, hk, j, c] for c in range(q.shape[3])))
          for j in range(Nk) if not (causal and j > i + Nk - Nq)]
    m = max(x for _, x in sc)
    w = [(j, math.exp(x - m)) for j, x in sc]
    z = sum(e for _, e in w)
    return [sum(e * v[b, hk, j, c] for j, e in w) / z for c in range(v.shape[3])], m + math.log(z)


def pin_rect_brute_force(fwd):
    for (B, H, Hkv, Nq, Nk, d, seed) in ((1, 2, 1, 1, 7, 3, 1), (1, 4, 2, 3, 8, 2, 2),
                                         (2, 2, 2, 5, 5, 3, 3), (1, 3, 3, 2, 9, 4, 4)):
        q = rand((B, H, Nq, d), seed)
        k = rand((B, Hkv, Nk, d), seed + 50)
        v = rand((B, Hkv, Nk, d), seed + 60)
        for causal in (False, True):
            O, L = fwd(q, k, v, causal, 0.8)
            for b in range(B):
                for h in range(H):
                    for i in range(Nq):
                        o, l = _row(q, k, v, b, h, i, H // Hkv, causal, 0.8)
                        if not (np.allclose(O[b, h, i], o, atol=1e-12) and abs(L[b, h, i] - l) < 1e-12):
                            return f"row ({b},{h},{i}) disagrees (Nq={Nq}, Nk={Nk}, causal={causal})"
    return None


def pin_rect_is_tail_of_square(fwd):
    for (Nq, Nk, d, seed) in ((1, 9, 4, 7), (4, 12, 3, 8), (12, 12, 5, 9), (3, 130, 8, 10)):
        qf = rand((2, 2, Nk, d), seed)
        k = rand((2, 2, Nk, d), seed + 1)
        v = rand((2, 2, Nk, d), seed + 2)
        for causal in (False, True):
            Of, Lf = attention_forward(qf, k, v, causal, 0.5)
            O, L = fwd(qf[:, :, Nk - Nq:], k, v, causal, 0.5)
            if not (np.allclose(O, Of[:, :, Nk - Nq:], atol=1e-12) and
                    np.allclose(L, Lf[:, :, Nk - Nq:], atol=1e-12)):
                return f"not the tail of the square attention (Nq={Nq}, Nk={Nk}, causal={causal})"
    return None


PINS = [pin_rect_brute_force, pin_rect_is_tail_of_square]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_rect_pin(pin):
    assert pin(attention_forward_rect) is None


def test_rect_rejects_causal_with_more_queries_than_keys():
    with pytest.raises(ValueError):
        attention_forward_rect(rand((1, 1, 5, 2), 0), rand((1, 1, 3, 2), 1), rand((1, 1, 3, 2), 2),
                               True, 1.0)


def _mut(offset_fn, tiled=False):
    def fwd(q, k, v, causal, scale):
        B, H, Nq, _ = q.shape
        Nk = k.shape[2]
        G = H // k.shape[1]
        O = np.empty((B, H, Nq, v.shape[-1]))
        L = np.empty((B, H, Nq))
        for b in range(B):
            for h in range(H):
                hk = h % k.shape[1] if tiled else h // G
                s = scale * (q[b, h] @ k[b, hk].T)
                if causal:
                    s = np.where(np.arange(Nk)[None, :] > (np.arange(Nq)[:, None] +
                                                          offset_fn(Nq, Nk)), -np.inf, s)
                m = s.max(axis=1, keepdims=True)
                e = np.exp(s - m)
                O[b, h] = (e / e.sum(axis=1, keepdims=True)) @ v[b, hk]
                L[b, h] = (m + np.log(e.sum(axis=1, keepdims=True)))[:, 0]
        return O, L
    return fwd


MUTANTS = [
    ("top_left_alignment", _mut(lambda nq, nk: 0)),
    ("offset_off_by_one", _mut(lambda nq, nk: nk - nq - 1)),
    ("head_mapping_tiled", _mut(lambda nq, nk: nk - nq, tiled=True)),
]


@pytest.mark.parametrize("name,fwd", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_rect_planted_mistake_is_caught(name, fwd):
    assert any(p(fwd) for p in PINS), f"planted mistake {name} passed every pin"


def test_rect_agrees_with_grouped_oracle_on_square_shapes():
    """Where both apply (Nq = Nk, grouped heads) the rectangular and the grouped oracle -- pinned
    separately -- must give the same result."""
    from oracle import attention_forward_gqa
    for (H, Hkv, N, d, seed) in ((4, 2, 7, 3, 70), (6, 1, 5, 4, 71), (3, 3, 9, 2, 72)):
        q = rand((2, H, N, d), seed)
        k = rand((2, Hkv, N, d), seed + 1)
        v = rand((2, Hkv, N, d), seed + 2)
        for causal in (False, True):
            O1, L1 = attention_forward_rect(q, k, v, causal, 0.7)
            O2, L2 = attention_forward_gqa(q, k, v, causal, 0.7)
            assert np.allclose(O1, O2, atol=1e-12) and np.allclose(L1, L2, atol=1e-12)
