"""Split-key forward (fa_fwd_splitkv: key ranges as separate work units, partial outputs merged by
their logsumexps) against the fp64 rectangular oracle, with the forward tolerances.

Cases: decoding (one query against a ragged key cache), a few queries with grouped heads, a
prefill chunk whose early queries see none of the keys of the later ranges (their partials are
empty and must weigh nothing), requests beyond the number of key tiles, every head dim, both
masks.  One range on square inputs must reproduce fa_fwd bit for bit (same kernel, same work)."""
import numpy as np
import pytest

import attn_inputs as ai
from oracle import attention_forward_rect
from parity import assert_fwd, to_np

pytestmark = pytest.mark.gpu


def inputs(B, H, Hkv, Nq, Nk, d, seed):
    import torch
    qb = ai.make_inputs(B, H, Nq, d, seed=seed, with_do=False)["q"]
    kv = ai.make_inputs(B, Hkv, Nk, d, seed=seed + 1, with_do=False)
    to_dev = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    dev = {"q": to_dev(qb), "k": to_dev(kv["k"]), "v": to_dev(kv["v"])}
    f64 = {"q": ai.bf16_bits_to_f64(qb), "k": ai.bf16_bits_to_f64(kv["k"]),
           "v": ai.bf16_bits_to_f64(kv["v"])}
    return dev, f64


def check(B, H, Hkv, Nq, Nk, d, causal, splits, seed=0):
    import torch
    import exact_io_aware_43_b200 as fa
    dev, f64 = inputs(B, H, Hkv, Nq, Nk, d, seed)
    s = ai.default_scale(d)
    o, lse = fa.forward_splitkv(dev["q"], dev["k"], dev["v"], causal, s, splits=splits)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == 0
    O, L = attention_forward_rect(f64["q"], f64["k"], f64["v"], causal, s)
    assert_fwd(to_np(o), O, to_np(lse), L,
               f"B={B} H={H} H_kv={Hkv} Nq={Nq} Nk={Nk} d={d} causal={causal} splits={splits}")


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("splits", [1, 3, 8, 100])
def test_decode_one_query(d, causal, splits):
    check(2, 4, 4, 1, 1000, d, causal, splits, seed=d + splits)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("splits", [1, 3, 8])
def test_decode_grouped_heads_packed(d, causal, splits):
    """G = 4 query heads per key/value head, one query each: the group shares one query tile."""
    check(2, 8, 2, 1, 1000, d, causal, splits, seed=40 + d + splits)


@pytest.mark.parametrize("H,Hkv,Nq", [(16, 1, 8), (16, 1, 9), (6, 2, 5)])
def test_packing_limits(H, Hkv, Nq):
    """MQA with G * Nq = 128 rows exactly, one row over the limit (unpacked), and G = 3."""
    check(1, H, Hkv, Nq, 777, 128, True, 4, seed=H + Nq)


@pytest.mark.parametrize("causal", [False, True])
def test_few_queries_grouped_heads(causal):
    check(1, 8, 2, 16, 4096, 128, causal, 8, seed=3)


@pytest.mark.parametrize("d", [64, 128])
def test_prefill_chunk_with_empty_ranges(d):
    """Nq = 300 queries at the end of Nk = 700 keys in 3 ranges of 256 keys: query 0 sees keys
    0..400 only, so the last range holds nothing it may see."""
    check(1, 2, 2, 300, 700, d, True, 3, seed=5)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_prefill_with_wholly_invisible_ranges(d):
    """Nq = 1000 queries at the end of Nk = 1100 keys, one range per 128-key tile: the first
    query blocks see keys up to about 100 + 255 only, so most of the later ranges give them no
    key at all -- whole work units are empty and are skipped."""
    check(1, 2, 1, 1000, 1100, d, True, 9, seed=11)


def test_long_keys_many_ranges():
    check(1, 2, 1, 64, 16384, 128, True, 32, seed=6)


def test_one_range_on_square_inputs_matches_fa_fwd():
    import torch
    import exact_io_aware_43_b200 as fa
    B, H, N, d = 1, 2, 640, 128
    dev, _ = inputs(B, H, H, N, N, d, 7)
    for causal in (False, True):
        o1, l1 = fa.forward(dev["q"], dev["k"], dev["v"], causal)
        o2, l2 = fa.forward_splitkv(dev["q"], dev["k"], dev["v"], causal, splits=1)
        torch.cuda.synchronize()
        assert torch.equal(o1, o2) and torch.equal(l1, l2)
