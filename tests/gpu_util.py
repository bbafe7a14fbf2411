"""Helpers for the GPU parity tests: seeded inputs to CUDA tensors, oracle on chosen heads."""
import numpy as np

import attn_inputs as ai


def cuda_inputs(B, H, N, d, seed=0, sigma_qk=1.0, with_do=True, kv_heads=None):
    import torch
    x = ai.make_inputs(B, H, N, d, seed=seed, sigma_qk=sigma_qk, with_do=with_do,
                       kv_heads=kv_heads)
    dev = {k: torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).cuda() for k, v in x.items()}
    f64 = {k: ai.bf16_bits_to_f64(v) for k, v in x.items()}
    return dev, f64
