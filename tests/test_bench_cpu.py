"""The bookkeeping behind bench.py's roofline figures, on the CPU: the algorithmic bytes of a
decode step counted from the 4B-class architecture (shapes only, meta tensors), and the DRAM
traffic taken from the committed ncu summary."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from block_diffusion_decoding_denoising_b200 import gen  # noqa: E402


def _meta_weights(cfg):
    import torch
    flat = {name: torch.empty(shape, dtype=torch.bfloat16, device="meta") for name, shape, _ in gen.weight_shapes(cfg)}
    return gen._nest(flat, cfg)


def test_step_bytes_match_the_architecture():
    cfg = gen.config_4b()
    d, hq, hkv, hd, F, V, nl = (cfg[k] for k in ("d", "n_q_heads", "n_kv_heads", "head_dim", "ffn", "vocab",
                                                 "n_layers"))
    # per layer: two RMSNorm gains, QKV, O, gate and up, down (bf16)
    qkv = (hq + 2 * hkv) * hd * d
    layer = 2 * (2 * d + qkv + d * hq * hd + 2 * F * d + d * F)
    kv_per_pos = 2 * hkv * hd * 2 * nl  # K and V of every layer, bf16
    mean_L = bench.PROMPT + bench.GEN / 2
    round_b = nl * layer + V * d * 2 + d * d * 2 + d * 2 + kv_per_pos * mean_L
    # a KV-fill forward: no adapter, no LM head, the last layer only up to its QKV projection
    fill_b = (nl - 1) * layer + 2 * (d + qkv) + kv_per_pos * (nl - 1) / nl * mean_L
    total, r, f = bench.step_algorithmic_bytes(cfg, _meta_weights(cfg), rounds=384, fills=1)
    assert r == round_b and f == fill_b
    assert total == 384 * round_b + fill_b
    # the weight part of a round: 36 layers + E + W_a (+ the final gain), about 8.058 GB
    assert abs(round_b - kv_per_pos * mean_L - 8.058e9) < 1e6


def test_traffic_comes_from_the_committed_profile():
    assert bench.profile_traffic("k_gemm_tc_9728x2560_t32.md") == 50378496.0
    assert bench.profile_traffic("no_such_profile.md") is None
