"""Seeded synthetic inputs shared by the CUDA path, the tests and the benchmark.

This module holds no arithmetic of the decoding method: it only draws numbers and
shapes them.  Two generators:

* ``normal_np`` -- SplitMix64 (counter form: output i of the stream seeded with s is
  mix64(s + (i + 1) * 0x9E3779B97F4A7C15)) followed by Box-Muller in float64, then
  rounded to bf16 (round-to-nearest-even).  Used for the small model shapes.
* ``normal_torch`` -- torch's seeded Philox generator on the target device, for the
  4B-class tensors that are too large to draw on the host in reasonable time.

Every tensor has its own sub-seed ``tensor_seed(seed, index)`` so that tensors can be
drawn independently; the index order is: embed, w_adapter, final_norm, then per layer
attn_norm, w_qkv, w_o, mlp_norm, w_gate, w_up, w_down, then the prompt.

The model shapes follow the block-diffusion workloads: a tiny one-layer model, the
4B-class dense model (36 layers, d=2560, GQA 32/8, head_dim 128, MLP 9728, V=151936),
and its NVFP4-MLP/LM-head variant.
"""
from __future__ import annotations

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def _mix64(z):
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def splitmix64(seed: int, n: int, offset: int = 0) -> np.ndarray:
    """Outputs offset .. offset+n-1 of SplitMix64 seeded with `seed`."""
    with np.errstate(over="ignore"):
        i = np.arange(offset + 1, offset + n + 1, dtype=np.uint64)
        return _mix64(np.uint64(seed) + i * _GAMMA)


def tensor_seed(seed: int, index: int) -> int:
    with np.errstate(over="ignore"):
        return int(_mix64(np.array([np.uint64(seed) * np.uint64(1000003) + np.uint64(index)],
                                   dtype=np.uint64))[0])


def uniform_np(seed: int, n: int) -> np.ndarray:
    """n doubles in [0, 1) from the top 53 bits of SplitMix64."""
    return (splitmix64(seed, n) >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)


def normal_np(seed: int, n: int, std: float = 1.0, mean: float = 0.0) -> np.ndarray:
    """n N(mean, std^2) doubles by Box-Muller on consecutive uniform pairs."""
    m = (n + 1) // 2
    u = uniform_np(seed, 2 * m)
    u1 = 1.0 - u[0::2]            # (0, 1]
    u2 = u[1::2]
    r = np.sqrt(-2.0 * np.log(u1))
    z = np.empty(2 * m)
    z[0::2] = r * np.cos(2.0 * np.pi * u2)
    z[1::2] = r * np.sin(2.0 * np.pi * u2)
    return mean + std * z[:n]


def bf16_bits(x) -> np.ndarray:
    """float array -> bf16 bit patterns (uint16), round-to-nearest-even via float32."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    r = ((u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16))
    return r.astype(np.uint16).reshape(f.shape)


def bf16_to_f64(bits) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def uniform_tokens_np(seed: int, n: int, vocab_lo: int, vocab_hi: int) -> np.ndarray:
    """n token ids uniform in [vocab_lo, vocab_hi)."""
    u = splitmix64(seed, n)
    return (vocab_lo + (u % np.uint64(vocab_hi - vocab_lo)).astype(np.int64)).astype(np.int32)


# ---------------------------------------------------------------- model configurations
def config_tiny(block_size: int = 8, max_ctx: int = 128) -> dict:
    """Tiny oracle-scale model: 1 layer, d=64, 2 q / 1 kv head, head_dim 32, MLP 4d, V=512."""
    return dict(n_layers=1, d=64, n_q_heads=2, n_kv_heads=1, head_dim=32, ffn=256, vocab=512,
                mask_id=511, max_ctx=max_ctx, block_size=block_size, rope_theta=10000.0,
                rms_eps=1e-6, weight_fmt=0)


def config_4b(block_size: int = 32, max_ctx: int = 4608 + 64, n_layers: int = 36,
              weight_fmt: int = 0) -> dict:
    """4B-class dense model: d=2560, GQA 32/8, head_dim 128, SiLU MLP 9728, V=151936."""
    return dict(n_layers=n_layers, d=2560, n_q_heads=32, n_kv_heads=8, head_dim=128, ffn=9728,
                vocab=151936, mask_id=151935, max_ctx=max_ctx, block_size=block_size,
                rope_theta=1.0e6, rms_eps=1e-6, weight_fmt=weight_fmt)


def weight_shapes(cfg: dict):
    """(name, shape, kind) in stream order; kind is 'norm' (gains, all ones) or 'w'."""
    d, hq, hkv, hd, F, V = (cfg[k] for k in ("d", "n_q_heads", "n_kv_heads", "head_dim", "ffn", "vocab"))
    out = [("embed", (V, d), "w"), ("w_adapter", (d, d), "w"), ("final_norm", (d,), "norm")]
    for li in range(cfg["n_layers"]):
        out += [(f"layers.{li}.attn_norm", (d,), "norm"),
                (f"layers.{li}.w_qkv", ((hq + 2 * hkv) * hd, d), "w"),
                (f"layers.{li}.w_o", (d, hq * hd), "w"),
                (f"layers.{li}.mlp_norm", (d,), "norm"),
                (f"layers.{li}.w_gate", (F, d), "w"),
                (f"layers.{li}.w_up", (F, d), "w"),
                (f"layers.{li}.w_down", (d, F), "w")]
    return out


def _nest(flat: dict, cfg: dict) -> dict:
    w = {k: flat[k] for k in ("embed", "w_adapter", "final_norm")}
    w["layers"] = []
    for li in range(cfg["n_layers"]):
        p = f"layers.{li}."
        w["layers"].append({k[len(p):]: v for k, v in flat.items() if k.startswith(p)})
    return w


def model_weights_np(cfg: dict, seed: int = 0, std: float = 0.02, embed_std: float | None = None) -> dict:
    """All weights as bf16 bit arrays (numpy), drawn with normal_np.  Norm gains are 1."""
    flat = {}
    for idx, (name, shape, kind) in enumerate(weight_shapes(cfg)):
        n = int(np.prod(shape))
        if kind == "norm":
            flat[name] = bf16_bits(np.ones(shape))
        else:
            sd = embed_std if (name == "embed" and embed_std is not None) else std
            flat[name] = bf16_bits(normal_np(tensor_seed(seed, idx), n, sd).reshape(shape))
    return _nest(flat, cfg)


def tiny_model(seed: int = 0, block_size: int = 8, max_ctx: int = 128, std: float = 0.02):
    """Config of the tiny model plus its weights: N(0, std) (0.02 by default), E rows
    N(0,1)/sqrt(d) x gain 8.  With std = 0.02 the single layer barely moves the residual
    stream, so all masked positions of a block see almost the same distribution; the
    variant std = 1/sqrt(d) makes positions distinct and exercises threshold commits."""
    cfg = config_tiny(block_size=block_size, max_ctx=max_ctx)
    w = model_weights_np(cfg, seed, std=std, embed_std=8.0 / np.sqrt(cfg["d"]))
    return cfg, w


def prompt_np(cfg: dict, n: int, seed: int = 0) -> np.ndarray:
    """Uniform random prompt over the non-mask vocabulary."""
    idx = len(weight_shapes(cfg))
    return uniform_tokens_np(tensor_seed(seed, idx), n, 0, cfg["vocab"] - 1)


# ---------------------------------------------------------------- device generation
def normal_torch(seed: int, shape, std: float, device, dtype=None):
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed & 0x7FFFFFFFFFFFFFFF)
    t = torch.randn(tuple(shape), generator=g, device=device, dtype=torch.float32)
    t.mul_(std)
    return t.to(dtype or torch.bfloat16)


def model_weights_torch(cfg: dict, seed: int = 0, std: float = 0.02, device="cuda",
                        embed_std: float | None = None) -> dict:
    """Same layout as model_weights_np, as bf16 torch tensors drawn on `device`."""
    import torch
    flat = {}
    for idx, (name, shape, kind) in enumerate(weight_shapes(cfg)):
        if kind == "norm":
            flat[name] = torch.ones(shape, dtype=torch.bfloat16, device=device)
        else:
            sd = embed_std if (name == "embed" and embed_std is not None) else std
            flat[name] = normal_torch(tensor_seed(seed, idx), shape, sd, device)
    return _nest(flat, cfg)


def torch_to_bits(t) -> np.ndarray:
    """bf16 torch tensor -> numpy uint16 bit array (host copy)."""
    import torch
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def lmhead_inputs_torch(B: int, d: int, V: int, seed: int = 0, device="cuda"):
    """Single-round LM-head workload: hidden H ~ N(0,1), E ~ N(0,0.02), W_a ~ N(0,0.02),
    and a previous-round distribution drawn as normalised exponentials of N(0,3) scores."""
    import torch
    H = normal_torch(tensor_seed(seed, 0), (B, d), 1.0, device, torch.float32)
    E = normal_torch(tensor_seed(seed, 1), (V, d), 0.02, device)
    Wa = normal_torch(tensor_seed(seed, 2), (d, d), 0.02, device)
    z = normal_torch(tensor_seed(seed, 3), (B, V), 3.0, device, torch.float32)
    z = torch.exp(z - z.max(dim=1, keepdim=True).values)
    P = (z / z.sum(dim=1, keepdim=True)).to(torch.bfloat16)
    return H, E, Wa, P


def attention_inputs_torch(B: int, L: int, n_q_heads: int = 32, n_kv_heads: int = 8,
                           head_dim: int = 128, max_ctx: int | None = None, seed: int = 0,
                           device="cuda"):
    """q [B][Hq][hd] and a K/V cache [Hkv][max_ctx][hd] with rows [0, L+B) ~ N(0,1), bf16."""
    import torch
    mc = max_ctx or (L + B)
    q = normal_torch(tensor_seed(seed, 10), (B, n_q_heads, head_dim), 1.0, device)
    k = torch.zeros((n_kv_heads, mc, head_dim), dtype=torch.bfloat16, device=device)
    v = torch.zeros_like(k)
    k[:, :L + B] = normal_torch(tensor_seed(seed, 11), (n_kv_heads, L + B, head_dim), 1.0, device)
    v[:, :L + B] = normal_torch(tensor_seed(seed, 12), (n_kv_heads, L + B, head_dim), 1.0, device)
    return q, k, v
