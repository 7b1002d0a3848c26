"""Seeded synthetic inputs for the LLaMA pre-norm decoder block.

This module only draws random numbers and names the workload shapes. It holds
none of the block's arithmetic, so both the fp64 oracle (``oracle/``) and the
CUDA library (``llama_pre_norm_b200``) can be fed from it without sharing any
code path.

Every tensor is drawn on the CPU with ``torch.Generator`` and rounded to the
compute dtype *before* it is handed out, so the oracle (which widens the values
exactly to float64) and the GPU see bit-identical inputs.

Seeds: 0 for the weights, 1 for the block input X, 2 for the KV cache, and
1000 + s for the new token of decode step s.

Weight layout follows ``nn.Linear``: ``[out_features, in_features]``, as in the
``LlamaAttention`` / ``LlamaMLP`` modules of the "LMDrive 大语言模型（LLM）核心推理单元"
page (§2.3, §2.4).
"""

from __future__ import annotations

from dataclasses import dataclass, field, replace

import torch

SEED_WEIGHTS = 0
SEED_X = 1
SEED_CACHE = 2
SEED_DECODE_BASE = 1000


@dataclass(frozen=True)
class BlockConfig:
    """Shape and numerics of one decoder block workload."""

    name: str
    d: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    f: int
    B: int
    T: int
    dtype: str  # "f32" or "bf16"
    eps: float = 1e-6
    rope_base: float = 10000.0
    # decode workloads: cached prefix length and number of decode steps
    cache_len: int = 0
    decode_steps: int = 0
    # RMSNorm gains: "ones" (module init) or "1+N(0,0.1)"
    gain: str = "ones"
    weight_std: float = 0.02
    tags: tuple = field(default_factory=tuple)

    @property
    def n_rep(self) -> int:
        return self.n_heads // self.n_kv_heads

    @property
    def qkv_dim(self) -> int:
        return (self.n_heads + 2 * self.n_kv_heads) * self.head_dim

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def with_(self, **kw) -> "BlockConfig":
        return replace(self, **kw)


# The five workloads: an fp32 tiny block, LLaMA-7B / 13B / 70B-shaped bf16
# blocks (d, f from the per-model table of the "深入解析Llama MLP模块" page, §3.2),
# and KV-cache decode on the 7B-shaped block.
TINY_F32 = BlockConfig("tiny-f32", d=256, n_heads=4, n_kv_heads=4, head_dim=64, f=688,
                       B=1, T=64, dtype="f32", gain="1+N(0,0.1)")
LLAMA7B = BlockConfig("llama7b-prefill", d=4096, n_heads=32, n_kv_heads=32, head_dim=128,
                      f=11008, B=1, T=2048, dtype="bf16")
LLAMA13B = BlockConfig("llama13b-prefill", d=5120, n_heads=40, n_kv_heads=40, head_dim=128,
                       f=13824, B=4, T=1024, dtype="bf16")
LLAMA70B = BlockConfig("llama70b-gqa-prefill", d=8192, n_heads=64, n_kv_heads=8, head_dim=128,
                       f=28672, B=1, T=4096, dtype="bf16")
DECODE7B = BlockConfig("llama7b-decode", d=4096, n_heads=32, n_kv_heads=32, head_dim=128,
                       f=11008, B=32, T=1, dtype="bf16", cache_len=4096, decode_steps=128)

CONFIGS = {c.name: c for c in (TINY_F32, LLAMA7B, LLAMA13B, LLAMA70B, DECODE7B)}


def _normal(shape, std, gen, dtype):
    t = torch.empty(shape, dtype=torch.float32)
    t.normal_(0.0, std, generator=gen)
    return t.to(dtype)


def make_weights(cfg: BlockConfig, seed: int = SEED_WEIGHTS) -> dict:
    """Random-init weights of one block, ``nn.Linear`` layout ``[out, in]``.

    Returns CPU tensors in the compute dtype: wq, wk, wv, wo, w_gate, w_up,
    w_down, g_attn, g_mlp.
    """
    gen = torch.Generator().manual_seed(seed)
    dt = cfg.torch_dtype
    hd = cfg.head_dim
    s = cfg.weight_std
    w = {
        "wq": _normal((cfg.n_heads * hd, cfg.d), s, gen, dt),
        "wk": _normal((cfg.n_kv_heads * hd, cfg.d), s, gen, dt),
        "wv": _normal((cfg.n_kv_heads * hd, cfg.d), s, gen, dt),
        "wo": _normal((cfg.d, cfg.n_heads * hd), s, gen, dt),
        "w_gate": _normal((cfg.f, cfg.d), s, gen, dt),
        "w_up": _normal((cfg.f, cfg.d), s, gen, dt),
        "w_down": _normal((cfg.d, cfg.f), s, gen, dt),
    }
    if cfg.gain == "ones":
        w["g_attn"] = torch.ones(cfg.d, dtype=dt)
        w["g_mlp"] = torch.ones(cfg.d, dtype=dt)
    else:
        w["g_attn"] = (1.0 + _normal((cfg.d,), 0.1, gen, torch.float32)).to(dt)
        w["g_mlp"] = (1.0 + _normal((cfg.d,), 0.1, gen, torch.float32)).to(dt)
    return w


def make_x(cfg: BlockConfig, seed: int = SEED_X, T: int | None = None) -> torch.Tensor:
    """Block input X ~ N(0,1), shape [B, T, d], compute dtype."""
    gen = torch.Generator().manual_seed(seed)
    T = cfg.T if T is None else T
    return _normal((cfg.B, T, cfg.d), 1.0, gen, cfg.torch_dtype)


def make_cache(cfg: BlockConfig, t_max: int, seed: int = SEED_CACHE):
    """Pre-filled KV cache ~ N(0,1), shape [B, n_kv_heads, t_max, head_dim] each.

    Positions ``[0, cfg.cache_len)`` hold the synthetic prefix (taken as already
    rotated keys, since the cache stores keys after RoPE); the rest is zero.
    """
    gen = torch.Generator().manual_seed(seed)
    shape = (cfg.B, cfg.n_kv_heads, t_max, cfg.head_dim)
    k = torch.zeros(shape, dtype=cfg.torch_dtype)
    v = torch.zeros(shape, dtype=cfg.torch_dtype)
    L = cfg.cache_len
    k[:, :, :L] = _normal((cfg.B, cfg.n_kv_heads, L, cfg.head_dim), 1.0, gen, cfg.torch_dtype)
    v[:, :, :L] = _normal((cfg.B, cfg.n_kv_heads, L, cfg.head_dim), 1.0, gen, cfg.torch_dtype)
    return k, v


def make_decode_x(cfg: BlockConfig, step: int) -> torch.Tensor:
    """New-token input of decode step ``step``: [B, 1, d] ~ N(0,1)."""
    gen = torch.Generator().manual_seed(SEED_DECODE_BASE + step)
    return _normal((cfg.B, 1, cfg.d), 1.0, gen, cfg.torch_dtype)


def make_tensor(shape, seed: int, dtype: torch.dtype, std: float = 1.0,
                mean: float = 0.0) -> torch.Tensor:
    """Generic seeded N(mean, std) tensor, rounded to ``dtype``."""
    gen = torch.Generator().manual_seed(seed)
    t = torch.empty(shape, dtype=torch.float32)
    t.normal_(mean, std, generator=gen)
    return t.to(dtype)


def sample_rows(T: int, n: int, seed: int) -> list:
    """Sorted row indices: first, last, and n-2 seeded-random others (distinct)."""
    if n >= T:
        return list(range(T))
    gen = torch.Generator().manual_seed(seed)
    rest = torch.randperm(T - 2, generator=gen)[: n - 2] + 1
    return sorted({0, T - 1, *rest.tolist()})
