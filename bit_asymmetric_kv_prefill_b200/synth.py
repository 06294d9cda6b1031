"""Seeded synthetic workloads for the KIVI cache (random draws only).

This module holds no quantization or attention arithmetic: it only draws the
inputs that both the CUDA path and the CPU oracle consume, so that the two sides
see identical bits.  Shapes and value statistics follow the workloads the KIVI
pages describe: fixed outlier key channels ("KIVI Quantization Secures Llama-2
Accuracy at Two Bits", paragraph 2: key outliers sit in fixed channels, values
have none) and a heavy-tailed key mix (same paragraph: magnitudes up to ~7000
against a median near 0.3).

Draw order, per workload and seed: K then V for the prefill, each a standard
normal fp32 tensor, scaled per channel, then cast to the cache dtype.  Decode
step s draws (k_t, v_t, q) from a generator seeded with 1000 + s.  Outlier
channel choices use their own generator (seed 7 + seed) so that they do not
shift the main stream.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H_q: int
    H_kv: int
    D: int
    T: int
    G: int = 32
    R: int = 128
    dtype: str = "bf16"          # cache / input dtype: "bf16" or "fp16"
    steps: int = 0               # decode steps, each appending one token
    layers: int = 1
    keys: str = "outlier"        # "outlier" (fixed channels x scale) or "heavy"
    outlier_channels: tuple = ()  # explicit channels, same for every head
    outliers_per_head: int = 0   # else: this many seeded channels per kv head
    outlier_scale: float = 1.0
    pre_rope: bool = False
    rope_theta: float = 10000.0

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float16

    @property
    def T_max(self) -> int:
        return self.T + self.steps


WORKLOADS = {
    # batch 1, 2 heads, head_dim 64, 256 tokens (128 quantized + 128 residual),
    # fp16, key channels 3 and 17 scaled x50, one decode query.
    "tiny": Workload("tiny", B=1, H_q=2, H_kv=2, D=64, T=256, dtype="fp16",
                     outlier_channels=(3, 17), outlier_scale=50.0),
    # Llama-2-7B layer shape: batch 8, 32 MHA heads, head_dim 128, 4096 tokens,
    # 4 seeded outlier key channels per head x100, 64 decode steps.
    "llama2_7b_layer": Workload("llama2_7b_layer", B=8, H_q=32, H_kv=32, D=128, T=4096,
                                steps=64, outliers_per_head=4, outlier_scale=100.0),
    # Llama-2-13B cache: batch 16, 40 layers x 40 kv heads, head_dim 128, 4096
    # tokens, heavy-tailed keys; one decode query per layer.
    "llama2_13b_cache": Workload("llama2_13b_cache", B=16, H_q=40, H_kv=40, D=128, T=4096,
                                 layers=40, keys="heavy"),
    # GQA Mistral-7B-like: batch 64, 32 query heads over 8 kv heads, 32768
    # tokens, 2 seeded outlier channels per kv head x200, 256 decode steps.
    "mistral_gqa": Workload("mistral_gqa", B=64, H_q=32, H_kv=8, D=128, T=32768, steps=256,
                            outliers_per_head=2, outlier_scale=200.0),
    # Long context: batch 1, 32/8 heads, 131072 tokens, keys quantized before
    # RoPE (theta 10000), heavy-tailed keys, 32 decode steps.
    "long_context": Workload("long_context", B=1, H_q=32, H_kv=8, D=128, T=131072, steps=32,
                             keys="heavy", pre_rope=True),
}


def scaled(w: Workload, **changes) -> Workload:
    """A smaller copy of a workload with the same value statistics."""
    return dataclasses.replace(w, **changes)


def _key_channel_scale(w: Workload, seed: int, device) -> torch.Tensor:
    """Per (kv head, channel) multiplier applied to keys: [H_kv, D] fp32."""
    g = torch.Generator().manual_seed(7 + seed)
    scale = torch.ones(w.H_kv, w.D)
    if w.keys == "heavy":
        # Body ~ N(0, 0.445^2) (median |x| ~ 0.3); 4 outlier channels per head
        # with magnitude 10^U(1, log10 1750), so max |k| reaches ~7000.
        scale *= 0.445
        for h in range(w.H_kv):
            ch = torch.randperm(w.D, generator=g)[:4]
            mag = 10.0 ** (1.0 + torch.rand(4, generator=g) * (math.log10(1750.0) - 1.0))
            scale[h, ch] = mag
    elif w.outlier_channels:
        for c in w.outlier_channels:
            scale[:, c] = w.outlier_scale
    elif w.outliers_per_head:
        for h in range(w.H_kv):
            ch = torch.randperm(w.D, generator=g)[:w.outliers_per_head]
            scale[h, ch] = w.outlier_scale
    return scale.to(device)


def _randn(shape, gen: torch.Generator, device) -> torch.Tensor:
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32)


def _gen(seed: int, device) -> torch.Generator:
    dev = torch.device(device)
    g = torch.Generator(device=dev) if dev.type == "cuda" else torch.Generator()
    return g.manual_seed(seed)


def prefill_inputs(w: Workload, seed: int = 0, device="cpu", T: Optional[int] = None):
    """K, V [B, H_kv, T, D] in the cache dtype."""
    T = w.T if T is None else T
    g = _gen(seed, device)
    ks = _key_channel_scale(w, seed, device)
    K = _randn((w.B, w.H_kv, T, w.D), g, device)
    K.mul_(ks[None, :, None, :])
    K = K.to(w.torch_dtype)
    V = _randn((w.B, w.H_kv, T, w.D), g, device).to(w.torch_dtype)
    return K, V


def step_inputs(w: Workload, step: int, seed: int = 0, device="cpu"):
    """(k_t, v_t) [B, H_kv, D] and q [B, H_q, D] for decode step `step`."""
    g = _gen(1000 + step + 100000 * seed, device)
    ks = _key_channel_scale(w, seed, device)
    k = (_randn((w.B, w.H_kv, w.D), g, device) * ks[None]).to(w.torch_dtype)
    v = _randn((w.B, w.H_kv, w.D), g, device).to(w.torch_dtype)
    q = _randn((w.B, w.H_q, w.D), g, device).to(w.torch_dtype)
    return k, v, q


def bits(t: torch.Tensor):
    """uint16 numpy view of a 2-byte tensor's bit patterns (host copy)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")
