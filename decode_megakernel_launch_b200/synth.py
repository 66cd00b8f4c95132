"""Seeded synthetic inputs for batch-1 Llama decode: model presets, weights, prompts, KV prefill.

This module only draws numbers. It holds none of the decode arithmetic (no quantiser, no norm,
no RoPE, no attention): the CPU oracle and the CUDA path both start from the tensors made here
and each applies the method in its own code.

Recipe (the same for every preset):
  * linear weights (wq, wk, wv, wo, w_gate, w_up, w_down, untied lm_head): N(0, 0.02) in fp32,
  * token embedding: N(0, 1), rounded to bf16 (it is stored in bf16),
  * RMSNorm gains: 1 + N(0, 0.02), rounded to bf16,
  * prompt ids: uniform integers in [0, vocab),
  * prefilled KV cache (8B-shaped and long-context presets): N(0, 1), rounded to bf16, treated as
    already-rotated keys and plain values,
  * first decode token of the prefilled presets: uniform in [0, vocab).

Each tensor has its own stream: numpy PCG64 seeded by SeedSequence([preset seed, crc32(name), block]),
one stream per block of 2**20 consecutive elements, so any tensor (or any layer) can be regenerated
alone, and the values do not depend on the number of threads used to draw them.

Shapes follow the HuggingFace Llama naming: wq [Hq*hd, d], wk/wv [Hkv*hd, d], wo [d, Hq*hd],
w_gate/w_up [ffn, d], w_down [d, ffn], embed/lm_head [V, d].
"""
from __future__ import annotations

import dataclasses
import os
import zlib
from concurrent.futures import ThreadPoolExecutor
from typing import Optional

import numpy as np
import torch

BLOCK = 1 << 20
LINEAR_STD = 0.02
GAIN_STD = 0.02


@dataclasses.dataclass(frozen=True)
class ModelConfig:
    """Dimensions and run recipe of one synthetic Llama-family model."""
    name: str
    seed: int
    n_layers: int
    d_model: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    ffn: int
    vocab: int
    tied: bool
    rope_theta: float
    rms_eps: float = 1e-5
    prompt_len: int = 0        # prompt tokens fed step by step from position 0
    prefill_len: int = 0       # KV positions 0..prefill_len-1 filled with N(0,1) before decoding
    decode_steps: int = 0      # greedy decode steps after the prompt / prefill
    compare_steps: int = 0     # decode steps the oracle is compared on
    weight_dtype: str = "int8"  # "int8" (W8A16), "int4" (W4A16) or "bf16"

    @property
    def max_seq(self) -> int:
        return self.prompt_len + self.prefill_len + self.decode_steps

    @property
    def qkv_rows(self) -> int:
        return (self.n_q_heads + 2 * self.n_kv_heads) * self.head_dim

    def with_(self, **kw) -> "ModelConfig":
        return dataclasses.replace(self, **kw)


PRESETS = {
    "tiny": ModelConfig("tiny", 0, 2, 256, 4, 2, 64, 704, 2048, False, 1e4,
                        prompt_len=16, decode_steps=32, compare_steps=32),
    "smollm135m": ModelConfig("smollm135m", 1, 30, 576, 9, 3, 64, 1536, 49152, True, 1e5,
                              prompt_len=128, decode_steps=256, compare_steps=256),
    "llama1b": ModelConfig("llama1b", 2, 16, 2048, 32, 8, 64, 8192, 128256, True, 5e5,
                           prompt_len=512, decode_steps=256, compare_steps=16),
    "llama8b": ModelConfig("llama8b", 3, 32, 4096, 32, 8, 128, 14336, 128256, False, 5e5,
                           prefill_len=1024, decode_steps=128, compare_steps=4),
    "llama1b_long4k": ModelConfig("llama1b_long4k", 4, 16, 2048, 32, 8, 64, 8192, 128256, True, 5e5,
                                  prefill_len=4096, decode_steps=64, compare_steps=4),
    "llama1b_long16k": ModelConfig("llama1b_long16k", 4, 16, 2048, 32, 8, 64, 8192, 128256, True, 5e5,
                                   prefill_len=16384, decode_steps=64, compare_steps=4),
    "llama1b_long32k": ModelConfig("llama1b_long32k", 4, 16, 2048, 32, 8, 64, 8192, 128256, True, 5e5,
                                   prefill_len=32768, decode_steps=64, compare_steps=4),
}
# W4A16 variants of the same shapes (int4 weight-only, per-row bf16 scales).
for _n in ("tiny", "llama1b", "llama8b"):
    PRESETS[_n + "_int4"] = PRESETS[_n].with_(name=_n + "_int4", weight_dtype="int4")


def preset(name: str, **overrides) -> ModelConfig:
    cfg = PRESETS[name]
    return cfg.with_(**overrides) if overrides else cfg


def _stream(seed: int, name: str, block: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, zlib.crc32(name.encode()), block])))


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def normal(seed: int, name: str, shape, std: float = 1.0, mean: float = 0.0) -> torch.Tensor:
    """fp32 tensor of N(mean, std^2) draws; element i comes from block i // BLOCK of its own stream."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.float32)
    nblk = (n + BLOCK - 1) // BLOCK

    def fill(b: int) -> None:
        lo, hi = b * BLOCK, min(n, (b + 1) * BLOCK)
        z = _stream(seed, name, b).standard_normal(hi - lo, dtype=np.float32)
        if std != 1.0:
            z *= np.float32(std)
        if mean != 0.0:
            z += np.float32(mean)
        out[lo:hi] = z

    if nblk == 1:
        fill(0)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(fill, range(nblk)))
    return torch.from_numpy(out).view(*shape)


def uniform_ids(seed: int, name: str, n: int, vocab: int) -> list:
    return [int(v) for v in _stream(seed, name, 0).integers(0, vocab, size=n)]


# ----------------------------------------------------------------------------------------------
# Named tensors of one model.

LINEARS = ("wq", "wk", "wv", "wo", "w_gate", "w_up", "w_down")


def linear_shape(cfg: ModelConfig, which: str):
    d, hd = cfg.d_model, cfg.head_dim
    return {
        "wq": (cfg.n_q_heads * hd, d),
        "wk": (cfg.n_kv_heads * hd, d),
        "wv": (cfg.n_kv_heads * hd, d),
        "wo": (d, cfg.n_q_heads * hd),
        "w_gate": (cfg.ffn, d),
        "w_up": (cfg.ffn, d),
        "w_down": (d, cfg.ffn),
        "lm_head": (cfg.vocab, d),
    }[which]


def linear(cfg: ModelConfig, layer: Optional[int], which: str) -> torch.Tensor:
    """fp32 linear weight, N(0, 0.02). `layer` is None for lm_head."""
    name = "lm_head" if which == "lm_head" else f"layers.{layer}.{which}"
    return normal(cfg.seed, name, linear_shape(cfg, which), std=LINEAR_STD)


def embedding(cfg: ModelConfig) -> torch.Tensor:
    """bf16 [V, d] token embedding, N(0, 1)."""
    return normal(cfg.seed, "embed", (cfg.vocab, cfg.d_model)).to(torch.bfloat16)


def norm_gain(cfg: ModelConfig, layer: Optional[int], which: str) -> torch.Tensor:
    """bf16 [d] RMSNorm gain 1 + N(0, 0.02); which in {attn_norm, ffn_norm, final_norm}."""
    name = "final_norm" if which == "final_norm" else f"layers.{layer}.{which}"
    return normal(cfg.seed, name, (cfg.d_model,), std=GAIN_STD, mean=1.0).to(torch.bfloat16)


def prompt_ids(cfg: ModelConfig) -> list:
    return uniform_ids(cfg.seed, "prompt", cfg.prompt_len, cfg.vocab)


def first_decode_token(cfg: ModelConfig) -> int:
    """Token fed at the first decode position of a prefilled preset."""
    return uniform_ids(cfg.seed, "first_token", 1, cfg.vocab)[0]


def kv_prefill(cfg: ModelConfig, layer: int, which: str) -> torch.Tensor:
    """bf16 [Hkv, prefill_len, hd] prefilled keys (which='k') or values ('v'), N(0, 1)."""
    shape = (cfg.n_kv_heads, cfg.prefill_len, cfg.head_dim)
    return normal(cfg.seed, f"layers.{layer}.{which}_prefill", shape).to(torch.bfloat16)
