"""CPU oracle for one batch-1 Llama-family decode step on W8A16 (or W4A16, or bf16) weights.

TEST INFRASTRUCTURE ONLY. This module is the slow, plain reference that the CUDA path is checked
against. Only the tests, the smoke check and the bench's CPU-baseline leg may import it; the product
path never does, and it shares no code with the CUDA library (it reads only the seeded inputs from
`decode_megakernel_launch_b200.synth`, which hold no decode arithmetic).

What it computes. "AutoMegaKernel: A Statically-Checked Agent Harness for Self-Retargeting Megakernel
Synthesis" (abstract) compiles the *whole forward pass* of a HuggingFace Llama-family model for
*greedy decode*, and its int8 variant is weight-only (W8A16); the technical summary ("Problem
Statement") fixes the workload as single-stream autoregressive decoding at batch size 1, and
"Key Contributions" says the megakernel matches eager execution, so the result has a plain
definition and this oracle writes that definition out:

  x = E[token]
  per layer:  n = RMSNorm(x) * g1;  q, k, v = Wq n, Wk n, Wv n;  RoPE(q, k) at pos;
              K[pos], V[pos] = bf16(k), bf16(v);  o = GQA softmax attention over positions 0..pos;
              x += Wo o;  n2 = RMSNorm(x) * g2;  x += Wd (silu(Wg n2) * (Wu n2))
  logits = W_head RMSNorm(x) * g_f;  next = argmax(logits), lowest index on ties.

Readings where the pages are silent (each is also listed in the design notes):
  * RoPE is the HuggingFace Llama rotate-half form: pairs (i, i + hd/2), inv_freq_i = theta^(-2i/hd),
    angles in float64, no rope scaling.
  * W8A16 quantiser: per output row, s = bf16_rne(max|w| / 127), q = clamp(rne(w / s), -127, 127);
    the scale is rounded before q is formed, so dequantisation q * s is exact in fp32. A row of
    zeros (or a scale that rounds to 0) gets s = 0, q = 0.
  * W4A16 (the technical summary, "Key Contributions", lists a lossy int4 weight-only variant with
    2.42x less weight traffic): the same per-row symmetric scheme with 7 in place of 127, q in
    [-7, 7]. The pages give no group size; per-row scales with the tied embedding left in bf16
    come within 1 % of that 2.42x reduction over bf16 for the 1B-shaped model (2.44x).
  * Everything is fp32 except the tensors that are stored in bf16: embedding, gains, scales,
    bf16 weights and the KV cache.
  * Attention is causal and includes the current position; scale 1/sqrt(hd); query head i reads
    KV head i // (Hq / Hkv).
  * A tied LM head reads the bf16 embedding table itself.

Precision: fp32 (torch CPU float32 ops; matmul is the library routine). RoPE tables in float64.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Tuple

import torch

from decode_megakernel_launch_b200 import synth

F32 = torch.float32


# ----------------------------------------------------------------------------------------------
# Elementary operations.

def bf16_round(x: torch.Tensor) -> torch.Tensor:
    """Round fp32 values to the nearest bf16 (ties to even) and return them as fp32."""
    return x.to(F32).to(torch.bfloat16).to(F32)


def quantize_rows(w: torch.Tensor, qmax: int = 127) -> Tuple[torch.Tensor, torch.Tensor]:
    """Per-output-row symmetric weight quantiser: W8A16 with qmax = 127 (the abstract's int8
    weight-only variant), W4A16 with qmax = 7 (the int4 weight-only variant of the technical
    summary, "Key Contributions").

    Returns (q int8 [rows, cols], s fp32 [rows] holding bf16 values) with
    s = bf16_rne(max|w_row| / qmax) and q = clamp(round_half_even(w / s), -qmax, qmax).
    """
    w = w.to(F32)
    amax = w.abs().amax(dim=1)
    s = bf16_round(amax / float(qmax))
    safe = torch.where(s > 0, s, torch.ones_like(s))
    q = torch.round(w / safe[:, None]).clamp_(-qmax, qmax)
    q = torch.where((s > 0)[:, None], q, torch.zeros_like(q))
    return q.to(torch.int8), s


def dequantize(q: torch.Tensor, s: torch.Tensor) -> torch.Tensor:
    """W = f32(q) * f32(s) per row; exact in fp32 (|q| <= 127 times a bf16 scale)."""
    return q.to(F32) * s.to(F32)[:, None]


def rmsnorm(x: torch.Tensor, g: torch.Tensor, eps: float) -> torch.Tensor:
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) * g (the Llama layer norm)."""
    x = x.to(F32)
    ms = (x * x).mean(dim=-1, keepdim=True)
    return x / torch.sqrt(ms + eps) * g.to(F32)


def rope_cos_sin(pos: int, head_dim: int, theta: float) -> Tuple[torch.Tensor, torch.Tensor]:
    """cos/sin of the rotate-half RoPE angles pos * theta^(-2i/hd), i < hd/2, formed in float64."""
    i = torch.arange(head_dim // 2, dtype=torch.float64)
    inv_freq = theta ** (-2.0 * i / head_dim)
    ang = float(pos) * inv_freq
    return torch.cos(ang).to(F32), torch.sin(ang).to(F32)


def rope(x: torch.Tensor, pos: int, theta: float) -> torch.Tensor:
    """Rotate-half RoPE of x [..., hd] at one position: pairs (i, i + hd/2)."""
    hd = x.shape[-1]
    c, s = rope_cos_sin(pos, hd, theta)
    x1, x2 = x[..., : hd // 2], x[..., hd // 2:]
    return torch.cat([x1 * c - x2 * s, x2 * c + x1 * s], dim=-1)


def silu(z: torch.Tensor) -> torch.Tensor:
    """silu(z) = z / (1 + exp(-z))."""
    return z / (1.0 + torch.exp(-z))


def gemv(w: torch.Tensor, x: torch.Tensor) -> torch.Tensor:
    """y = W x (library matmul, fp32)."""
    return torch.matmul(w.to(F32), x.to(F32))


def gemv_naive(w: torch.Tensor, x: torch.Tensor) -> List[float]:
    """y_r = sum_k W[r][k] x[k] as a plain double loop in Python floats (pins `gemv` on tiny shapes)."""
    rows, cols = w.shape
    wl, xl = w.tolist(), x.tolist()
    out = []
    for r in range(rows):
        acc = 0.0
        for k in range(cols):
            acc += wl[r][k] * xl[k]
        out.append(acc)
    return out


def attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor) -> torch.Tensor:
    """Grouped-query softmax attention of one decode position.

    q [Hq, hd]; k, v [Hkv, P, hd] holding the P visible positions (0..pos). Query head i reads KV
    head i // (Hq / Hkv). Scores q.k / sqrt(hd), softmax with the maximum subtracted, o = p @ v.
    """
    hq, hd = q.shape
    hkv = k.shape[0]
    group = hq // hkv
    out = torch.empty(hq, hd, dtype=F32)
    for i in range(hq):
        h = i // group
        s = torch.matmul(k[h], q[i]) / math.sqrt(hd)
        p = torch.exp(s - s.max())
        p = p / p.sum()
        out[i] = torch.matmul(p, v[h])
    return out


def argmax_lowest(logits: torch.Tensor) -> int:
    """Greedy token: index of the largest logit, the lowest such index on ties. NaN is an error."""
    if not torch.isfinite(logits).all():
        raise ValueError("non-finite logits")
    m = logits.max()
    return int(torch.nonzero(logits == m)[0, 0])


def top2_margin(logits: torch.Tensor) -> float:
    """Largest logit minus the second largest (0 on a tie)."""
    t = torch.topk(logits.to(F32), 2).values
    return float(t[0] - t[1])


# ----------------------------------------------------------------------------------------------
# Model weights as the oracle holds them.

class OracleModel:
    """Weights of one synthetic model, quantised (W8A16) or bf16-rounded by the oracle's own code.

    For W8A16 the oracle keeps (q, s) and dequantises a matrix each time it is used, so the
    8B-shaped model needs ~8 GB of host memory instead of 32 GB.
    `zero` lists linear names ("wo", "w_down", ...) that are replaced by zeros before quantising
    (used by the closed-form special-case checks).
    """

    def __init__(self, cfg: synth.ModelConfig, zero: Tuple[str, ...] = (), keep_dequantized: Optional[bool] = None):
        self.cfg = cfg
        self.embed = synth.embedding(cfg).to(F32)
        self.final_norm = synth.norm_gain(cfg, None, "final_norm").to(F32)
        self.attn_norm = [synth.norm_gain(cfg, l, "attn_norm").to(F32) for l in range(cfg.n_layers)]
        self.ffn_norm = [synth.norm_gain(cfg, l, "ffn_norm").to(F32) for l in range(cfg.n_layers)]
        self.qmax = 7 if cfg.weight_dtype == "int4" else 127
        n_params = cfg.n_layers * (cfg.qkv_rows + 3 * cfg.ffn + cfg.n_q_heads * cfg.head_dim) * cfg.d_model
        self.keep_dq = (n_params < 400_000_000) if keep_dequantized is None else keep_dequantized
        self._store: Dict[Tuple[Optional[int], str], tuple] = {}
        for l in range(cfg.n_layers):
            for which in synth.LINEARS:
                self._store[(l, which)] = self._prepare(synth.linear(cfg, l, which), which in zero)
        if not cfg.tied:
            self._store[(None, "lm_head")] = self._prepare(synth.linear(cfg, None, "lm_head"), "lm_head" in zero)

    def _prepare(self, w: torch.Tensor, zero: bool) -> tuple:
        if zero:
            w = torch.zeros_like(w)
        if self.cfg.weight_dtype == "bf16":
            return ("w", bf16_round(w))
        q, s = quantize_rows(w, self.qmax)
        if self.keep_dq:
            return ("w", dequantize(q, s))
        return ("qs", q, s)

    def weight(self, layer: Optional[int], which: str) -> torch.Tensor:
        """fp32 weight matrix as the method uses it (dequantised int8 or bf16 values)."""
        if which == "lm_head" and self.cfg.tied:
            return self.embed
        ent = self._store[(layer, which)]
        return ent[1] if ent[0] == "w" else dequantize(ent[1], ent[2])

    def quantized(self, layer: Optional[int], which: str) -> Tuple[torch.Tensor, torch.Tensor]:
        """(q, s) of a quantised matrix (int8 values; within [-7, 7] for W4A16), recomputed from
        the seeded weight."""
        w = synth.linear(self.cfg, layer, which)
        return quantize_rows(w, self.qmax)


class OracleKV:
    """KV cache: per layer K, V [Hkv, max_seq, hd] fp32 holding bf16-rounded values.

    `store` is the rounding applied when a new key/value is written (bf16 by default; the
    HuggingFace cross-check passes the identity to keep fp32).
    """

    def __init__(self, cfg: synth.ModelConfig, max_seq: Optional[int] = None, store=bf16_round):
        self.cfg = cfg
        ms = max_seq or cfg.max_seq
        shape = (cfg.n_kv_heads, ms, cfg.head_dim)
        self.k = [torch.zeros(shape, dtype=F32) for _ in range(cfg.n_layers)]
        self.v = [torch.zeros(shape, dtype=F32) for _ in range(cfg.n_layers)]
        self.store = store

    def prefill_synthetic(self) -> None:
        """Load the seeded N(0,1) bf16 prefix into positions 0..prefill_len-1."""
        p = self.cfg.prefill_len
        for l in range(self.cfg.n_layers):
            self.k[l][:, :p] = synth.kv_prefill(self.cfg, l, "k").to(F32)
            self.v[l][:, :p] = synth.kv_prefill(self.cfg, l, "v").to(F32)


# ----------------------------------------------------------------------------------------------
# One decode step and a full causal forward.

def decode_step(model: OracleModel, kv: OracleKV, token: int, pos: int) -> torch.Tensor:
    """Logits [V] of one batch-1 decode step; writes K/V at `pos` and attends over 0..pos."""
    cfg = model.cfg
    hq, hkv, hd = cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim
    x = model.embed[token].clone()
    for l in range(cfg.n_layers):
        n = rmsnorm(x, model.attn_norm[l], cfg.rms_eps)
        q = gemv(model.weight(l, "wq"), n).view(hq, hd)
        k = gemv(model.weight(l, "wk"), n).view(hkv, hd)
        v = gemv(model.weight(l, "wv"), n).view(hkv, hd)
        q = rope(q, pos, cfg.rope_theta)
        k = rope(k, pos, cfg.rope_theta)
        kv.k[l][:, pos] = kv.store(k)
        kv.v[l][:, pos] = kv.store(v)
        o = attention(q, kv.k[l][:, : pos + 1], kv.v[l][:, : pos + 1])
        x = x + gemv(model.weight(l, "wo"), o.reshape(-1))
        n2 = rmsnorm(x, model.ffn_norm[l], cfg.rms_eps)
        a = silu(gemv(model.weight(l, "w_gate"), n2)) * gemv(model.weight(l, "w_up"), n2)
        x = x + gemv(model.weight(l, "w_down"), a)
    nf = rmsnorm(x, model.final_norm, cfg.rms_eps)
    return gemv(model.weight(None, "lm_head"), nf)


def full_forward(model: OracleModel, tokens: List[int], start: int = 0, prefix: Optional[OracleKV] = None,
                 store=bf16_round, kv_out: Optional[OracleKV] = None) -> torch.Tensor:
    """Logits [T, V] of a causal forward over `tokens` at positions start..start+T-1, all at once.

    A second, independent formulation: every position's q/k/v in one matmul per layer, then a masked
    [T, start+T] softmax per head. Keys/values of the new positions pass through `store` exactly as
    the step-wise cache does; positions < start come from `prefix`. If `kv_out` is given, the stored
    keys/values of positions 0..start+T-1 are written into it (a prompt's cache in one pass).
    """
    cfg = model.cfg
    hq, hkv, hd = cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim
    group = hq // hkv
    T = len(tokens)
    P = start + T
    x = model.embed[torch.tensor(tokens)].clone()                       # [T, d]
    positions = list(range(start, P))
    for l in range(cfg.n_layers):
        n = rmsnorm(x, model.attn_norm[l], cfg.rms_eps)                  # [T, d]
        q = (n @ model.weight(l, "wq").T).view(T, hq, hd)
        k = (n @ model.weight(l, "wk").T).view(T, hkv, hd)
        v = (n @ model.weight(l, "wv").T).view(T, hkv, hd)
        q = torch.stack([rope(q[t], positions[t], cfg.rope_theta) for t in range(T)])
        k = torch.stack([rope(k[t], positions[t], cfg.rope_theta) for t in range(T)])
        kk = torch.zeros(hkv, P, hd, dtype=F32)
        vv = torch.zeros(hkv, P, hd, dtype=F32)
        if start:
            kk[:, :start] = prefix.k[l][:, :start]
            vv[:, :start] = prefix.v[l][:, :start]
        kk[:, start:] = store(k).permute(1, 0, 2)
        vv[:, start:] = store(v).permute(1, 0, 2)
        if kv_out is not None:
            kv_out.k[l][:, :P] = kk
            kv_out.v[l][:, :P] = vv
        mask = torch.arange(P)[None, :] <= torch.tensor(positions)[:, None]   # [T, P]
        o = torch.empty(T, hq, hd, dtype=F32)
        for i in range(hq):
            h = i // group
            s = (q[:, i] @ kk[h].T) / math.sqrt(hd)                          # [T, P]
            s = s.masked_fill(~mask, float("-inf"))
            p = torch.softmax(s, dim=-1)
            o[:, i] = p @ vv[h]
        x = x + o.reshape(T, -1) @ model.weight(l, "wo").T
        n2 = rmsnorm(x, model.ffn_norm[l], cfg.rms_eps)
        a = silu(n2 @ model.weight(l, "w_gate").T) * (n2 @ model.weight(l, "w_up").T)
        x = x + a @ model.weight(l, "w_down").T
    nf = rmsnorm(x, model.final_norm, cfg.rms_eps)
    return nf @ model.weight(None, "lm_head").T


def teacher_forced(model: OracleModel, kv: OracleKV, tokens: List[int], start: int) -> List[torch.Tensor]:
    """Logits of decode steps feeding tokens[i] at position start + i (the GPU's own token chain)."""
    return [decode_step(model, kv, t, start + i) for i, t in enumerate(tokens)]
