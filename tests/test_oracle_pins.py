"""Pins of the CPU oracle to things other than itself (no GPU needed).

Each check below ties one oracle function to a closed form, an invariant, a brute-force evaluation
in Python floats, or an independent library implementation (HuggingFace `LlamaForCausalLM`, whose
decoder layer is the Llama-family forward pass the megakernel pages compile). The mutant tests at the
end plant plausible mistakes in the oracle and check that these pins catch them.
"""
import math
import struct

import pytest
import torch

from decode_megakernel_launch_b200 import synth
from oracle import llama_decode as O

SMALL = synth.ModelConfig("pin", seed=11, n_layers=2, d_model=48, n_q_heads=4, n_kv_heads=2, head_dim=16,
                          ffn=80, vocab=96, tied=False, rope_theta=1e4, prompt_len=6, decode_steps=4)


# ---------------------------------------------------------------------------------------------
# bf16 rounding and the quantiser, against bit-level Python.

def _f32(x):
    return struct.unpack("<f", struct.pack("<f", x))[0]


def _bf16_rne_py(x):
    u = struct.unpack("<I", struct.pack("<f", x))[0]
    u = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return struct.unpack("<f", struct.pack("<I", u & 0xFFFFFFFF))[0]


def test_bf16_round_matches_bitwise_rne():
    g = torch.Generator().manual_seed(0)
    x = torch.randn(2000, generator=g) * torch.exp(torch.randn(2000, generator=g) * 4)
    # include exact ties: mantissa low half == 0x8000 with even and odd upper halves
    ties = [struct.unpack("<f", struct.pack("<I", u))[0] for u in (0x3F808000, 0x3F818000, 0xC0408000, 0x40C18000)]
    x = torch.cat([x, torch.tensor(ties)])
    got = O.bf16_round(x).tolist()
    want = [_bf16_rne_py(v) for v in x.tolist()]
    assert got == want


def _quantize_py(row, qmax=127):
    amax = max(abs(v) for v in row)
    s = _bf16_rne_py(_f32(amax / float(qmax)))
    if s == 0.0:
        return [0] * len(row), 0.0
    q = [max(-qmax, min(qmax, round(_f32(v / s)))) for v in row]
    return q, s


def test_quantizer_brute_force():
    g = torch.Generator().manual_seed(1)
    w = torch.randn(7, 33, generator=g) * 0.02
    w[3] = 0.0                      # zero row
    w[4, 5] = 0.5                   # outlier row
    w[5] = torch.linspace(-1, 1, 33)
    q, s = O.quantize_rows(w)
    for r in range(w.shape[0]):
        qr, sr = _quantize_py([_f32(v) for v in w[r].tolist()])
        assert q[r].tolist() == qr
        assert s[r].item() == sr


def test_quantizer_int4_brute_force():
    """W4A16 reading: the same per-row scheme with qmax = 7, against pure-Python rounding."""
    g = torch.Generator().manual_seed(2)
    w = torch.randn(9, 40, generator=g) * 0.02
    w[2] = 0.0
    w[6, 1] = -0.3
    w[7] = torch.linspace(-0.7, 0.7, 40)        # ties of w/s at +-0.5 steps
    q, s = O.quantize_rows(w, 7)
    for r in range(w.shape[0]):
        qr, sr = _quantize_py([_f32(v) for v in w[r].tolist()], 7)
        assert q[r].tolist() == qr
        assert s[r].item() == sr


def test_quantizer_int4_bounds_and_exact_dequant():
    w = synth.normal(6, "q4bounds", (64, 512), std=0.02)
    q, s = O.quantize_rows(w, 7)
    assert int(q.min()) >= -7 and int(q.max()) <= 7
    assert set(q.abs().amax(dim=1).tolist()) <= {6, 7}
    assert torch.equal(O.bf16_round(s), s)
    deq = O.dequantize(q, s)
    assert torch.equal(deq.double(), q.double() * s.double()[:, None])
    err = (w - deq).abs()
    unclamped = (w / s[:, None]).abs() <= 7
    assert bool((err[unclamped] <= (s[:, None] / 2).expand_as(w)[unclamped] * (1 + 1e-6)).all())
    # the oracle model uses this quantiser for int4 configs
    cfg = synth.preset("tiny_int4")
    m = O.OracleModel(cfg)
    q2, s2 = m.quantized(0, "wo")
    assert int(q2.abs().max()) <= 7
    assert torch.equal(m.weight(0, "wo"), O.dequantize(q2, s2))


def test_quantizer_bounds_and_exact_dequant():
    w = synth.normal(5, "qbounds", (64, 512), std=0.02)
    q, s = O.quantize_rows(w)
    assert int(q.min()) >= -127 and int(q.max()) <= 127
    amax_q = q.abs().amax(dim=1)
    assert set(amax_q.tolist()) <= {126, 127}
    # scales are bf16 values
    assert torch.equal(O.bf16_round(s), s)
    deq = O.dequantize(q, s)
    # exact in fp32: the float64 product equals the fp32 product
    assert torch.equal(deq.double(), q.double() * s.double()[:, None])
    err = (w - deq).abs()
    unclamped = (w / s[:, None]).abs() <= 127
    assert bool((err[unclamped] <= (s[:, None] / 2).expand_as(w)[unclamped] * (1 + 1e-6)).all())


# ---------------------------------------------------------------------------------------------
# RMSNorm, RoPE, silu.

def test_rmsnorm_constant_vector_closed_form():
    d, c, eps = 64, 3.0, 1e-5
    g = synth.norm_gain(SMALL, 0, "attn_norm").to(torch.float32)[:48]
    x = torch.full((48,), c)
    got = O.rmsnorm(x, g, eps)
    want = torch.tensor([c / math.sqrt(c * c + eps) * gi for gi in g.tolist()])
    assert torch.allclose(got, want, rtol=1e-6, atol=0)


def test_rmsnorm_brute_force_and_scale_invariance():
    x = synth.normal(6, "rms", (100,))
    g = synth.normal(6, "rmsg", (100,), std=0.1, mean=1.0)
    xl, gl = x.tolist(), g.tolist()
    rms = math.sqrt(sum(v * v for v in xl) / len(xl) + 1e-5)
    want = torch.tensor([v / rms * gi for v, gi in zip(xl, gl)])
    assert torch.allclose(O.rmsnorm(x, g, 1e-5), want, rtol=2e-6, atol=1e-7)
    assert torch.allclose(O.rmsnorm(x * 1000.0, g, 1e-5), O.rmsnorm(x, g, 1e-5), rtol=1e-5)


def test_rope_identity_at_pos0_and_2d_rotation():
    x = synth.normal(7, "rope", (3, 16))
    assert torch.equal(O.rope(x, 0, 1e4), x)
    # head_dim 2: the textbook 2-D rotation by angle pos (inv_freq = theta^0 = 1)
    a, b = 0.3, -1.7
    for pos in (1, 5, 100):
        got = O.rope(torch.tensor([[a, b]]), pos, 1e4)[0].tolist()
        want = [a * math.cos(pos) - b * math.sin(pos), b * math.cos(pos) + a * math.sin(pos)]
        assert got == pytest.approx(want, rel=1e-6, abs=1e-6)


def test_rope_frequencies_pairs_and_norm():
    hd, theta = 8, 1e4
    x = synth.normal(8, "rope2", (hd,))
    pos = 3
    y = O.rope(x[None], pos, theta)[0]
    for i in range(hd // 2):
        # pair (i, i + hd/2) rotates by pos * theta^(-2i/hd) and keeps its norm
        a0 = math.atan2(x[i + hd // 2].item(), x[i].item())
        a1 = math.atan2(y[i + hd // 2].item(), y[i].item())
        ang = (a1 - a0) % (2 * math.pi)
        want = (pos * theta ** (-2 * i / hd)) % (2 * math.pi)
        assert min(abs(ang - want), 2 * math.pi - abs(ang - want)) < 1e-5
        assert math.hypot(y[i], y[i + hd // 2]) == pytest.approx(math.hypot(x[i], x[i + hd // 2]), rel=1e-6)


def test_rope_relative_position():
    q = synth.normal(9, "rq", (64,))
    k = synth.normal(9, "rk", (64,))
    dots = [float(O.rope(q[None], m, 5e5)[0] @ O.rope(k[None], n, 5e5)[0]) for m, n in ((7, 3), (107, 103), (1007, 1003))]
    assert dots[0] == pytest.approx(dots[1], rel=1e-4) and dots[0] == pytest.approx(dots[2], rel=1e-4)


def test_rope_matches_huggingface_apply_rotary():
    from transformers.models.llama.modeling_llama import apply_rotary_pos_emb
    hd, theta, pos = 64, 5e5, 37
    q = synth.normal(10, "hq", (1, 4, 1, hd))
    k = synth.normal(10, "hk", (1, 2, 1, hd))
    inv = 1.0 / (theta ** (torch.arange(0, hd, 2, dtype=torch.float64) / hd))
    ang = pos * inv
    emb = torch.cat([ang, ang])
    cos, sin = emb.cos().float()[None, None], emb.sin().float()[None, None]
    hq, hk = apply_rotary_pos_emb(q, k, cos[0], sin[0], unsqueeze_dim=0)
    assert torch.allclose(O.rope(q[0, :, 0], pos, theta), hq[0, :, 0], rtol=1e-6, atol=1e-6)
    assert torch.allclose(O.rope(k[0, :, 0], pos, theta), hk[0, :, 0], rtol=1e-6, atol=1e-6)


def test_silu():
    z = torch.tensor([0.0, 1.0, -2.5, 30.0, -30.0])
    assert torch.allclose(O.silu(z), z * torch.sigmoid(z), rtol=1e-6, atol=1e-12)
    assert O.silu(torch.tensor([0.0])).item() == 0.0


# ---------------------------------------------------------------------------------------------
# GEMV and attention.

def test_gemv_against_triple_loop():
    w = synth.normal(12, "gw", (9, 37))
    x = synth.normal(12, "gx", (37,))
    assert O.gemv(w, x).tolist() == pytest.approx(O.gemv_naive(w, x), rel=1e-5, abs=1e-5)


def _attention_py(q, k, v):
    hq, hd = len(q), len(q[0])
    hkv = len(k)
    out = []
    for i in range(hq):
        h = i // (hq // hkv)
        s = [sum(a * b for a, b in zip(q[i], kj)) / math.sqrt(hd) for kj in k[h]]
        m = max(s)
        e = [math.exp(t - m) for t in s]
        z = sum(e)
        out.append([sum(e[j] / z * k_[d] for j, k_ in enumerate(v[h])) for d in range(hd)])
    return out


def test_attention_brute_force_gqa():
    q = synth.normal(13, "aq", (6, 8))
    k = synth.normal(13, "ak", (2, 5, 8)) * 2
    v = synth.normal(13, "av", (2, 5, 8))
    got = O.attention(q, k, v)
    want = _attention_py(q.tolist(), k.tolist(), v.tolist())
    assert torch.allclose(got, torch.tensor(want), rtol=1e-5, atol=1e-6)


def test_attention_special_cases():
    q = synth.normal(14, "sq", (4, 8))
    v = synth.normal(14, "sv", (2, 1, 8))
    k = synth.normal(14, "sk", (2, 1, 8))
    o = O.attention(q, k, v)                      # one position: o = v of the head's KV group
    assert torch.allclose(o[:2], v[0].expand(2, 8)) and torch.allclose(o[2:], v[1].expand(2, 8))
    k_eq = torch.ones(2, 6, 8)
    v6 = synth.normal(14, "sv6", (2, 6, 8))
    o = O.attention(q, k_eq, v6)                  # equal keys: uniform weights, o = mean(v)
    assert torch.allclose(o[0], v6[0].mean(0), atol=1e-6) and torch.allclose(o[3], v6[1].mean(0), atol=1e-6)


def test_argmax_lowest_on_ties():
    assert O.argmax_lowest(torch.tensor([1.0, 3.0, 2.0, 3.0])) == 1
    with pytest.raises(ValueError):
        O.argmax_lowest(torch.tensor([1.0, float("nan")]))


# ---------------------------------------------------------------------------------------------
# The token gate. Greedy decode is exact ("Experimental Results", "Correctness & Portability" of the
# technical summary: token-for-token agreement), and the GPU tests require the GPU's token to equal
# the oracle's wherever the oracle's top-1 minus top-2 logit exceeds 0.1, so that margin is pinned to
# a plain Python sort of the same float values (ties at the top give 0).

def _top2_margin_py(values):
    s = sorted((float(v) for v in values), reverse=True)
    return s[0] - s[1]


def _top2_cases():
    g = torch.Generator().manual_seed(5)
    yield torch.tensor([1.0, 3.0, 2.0, 3.0])                     # tie at the top: 0
    yield torch.tensor([-5.0, -1.5, -9.0, -1.25])                # all negative: 0.25
    yield torch.tensor([7.0, 7.0, 7.0])                          # all equal: 0
    yield torch.tensor([0.0, 100.0])                             # two logits: 100
    yield torch.tensor([2.0, 2.05, -3.0, 1.0])                   # a near tie: 0.05
    yield torch.randn(128256, generator=g) * 3.0                # a vocabulary of the 1B / 8B shapes
    big = torch.randn(50000, generator=g)
    big[123], big[40000] = 9.0, 8.75                             # a clear runner-up far from the top
    yield big


def _top2_agrees(fn):
    return all(math.isclose(fn(t), _top2_margin_py(t.tolist()), rel_tol=0.0, abs_tol=1e-5) for t in _top2_cases())


def test_top2_margin_matches_a_python_sort():
    assert _top2_agrees(O.top2_margin)
    assert O.top2_margin(torch.tensor([1.0, 3.0, 2.0, 3.0])) == 0.0


@pytest.mark.parametrize("fn", [
    lambda t: float(t.max() - t.min()),                                      # top minus bottom
    lambda t: float(torch.topk(t.abs(), 2).values[0] - torch.topk(t.abs(), 2).values[1]),   # magnitudes
    lambda t: (lambda m: m if m > 0.1 else 0.0)(O.top2_margin(t)),           # near ties dropped
    lambda t: (lambda u: float(u[-1] - u[-2]) if len(u) > 1 else 0.0)(torch.unique(t)),  # distinct values
    lambda t: float(torch.sort(t).values[1] - torch.sort(t).values[0]),      # the bottom two
], ids=["max_minus_min", "abs", "zero_near_ties", "distinct", "bottom_two"])
def test_top2_margin_pin_catches_planted_mistakes(fn):
    assert not _top2_agrees(fn)


# ---------------------------------------------------------------------------------------------
# Whole step: incremental == full causal forward; closed-form special case; HuggingFace Llama.

def test_incremental_equals_full_causal_forward():
    m = O.OracleModel(SMALL)
    toks = synth.prompt_ids(SMALL)
    kv = O.OracleKV(SMALL)
    inc = torch.stack(O.teacher_forced(m, kv, toks, 0))
    full = O.full_forward(m, toks)
    rel = (inc - full).norm() / full.norm()
    assert rel < 2e-6


def test_incremental_equals_full_with_prefilled_cache():
    cfg = SMALL.with_(prompt_len=0, prefill_len=5, decode_steps=4)
    m = O.OracleModel(cfg)
    kv = O.OracleKV(cfg)
    kv.prefill_synthetic()
    toks = [3, 90, 17, 42]
    prefix = O.OracleKV(cfg)
    prefix.prefill_synthetic()
    full = O.full_forward(m, toks, start=5, prefix=prefix)
    inc = torch.stack(O.teacher_forced(m, kv, toks, 5))
    assert (inc - full).norm() / full.norm() < 2e-6


def test_zero_mixers_closed_form():
    # With Wo = Wd = 0 the residual stream stays at the embedding: logits = W_head rmsnorm(E[t]) g_f.
    m = O.OracleModel(SMALL, zero=("wo", "w_down"))
    kv = O.OracleKV(SMALL)
    tok = 17
    got = O.decode_step(m, kv, tok, 0)
    e = synth.embedding(SMALL).double()[tok]
    gf = synth.norm_gain(SMALL, None, "final_norm").double()
    n = e / torch.sqrt((e * e).mean() + SMALL.rms_eps) * gf
    q, s = O.quantize_rows(synth.linear(SMALL, None, "lm_head"))
    want = (q.double() * s.double()[:, None]) @ n
    assert torch.allclose(got.double(), want, rtol=1e-5, atol=1e-5)


def _hf_model(om: O.OracleModel):
    from transformers import LlamaConfig, LlamaForCausalLM
    c = om.cfg
    hc = LlamaConfig(vocab_size=c.vocab, hidden_size=c.d_model, intermediate_size=c.ffn,
                     num_hidden_layers=c.n_layers, num_attention_heads=c.n_q_heads,
                     num_key_value_heads=c.n_kv_heads, head_dim=c.head_dim, rms_norm_eps=c.rms_eps,
                     rope_theta=c.rope_theta, tie_word_embeddings=c.tied, attention_bias=False, mlp_bias=False,
                     max_position_embeddings=4096, attn_implementation="eager")
    hf = LlamaForCausalLM(hc).eval()
    sd = {"model.embed_tokens.weight": om.embed, "model.norm.weight": om.final_norm}
    names = {"wq": "self_attn.q_proj", "wk": "self_attn.k_proj", "wv": "self_attn.v_proj", "wo": "self_attn.o_proj",
             "w_gate": "mlp.gate_proj", "w_up": "mlp.up_proj", "w_down": "mlp.down_proj"}
    for l in range(c.n_layers):
        for k_, n_ in names.items():
            sd[f"model.layers.{l}.{n_}.weight"] = om.weight(l, k_)
        sd[f"model.layers.{l}.input_layernorm.weight"] = om.attn_norm[l]
        sd[f"model.layers.{l}.post_attention_layernorm.weight"] = om.ffn_norm[l]
    sd["lm_head.weight"] = om.weight(None, "lm_head")
    missing, unexpected = hf.load_state_dict(sd, strict=False)
    assert not unexpected and all("rotary" in m_ for m_ in missing), (missing, unexpected)
    return hf


@pytest.mark.parametrize("cfg", [SMALL, synth.preset("tiny"), SMALL.with_(tied=True, name="pin_tied")],
                         ids=["small", "tiny", "small_tied"])
def test_matches_huggingface_llama(cfg):
    om = O.OracleModel(cfg)
    toks = synth.prompt_ids(cfg)[:8] if cfg.prompt_len else [1, 2, 3]
    hf = _hf_model(om)
    with torch.no_grad():
        ref = hf(torch.tensor([toks])).logits[0].float()
    ident = lambda t: t.to(torch.float32)
    kv = O.OracleKV(cfg, max_seq=len(toks), store=ident)
    inc = torch.stack(O.teacher_forced(om, kv, toks, 0))
    full = O.full_forward(om, toks, store=ident)
    for got in (inc, full):
        assert (got - ref).norm() / ref.norm() < 2e-5
        assert (got - ref).abs().max() < 1e-4 * ref.abs().max()


# ---------------------------------------------------------------------------------------------
# Planted mistakes (in the oracle, on the CPU) must be caught by the pins above.

def _hf_agrees(cfg=SMALL):
    om = O.OracleModel(cfg)
    toks = [5, 60, 7, 33, 2]
    hf = _hf_model(om)
    with torch.no_grad():
        ref = hf(torch.tensor([toks])).logits[0].float()
    kv = O.OracleKV(cfg, max_seq=len(toks), store=lambda t: t.to(torch.float32))
    inc = torch.stack(O.teacher_forced(om, kv, toks, 0))
    return float((inc - ref).norm() / ref.norm()) < 2e-5


def _mut_rope_interleaved(x, pos, theta):
    hd = x.shape[-1]
    c, s = O.rope_cos_sin(pos, hd, theta)
    x1, x2 = x[..., 0::2], x[..., 1::2]
    out = torch.empty_like(x)
    out[..., 0::2] = x1 * c - x2 * s
    out[..., 1::2] = x2 * c + x1 * s
    return out


def _mut_rope_sign(x, pos, theta):
    hd = x.shape[-1]
    c, s = O.rope_cos_sin(pos, hd, theta)
    x1, x2 = x[..., : hd // 2], x[..., hd // 2:]
    return torch.cat([x1 * c + x2 * s, x2 * c - x1 * s], dim=-1)


def _mut_attention_no_scale(q, k, v):
    hq, hd = q.shape
    return O.__dict__["_orig_attention"](q * math.sqrt(hd), k, v)


def _mut_attention_wrong_group(q, k, v):
    hq, hd = q.shape
    hkv = k.shape[0]
    out = torch.empty(hq, hd)
    for i in range(hq):
        h = i % hkv
        s = torch.matmul(k[h], q[i]) / math.sqrt(hd)
        p = torch.softmax(s, 0)
        out[i] = p @ v[h]
    return out


def _mut_rmsnorm_no_eps_mean(x, g, eps):
    x = x.to(torch.float32)
    return x / torch.sqrt((x * x).sum(-1, keepdim=True) + eps) * g


def _mut_silu_sigmoid(z):
    return 1.0 / (1.0 + torch.exp(-z))


@pytest.mark.parametrize("name,fn", [
    ("rope", _mut_rope_interleaved), ("rope", _mut_rope_sign), ("attention", _mut_attention_no_scale),
    ("attention", _mut_attention_wrong_group), ("rmsnorm", _mut_rmsnorm_no_eps_mean), ("silu", _mut_silu_sigmoid),
], ids=["rope_interleaved", "rope_sign", "attn_no_scale", "attn_wrong_group", "rmsnorm_sum", "silu_sigmoid"])
def test_planted_mistake_is_caught(monkeypatch, name, fn):
    assert _hf_agrees()
    monkeypatch.setitem(O.__dict__, "_orig_attention", O.attention)
    monkeypatch.setattr(O, name, fn)
    assert not _hf_agrees()
