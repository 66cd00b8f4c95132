"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the same seeded inputs."""
import ctypes as C

import pytest
import torch

from decode_megakernel_launch_b200 import synth
from oracle import llama_decode as O

pytestmark = pytest.mark.gpu

from tests.decode_harness import compare_logits, first_argmax, run_and_compare, run_gpu_chain  # noqa: E402


def _amk():
    from decode_megakernel_launch_b200 import amk, runtime
    return amk, runtime


# ---------------------------------------------------------------------------------------------
# Packer: integer work, bit-exact against the oracle's quantiser.

def _edge_rows(rows, cols, seed):
    w = synth.normal(seed, "packer", (rows, cols), std=0.02)
    w[0] = 0.0                                   # zero row -> s = 0, q = 0
    w[1] = 1e-39                                 # scale underflows to 0 in bf16
    w[2, 3] = 7.5                                # one outlier
    w[3] = torch.linspace(-3, 3, cols)           # ties of w/s
    w[4] = -w[4].abs()
    return w


@pytest.mark.parametrize("src_dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [(37, 64), (300, 576), (8, 14336)])
def test_packer_int8_bit_exact(src_dtype, shape):
    amk, rt = _amk()
    w = _edge_rows(*shape, seed=shape[0])
    if src_dtype == "bf16":
        w = w.to(torch.bfloat16).float()
    src = (w if src_dtype == "f32" else w.to(torch.bfloat16)).cuda().contiguous()
    packed, scales = rt.pack(amk.AMK_ROLE_PLAIN, None, src, amk.AMK_W_INT8)
    torch.cuda.synchronize()
    q_ref, s_ref = O.quantize_rows(w)
    q = packed.cpu().view(torch.int8).view(shape)
    assert torch.equal(q, q_ref)
    assert torch.equal(scales.cpu().float(), s_ref)


def _unpack_int4(packed: torch.Tensor, rows: int, cols: int) -> torch.Tensor:
    """Byte j of a row holds element 2j in its low nibble and 2j + 1 in its high one, each + 8."""
    b = packed.cpu().view(rows, cols // 2).to(torch.int16)
    q = torch.empty(rows, cols, dtype=torch.int16)
    q[:, 0::2] = (b & 15) - 8
    q[:, 1::2] = (b >> 4) - 8
    return q.to(torch.int8)


@pytest.mark.parametrize("src_dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [(37, 64), (300, 576), (8, 14336)])
def test_packer_int4_bit_exact(src_dtype, shape):
    amk, rt = _amk()
    w = _edge_rows(*shape, seed=shape[0] + 1)
    if src_dtype == "bf16":
        w = w.to(torch.bfloat16).float()
    src = (w if src_dtype == "f32" else w.to(torch.bfloat16)).cuda().contiguous()
    packed, scales = rt.pack(amk.AMK_ROLE_PLAIN, None, src, amk.AMK_W_INT4)
    torch.cuda.synchronize()
    assert packed.numel() == shape[0] * shape[1] // 2
    q_ref, s_ref = O.quantize_rows(w, 7)
    assert torch.equal(_unpack_int4(packed, *shape), q_ref)
    assert torch.equal(scales.cpu().float(), s_ref)


def test_packer_int4_rejects_odd_rows():
    amk, rt = _amk()
    with pytest.raises(ValueError):
        rt.pack(amk.AMK_ROLE_PLAIN, None, torch.ones(4, 5, device="cuda"), amk.AMK_W_INT4)


@pytest.mark.parametrize("role", ["qkv", "gate_up"])
def test_packer_row_order(role):
    amk, rt = _amk()
    cfg = synth.preset("tiny")
    dims = rt.dims_of(cfg)
    rows = cfg.qkv_rows if role == "qkv" else 2 * cfg.ffn
    r = amk.AMK_ROLE_QKV if role == "qkv" else amk.AMK_ROLE_GATE_UP
    w = synth.normal(3, "rows" + role, (rows, cfg.d_model), std=0.02)
    packed, scales = rt.pack(r, dims, w.cuda(), amk.AMK_W_INT8)
    torch.cuda.synchronize()
    q_ref, s_ref = O.quantize_rows(w)
    q = packed.cpu().view(torch.int8).view(rows, cfg.d_model)
    src = [amk.amk_packed_row_source(r, C.byref(dims), rows, i) for i in range(rows)]
    assert torch.equal(q, q_ref[src]) and torch.equal(scales.cpu().float(), s_ref[src])


def test_packer_bf16():
    amk, rt = _amk()
    w = _edge_rows(40, 128, seed=9)
    packed, scales = rt.pack(amk.AMK_ROLE_PLAIN, None, w.cuda(), amk.AMK_W_BF16)
    torch.cuda.synchronize()
    assert scales is None
    got = packed.cpu().view(torch.bfloat16).view(40, 128).float()
    assert torch.equal(got, O.bf16_round(w))


# ---------------------------------------------------------------------------------------------
# Whole decode step.

def test_tiny_megakernel_parity():
    res = run_and_compare(synth.preset("tiny"), compare_prompt=True)
    res.assert_ok()
    assert len(res.checks) == 16 + 32


def test_tiny_int4_megakernel_parity():
    res = run_and_compare(synth.preset("tiny_int4"), compare_prompt=True)
    res.assert_ok()
    assert len(res.checks) == 16 + 32


def test_tiny_int4_unfused_equals_megakernel_bitwise():
    amk, rt = _amk()
    cfg = synth.preset("tiny_int4")
    m = rt.DeviceModel(cfg)
    _, fed_a, kept_a, _ = run_gpu_chain(m, cfg, 16, 16)
    m.k_cache.zero_(); m.v_cache.zero_()
    _, fed_b, kept_b, _ = run_gpu_chain(m, cfg, 16, 16, unfused=True)
    m.close()
    assert fed_a == fed_b
    assert all(torch.equal(a, b) for a, b in zip(kept_a, kept_b))


def test_tiny_unfused_equals_megakernel_bitwise():
    amk, rt = _amk()
    cfg = synth.preset("tiny")
    m = rt.DeviceModel(cfg)
    _, fed_a, kept_a, nxt_a = run_gpu_chain(m, cfg, 32, 32)
    m.k_cache.zero_(); m.v_cache.zero_()
    _, fed_b, kept_b, nxt_b = run_gpu_chain(m, cfg, 32, 32, unfused=True)
    m.close()
    assert fed_a == fed_b and nxt_a == nxt_b
    for a, b in zip(kept_a, kept_b):
        assert torch.equal(a, b)


def test_tiny_unfused_parity():
    run_and_compare(synth.preset("tiny"), unfused=True).assert_ok()


def test_device_token_feedback_matches_host_loop():
    amk, rt = _amk()
    cfg = synth.preset("tiny")
    m = rt.DeviceModel(cfg)
    _, fed_a, kept_a, _ = run_gpu_chain(m, cfg, 32, 32)
    m.k_cache.zero_(); m.v_cache.zero_()
    _, fed_b, kept_b, _ = run_gpu_chain(m, cfg, 32, 32, feedback=True)
    m.close()
    assert fed_a == fed_b
    assert all(torch.equal(a, b) for a, b in zip(kept_a, kept_b))


def test_deterministic_across_runs():
    amk, rt = _amk()
    cfg = synth.preset("smollm135m", decode_steps=8)
    m = rt.DeviceModel(cfg)
    runs = []
    for _ in range(2):
        m.k_cache.zero_(); m.v_cache.zero_()
        runs.append(run_gpu_chain(m, cfg, 8, 8)[2])
    m.close()
    assert all(torch.equal(a, b) for a, b in zip(*runs))


@pytest.mark.parametrize("opts", [dict(grid=1), dict(grid=7), dict(grid=37, kv_block=1), dict(kv_block=4, max_kv_chunks=3)],
                         ids=["grid1", "grid7", "grid37_kv1", "kv4_c3"])
def test_tiny_launch_shapes(opts):
    run_and_compare(synth.preset("tiny"), options=opts).assert_ok()


ODD = [
    # group 3, d and ffn not multiples of 128, vocab not a multiple of anything
    synth.ModelConfig("odd_g3", 21, 3, 320, 6, 2, 64, 448, 1000, False, 1e4, prompt_len=9, decode_steps=12,
                      compare_steps=12),
    # head_dim 128, one KV head (group 4), tied head
    synth.ModelConfig("odd_hd128", 22, 2, 256, 4, 1, 128, 512, 777, True, 5e5, prompt_len=5, decode_steps=70,
                      compare_steps=70),
    # bf16 weights, group 1 (MHA)
    synth.ModelConfig("odd_bf16", 23, 2, 192, 3, 3, 64, 320, 515, False, 1e4, prompt_len=7, decode_steps=10,
                      compare_steps=10, weight_dtype="bf16"),
    # int4 weights with an int4 LM head, FFN of 3 x 256, odd vocab
    synth.ModelConfig("odd_int4", 24, 3, 512, 4, 2, 64, 768, 1001, False, 1e4, prompt_len=9, decode_steps=12,
                      compare_steps=12, weight_dtype="int4"),
    # int4 weights with a tied (bf16) head, head_dim 128, one KV head
    synth.ModelConfig("odd_int4_tied", 25, 2, 256, 2, 1, 128, 1280, 515, True, 5e5, prompt_len=5,
                      decode_steps=20, compare_steps=20, weight_dtype="int4"),
    # int4 rows that no whole number of warps covers: d 320 (160 bytes), ffn 448 (224 bytes)
    synth.ModelConfig("odd_int4_k320", 26, 2, 320, 5, 5, 64, 448, 999, False, 1e4, prompt_len=6,
                      decode_steps=10, compare_steps=10, weight_dtype="int4"),
]


@pytest.mark.parametrize("cfg", ODD, ids=[c.name for c in ODD])
def test_odd_shapes(cfg):
    run_and_compare(cfg, compare_prompt=True).assert_ok()


def test_first_and_last_position():
    amk, rt = _amk()
    cfg = synth.preset("tiny")
    # a one-position cache: pos 0 is both the first and the last valid position
    m = rt.DeviceModel(cfg, max_seq=1)
    m.step(5, 0)
    torch.cuda.synchronize()
    g = m.logits.cpu()
    nt = int(m.next_token.item())
    m.close()
    om = O.OracleModel(cfg)
    ref = O.decode_step(om, O.OracleKV(cfg, max_seq=1), 5, 0)
    c = compare_logits(g, ref, nt, 0, 0)
    assert c.ok, c
    assert nt == first_argmax(g)


def test_invalid_step_arguments_are_rejected_before_launch():
    amk, rt = _amk()
    cfg = synth.preset("tiny")
    m = rt.DeviceModel(cfg)
    st = torch.cuda.current_stream().cuda_stream
    for tok, pos in ((cfg.vocab, 0), (-2, 0), (0, cfg.max_seq), (0, -1)):
        assert amk.amk_decode_step(m.handle, tok, pos, m.logits.data_ptr(), m.next_token.data_ptr(), st) == amk.AMK_ERR_INVALID_ARG
    assert amk.amk_decode_step(m.handle, 0, 0, None, None, st) == amk.AMK_ERR_INVALID_ARG
    # logits_out may be NULL: only the next token is produced
    assert amk.amk_decode_step(m.handle, 3, 0, None, m.next_token.data_ptr(), st) == 0
    torch.cuda.synchronize()
    assert 0 <= int(m.next_token.item()) < cfg.vocab
    m.close()


def test_expired_wait_reports_timeout_and_context_survives():
    amk, rt = _amk()
    cfg = synth.preset("tiny")
    m = rt.DeviceModel(cfg, options=dict(test_drop_signal=3, timeout_ms=100))
    m.step(1, 0)
    torch.cuda.synchronize()
    rc, detail = m.status()
    assert rc == amk.AMK_ERR_DEVICE_TIMEOUT and (detail >> 16) & 0xFF == 1
    st = torch.cuda.current_stream().cuda_stream
    assert amk.amk_decode_step(m.handle, 1, 1, None, m.next_token.data_ptr(), st) == amk.AMK_ERR_DEVICE_TIMEOUT
    m.close()
    # the CUDA context is still usable: a fresh handle decodes correctly
    run_and_compare(synth.preset("tiny"), decode_steps=4, compare_steps=4).assert_ok()


def test_trace_records_every_task():
    amk, rt = _amk()
    cfg = synth.preset("tiny")
    m = rt.DeviceModel(cfg, options=dict(trace=1))
    m.step(1, 0)
    tr = m.trace()
    info = m.plan_info()
    m.close()
    done = tr[tr[:, 3] > 0]
    assert len(done) == info.n_tasks
    assert (done[:, 3] >= done[:, 1]).all()
    bd = rt.stage_breakdown(tr)
    assert bd["stages"] == 5 * cfg.n_layers + 1
    assert bd["span_us"] > 0 and abs(sum(bd["us"].values()) - bd["span_us"]) < 1e-6


# ---------------------------------------------------------------------------------------------
# Full-size configurations.

def test_smollm135m_parity_every_step():
    res = run_and_compare(synth.preset("smollm135m"), compare_prompt=True)
    res.assert_ok()
    assert len(res.checks) == 128 + 256


@pytest.mark.parametrize("wdt", ["int8", "bf16", "int4"])
def test_llama1b_parity(wdt):
    run_and_compare(synth.preset("llama1b", weight_dtype=wdt)).assert_ok()


@pytest.mark.slow
@pytest.mark.parametrize("wdt", ["int8", "bf16", "int4"])
def test_llama8b_parity(wdt):
    run_and_compare(synth.preset("llama8b", weight_dtype=wdt)).assert_ok()


@pytest.mark.slow
@pytest.mark.parametrize("name", ["llama1b_long4k", "llama1b_long16k", "llama1b_long32k"])
def test_long_context_parity(name):
    run_and_compare(synth.preset(name)).assert_ok()
