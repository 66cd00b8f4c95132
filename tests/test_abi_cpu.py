"""C-ABI checks that need no GPU: the library loads, exports every declared call, and its host-only
logic (packed row order, byte model, argument checks, the static task-list checker) behaves."""
import ctypes as C

import pytest

from decode_megakernel_launch_b200 import synth

amk = pytest.importorskip("decode_megakernel_launch_b200.amk", reason="libamk.so not built")
from decode_megakernel_launch_b200.runtime import dims_of  # noqa: E402

CONFIGS = ["tiny", "smollm135m", "llama1b", "llama8b", "llama1b_long32k", "tiny_int4", "llama1b_int4",
           "llama8b_int4"]


def test_every_declared_symbol_is_exported():
    names = amk.exported_symbols_in_header()
    assert "amk_decode_step" in names and "amk_create" in names
    for n in names:
        assert hasattr(amk.lib, n), n


def test_packed_bytes():
    assert amk.amk_packed_bytes(6144, 4096, amk.AMK_W_INT8) == 6144 * 4096
    assert amk.amk_packed_bytes(6144, 4096, amk.AMK_W_BF16) == 2 * 6144 * 4096
    assert amk.amk_packed_bytes(6144, 4096, amk.AMK_W_INT4) == 6144 * 4096 // 2
    assert amk.amk_packed_bytes(3, 5, amk.AMK_W_INT4) == 0          # two nibbles per byte: even rows only
    assert amk.amk_packed_bytes(-1, 4, amk.AMK_W_INT8) == 0
    assert amk.amk_packed_bytes(4, 4, 7) == 0


def test_packed_row_order_is_a_pairing_permutation():
    cfg = synth.preset("llama8b")
    d = dims_of(cfg)
    rows = cfg.qkv_rows
    src = [amk.amk_packed_row_source(amk.AMK_ROLE_QKV, C.byref(d), rows, r) for r in range(rows)]
    assert sorted(src) == list(range(rows))
    hd = cfg.head_dim
    for r in range(0, rows, 2):
        head = r // hd
        i = (r % hd) // 2
        assert src[r] == head * hd + i and src[r + 1] == head * hd + i + hd // 2
    gu = [amk.amk_packed_row_source(amk.AMK_ROLE_GATE_UP, C.byref(d), 2 * cfg.ffn, r) for r in range(2 * cfg.ffn)]
    assert gu[:4] == [0, cfg.ffn, 1, cfg.ffn + 1] and sorted(gu) == list(range(2 * cfg.ffn))
    assert amk.amk_packed_row_source(amk.AMK_ROLE_O, C.byref(d), 10, 7) == 7
    assert amk.amk_packed_row_source(amk.AMK_ROLE_QKV, None, rows, 0) == -1
    assert amk.amk_packed_row_source(amk.AMK_ROLE_PLAIN, None, 10, 10) == -1


def test_step_bytes_model():
    cfg = synth.preset("llama8b")
    d = dims_of(cfg)
    b = amk.amk_step_bytes(C.byref(d), 1023)
    L, dm, ffn, V = 32, 4096, 14336, 128256
    w = L * ((6144 + 4096) * dm + 2 * ffn * dm + dm * ffn) + V * dm
    scales = 2 * (L * (6144 + dm + 2 * ffn + dm) + V)
    kv = 2 * L * 8 * 1024 * 128 * 2
    assert b == w + scales + dm * 2 + (2 * L + 1) * dm * 2 + kv
    assert 7.5e9 < b < 7.8e9
    d.weight_dtype = amk.AMK_W_BF16
    assert amk.amk_step_bytes(C.byref(d), 1023) > 1.9 * b
    d.weight_dtype = amk.AMK_W_INT4
    assert amk.amk_step_bytes(C.byref(d), 1023) == w // 2 + scales + dm * 2 + (2 * L + 1) * dm * 2 + kv
    assert amk.amk_step_bytes(None, 0) == 0


def test_step_bytes_int4_tied_head_stays_bf16():
    # 1B shape, tied head: the head reads the bf16 embedding table, the layers read nibbles
    d = dims_of(synth.preset("llama1b_int4"))
    L, dm, ffn, V, qkv = 16, 2048, 8192, 128256, 3072
    w = L * ((qkv + dm) * dm + 3 * ffn * dm)
    scales = 2 * L * (qkv + dm + 2 * ffn + dm)
    assert amk.amk_step_bytes(C.byref(d), 0) == w // 2 + scales + V * dm * 2 + dm * 2 + (2 * L + 1) * dm * 2 \
        + 2 * L * 8 * 64 * 2
    d8 = dims_of(synth.preset("llama1b", weight_dtype="bf16"))
    # weight bytes fall by about the 2.42x the int4 variant is quoted with (per-row scales: 2.44x)
    assert 2.40 < amk.amk_step_bytes(C.byref(d8), 0) / amk.amk_step_bytes(C.byref(d), 0) < 2.46


@pytest.mark.parametrize("name", CONFIGS)
@pytest.mark.parametrize("grid", [148, 132, 16, 3])
def test_plan_accepted(name, grid):
    rc, msg = amk.plan_check(dims_of(synth.preset(name)), grid)
    assert rc == amk.AMK_OK, msg


@pytest.mark.parametrize("mutation", [1, 2, 3, 4, 5])
@pytest.mark.parametrize("name", ["tiny", "llama8b"])
def test_plan_defects_rejected(name, mutation):
    rc, msg = amk.plan_check(dims_of(synth.preset(name)), 148, mutation)
    assert rc == amk.AMK_ERR_PLAN, msg
    assert msg and msg != "ok"


def test_unsupported_dims_rejected():
    d = dims_of(synth.preset("tiny"))
    d.head_dim = 96
    assert amk.plan_check(d, 148)[0] == amk.AMK_ERR_UNSUPPORTED


def test_int4_rows_need_only_the_common_multiple_of_64():
    # int4 rows that no whole number of warps covers run with the last warp partly idle
    d = dims_of(synth.preset("tiny_int4"))
    assert amk.plan_check(d, 148)[0] == amk.AMK_OK
    for k in (704, 320, 64):
        d.ffn = k
        assert amk.plan_check(d, 148)[0] == amk.AMK_OK, k
    d.ffn = 672 + 2                                   # not a multiple of 64
    assert amk.plan_check(d, 148)[0] == amk.AMK_ERR_UNSUPPORTED
    d.ffn = 704
    d.weight_dtype = amk.AMK_W_INT8
    assert amk.plan_check(d, 148)[0] == amk.AMK_OK
    d = dims_of(synth.preset("tiny"))
    d.n_q_heads = 16          # group of 8
    assert amk.plan_check(d, 148)[0] == amk.AMK_ERR_UNSUPPORTED
    d = dims_of(synth.preset("tiny"))
    d.ffn = 700
    assert amk.plan_check(d, 148)[0] == amk.AMK_ERR_UNSUPPORTED
    d = dims_of(synth.preset("tiny"))
    d.n_layers = 0
    assert amk.plan_check(d, 148)[0] == amk.AMK_ERR_INVALID_ARG


def test_argument_errors_before_any_launch():
    h = C.c_void_p()
    assert amk.amk_create(None, None, None, C.byref(h)) == amk.AMK_ERR_INVALID_ARG
    assert amk.amk_create(None, None, None, None) == amk.AMK_ERR_INVALID_ARG
    assert amk.amk_decode_step(None, 0, 0, None, None, None) == amk.AMK_ERR_INVALID_ARG
    assert amk.amk_decode_step_unfused(None, 0, 0, None, None, None) == amk.AMK_ERR_INVALID_ARG
    assert amk.amk_status(None, None) == amk.AMK_ERR_INVALID_ARG
    d = dims_of(synth.preset("tiny"))
    assert amk.amk_pack_weight(amk.AMK_ROLE_QKV, C.byref(d), None, 0, 512, 256, 0, None, None, None) == amk.AMK_ERR_INVALID_ARG
    # wrong shape for the role is rejected on the host
    assert amk.amk_pack_weight(amk.AMK_ROLE_QKV, C.byref(d), 16, 0, 100, 256, 0, 16, 16, None) == amk.AMK_ERR_INVALID_ARG
    assert amk.amk_pack_weight(amk.AMK_ROLE_PLAIN, None, 16, 0, 4, 4, 0, 16, None, None) == amk.AMK_ERR_INVALID_ARG
    assert amk.amk_trace_read(None, None, 0) == amk.AMK_ERR_INVALID_ARG


def test_trace_op_codes_match_the_kernel():
    import os
    import re
    text = open(os.path.join(os.path.dirname(amk.HEADER), "..", "decode_megakernel_launch_b200", "csrc",
                             "amk_internal.h")).read()
    enum = {m.group(1): int(m.group(2)) for m in re.finditer(r"\bOP_(\w+)\s*=\s*(\d+)", text)}
    for name in ("QKV", "ATTN", "O", "GU", "DOWN", "LM"):
        assert getattr(amk, "AMK_OP_" + name) == enum[name], name


def test_stage_breakdown_of_a_synthetic_trace():
    import numpy as np
    from decode_megakernel_launch_b200.runtime import stage_breakdown

    def rec(op, layer, ti, t0, t1, t2):
        return [(op << 32) | (layer << 16) | ti, t0, t1, t2]
    # two CTAs, one layer: QKV ends at 3000 ns (slowest CTA), ATTN at 7000, O 9000, GU 15000, DOWN
    # 18000, LM 21000; the step starts at 1000 (first wait-start); one unused (zero) record
    tr = np.array([rec(1, 0, 0, 1000, 1500, 2500), rec(1, 0, 0, 1200, 1600, 3000),
                   rec(2, 0, 1, 3100, 3200, 7000), rec(2, 0, 1, 3000, 3300, 5000),
                   rec(3, 0, 2, 7000, 7100, 9000), rec(4, 0, 3, 9000, 9100, 15000),
                   rec(5, 0, 4, 15000, 15100, 18000), rec(6, 0, 5, 18000, 18100, 21000),
                   [0, 0, 0, 0]], dtype=np.uint64)
    bd = stage_breakdown(tr)
    assert bd["stages"] == 6
    assert bd["us"] == {"qkv": 2.0, "attn": 4.0, "o": 2.0, "gu": 6.0, "down": 3.0, "lm": 3.0}
    assert bd["span_us"] == 20.0 == sum(bd["us"].values())
    assert stage_breakdown(np.zeros((3, 4), dtype=np.uint64))["stages"] == 0


def test_step_byte_model_reproduces_the_pages_ratios():
    import json
    import os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_ratios.json")))
    b8 = amk.amk_step_bytes(C.byref(dims_of(synth.preset("llama1b"))), 0)
    b16 = amk.amk_step_bytes(C.byref(dims_of(synth.preset("llama1b", weight_dtype="bf16"))), 0)
    b4 = amk.amk_step_bytes(C.byref(dims_of(synth.preset("llama1b_int4"))), 0)
    r = g["int8_over_bf16_step_bytes"]
    assert abs(b8 / b16 - r["value"]) <= r["tolerance"], b8 / b16
    r = g["bf16_over_int4_weight_bytes"]
    assert abs(b16 / b4 - r["value"]) <= r["tolerance"], b16 / b4
