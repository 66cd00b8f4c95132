"""Knob sweep: host-side search logic, the correctness gate and variant builds (no GPU)."""
import os

import pytest
import torch

from decode_megakernel_launch_b200 import build as B
from decode_megakernel_launch_b200 import sweep as S


def test_compile_defaults_match_the_header():
    d = S.compile_defaults()
    assert d["AMK_SLOT_BYTES"] == 65536 and d["AMK_SLOTS"] == 3 and d["AMK_INFLIGHT"] == 1
    assert set(d) == set(B.TUNABLE)
    for k, v in d.items():
        assert v in B.TUNABLE[k], (k, v)


def test_parse_knob_checks_names_and_values():
    assert S.parse_knob("kv_block=32,128") == ("kv_block", [32, 128])
    assert S.parse_knob("AMK_PF_ITEMS=6,12") == ("AMK_PF_ITEMS", [6, 12])
    for bad in ("kv_block", "kv_block=", "AMK_NOT_A_KNOB=1", "AMK_SLOTS=9", "grid=-1"):
        with pytest.raises(ValueError):
            S.parse_knob(bad)


def test_single_candidates_start_with_the_default_and_skip_default_values():
    c = S.single_candidates([("kv_block", [0, 32]), ("AMK_PF_ITEMS", [10, 6]), ("grid", [144])])
    keys = [S.candidate_key(x) for x in c]
    assert keys == ["default", "kv_block=32", "AMK_PF_ITEMS=6", "grid=144"]


def _res(key, runtime, compile_, ms, correct=True):
    return {"key": key, "runtime": runtime, "compile": compile_, "ms": ms, "correct": correct}


def test_keep_rule_needs_correctness_and_one_percent():
    rs = [_res("default", {}, {}, 2.000),
          _res("a", {"kv_block": 32}, {}, 1.985),           # 0.75 % faster: not kept
          _res("b", {"grid": 144}, {}, 1.970),              # 1.5 % faster: kept
          _res("c", {}, {"AMK_PF_ITEMS": 6}, 1.900, False),  # faster but wrong: not kept
          _res("d", {}, {"AMK_INFLIGHT": 3}, None, False)]   # failed
    S.decide(rs)
    assert [r["keep"] for r in rs] == [False, False, True, False, False]
    assert rs[2]["speedup"] == pytest.approx(2.0 / 1.97)


def test_combined_candidate_takes_the_best_kept_value_per_knob():
    rs = [_res("default", {}, {}, 2.0),
          _res("g1", {"grid": 144}, {}, 1.96), _res("g2", {"grid": 132}, {}, 1.95),
          _res("p", {}, {"AMK_PF_ITEMS": 6}, 1.97), _res("k", {"kv_block": 32}, {}, 2.1)]
    S.decide(rs)
    c = S.combined_candidate(rs)
    assert c == {"runtime": {"grid": 132}, "compile": {"AMK_PF_ITEMS": 6}}
    assert S.combined_candidate(rs[:3]) is None       # one knob only


def test_agreement_gate_catches_small_planted_errors():
    g = torch.Generator().manual_seed(0)
    ref = [torch.randn(1000, generator=g) for _ in range(4)]
    ok, rel, bad = S.agreement(ref, [r.clone() for r in ref])
    assert ok and rel == 0.0 and bad == 0
    noisy = [r + 1e-5 * torch.randn(1000, generator=g) for r in ref]
    assert S.agreement(ref, noisy)[0]
    # a dropped term (one logit off by 10 %) exceeds the relative L2 bound
    off = [r.clone() for r in ref]
    off[2] = off[2] * 1.1
    assert not S.agreement(ref, off)[0]
    # a different greedy token with a clear margin fails even when the L2 change is tiny
    big = torch.randn(100000, generator=g) * 10.0
    big[5], big[7] = 100.0, 99.8                      # margin 0.2 > 0.1
    swapped = big.clone()
    swapped[5], swapped[7] = 99.8, 100.0
    ok, rel, bad = S.agreement([big], [swapped])
    assert rel < S.REL_L2_MAX and bad == 1 and not ok
    near = big.clone()
    near[7] = 99.95                                   # margin 0.05: a swap there is allowed
    near_sw = near.clone()
    near_sw[5], near_sw[7] = 99.95, 100.0
    assert S.agreement([near], [near_sw])[0]
    nan = [r.clone() for r in ref]
    nan[0][3] = float("nan")
    assert not S.agreement(ref, nan)[0]
    assert not S.agreement(ref, ref[:3])[0]


def test_variant_tag_and_defines():
    assert B.variant_tag({}) == "default"
    assert B.variant_tag({"AMK_PF_ITEMS": 6, "AMK_INFLIGHT": 3}) == "inflight-3_pf_items-6"
    with pytest.raises(ValueError):
        B.check_defines({"AMK_SLOT_BYTES": 1000})


def test_variant_library_builds_and_loads_its_symbols():
    import ctypes as C
    path = B.build_variant({"AMK_PF_ITEMS": 6})
    assert os.path.basename(path) == "libamk_pf_items-6.so" and os.path.exists(path)
    lib = C.CDLL(path)
    assert hasattr(lib, "amk_decode_step") and hasattr(lib, "amk_create")


def test_oversized_ring_is_rejected_by_the_kernel_checks():
    # 4 x 64 KB slots exceed one CTA's shared memory: the static check stops the build
    import subprocess
    with pytest.raises(subprocess.CalledProcessError):
        B.build_variant({"AMK_SLOTS": 4}, force=True)
