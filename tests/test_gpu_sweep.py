"""Knob sweep end to end on the GPU: every candidate passes the correctness gate against the default
build, and the report carries timings and keep decisions."""
import pytest

from decode_megakernel_launch_b200 import sweep as S

pytestmark = pytest.mark.gpu


def test_sweep_on_tiny_runs_runtime_and_compile_knobs():
    rep = S.sweep([("kv_block", [16]), ("AMK_PF_ITEMS", [6])], "tiny", steps=10, warmup=3, check_steps=6)
    res = rep["results"]
    assert [r["key"] for r in res[:3]] == ["default", "kv_block=16", "AMK_PF_ITEMS=6"]
    assert res[0]["rel_l2"] == 0.0 and res[0]["keep"] is False
    for r in res:
        assert r["correct"], r
        assert r["ms"] > 0 and r["status"] == 0
        assert r["rel_l2"] <= S.REL_L2_MAX and r["token_mismatches"] == 0
    assert rep["recommended"] is None or rep["recommended"]["speedup"] >= 1.0 + S.KEEP_GAIN - 1e-9
