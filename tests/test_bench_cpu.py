"""bench.py pieces that need no GPU: the CPU baseline and the reference arm's JSON line."""
import json
import os
import subprocess
import sys

import bench
from decode_megakernel_launch_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_oracle_baseline_times_full_depth_steps():
    tps, secs, sample, cores = bench.oracle_tokens_per_s(synth.preset("tiny"), steps=2)
    assert tps > 0 and cores >= 1 and secs > 0
    assert "full 2-layer tiny-shaped" in sample and "2 timed greedy step(s) from position 16" in sample


def test_oracle_decoder_follows_the_oracle_greedy_chain():
    # the timed steps are the oracle's own greedy chain from the prompt: same tokens as decode_step
    from oracle import llama_decode as O
    cfg = synth.preset("tiny")
    dec = bench.OracleDecoder(cfg)
    om, kv = O.OracleModel(cfg), O.OracleKV(cfg)
    tok = O.argmax_lowest(O.full_forward(om, synth.prompt_ids(cfg), kv_out=kv)[-1])
    assert dec.token == tok
    for s in range(3):
        dec.step()
        tok = O.argmax_lowest(O.decode_step(om, kv, tok, cfg.prompt_len + s))
        assert dec.token == tok


def test_reference_arm_prints_one_contract_line():
    p = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--config", "tiny", "--steps", "2",
                        "--warmup", "3"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["steps"] == 2 and d["warmup"] == 3 and d["higher_is_better"] is True
    assert d["metric"] == bench.metric_for(synth.preset("tiny"))
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["workload"]


def test_kernel_hash_ignores_comments_but_not_code(tmp_path, monkeypatch):
    # the DRAM-traffic ratio stays attached to counters taken on the same code: a comment edit keeps
    # the hash, a code edit changes it
    import shutil
    src = os.path.join(ROOT, "decode_megakernel_launch_b200", "csrc")
    dst = tmp_path / "decode_megakernel_launch_b200" / "csrc"
    shutil.copytree(src, dst)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    h0 = bench._kernel_hash()
    dev = dst / "amk_device.cu"
    text = dev.read_text()
    dev.write_text("// an added comment line\n" + text.replace("namespace amk {", "namespace amk {  /* inline */", 1))
    assert bench._kernel_hash() == h0
    dev.write_text(text + "\nstatic int amk_hash_probe = 1;\n")
    assert bench._kernel_hash() != h0


def test_traffic_ratio_is_reported_only_for_the_captured_sources():
    with open(os.path.join(ROOT, "profiles", "decode_kernel_dram_traffic.json")) as f:
        ent = json.load(f)["workloads"]["llama8b"]
    t = bench._dram_traffic("llama8b", 1e9)
    if ent["kernel"] == bench._kernel_hash():
        assert t == ent["ratio"] * 1e9
    else:
        assert t is None
