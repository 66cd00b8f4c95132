"""Knob sweep of the persistent decode kernel.

The pages' schedule search tunes a fixed set of knobs (GEMV tile rows, attention KV block, pipeline
depth, threads) and keeps a change only when the result is still correct and at least 1 % faster.
This module does that search without an agent, over this kernel's own knobs:

* runtime options of `amk_create` (`amk_options`): `grid`, `kv_block`, `max_kv_chunks`;
* compile-time macros of the kernel (`build.TUNABLE`: ring slot size and depth, bulk copies in
  flight, L2 warm-up items and pacing, GEMV row batch), each value built as a variant library.

Search: the default build and options first, then every listed value of every knob alone
(coordinate search around the default), then the best kept value of each knob together. Each
library runs in its own process (a variant is loaded through AMK_LIB), which times every runtime
option set on one resident model.

Correctness gate: every candidate decodes the same teacher-forced token sequence as the default
(seeded token ids, the workload's first decode positions) and its logits must agree with the
default's: relative L2 difference <= 1e-3 per step and the same greedy token wherever the default's
top-2 margin exceeds 0.1. The default build itself is held to the oracle by the parity tests, so
agreement with it is agreement with the oracle within the parity tolerance.

Timing: CUDA events around K launches with device-side token feedback (the bench's loop), median of
three repeats; weights of the target workloads exceed L2, so no flush is needed between launches.

Usage (on a machine with a GPU):
    python -m decode_megakernel_launch_b200.sweep --config llama8b \\
        --knob kv_block=32,128 --knob AMK_PF_ITEMS=6,12 --out sweep.json
"""
from __future__ import annotations

import argparse
import json
import os
import re
import shutil
import subprocess
import sys
import tempfile
from typing import Dict, List, Optional, Tuple

from . import build as B

RUNTIME_KNOBS = ("grid", "kv_block", "max_kv_chunks")
REL_L2_MAX = 1e-3       # candidate vs default logits, per step
MARGIN = 0.1            # greedy tokens must match where the default's top-2 margin exceeds this
KEEP_GAIN = 0.01        # a kept setting is at least 1 % faster than the default


# ------------------------------------------------------------------------------------------------
# Host-side logic (no GPU)

def compile_defaults() -> Dict[str, int]:
    """Default values of the compile-time knobs, read from the kernel's header."""
    text = open(os.path.join(B.PKG, "csrc", "amk_internal.h")).read()
    out = {}
    for name in B.TUNABLE:
        m = re.search(r"#ifndef\s+%s\s*\n\s*#define\s+%s\s+(-?\d+)" % (name, name), text)
        if m:
            out[name] = int(m.group(1))
    return out


def parse_knob(spec: str) -> Tuple[str, List[int]]:
    """'kv_block=32,128' -> ('kv_block', [32, 128]); checks the name and the values."""
    if "=" not in spec:
        raise ValueError(f"knob spec {spec!r}: expected NAME=v1,v2,...")
    name, vals = spec.split("=", 1)
    name = name.strip()
    values = [int(v) for v in vals.split(",") if v.strip()]
    if not values:
        raise ValueError(f"knob {name}: no values")
    if name in RUNTIME_KNOBS:
        if any(v < 0 for v in values):
            raise ValueError(f"knob {name}: values must be >= 0 (0 = the library's default)")
    else:
        B.check_defines({name: v for v in values})
    return name, values


def candidate_key(c: dict) -> str:
    parts = [f"{k}={v}" for k, v in sorted(c["compile"].items())] + [f"{k}={v}" for k, v in sorted(c["runtime"].items())]
    return ",".join(parts) or "default"


def single_candidates(knobs: List[Tuple[str, List[int]]]) -> List[dict]:
    """The default, then each knob value alone; values equal to the default are skipped."""
    cdef = compile_defaults()
    out = [{"runtime": {}, "compile": {}}]
    seen = {candidate_key(out[0])}
    for name, values in knobs:
        for v in values:
            if name in RUNTIME_KNOBS:
                c = {"runtime": {name: v} if v != 0 else {}, "compile": {}}
            else:
                c = {"runtime": {}, "compile": {name: v} if cdef.get(name) != v else {}}
            k = candidate_key(c)
            if k not in seen:
                seen.add(k)
                out.append(c)
    return out


def combined_candidate(results: List[dict]) -> Optional[dict]:
    """The fastest kept value of each knob together, if at least two knobs have one."""
    best: Dict[str, dict] = {}
    for r in results:
        if not r.get("keep"):
            continue
        knob_items = list(r["runtime"].items()) + list(r["compile"].items())
        if len(knob_items) != 1:
            continue
        name = knob_items[0][0]
        if name not in best or r["ms"] < best[name]["ms"]:
            best[name] = r
    if len(best) < 2:
        return None
    c = {"runtime": {}, "compile": {}}
    for r in best.values():
        c["runtime"].update(r["runtime"])
        c["compile"].update(r["compile"])
    return c


def agreement(ref: List, got: List) -> Tuple[bool, float, int]:
    """(agrees, worst relative L2 difference, greedy-token mismatches where the margin is clear)
    of two lists of per-step logits (torch tensors)."""
    import torch
    worst, bad = 0.0, 0
    if len(ref) != len(got):
        return False, float("inf"), len(ref)
    for a, b in zip(ref, got):
        a, b = a.double(), b.double()
        if not bool(torch.isfinite(b).all()):
            return False, float("inf"), bad
        rel = float((a - b).norm() / max(float(a.norm()), 1e-30))
        worst = max(worst, rel)
        top = torch.topk(a, 2).values
        if float(top[0] - top[1]) > MARGIN and int(torch.argmax(a)) != int(torch.argmax(b)):
            bad += 1
    return worst <= REL_L2_MAX and bad == 0, worst, bad


def decide(results: List[dict]) -> None:
    """Marks `keep` on each result: correct and at least KEEP_GAIN faster than the default (the
    first result). The default itself is never 'kept'."""
    base = results[0]["ms"]
    for i, r in enumerate(results):
        r["keep"] = bool(i > 0 and r.get("correct") and r.get("ms") is not None
                         and r["ms"] <= base * (1.0 - KEEP_GAIN))
        if r.get("ms") is not None and base:
            r["speedup"] = base / r["ms"]


# ------------------------------------------------------------------------------------------------
# Worker: one library, several runtime option sets, one resident model (needs a GPU)

def _worker(args) -> None:
    import torch
    from . import amk, synth
    from .runtime import DeviceModel
    cfg = synth.preset(args.config)
    opts_list = json.loads(args.options)
    start = cfg.prefill_len + cfg.prompt_len
    span = cfg.decode_steps
    m = DeviceModel(cfg, options=opts_list[0])
    if cfg.prompt_len:
        for i, t in enumerate(synth.prompt_ids(cfg)):
            m.step(t, i)
    check_ids = synth.uniform_ids(cfg.seed, "sweep-check", args.check_steps, cfg.vocab)
    out = []
    for j, opts in enumerate(opts_list):
        if j:
            m.close()
            m._create(opts)
        logits = []
        for i, t in enumerate(check_ids):
            m.step(t, start + (i % span))
            logits.append(m.logits.detach().cpu().clone())
        stream = torch.cuda.current_stream()
        m.next_token.fill_(1)
        for k in range(args.warmup):
            m.step(-1 if k else 1, start + (k % span))
        times = []
        for _ in range(3):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            e0.record(stream)
            for k in range(args.steps):
                m.step(-1, start + ((args.warmup + k) % span))
            e1.record(stream)
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1) / args.steps)
        rc, detail = m.status()
        path = os.path.join(args.tmp, f"logits_{j}.pt")
        torch.save(logits, path)
        out.append({"ms": sorted(times)[1], "status": rc, "detail": detail, "logits": path,
                    "lib": amk.LIB_PATH})
    m.close()
    with open(args.result, "w") as f:
        json.dump(out, f)


def _run_library(compile_defs: dict, runtime_sets: List[dict], cfg_name: str, steps: int, warmup: int,
                 check_steps: int, tmp: str) -> List[dict]:
    """Builds the library variant and times every runtime option set on it in a child process."""
    try:
        lib = B.build_variant(compile_defs)
    except (subprocess.CalledProcessError, ValueError) as e:
        return [{"error": f"build failed: {type(e).__name__}"} for _ in runtime_sets]
    sub = tempfile.mkdtemp(prefix="lib_", dir=tmp)
    result = os.path.join(sub, "result.json")
    env = dict(os.environ, AMK_LIB=lib)
    cmd = [sys.executable, "-m", "decode_megakernel_launch_b200.sweep", "--worker", "--config", cfg_name,
           "--options", json.dumps(runtime_sets), "--steps", str(steps), "--warmup", str(warmup),
           "--check-steps", str(check_steps), "--tmp", sub, "--result", result]
    p = subprocess.run(cmd, env=env, cwd=os.path.dirname(B.PKG), capture_output=True, text=True)
    if p.returncode != 0:
        tail = (p.stderr or p.stdout).strip().splitlines()[-1:] or ["?"]
        return [{"error": f"worker exit {p.returncode}: {tail[0][:200]}"} for _ in runtime_sets]
    return json.load(open(result))


def evaluate(cands: List[dict], cfg_name: str, steps: int, warmup: int, check_steps: int, tmp: str,
             ref_logits=None) -> Tuple[List[dict], list]:
    """Runs the candidates (grouped by library); the first candidate is the reference unless
    `ref_logits` is given. Returns (results in candidate order, reference logits)."""
    import torch
    groups: Dict[str, List[int]] = {}
    for i, c in enumerate(cands):
        groups.setdefault(json.dumps(c["compile"], sort_keys=True), []).append(i)
    raw: List[Optional[dict]] = [None] * len(cands)
    for key, idx in groups.items():
        rs = _run_library(json.loads(key), [cands[i]["runtime"] for i in idx], cfg_name, steps, warmup,
                          check_steps, tmp)
        for i, r in zip(idx, rs):
            raw[i] = r
    results = []
    for c, r in zip(cands, raw):
        res = {"key": candidate_key(c), "runtime": c["runtime"], "compile": c["compile"]}
        if "error" in r:
            res.update(correct=False, ms=None, error=r["error"])
        else:
            logits = torch.load(r["logits"])
            if ref_logits is None:
                ref_logits = logits
            ok, rel, bad = agreement(ref_logits, logits)
            ok = ok and r["status"] == 0
            res.update(correct=ok, ms=r["ms"], rel_l2=rel, token_mismatches=bad, status=r["status"])
        results.append(res)
    return results, ref_logits


def sweep(knobs: List[Tuple[str, List[int]]], cfg_name: str, steps: int = 100, warmup: int = 5,
          check_steps: int = 8) -> dict:
    """Full search; returns the report (also what `--out` writes)."""
    tmp = tempfile.mkdtemp(prefix="amk_sweep_")
    try:
        cands = single_candidates(knobs)
        results, ref = evaluate(cands, cfg_name, steps, warmup, check_steps, tmp)
        if results[0].get("ms") is None or not results[0].get("correct"):
            raise RuntimeError(f"the default configuration failed: {results[0]}")
        decide(results)
        comb = combined_candidate(results)
        if comb is not None:
            # time the default again beside the combination, so both share one measurement window
            again, _ = evaluate([{"runtime": {}, "compile": {}}, comb], cfg_name, steps, warmup, check_steps, tmp, ref)
            decide(again)
            results.append(dict(again[1], combined=True, default_ms_same_run=again[0]["ms"]))
    finally:
        shutil.rmtree(tmp, ignore_errors=True)
    kept = [r for r in results if r.get("keep")]
    best = min(kept, key=lambda r: r["ms"] / (r.get("default_ms_same_run") or results[0]["ms"])) if kept else None
    return {"config": cfg_name, "steps": steps, "warmup": warmup, "check_steps": check_steps,
            "rule": f"correct (rel L2 <= {REL_L2_MAX} vs default, same greedy tokens where margin > {MARGIN}) "
                    f"and >= {KEEP_GAIN:.0%} faster",
            "compile_defaults": compile_defaults(), "results": results,
            "recommended": None if best is None else {"runtime": best["runtime"], "compile": best["compile"],
                                                       "speedup": best.get("speedup")}}


def main(argv=None) -> None:
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--config", default="llama8b")
    ap.add_argument("--knob", action="append", default=[], help="NAME=v1,v2 (runtime option or kernel macro)")
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--check-steps", type=int, default=8)
    ap.add_argument("--out", default=None)
    ap.add_argument("--worker", action="store_true", help=argparse.SUPPRESS)
    ap.add_argument("--options", default="[{}]", help=argparse.SUPPRESS)
    ap.add_argument("--tmp", default=None, help=argparse.SUPPRESS)
    ap.add_argument("--result", default=None, help=argparse.SUPPRESS)
    args = ap.parse_args(argv)
    if args.worker:
        _worker(args)
        return
    knobs = [parse_knob(k) for k in args.knob]
    rep = sweep(knobs, args.config, args.steps, args.warmup, args.check_steps)
    for r in rep["results"]:
        ms = "   failed" if r.get("ms") is None else f"{r['ms']:.4f} ms"
        print(f"{r['key']:40s} {ms}  correct={r.get('correct')}  keep={r.get('keep')}"
              f"  speedup={r.get('speedup', float('nan')):.4f}" + ("  (combined)" if r.get("combined") else ""))
    print("recommended:", json.dumps(rep["recommended"]))
    if args.out:
        with open(args.out, "w") as f:
            json.dump(rep, f, indent=1)


if __name__ == "__main__":
    main()
