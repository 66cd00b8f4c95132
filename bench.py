"""Batch-1 decode benchmark: tokens/s and achieved HBM bandwidth of the persistent decode kernel.

Default workload: the Llama-3-8B-shaped synthetic model with W8A16 weights (int8 per output row,
bf16 scales), KV cache prefilled with N(0,1) bf16 values for positions 0..1023, greedy decode at
positions 1024..1151 (cycled when more steps are timed). One step = one token = one launch of the
persistent kernel over the whole forward pass. Weights (7.65 GB) are far larger than L2 (126 MB),
so no L2 flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--config NAME]

With --gpus N > 1 the script is launched by torch.distributed.run; each rank runs an independent
replica on its own GPU (the decode step does not shard), and rank 0 prints one JSON line whose value
is the sum over ranks of tokens decoded divided by the slowest rank's time.
`--impl reference` times the CPU oracle (the slow plain definition) on the host cores instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "batch-1 decode tokens/s (W8A16) and achieved HBM GB/s vs B200 peak"
DTYPE_TEXT = {"int8": "w8a16: int8 weights (bf16 row scales) x bf16 activations, quantised in the GEMV to int16 "
                      "per 16 elements (fp32 scale), exact int32 dot per 16 elements, fp32 accumulate; fp32 residual",
              "int4": "w4a16: int4 weights (bf16 row scales) x bf16 activations, quantised in the GEMV to int16 "
                      "per 32 elements (fp32 scale), exact int32 dot per 32 elements, fp32 accumulate; fp32 residual",
              "bf16": "bf16 weights x bf16 activations, fp32 accumulate; fp32 residual"}
# Every named shape, measured in the same run after the headline workload (bounded windows).
CONFIG_SET = [("smollm135m", {}), ("llama1b", {}), ("llama1b", {"weight_dtype": "bf16"}),
              ("llama8b", {"weight_dtype": "bf16"}), ("llama8b_int4", {}), ("llama1b_long4k", {}),
              ("llama1b_long16k", {}), ("llama1b_long32k", {})]
L2_BYTES = 126e6
# shapes whose oracle steps the bench also times on the host cores (a bounded sample: about a minute)
ORACLE_TIMED = ("smollm135m", "llama1b", "llama1b_long4k", "llama1b_long16k", "llama1b_long32k")


def metric_for(cfg) -> str:
    """The headline metric names the W8A16 workload; other weight dtypes say theirs instead."""
    tag = {"int8": "W8A16", "int4": "W4A16", "bf16": "bf16 weights"}[cfg.weight_dtype]
    return METRIC.replace("W8A16", tag)
FALLBACK_HBM_GBS = 6650.0


def _peak_hbm():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, copy bandwidth)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback (earlier copy measurement on this pool)"


def _workload_name(cfg):
    if cfg.prefill_len:
        return (f"{cfg.name}-shaped {cfg.weight_dtype} batch-1 greedy decode, KV prefilled 0..{cfg.prefill_len - 1}, "
                f"positions {cfg.prefill_len}..{cfg.prefill_len + cfg.decode_steps - 1}")
    return (f"{cfg.name}-shaped {cfg.weight_dtype} batch-1 greedy decode after a {cfg.prompt_len}-token prompt, "
            f"positions {cfg.prompt_len}..{cfg.prompt_len + cfg.decode_steps - 1}")


# ------------------------------------------------------------------------------------------------
# clocks during the timed region

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.out,
                                         stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc:
            time.sleep(0.15)
            self.proc.terminate()
            self.proc.wait(timeout=10)

    def summary(self):
        try:
            self.out.flush()
            rows = [l.split(",") for l in open(self.out.name).read().strip().splitlines() if l.strip()]
            os.unlink(self.out.name)
        except Exception:
            rows = []
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx = max(mx, float(r[2]))
                for n, v in zip(names, r[5:9]):
                    if v.strip().lower() == "active":
                        reasons.add(n)
            except (ValueError, IndexError):
                continue
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx or None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------------------------
# CPU baseline: the oracle as it stands, full-depth decode steps of the workload

class OracleDecoder:
    """The oracle as it stands, at full depth on the workload's own shape: an OracleModel (weights held
    as int8 / int4 codes plus scales and dequantised per use), a KV cache filled like the GPU's
    (the seeded prefill, or the prompt in one batched causal pass), then greedy decode steps at the
    workload's positions, cycling through its decode span like the GPU bench."""

    def __init__(self, cfg):
        import torch
        from oracle import llama_decode as O
        from decode_megakernel_launch_b200 import synth
        t0 = time.time()
        self.O, self.cfg = O, cfg
        self.threads = torch.get_num_threads()
        self.model = O.OracleModel(cfg, keep_dequantized=False)
        self.kv = O.OracleKV(cfg)
        self.start = cfg.prefill_len + cfg.prompt_len
        if cfg.prefill_len:
            self.kv.prefill_synthetic()
            self.token = synth.first_decode_token(cfg)
        else:
            ids = synth.prompt_ids(cfg)
            self.token = O.argmax_lowest(O.full_forward(self.model, ids, kv_out=self.kv)[-1])
        self.k = 0
        self.setup_s = time.time() - t0

    def step(self) -> float:
        """One full decode step; returns its wall time in seconds."""
        pos = self.start + self.k % max(1, self.cfg.decode_steps)
        t0 = time.perf_counter()
        logits = self.O.decode_step(self.model, self.kv, self.token, pos)
        dt = time.perf_counter() - t0
        self.token = self.O.argmax_lowest(logits)
        self.k += 1
        return dt

    def describe(self, n_timed: int) -> str:
        c = self.cfg
        return (f"oracle decode_step (torch CPU fp32, {self.threads} threads) on the full {c.n_layers}-layer "
                f"{c.name}-shaped model: {n_timed} timed greedy step(s) from position {self.start} "
                f"(model and cache set-up of {self.setup_s:.0f} s not timed)")


def oracle_tokens_per_s(cfg, steps=None):
    """(tokens/s on all host threads, seconds spent, sample description, threads): the wall time of
    the oracle's decode steps on the steps the parity tests compare (the workload's compare_steps;
    8B-shaped: the first 4)."""
    t_all = time.time()
    dec = OracleDecoder(cfg)
    n = steps or max(1, cfg.compare_steps)
    times = [dec.step() for _ in range(n)]
    return n / sum(times), time.time() - t_all, dec.describe(n), dec.threads


# ------------------------------------------------------------------------------------------------

def run_reference(args, cfg, rank, world):
    """The reference arm: the CPU oracle, W untimed and K timed full-depth decode steps of the same
    workload on the host cores (rank 0 only)."""
    if rank != 0:
        return
    dec = OracleDecoder(cfg)
    for _ in range(args.warmup):
        dec.step()
    timed = [dec.step() for _ in range(args.steps)]
    value = args.steps / sum(timed)
    line = {"impl": "reference", "metric": metric_for(cfg), "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 / value, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": _workload_name(cfg)},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": dec.threads, "kind": "oracle",
                             "sample": dec.describe(args.steps)},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


def measure_config(cfg, peak, steps=32, warmup=8, ablation_steps=4):
    """One named shape in a bounded window: tokens/s, per-token latency p50/p99, algorithmic bytes, GB/s
    and its fraction of the HBM peak, the op-per-kernel ablation, and the critical path per op of one
    traced step (for the long-context shapes also the attention share of bytes and of time)."""
    import torch
    from decode_megakernel_launch_b200 import synth
    from decode_megakernel_launch_b200.runtime import DeviceModel, stage_breakdown
    t0 = time.time()
    model = DeviceModel(cfg)
    if cfg.prompt_len:
        for i, t in enumerate(synth.prompt_ids(cfg)):
            model.step(t, i)
    start = cfg.prefill_len + cfg.prompt_len
    span = max(1, cfg.decode_steps)
    pos_of = lambda k: start + k % span
    model.next_token.fill_(1)
    for k in range(warmup):
        model.step(-1 if k else 1, pos_of(k))
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for k in range(steps):
        ev[k][0].record()
        model.step(-1, pos_of(warmup + k))
        ev[k][1].record()
    torch.cuda.synchronize()
    per = sorted(a.elapsed_time(b) for a, b in ev)
    rc, detail = model.status()
    if rc != 0:
        raise RuntimeError(f"{cfg.name}: device status {rc} detail {detail:#x}")
    ms = sum(per) / len(per)
    by = sum(model.step_bytes(pos_of(warmup + k)) for k in range(steps)) / steps
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record()
    for k in range(ablation_steps):
        model.step(-1, pos_of(k), unfused=True)
    a1.record()
    torch.cuda.synchronize()
    out = {"workload": _workload_name(cfg), "tokens_per_s": 1000.0 / ms, "ms_per_token": ms, "p50_ms": per[len(per) // 2],
           "p99_ms": per[min(len(per) - 1, int(0.99 * len(per)))], "bytes_per_step": by,
           "achieved_gbs": by / (ms / 1e3) / 1e9, "frac": by / (ms / 1e3) / 1e9 / peak,
           "unfused_ms_per_token": a0.elapsed_time(a1) / ablation_steps, "steps": steps}
    if by < 2 * L2_BYTES:
        out["l2_note"] = (f"{by / 1e6:.0f} MB per token against a {L2_BYTES / 1e6:.0f} MB L2: weights stay partly "
                          "L2-resident between steps, so GB/s may exceed what HBM alone gives")
    try:
        model.close()
        model._create(dict(trace=1))
        model.next_token.fill_(1)
        for k in range(3):
            model.step(-1 if k else 1, pos_of(k))
        bd = stage_breakdown(model.trace())
        out["stage_us"] = {k: round(v, 1) for k, v in bd["us"].items()}
        out["span_us"] = round(bd["span_us"], 1)
        if cfg.prefill_len >= 4096:
            kv = 2.0 * cfg.n_layers * cfg.n_kv_heads * (pos_of(2) + 1) * cfg.head_dim * 2
            out["attention_share"] = {"bytes": kv / model.step_bytes(pos_of(2)),
                                      "time": bd["us"].get("attn", 0.0) / max(bd["span_us"], 1e-9)}
    except Exception as e:  # diagnostics only
        out["stage_us"] = f"unavailable: {type(e).__name__}"
    model.close()
    del model
    torch.cuda.empty_cache()
    out["seconds"] = round(time.time() - t0, 1)
    return out


def max_over_ranks(x: float, device) -> float:
    """The largest of every rank's value: a replica job ends with its slowest rank, so device-timed
    regions are reduced with MAX (identity without an initialised process group of > 1 rank)."""
    import torch
    import torch.distributed as td
    if not (td.is_available() and td.is_initialized()) or td.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    td.all_reduce(t, op=td.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, steps_per_rank: int, max_ms: float) -> float:
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return world * steps_per_rank / (max_ms / 1000.0)


def run_gpu(args, cfg, rank, world, local_rank):
    import ctypes as C
    import torch
    from decode_megakernel_launch_b200 import amk
    from decode_megakernel_launch_b200.runtime import DeviceModel
    torch.cuda.set_device(local_rank)
    dist = world > 1
    if dist:
        import torch.distributed as td

    start = cfg.prefill_len + cfg.prompt_len
    span = cfg.decode_steps
    t_setup = time.time()
    model = DeviceModel(cfg, options=dict(kv_block=args.kv_block) if args.kv_block else None)
    if cfg.prompt_len:            # fill the prompt's KV once (positions 0..P-1)
        for i, t in enumerate(__import__("decode_megakernel_launch_b200.synth", fromlist=["x"]).prompt_ids(cfg)):
            model.step(t, i)
        torch.cuda.synchronize()
    setup_s = time.time() - t_setup
    stream = torch.cuda.current_stream()
    first_tok = 1
    model.next_token.fill_(first_tok)

    def pos_of(k):
        return start + (k % span)

    # warm-up (device feedback: token read from the previous step's next_token)
    for k in range(args.warmup):
        model.step(-1 if k else first_tok, pos_of(k))
    torch.cuda.synchronize()

    # ---- timed region: K launches, one CUDA event pair per launch on the launch stream ----
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        td.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clk:
        t_start.record(stream)
        for k in range(args.steps):
            ev[k][0].record(stream)
            model.step(-1, pos_of(args.warmup + k))
            ev[k][1].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize()
    if dist:
        td.barrier()
    elapsed_ms = t_start.elapsed_time(t_end)
    per = [a.elapsed_time(b) for a, b in ev]
    rc, detail = model.status()
    if rc != 0:
        raise RuntimeError(f"device status {rc} detail {detail:#x}")
    elapsed_ms = max_over_ranks(elapsed_ms, "cuda")
    value = job_throughput(world, args.steps, elapsed_ms)

    bytes_steps = [model.step_bytes(pos_of(args.warmup + k)) for k in range(args.steps)]
    avg_bytes = sum(bytes_steps) / len(bytes_steps)
    kernel_ms = sum(per) / len(per)
    peak, peak_src = _peak_hbm()
    achieved = avg_bytes / (kernel_ms / 1000.0) / 1e9

    # ---- end to end through the C ABI with host buffers: H2D token, step, D2H logits + token ----
    k_e2e = min(args.steps, span)
    h_tok = torch.empty(1, dtype=torch.int32, pin_memory=True)
    h_logits = torch.empty(cfg.vocab, dtype=torch.float32, pin_memory=True)
    h_next = torch.empty(1, dtype=torch.int32, pin_memory=True)
    d_tok = torch.empty(1, dtype=torch.int32, device="cuda")
    h_tok[0] = first_tok
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        td.barrier()
    torch.cuda.synchronize()
    w0 = time.perf_counter()
    e0.record(stream)
    for k in range(k_e2e):
        d_tok.copy_(h_tok, non_blocking=True)
        # the step reads its token from the device buffer (token_id -1), as a caller with a device-side
        # token would; the host token reaches it through the H2D copy above
        model.step(-1, pos_of(k), next_token=d_tok)
        h_logits.copy_(model.logits, non_blocking=True)
        h_next.copy_(d_tok, non_blocking=True)
        stream.synchronize()
        h_tok[0] = int(h_next[0])
    e1.record(stream)
    torch.cuda.synchronize()
    wall_e2e = time.perf_counter() - w0
    e2e_ms = e0.elapsed_time(e1)
    e2e_ms = max_over_ranks(e2e_ms, "cuda")
    e2e_value = job_throughput(world, k_e2e, e2e_ms)

    # ---- op-per-kernel ablation (same routines, one kernel per op), eager and CUDA-graph replay ----
    k_abl = min(args.steps, 32)
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    model.next_token.fill_(first_tok)
    for k in range(3):
        model.step(-1, pos_of(k), unfused=True)
    torch.cuda.synchronize()
    a0.record(stream)
    for k in range(k_abl):
        model.step(-1, pos_of(k), unfused=True)
    a1.record(stream)
    torch.cuda.synchronize()
    abl_ms = a0.elapsed_time(a1) / k_abl
    graph_ms = None
    try:
        g = torch.cuda.CUDAGraph()
        gs = torch.cuda.Stream()
        pos_g = pos_of(0)
        with torch.cuda.graph(g, stream=gs):
            model.step(-1, pos_g, stream=gs, unfused=True)
        torch.cuda.synchronize()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for _ in range(k_abl):
            g.replay()
        g1.record(stream)
        torch.cuda.synchronize()
        graph_ms = g0.elapsed_time(g1) / k_abl
        del g
    except Exception as e:  # capture is optional context, never the headline
        graph_ms = f"unavailable: {type(e).__name__}"
    info = model.plan_info()

    # ---- one traced step, outside every timed region: what each op adds to the critical path ----
    try:
        from decode_megakernel_launch_b200.runtime import stage_breakdown
        model.close()
        model._create(dict(trace=1, **(dict(kv_block=args.kv_block) if args.kv_block else {})))
        model.next_token.fill_(first_tok)
        for k in range(3):
            model.step(-1 if k else first_tok, pos_of(k))
        bd = stage_breakdown(model.trace())
        stages = {"us": {k: round(v, 2) for k, v in bd["us"].items()}, "span_us": round(bd["span_us"], 2),
                  "position": pos_of(2), "what": "critical-path microseconds per op of one traced step "
                  "(%globaltimer: a stage adds the time from the previous stage's last CTA to its own)"}
    except Exception as e:  # diagnostics only
        stages = {"unavailable": f"{type(e).__name__}: {e}"[:200]}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        tps, secs, sample, cores = oracle_tokens_per_s(cfg)
        cpu = {"value": tps, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample,
               "seconds": round(secs, 1)}

    traffic = _dram_traffic(cfg.name, avg_bytes)
    # the headline model's device memory goes before the other shapes and the comparator load theirs
    model.close()
    del model
    import gc
    gc.collect()
    torch.cuda.empty_cache()
    configs = None
    if rank == 0 and world == 1 and not args.no_configs:
        from decode_megakernel_launch_b200 import synth as _synth
        configs = {}
        for name, over in CONFIG_SET:
            c = _synth.preset(name, **over)
            key = f"{name}_{c.weight_dtype}" if over else name
            try:
                configs[key] = measure_config(c, peak)
            except Exception as e:  # one shape failing must not hide the headline
                configs[key] = {"unavailable": f"{type(e).__name__}: {e}"[:200]}
    if configs is not None and not args.no_cpu_baseline:
        # the oracle on the host cores, per named shape, over the steps the parity tests compare
        # (135M all 256, 1B the first 16, long contexts the first 4 per length; the 8B-shaped first 4
        # are the headline's cpu_baseline)
        for key in ORACLE_TIMED:
            if key not in configs or "unavailable" in configs[key]:
                continue
            try:
                tps, secs, sample, cores = oracle_tokens_per_s(_synth.preset(key))
                configs[key]["cpu_oracle"] = {"tokens_per_s": tps, "ms_per_step": 1000.0 / tps, "cores": cores,
                                              "sample": sample, "seconds": round(secs, 1)}
            except Exception as e:  # a reported baseline, never the headline
                configs[key]["cpu_oracle"] = {"unavailable": f"{type(e).__name__}: {e}"[:200]}
    comparator = None
    if world == 1 and not args.no_comparator:
        try:
            comparator = run_bf16_comparator(cfg, min(args.steps, 64), 3)
        except Exception as e:  # context only, never the headline
            comparator = {"unavailable": f"{type(e).__name__}: {e}"[:200]}

    if rank == 0:
        srt = sorted(per)
        line = {
            "metric": metric_for(cfg), "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": DTYPE_TEXT[cfg.weight_dtype],
            "data": "synthetic (seeded random-init weights of the named shape, N(0,1) KV prefill)",
            "config": {"workload": _workload_name(cfg), "grid": info.grid, "threads": info.threads,
                       "smem_bytes": info.smem_bytes, "l2": "weights+KV per step far exceed the 126 MB L2; no flush",
                       "parallelism": "replicas" if world > 1 else "single GPU"},
            "p50_ms": srt[len(srt) // 2], "p99_ms": srt[min(len(srt) - 1, int(0.99 * len(srt)))],
            "bytes_per_step": avg_bytes, "achieved_gbs": achieved, "stage_us": stages,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                         "traffic": traffic, "peak_source": peak_src,
                         "spec_frac": achieved / 8000.0},
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": 4,
                    "d2h_bytes_per_step": 4 * cfg.vocab + 4, "wall_s": wall_e2e},
            "gpu_launches": args.steps,
            "clocks": clk.summary(),
            "unfused": {"ms_per_step": abl_ms, "tokens_per_s": 1000.0 / abl_ms,
                        "launches_per_step": 6 * cfg.n_layers + 2,
                        "graph_ms_per_step": graph_ms},
            "cpu_baseline": cpu,
            "bf16_cublas_graph": comparator,
            "configs": configs,
            "setup_s": round(setup_s, 1),
        }
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------------------------
# Comparator: the same decode step as plain torch bf16 ops (matmuls on cuBLAS), one CUDA graph.

class TorchBf16Step:
    """One batch-1 decode step written with torch bf16 tensors on the GPU, for comparison only: every
    linear is an `F.linear` (a cuBLAS GEMV), attention is `scaled_dot_product_attention` over the
    whole cache with a position mask, and the step is recorded once as a CUDA graph whose replays
    read the token and position from device tensors and advance them (greedy feedback), so a replay
    is one full decode step with no host work. It is not the product path and shares no code with it.

    `w` holds bf16 CUDA tensors in source row order: embed [V, d]; per layer lists attn_norm, ffn_norm
    [d], wqkv [(Hq + 2 Hkv) hd, d], wo [d, Hq hd], wgu [2 ffn, d] (gate rows then up rows),
    wd [d, ffn]; final_norm [d]; lm_head [V, d]. KV caches are bf16 [L][Hkv, max_seq, hd].
    """

    def __init__(self, cfg, w, max_seq, start, span):
        import torch
        self.cfg, self.w, self.max_seq = cfg, w, max_seq
        dev = w["embed"].device
        hd, L = cfg.head_dim, cfg.n_layers
        self.k = [torch.zeros(cfg.n_kv_heads, max_seq, hd, dtype=torch.bfloat16, device=dev) for _ in range(L)]
        self.v = [torch.zeros_like(t) for t in self.k]
        inv = torch.pow(torch.tensor(float(cfg.rope_theta), dtype=torch.float64),
                        -2.0 * torch.arange(hd // 2, dtype=torch.float64) / hd)
        ang = torch.arange(max_seq, dtype=torch.float64)[:, None] * inv[None, :]
        self.cos = ang.cos().float().to(dev)
        self.sin = ang.sin().float().to(dev)
        self.ar = torch.arange(max_seq, device=dev)
        self.tok = torch.zeros(1, dtype=torch.long, device=dev)
        self.pos = torch.zeros(1, dtype=torch.long, device=dev)
        self.logits = torch.zeros(cfg.vocab, dtype=torch.float32, device=dev)
        self.start, self.span = start, span
        self.graph = None

    def _rms(self, x, g):
        import torch
        return (x * torch.rsqrt(x.pow(2).mean(-1, keepdim=True) + self.cfg.rms_eps) * g.float()).to(torch.bfloat16)

    def _rope(self, t, cos, sin):
        import torch
        a, b = t[..., : t.shape[-1] // 2], t[..., t.shape[-1] // 2:]
        return torch.cat([a * cos - b * sin, b * cos + a * sin], dim=-1)

    def _step(self, advance):
        import torch
        import torch.nn.functional as F
        c, w = self.cfg, self.w
        hq, hkv, hd = c.n_q_heads, c.n_kv_heads, c.head_dim
        pos = self.pos
        cos, sin = self.cos.index_select(0, pos), self.sin.index_select(0, pos)
        bias = torch.where(self.ar <= pos, 0.0, float("-inf")).view(1, 1, 1, -1).to(torch.bfloat16)
        x = w["embed"].index_select(0, self.tok).float()
        for l in range(c.n_layers):
            qkv = F.linear(self._rms(x, w["attn_norm"][l]), w["wqkv"][l]).float()
            q = self._rope(qkv[:, : hq * hd].view(hq, hd), cos, sin)
            k = self._rope(qkv[:, hq * hd: (hq + hkv) * hd].view(hkv, hd), cos, sin)
            v = qkv[:, (hq + hkv) * hd:].view(hkv, hd)
            self.k[l].index_copy_(1, pos, k.to(torch.bfloat16).unsqueeze(1))
            self.v[l].index_copy_(1, pos, v.to(torch.bfloat16).unsqueeze(1))
            o = F.scaled_dot_product_attention(q.to(torch.bfloat16).view(1, hq, 1, hd), self.k[l].unsqueeze(0),
                                               self.v[l].unsqueeze(0), attn_mask=bias, enable_gqa=True)
            x = x + F.linear(o.reshape(1, hq * hd), w["wo"][l]).float()
            gu = F.linear(self._rms(x, w["ffn_norm"][l]), w["wgu"][l]).float()
            a = F.silu(gu[:, : c.ffn]) * gu[:, c.ffn:]
            x = x + F.linear(a.to(torch.bfloat16), w["wd"][l]).float()
        self.logits.copy_(F.linear(self._rms(x, w["final_norm"]), w["lm_head"]).float()[0])
        if advance:
            self.tok.copy_(torch.argmax(self.logits).view(1))
            self.pos.copy_(self.start + torch.remainder(pos + 1 - self.start, self.span))

    def step_eager(self, token, pos):
        self.tok.fill_(token)
        self.pos.fill_(pos)
        self._step(advance=False)
        return self.logits

    def capture(self, token, pos):
        import torch
        self.tok.fill_(token)
        self.pos.fill_(pos)
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self._step(advance=False)            # library and kernel selection before capture
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self._step(advance=True)
        torch.cuda.synchronize()


def run_bf16_comparator(cfg, steps, warmup):
    """Times TorchBf16Step on random bf16 weights of `cfg`'s shape (values do not change the time;
    the step itself is checked against the oracle on a small model by the GPU tests)."""
    import torch
    dev = "cuda"
    gen = torch.Generator(device=dev).manual_seed(1234)

    def rnd(*shape, scale=0.02):
        return (torch.randn(*shape, generator=gen, device=dev, dtype=torch.float32) * scale).to(torch.bfloat16)

    c, L = cfg, cfg.n_layers
    qkv = (c.n_q_heads + 2 * c.n_kv_heads) * c.head_dim
    w = {"embed": rnd(c.vocab, c.d_model, scale=1.0), "final_norm": 1 + rnd(c.d_model),
         "attn_norm": [1 + rnd(c.d_model) for _ in range(L)], "ffn_norm": [1 + rnd(c.d_model) for _ in range(L)],
         "wqkv": [rnd(qkv, c.d_model) for _ in range(L)], "wo": [rnd(c.d_model, c.n_q_heads * c.head_dim) for _ in range(L)],
         "wgu": [rnd(2 * c.ffn, c.d_model) for _ in range(L)], "wd": [rnd(c.d_model, c.ffn) for _ in range(L)]}
    w["lm_head"] = w["embed"] if c.tied else rnd(c.vocab, c.d_model)
    start = c.prefill_len + c.prompt_len
    span = c.decode_steps
    m = TorchBf16Step(c, w, start + span, start, span)
    for l in range(L):
        m.k[l][:, :start] = torch.randn(c.n_kv_heads, start, c.head_dim, generator=gen, device=dev).to(torch.bfloat16)
        m.v[l][:, :start] = torch.randn(c.n_kv_heads, start, c.head_dim, generator=gen, device=dev).to(torch.bfloat16)
    m.capture(1, start)
    for _ in range(warmup):
        m.graph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        m.graph.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    wbytes = sum(t.numel() * 2 for k in ("wqkv", "wo", "wgu", "wd") for t in w[k])
    wbytes += (0 if c.tied else w["lm_head"].numel() * 2) + (c.vocab * c.d_model * 2 if c.tied else 0)
    kv_bytes = 2 * L * c.n_kv_heads * (start + span) * c.head_dim * 2
    out = {"what": "torch bf16 decode step (F.linear = cuBLAS GEMV, SDPA over the masked cache) replayed as one "
                   "CUDA graph; random bf16 weights of the same shape", "ms_per_step": ms, "tokens_per_s": 1000.0 / ms,
           "bytes_per_step": wbytes + kv_bytes, "achieved_gbs": (wbytes + kv_bytes) / (ms / 1000.0) / 1e9}
    del m, w
    torch.cuda.empty_cache()
    return out


def _dram_traffic(workload, algorithmic_bytes):
    """DRAM read+write bytes per launch: the measured traffic / algorithmic ratio recorded beside the
    ncu summary (profiles/decode_kernel_dram_traffic.json) times this launch's algorithmic bytes, or
    None when the ratio was taken on other kernel sources (or is missing)."""
    try:
        with open(os.path.join(ROOT, "profiles", "decode_kernel_dram_traffic.json")) as f:
            ent = json.load(f)["workloads"][workload]
        if ent["kernel"] == _kernel_hash():
            return float(ent["ratio"]) * algorithmic_bytes
    except (OSError, ValueError, KeyError, TypeError):
        return None
    return None


def _kernel_hash():
    """Hash of the kernel sources with comments and blank space removed, so that a comment edit does
    not disown counters taken on the same code."""
    import hashlib
    import re
    h = hashlib.sha1()
    for f in sorted(os.listdir(os.path.join(ROOT, "decode_megakernel_launch_b200", "csrc"))):
        text = open(os.path.join(ROOT, "decode_megakernel_launch_b200", "csrc", f), encoding="utf-8").read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(f.encode() + b"\0" + " ".join(text.split()).encode())
    return h.hexdigest()[:12]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    # defaults: 200 timed launches (8 warm-up) for the kernel; the reference arm (the CPU oracle, ~3 s
    # per full-depth 8B step) defaults to 20 (3 warm-up), so its run ends within a few minutes
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--impl", default="amk", choices=["amk", "reference"])
    ap.add_argument("--config", default="llama8b")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-comparator", action="store_true", help="skip the torch bf16 CUDA-graph comparator")
    ap.add_argument("--no-configs", action="store_true", help="skip the other named shapes (measured after the headline)")
    ap.add_argument("--kv-block", type=int, default=0, help="amk_options.kv_block (minimum positions per attention chunk)")
    ap.add_argument("--layers", type=int, default=0,
                    help="override the layer count (smaller cases for profiler captures; not a bench line)")
    args = ap.parse_args()
    if args.steps is None:
        args.steps = 20 if args.impl == "reference" else 200
    if args.warmup is None:
        args.warmup = 3 if args.impl == "reference" else 8
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    from decode_megakernel_launch_b200 import synth
    cfg = synth.preset(args.config)
    if args.layers:
        cfg = cfg.with_(n_layers=args.layers, name=f"{cfg.name}-{args.layers}layers")
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        run_reference(args, cfg, rank, world)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as td
        torch.cuda.set_device(local_rank)
        td.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    try:
        run_gpu(args, cfg, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as td
            td.destroy_process_group()


if __name__ == "__main__":
    main()
