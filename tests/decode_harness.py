"""Shared GPU-vs-oracle harness: run the GPU greedy chain, teacher-force the oracle on it, compare.

Tolerances (per compared step, fp32 logits): relative L2 error <= 2e-2, max |delta| <= 5e-2 * max|logit|,
and the GPU's next token equal to the oracle's argmax whenever the oracle's top-1/top-2 margin > 0.1.
"""
from __future__ import annotations

import dataclasses
import time
from typing import List, Optional

import torch

from decode_megakernel_launch_b200 import synth
from oracle import llama_decode as O

REL_L2 = 2e-2
MAX_ABS_FRAC = 5e-2
MARGIN = 0.1


@dataclasses.dataclass
class StepCheck:
    step: int
    pos: int
    rel_l2: float
    max_abs_frac: float
    margin: float
    gpu_token: int
    ref_token: int

    @property
    def ok(self) -> bool:
        tok_ok = self.margin <= MARGIN or self.gpu_token == self.ref_token
        return self.rel_l2 <= REL_L2 and self.max_abs_frac <= MAX_ABS_FRAC and tok_ok


def compare_logits(gpu: torch.Tensor, ref: torch.Tensor, gpu_token: int, step: int, pos: int) -> StepCheck:
    gpu = gpu.double()
    ref = ref.double()
    rel = float((gpu - ref).norm() / ref.norm())
    mab = float((gpu - ref).abs().max() / ref.abs().max())
    return StepCheck(step, pos, rel, mab, O.top2_margin(ref.float()), gpu_token, O.argmax_lowest(ref.float()))


def first_argmax(x: torch.Tensor) -> int:
    m = x.max()
    return int(torch.nonzero(x == m)[0, 0])


@dataclasses.dataclass
class RunResult:
    checks: List[StepCheck]
    tokens: List[int]              # tokens fed at the decode positions (GPU chain)
    decode_logits: List[torch.Tensor]
    gpu_seconds: float
    oracle_seconds: float

    @property
    def gated(self) -> int:
        """Compared steps whose oracle top-1/top-2 margin exceeds MARGIN, i.e. whose greedy token was
        required to match the oracle's."""
        return sum(c.margin > MARGIN for c in self.checks)

    def assert_ok(self, min_gated: int = 1):
        bad = [c for c in self.checks if not c.ok]
        assert not bad, f"{len(bad)} of {len(self.checks)} steps out of tolerance, first: {bad[0]}"
        # a run where no step armed the token check would pass even with a broken margin or argmax
        assert self.gated >= min_gated, f"only {self.gated} of {len(self.checks)} steps had their token checked"


def run_gpu_chain(model, cfg: synth.ModelConfig, decode_steps: int, keep: int, unfused: bool = False,
                  feedback: bool = False, prompt_logits: bool = False):
    """Feeds the prompt (or starts after the prefill), then decodes greedily on the GPU.

    Returns (prompt logits [P, V] or None, fed decode tokens, logits of the first `keep` decode steps).
    """
    dev = model.device
    P = cfg.prompt_len
    plog = torch.empty(P, cfg.vocab, dtype=torch.float32, device=dev) if (prompt_logits and P) else None
    nt = model.next_token
    for i, t in enumerate(synth.prompt_ids(cfg)):
        model.step(t, i, logits=plog[i] if plog is not None else model.logits, unfused=unfused)
    start = P + cfg.prefill_len
    if P:
        tok = int(nt.item())
    else:
        tok = synth.first_decode_token(cfg)
    fed, kept = [], []
    out = torch.empty(max(keep, 1), cfg.vocab, dtype=torch.float32, device=dev)
    for s in range(decode_steps):
        fed.append(tok)
        lg = out[s] if s < keep else model.logits
        if feedback and s > 0:
            model.step(-1, start + s, logits=lg, unfused=unfused)
        else:
            model.step(tok, start + s, logits=lg, unfused=unfused)
        tok = int(nt.item())
    torch.cuda.synchronize(dev)
    kept = [out[s].cpu() for s in range(min(keep, decode_steps))]
    final_next = tok
    return (plog.cpu() if plog is not None else None), fed, kept, final_next


def run_and_compare(cfg: synth.ModelConfig, options: Optional[dict] = None, unfused: bool = False,
                    feedback: bool = False, decode_steps: Optional[int] = None, compare_steps: Optional[int] = None,
                    compare_prompt: bool = False, model=None) -> RunResult:
    from decode_megakernel_launch_b200.runtime import DeviceModel
    decode_steps = cfg.decode_steps if decode_steps is None else decode_steps
    compare_steps = cfg.compare_steps if compare_steps is None else compare_steps
    own = model is None
    t0 = time.time()
    if own:
        model = DeviceModel(cfg, options=options)
    plog, fed, kept, _ = run_gpu_chain(model, cfg, decode_steps, compare_steps, unfused=unfused, feedback=feedback,
                                       prompt_logits=compare_prompt)
    gtoks = [first_argmax(k) for k in kept]
    rc = model.status()[0]
    assert rc == 0, f"device status {model.status()}"
    if own:
        model.close()
        del model
    torch.cuda.empty_cache()
    t1 = time.time()

    om = O.OracleModel(cfg)
    kv = O.OracleKV(cfg)
    checks = []
    start = cfg.prompt_len + cfg.prefill_len
    if cfg.prefill_len:
        kv.prefill_synthetic()
    if cfg.prompt_len:
        full = O.full_forward(om, synth.prompt_ids(cfg), kv_out=kv)
        if plog is not None:
            for i in range(cfg.prompt_len):
                checks.append(compare_logits(plog[i], full[i], first_argmax(plog[i]), -1, i))
    t2 = time.time()
    for s in range(compare_steps):
        ref = O.decode_step(om, kv, fed[s], start + s)
        c = compare_logits(kept[s], ref, gtoks[s], s, start + s)
        # the kernel's own next token is the argmax of its logits (lowest index on ties)
        nxt = fed[s + 1] if s + 1 < len(fed) else None
        if nxt is not None:
            assert nxt == gtoks[s], f"step {s}: kernel next token {nxt} != argmax of its logits {gtoks[s]}"
        checks.append(c)
    t3 = time.time()
    return RunResult(checks, fed, kept, t1 - t0, (t3 - t2))
