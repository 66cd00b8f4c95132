"""GPU: the torch bf16 CUDA-graph comparator in bench.py computes the same decode step as the oracle.

The comparator is context for the bench line, not the product path; this checks that its timing is
the timing of a real decode step (same function, bf16 tolerances) and that a graph replay equals the
eager step it was recorded from.
"""
import pytest
import torch

from decode_megakernel_launch_b200 import synth
from oracle import llama_decode as O

pytestmark = pytest.mark.gpu

REL_L2 = 2e-2           # the decode step's tolerance; bf16 weights and activations stay well inside it


def _comparator_from_oracle(cfg, model, max_seq, start, span):
    import bench
    dev = "cuda"
    b = lambda t: t.to(torch.bfloat16).to(dev)  # noqa: E731
    L = cfg.n_layers
    w = {"embed": b(model.embed), "final_norm": b(model.final_norm),
         "attn_norm": [b(g) for g in model.attn_norm], "ffn_norm": [b(g) for g in model.ffn_norm],
         "wqkv": [b(torch.cat([model.weight(l, "wq"), model.weight(l, "wk"), model.weight(l, "wv")])) for l in range(L)],
         "wo": [b(model.weight(l, "wo")) for l in range(L)],
         "wgu": [b(torch.cat([model.weight(l, "w_gate"), model.weight(l, "w_up")])) for l in range(L)],
         "wd": [b(model.weight(l, "w_down")) for l in range(L)],
         "lm_head": b(model.weight(None, "lm_head"))}
    return bench.TorchBf16Step(cfg, w, max_seq, start, span)


def _rel_l2(a, b):
    return float((a - b).norm() / b.norm())


def test_bf16_comparator_matches_oracle_stepwise():
    cfg = synth.preset("tiny")
    model = O.OracleModel(cfg)
    kv = O.OracleKV(cfg)
    toks = synth.prompt_ids(cfg)[:12]
    comp = _comparator_from_oracle(cfg, model, cfg.max_seq, len(toks), 4)
    for pos, tok in enumerate(toks):
        want = O.decode_step(model, kv, int(tok), pos)
        got = comp.step_eager(int(tok), pos).cpu()
        assert torch.isfinite(got).all()
        assert _rel_l2(got, want) <= REL_L2, (pos, _rel_l2(got, want))


def test_bf16_comparator_graph_replay_equals_eager_step():
    cfg = synth.preset("tiny")
    model = O.OracleModel(cfg)
    toks = synth.prompt_ids(cfg)[:6]
    comp = _comparator_from_oracle(cfg, model, cfg.max_seq, 5, 4)
    for pos, tok in enumerate(toks[:5]):
        comp.step_eager(int(tok), pos)
    eager = comp.step_eager(int(toks[5]), 5).clone()
    comp.capture(int(toks[5]), 5)     # records the step at (token, 5) with greedy feedback
    comp.tok.fill_(int(toks[5]))
    comp.pos.fill_(5)
    comp.graph.replay()
    torch.cuda.synchronize()
    assert torch.allclose(comp.logits, eager, rtol=1e-5, atol=1e-5)
    assert int(comp.pos.item()) == 6   # advanced inside the graph (start 5, span 4)
    assert int(comp.tok.item()) == int(torch.argmax(eager).item())
