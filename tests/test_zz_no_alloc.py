"""amk_decode_step_noalloc against amk_decode_step.

The no-allocation entry point serves callers that can't call cudaMalloc: a plugin whose host
framework's memory pool owns the device memory (an outside allocation fails near the pool's limit or
is forbidden by its policy), or a latency-critical loop where cudaMalloc/cudaFree may synchronize the
device. It keeps its state in one fixed 4 MiB static device array instead of allocating, and launches
the same kernel on the same plan as amk_decode_step, so its results must be bit-identical: these tests
call both through the C ABI on the same inputs, step after step (every call after the first reuses
the array the previous call left), and compare logits, next token and the K/V rows each call writes.
They also check that dims needing more than the array are rejected before any launch, and that a
reload of the array is refused while the stream is capturing.
This file is collected last on purpose, and each test also passes alone in a fresh process.
"""
import ctypes as C

import pytest
import torch

from decode_megakernel_launch_b200 import synth

pytestmark = pytest.mark.gpu

CASES = {
    "tiny_int8": synth.preset("tiny"),
    "tiny_int4": synth.preset("tiny_int4"),
    "tiny_bf16": synth.preset("tiny", weight_dtype="bf16"),
    # a prefilled cache: decoding starts at position 40 over 40 seeded N(0,1) keys and values
    "tiny_prefilled": synth.preset("tiny").with_(name="tiny_prefilled", prompt_len=0, prefill_len=40,
                                                  decode_steps=12, compare_steps=12),
    "smollm135m": synth.preset("smollm135m", decode_steps=8),   # tied head, odd row sizes
}


def _weights(model, k_cache, v_cache):
    from decode_megakernel_launch_b200 import amk
    keep = []

    def arr(ts):
        a = (C.c_void_p * len(ts))(*[None if t is None else t.data_ptr() for t in ts])
        keep.append(a)
        return C.cast(a, C.POINTER(C.c_void_p))

    i8 = model.dims.weight_dtype != amk.AMK_W_BF16   # quantised: per-row scales
    w = amk.amk_weights(
        model.embed.data_ptr(), arr(model.attn_norm), arr(model.ffn_norm), model.final_norm.data_ptr(),
        arr(model.w["qkv"]), arr(model.w["o"]), arr(model.w["gu"]), arr(model.w["down"]),
        None if model.lm_w is None else model.lm_w.data_ptr(),
        arr(model.s["qkv"]) if i8 else None, arr(model.s["o"]) if i8 else None,
        arr(model.s["gu"]) if i8 else None, arr(model.s["down"]) if i8 else None,
        None if model.lm_s is None else model.lm_s.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr())
    return w, keep


@pytest.mark.parametrize("name", list(CASES))
def test_noalloc_is_bitwise_equal_to_decode_step_call_after_call(name):
    from decode_megakernel_launch_b200 import amk
    from decode_megakernel_launch_b200.runtime import DeviceModel
    cfg = CASES[name]
    model = DeviceModel(cfg)
    # the no-allocation calls get their own copy of the cache (prefilled part included)
    k2, v2 = model.k_cache.clone(), model.v_cache.clone()
    w2, keep = _weights(model, k2, v2)
    dims = model.dims
    lg_a = torch.empty(cfg.vocab, dtype=torch.float32, device="cuda")
    lg_b = torch.empty_like(lg_a)
    nt_a = torch.zeros(1, dtype=torch.int32, device="cuda")
    nt_b = torch.zeros_like(nt_a)
    stream = torch.cuda.current_stream().cuda_stream
    # the prompt (or the first decode token) and then the greedy chain of the handle-based calls
    tokens = synth.prompt_ids(cfg) if cfg.prompt_len else [synth.first_decode_token(cfg)]
    start = cfg.prefill_len
    n_steps = 10
    assert start + n_steps <= cfg.max_seq
    tok = tokens[0]
    for s in range(n_steps):
        pos = start + s
        model.step(tok, pos, logits=lg_a, next_token=nt_a)
        rc = amk.amk_decode_step_noalloc(C.byref(dims), C.byref(w2), tok, pos, lg_b.data_ptr(), nt_b.data_ptr(), stream)
        assert rc == amk.AMK_OK
        torch.cuda.synchronize()
        assert torch.equal(lg_a, lg_b), f"step {s}: logits differ (max {float((lg_a - lg_b).abs().max()):.3e})"
        assert int(nt_b.item()) == int(nt_a.item())
        assert torch.equal(k2[:, :, pos], model.k_cache[:, :, pos]) and torch.equal(v2[:, :, pos], model.v_cache[:, :, pos])
        tok = tokens[s + 1] if s + 1 < len(tokens) else int(nt_a.item())
    assert model.status()[0] == 0
    model.close()
    del keep


def test_noalloc_rejects_dims_beyond_its_scratch_and_reloads_under_capture():
    from decode_megakernel_launch_b200 import amk
    from decode_megakernel_launch_b200.runtime import DeviceModel
    cfg = synth.preset("tiny")
    model = DeviceModel(cfg)
    w, keep = _weights(model, model.k_cache, model.v_cache)
    big = amk.amk_dims.from_buffer_copy(model.dims)
    big.max_seq = 200000          # RoPE table alone would need ~51 MB
    nt = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    rc = amk.amk_decode_step_noalloc(C.byref(big), C.byref(w), 1, 0, None, nt.data_ptr(), stream)
    assert rc == amk.AMK_ERR_SCRATCH_LIMIT
    assert amk.amk_decode_step_noalloc(C.byref(model.dims), C.byref(w), cfg.vocab, 0, None, nt.data_ptr(),
                                       stream) == amk.AMK_ERR_INVALID_ARG
    torch.cuda.synchronize()
    # the array holds another model now (or nothing): a call that would reload it while the stream
    # captures is refused before anything is enqueued, and the capture stays valid
    other = amk.amk_dims.from_buffer_copy(model.dims)
    other.max_seq = model.dims.max_seq - 1
    cs = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cs):
        rc = amk.amk_decode_step_noalloc(C.byref(other), C.byref(w), 1, 0, None, nt.data_ptr(), cs.cuda_stream)
    assert rc == amk.AMK_ERR_INVALID_ARG
    del g
    torch.cuda.synchronize()
    model.close()
    del keep
