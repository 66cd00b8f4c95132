"""amk_decode_step_noalloc against amk_decode_step.

The no-allocation entry point serves callers that can't call cudaMalloc (a plugin whose host
framework's memory pool owns the device memory, or a latency-critical loop where cudaMalloc/cudaFree
may synchronize the device): it keeps its state in a fixed 4 MiB static device array instead of
allocating. These tests call it through the C ABI and check its logits and next token against the
existing handle-based entry point on two calls in a row, within the parity tolerances used everywhere
else, and check that dims needing more than the array are rejected before any launch.
This file is collected last on purpose, and each test also passes alone in a fresh process.
"""
import ctypes as C

import pytest
import torch

from decode_megakernel_launch_b200 import synth

pytestmark = pytest.mark.gpu

REL_L2 = 2e-2
MAX_ABS_FRAC = 5e-2


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


@pytest.mark.parametrize("name", ["tiny", "smollm135m", "tiny_int4"])
def test_noalloc_matches_decode_step_on_two_calls(name):
    from decode_megakernel_launch_b200 import amk
    from decode_megakernel_launch_b200.runtime import DeviceModel
    cfg = synth.preset(name)
    model = DeviceModel(cfg)
    k2, v2 = torch.zeros_like(model.k_cache), torch.zeros_like(model.v_cache)
    w2, keep = _weights(model, k2, v2)
    dims = model.dims
    lg_a = torch.empty(cfg.vocab, dtype=torch.float32, device="cuda")
    lg_b = torch.empty_like(lg_a)
    nt_a = torch.zeros(1, dtype=torch.int32, device="cuda")
    nt_b = torch.zeros_like(nt_a)
    stream = torch.cuda.current_stream().cuda_stream
    tok = 7
    for pos in (0, 1):
        model.step(tok, pos, logits=lg_a, next_token=nt_a)
        rc = amk.amk_decode_step_noalloc(C.byref(dims), C.byref(w2), tok, pos, lg_b.data_ptr(), nt_b.data_ptr(), stream)
        assert rc == amk.AMK_OK
        torch.cuda.synchronize()
        a, b = lg_a.double().cpu(), lg_b.double().cpu()
        assert float((b - a).norm() / a.norm()) <= REL_L2
        assert float((b - a).abs().max() / a.abs().max()) <= MAX_ABS_FRAC
        assert int(nt_b.item()) == int(nt_a.item())
        assert torch.equal(k2[:, :, pos], model.k_cache[:, :, pos]) and torch.equal(v2[:, :, pos], model.v_cache[:, :, pos])
        tok = int(nt_a.item())
    model.close()
    del keep


def test_noalloc_rejects_dims_beyond_its_scratch():
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
    model.close()
    del keep
