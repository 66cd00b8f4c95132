"""Device-side model setup and the decode calls, on top of the C ABI.

PyTorch is used only to hold device memory and streams: the seeded weights from `synth` are copied
to the GPU, packed there by `amk_pack_weight` (the library's own quantiser / bf16 packer), and the
pointers are handed to `amk_create`. Each decode step is one `amk_decode_step` call.
"""
from __future__ import annotations

import ctypes as C
from typing import List, Optional

import torch

from . import amk
from . import synth


def weight_kind(name: str) -> int:
    """AMK_W_* code of a weight dtype name ("int8", "int4" or "bf16")."""
    return {"int8": amk.AMK_W_INT8, "int4": amk.AMK_W_INT4, "bf16": amk.AMK_W_BF16}[name]


def dims_of(cfg: synth.ModelConfig, max_seq: Optional[int] = None) -> amk.amk_dims:
    return amk.amk_dims(cfg.n_layers, cfg.d_model, cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, cfg.ffn, cfg.vocab,
                        max_seq or cfg.max_seq, cfg.rope_theta, cfg.rms_eps, weight_kind(cfg.weight_dtype),
                        int(cfg.tied))


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _ptr_array(ts: List[Optional[torch.Tensor]]):
    arr = (C.c_void_p * len(ts))(*[_ptr(t) for t in ts])
    return arr, C.cast(arr, C.POINTER(C.c_void_p))


def pack(role: int, dims: amk.amk_dims, src: torch.Tensor, dst_dtype: int, stream=None):
    """Packs a device fp32/bf16 [rows, cols] source with the library packer; returns (packed, scales)."""
    assert src.is_cuda and src.is_contiguous() and src.dim() == 2
    rows, cols = src.shape
    src_dt = amk.AMK_SRC_F32 if src.dtype == torch.float32 else amk.AMK_SRC_BF16
    nbytes = amk.amk_packed_bytes(rows, cols, dst_dtype)
    if nbytes == 0:
        raise ValueError(f"cannot pack a [{rows}, {cols}] matrix as weight dtype {dst_dtype}")
    packed = torch.empty(nbytes, dtype=torch.uint8, device=src.device)
    quantised = dst_dtype != amk.AMK_W_BF16
    scales = torch.empty(rows, dtype=torch.bfloat16, device=src.device) if quantised else None
    amk.check(amk.amk_pack_weight(role, C.byref(dims) if dims is not None else None, src.data_ptr(), src_dt, rows, cols,
                                  dst_dtype, packed.data_ptr(), _ptr(scales), stream), "amk_pack_weight")
    return packed, scales


class DeviceModel:
    """One synthetic model resident on the current CUDA device, with its KV cache and an amk handle."""

    def __init__(self, cfg: synth.ModelConfig, max_seq: Optional[int] = None, options: Optional[dict] = None,
                 device: str = "cuda"):
        self.cfg = cfg
        self.max_seq = max_seq or cfg.max_seq
        self.dims = dims_of(cfg, self.max_seq)
        self.device = torch.device(device)
        dev = self.device
        wdt = self.dims.weight_dtype
        L, hd, hkv = cfg.n_layers, cfg.head_dim, cfg.n_kv_heads
        self.embed = synth.embedding(cfg).to(dev)
        self.final_norm = synth.norm_gain(cfg, None, "final_norm").to(dev)
        self.attn_norm = [synth.norm_gain(cfg, l, "attn_norm").to(dev) for l in range(L)]
        self.ffn_norm = [synth.norm_gain(cfg, l, "ffn_norm").to(dev) for l in range(L)]
        self.w = {k: [] for k in ("qkv", "o", "gu", "down")}
        self.s = {k: [] for k in ("qkv", "o", "gu", "down")}
        for l in range(L):
            src = torch.cat([synth.linear(cfg, l, "wq"), synth.linear(cfg, l, "wk"), synth.linear(cfg, l, "wv")]).to(dev)
            self._add("qkv", amk.AMK_ROLE_QKV, src, wdt)
            self._add("o", amk.AMK_ROLE_O, synth.linear(cfg, l, "wo").to(dev), wdt)
            src = torch.cat([synth.linear(cfg, l, "w_gate"), synth.linear(cfg, l, "w_up")]).to(dev)
            self._add("gu", amk.AMK_ROLE_GATE_UP, src, wdt)
            self._add("down", amk.AMK_ROLE_DOWN, synth.linear(cfg, l, "w_down").to(dev), wdt)
            del src
        self.lm_w = self.lm_s = None
        if not cfg.tied:
            self.lm_w, self.lm_s = pack(amk.AMK_ROLE_LM_HEAD, self.dims, synth.linear(cfg, None, "lm_head").to(dev), wdt)
        shape = (L, hkv, self.max_seq, hd)
        self.k_cache = torch.zeros(shape, dtype=torch.bfloat16, device=dev)
        self.v_cache = torch.zeros(shape, dtype=torch.bfloat16, device=dev)
        if cfg.prefill_len:
            self.load_prefill()
        self.logits = torch.empty(cfg.vocab, dtype=torch.float32, device=dev)
        self.next_token = torch.zeros(1, dtype=torch.int32, device=dev)
        torch.cuda.synchronize(dev)
        self.handle = None
        self._create(options or {})

    def _add(self, key, role, src, wdt):
        w, s = pack(role, self.dims, src, wdt)
        self.w[key].append(w)
        self.s[key].append(s)

    def load_prefill(self) -> None:
        p = self.cfg.prefill_len
        for l in range(self.cfg.n_layers):
            self.k_cache[l, :, :p] = synth.kv_prefill(self.cfg, l, "k").to(self.device)
            self.v_cache[l, :, :p] = synth.kv_prefill(self.cfg, l, "v").to(self.device)

    def _create(self, options: dict) -> None:
        keep = []

        def arr(ts):
            a, p = _ptr_array(ts)
            keep.append(a)
            return p

        i8 = self.dims.weight_dtype != amk.AMK_W_BF16   # quantised: per-row scales
        wts = amk.amk_weights(
            _ptr(self.embed), arr(self.attn_norm), arr(self.ffn_norm), _ptr(self.final_norm),
            arr(self.w["qkv"]), arr(self.w["o"]), arr(self.w["gu"]), arr(self.w["down"]), _ptr(self.lm_w),
            arr(self.s["qkv"]) if i8 else None, arr(self.s["o"]) if i8 else None,
            arr(self.s["gu"]) if i8 else None, arr(self.s["down"]) if i8 else None,
            _ptr(self.lm_s), self.k_cache.data_ptr(), self.v_cache.data_ptr())
        opt = amk.amk_options(**{k: int(v) for k, v in options.items()})
        h = C.c_void_p()
        amk.check(amk.amk_create(C.byref(self.dims), C.byref(wts), C.byref(opt), C.byref(h)), "amk_create")
        self.handle = h

    # -- decode ------------------------------------------------------------------------------------
    def step(self, token: int, pos: int, logits: Optional[torch.Tensor] = None, next_token: Optional[torch.Tensor] = None,
             stream: Optional[torch.cuda.Stream] = None, unfused: bool = False) -> None:
        """Enqueues one decode step (token -1 = read it from next_token) on `stream`."""
        lg = self.logits if logits is None else logits
        nt = self.next_token if next_token is None else next_token
        st = (stream or torch.cuda.current_stream(self.device)).cuda_stream
        fn = amk.amk_decode_step_unfused if unfused else amk.amk_decode_step
        amk.check(fn(self.handle, int(token), int(pos), _ptr(lg), nt.data_ptr(), st),
                  "amk_decode_step_unfused" if unfused else "amk_decode_step")

    def status(self):
        d = C.c_uint32()
        rc = amk.amk_status(self.handle, C.byref(d))
        return rc, d.value

    def plan_info(self) -> amk.amk_plan_info:
        info = amk.amk_plan_info()
        amk.check(amk.amk_plan_info_get(self.handle, C.byref(info)), "amk_plan_info_get")
        return info

    def step_bytes(self, pos: int) -> int:
        return int(amk.amk_step_bytes(C.byref(self.dims), pos))

    def trace(self, max_records: int = 1 << 20):
        import numpy as np
        w = amk.AMK_TRACE_WORDS
        buf = (C.c_uint64 * (w * max_records))()
        n = amk.amk_trace_read(self.handle, buf, max_records)
        if n < 0:
            raise amk.AmkError("amk_trace_read", n)
        return np.frombuffer(buf, dtype=np.uint64, count=w * n).reshape(n, w).copy()

    def close(self) -> None:
        if self.handle is not None:
            amk.amk_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


OP_NAMES = {amk.AMK_OP_QKV: "qkv", amk.AMK_OP_ATTN: "attn", amk.AMK_OP_O: "o", amk.AMK_OP_GU: "gu",
            amk.AMK_OP_DOWN: "down", amk.AMK_OP_LM: "lm"}


def stage_breakdown(trace) -> dict:
    """Critical-path time of each op over one traced step, from `DeviceModel.trace()` records.

    A stage (op, layer) ends when its last CTA is done; stages end in dependency order, so the time
    from one stage's end to the next stage's end is what that stage adds to the step. Returns
    {"us": {op name: summed microseconds}, "span_us": first wait-start to the last stage end,
    "stages": number of stages}.
    """
    import numpy as np
    tr = np.asarray(trace, dtype=np.uint64)
    tr = tr[tr[:, 3] > 0]
    if len(tr) == 0:
        return {"us": {}, "span_us": 0.0, "stages": 0}
    op = (tr[:, 0] >> np.uint64(32)).astype(np.int64)
    layer = ((tr[:, 0] >> np.uint64(16)) & np.uint64(0xFFFF)).astype(np.int64)
    start = int(tr[:, 1].min())
    ends = {}
    for o, l, t in zip(op, layer, tr[:, 3].astype(np.int64)):
        key = (int(o), int(l))
        ends[key] = max(ends.get(key, 0), int(t))
    out = {name: 0.0 for name in OP_NAMES.values()}
    prev = start
    for key, t in sorted(ends.items(), key=lambda kv: kv[1]):
        out[OP_NAMES.get(key[0], str(key[0]))] = out.get(OP_NAMES.get(key[0], str(key[0])), 0.0) + (t - prev) / 1e3
        prev = max(prev, t)
    return {"us": out, "span_us": (prev - start) / 1e3, "stages": len(ends)}

