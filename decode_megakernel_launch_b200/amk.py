"""ctypes binding of libamk (include/amk.h): same names, argument marshalling only.

Every computation runs in the CUDA library; this module only converts Python values and
torch tensors into the plain pointers and sizes of the C ABI. Importing it loads libamk.so
from the package directory and raises if the library is missing (there is no fallback).
"""
from __future__ import annotations

import ctypes as C
import os
import re

_PKG = os.path.dirname(os.path.abspath(__file__))
# AMK_LIB may name a variant build of the same library (build.build_variant: other compile-time
# knobs, same ABI); the default is the in-tree libamk.so.
LIB_PATH = os.environ.get("AMK_LIB") or os.path.join(_PKG, "libamk.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "amk.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built: run `python -c 'import __graft_entry__ as g; g.build()'` "
                      f"or `python decode_megakernel_launch_b200/build.py`")
lib = C.CDLL(LIB_PATH)


def _defines() -> dict:
    out = {}
    with open(HEADER) as f:
        for m in re.finditer(r"#define\s+(AMK_\w+)\s+(-?\d+)", f.read()):
            out[m.group(1)] = int(m.group(2))
    return out


globals().update(_defines())


class amk_dims(C.Structure):
    _fields_ = [("n_layers", C.c_int), ("d_model", C.c_int), ("n_q_heads", C.c_int), ("n_kv_heads", C.c_int),
                ("head_dim", C.c_int), ("ffn", C.c_int), ("vocab", C.c_int), ("max_seq", C.c_int),
                ("rope_theta", C.c_float), ("rms_eps", C.c_float), ("weight_dtype", C.c_int), ("tied_head", C.c_int)]


_PP = C.POINTER(C.c_void_p)


class amk_weights(C.Structure):
    _fields_ = [("embed", C.c_void_p), ("attn_norm", _PP), ("ffn_norm", _PP), ("final_norm", C.c_void_p),
                ("wqkv", _PP), ("wo", _PP), ("wgu", _PP), ("wdown", _PP), ("lm_head", C.c_void_p),
                ("sqkv", _PP), ("so", _PP), ("sgu", _PP), ("sdown", _PP), ("slm", C.c_void_p),
                ("k_cache", C.c_void_p), ("v_cache", C.c_void_p)]


class amk_options(C.Structure):
    _fields_ = [("grid", C.c_int), ("kv_block", C.c_int), ("max_kv_chunks", C.c_int), ("timeout_ms", C.c_int),
                ("trace", C.c_int), ("test_drop_signal", C.c_int)]


class amk_plan_info(C.Structure):
    _fields_ = [("grid", C.c_int), ("threads", C.c_int), ("smem_bytes", C.c_int), ("n_tasks", C.c_int),
                ("n_counters", C.c_int), ("kv_chunks_max", C.c_int), ("weight_bytes", C.c_uint64)]


def _sig(name, res, *args):
    f = getattr(lib, name)
    f.restype = res
    f.argtypes = list(args)
    return f


amk_packed_bytes = _sig("amk_packed_bytes", C.c_size_t, C.c_int, C.c_int, C.c_int)
amk_packed_row_source = _sig("amk_packed_row_source", C.c_int, C.c_int, C.POINTER(amk_dims), C.c_int, C.c_int)
amk_pack_weight = _sig("amk_pack_weight", C.c_int, C.c_int, C.POINTER(amk_dims), C.c_void_p, C.c_int, C.c_int,
                       C.c_int, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p)
amk_create = _sig("amk_create", C.c_int, C.POINTER(amk_dims), C.POINTER(amk_weights), C.POINTER(amk_options),
                  C.POINTER(C.c_void_p))
amk_destroy = _sig("amk_destroy", None, C.c_void_p)
amk_decode_step = _sig("amk_decode_step", C.c_int, C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p)
amk_decode_step_unfused = _sig("amk_decode_step_unfused", C.c_int, C.c_void_p, C.c_int, C.c_int, C.c_void_p,
                               C.c_void_p, C.c_void_p)
amk_decode_step_noalloc = _sig("amk_decode_step_noalloc", C.c_int, C.POINTER(amk_dims), C.POINTER(amk_weights),
                               C.c_int, C.c_int, C.c_void_p, C.c_void_p, C.c_void_p)
amk_status = _sig("amk_status", C.c_int, C.c_void_p, C.POINTER(C.c_uint32))
amk_last_cuda_error = _sig("amk_last_cuda_error", C.c_char_p)
amk_plan_info_get = _sig("amk_plan_info_get", C.c_int, C.c_void_p, C.POINTER(amk_plan_info))
amk_step_bytes = _sig("amk_step_bytes", C.c_uint64, C.POINTER(amk_dims), C.c_int)
amk_plan_check = _sig("amk_plan_check", C.c_int, C.POINTER(amk_dims), C.c_int, C.c_int, C.c_char_p, C.c_int)
amk_trace_read = _sig("amk_trace_read", C.c_int, C.c_void_p, C.POINTER(C.c_uint64), C.c_int)


class AmkError(RuntimeError):
    def __init__(self, where: str, code: int):
        detail = amk_last_cuda_error().decode(errors="replace")
        super().__init__(f"{where} failed with {code}{': ' + detail if detail else ''}")
        self.code = code


def check(code: int, where: str) -> None:
    if code != 0:
        raise AmkError(where, code)


def plan_check(dims: amk_dims, grid: int, mutation: int = 0):
    """(return code, checker message) of the static task-list check."""
    buf = C.create_string_buffer(512)
    rc = amk_plan_check(C.byref(dims), grid, mutation, buf, len(buf))
    return rc, buf.value.decode()


def exported_symbols_in_header() -> list:
    """Function names the public header declares."""
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"\b(amk_\w+)\s*\(", text)) - {"amk_dims", "amk_weights"})
