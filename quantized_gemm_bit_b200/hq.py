"""Thin ctypes binding of the C ABI in include/hq.h (libhq.so).

Argument marshalling only: every function here forwards raw pointers, sizes
and the caller's CUDA stream to the C entry point of the same name and turns
a non-OK status into an HQError.  No arithmetic of the method runs in
Python; if libhq.so is missing the first call raises instead of falling back
to anything else.

Device arrays are torch CUDA tensors (PyTorch supplies memory and streams);
host arrays for the packer are numpy arrays or CPU tensors.
"""

import ctypes
import os

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhq.so")

HQ_LAYOUT_VERSION = 1

HQ_OK = 0
HQ_ERR_INVALID_ARG = 1
HQ_ERR_UNSUPPORTED = 2
HQ_ERR_ALIGNMENT = 3
HQ_ERR_WORKSPACE_TOO_SMALL = 4
HQ_ERR_LAYOUT_VERSION = 5
HQ_ERR_CUDA = 6
HQ_ERR_DEVICE_TIMEOUT = 7
HQ_ERR_DEVICE_BAD_OFFSETS = 8
HQ_ERR_NO_DEVICE = 9

HQ_FMT_INT4 = 1
HQ_FMT_MXFP4 = 2
HQ_FMT_NVFP4 = 3
HQ_FMT_MXFP4_A16 = 4
HQ_FMT_INT3 = 5
HQ_FMT_INT2 = 6
HQ_FMT_INT8 = 7
HQ_FMT_MXINT4 = 8

# Every symbol include/hq.h declares.
EXPORTS = (
    "hq_layout_version", "hq_status_string", "hq_quant_desc_init", "hq_packed_size", "hq_pack_weights",
    "hq_workspace_size", "hq_gemm_w4a16", "hq_gemm_mxfp4_a8", "hq_gemm_nvfp4", "hq_quantize_fp8_rows",
    "hq_quantize_nvfp4_workspace_size", "hq_quantize_nvfp4", "hq_moe_topk", "hq_moe_topk_softmax",
    "hq_moe_permute_workspace_size", "hq_moe_permute", "hq_grouped_gemm_moe", "hq_moe_swiglu",
    "hq_moe_combine_workspace_size", "hq_moe_combine", "hq_check_device_status",
    "hq_debug_timeout_probe", "hq_gemm_w4a16_static", "hq_static_check_device_status",
    "hq_pack_weights_gated", "hq_grouped_gemm_moe_swiglu", "hq_tuning_table_set", "hq_plan_describe",
)


class QuantDesc(ctypes.Structure):
    _fields_ = [(f, ctypes.c_int32) for f in
                ("layout_version", "fmt", "n", "k", "group_size", "has_zero_point", "num_experts")]


class Tuning(ctypes.Structure):
    _fields_ = [(f, ctypes.c_int32) for f in
                ("tile_m", "tile_n", "tile_k", "stages", "split_k", "cta_group", "variant", "flags")]


HQ_TUNE_NO_EARLY_WEIGHTS = 1


class TuningEntry(ctypes.Structure):
    _fields_ = [(f, ctypes.c_int32) for f in ("fmt", "n", "k", "num_experts", "m_min", "m_max")] + \
               [("tuning", Tuning)]


class Plan(ctypes.Structure):
    _fields_ = [(f, ctypes.c_int32) for f in
                ("kernel", "tile_m", "grid", "split", "whole_tiles", "stages", "ring_stages", "from_table",
                 "cta_group")] + \
               [("workspace_bytes", ctypes.c_size_t)]


class HQError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


_lib = None


def lib():
    """Load libhq.so once; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m quantized_gemm_bit_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, sz, i32, st = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_int
        dp = ctypes.POINTER(QuantDesc)
        tp = ctypes.POINTER(Tuning)
        sig = {
            "hq_layout_version": (ctypes.c_int, []),
            "hq_status_string": (ctypes.c_char_p, [st]),
            "hq_quant_desc_init": (st, [dp, i32, i32, i32, i32, i32, i32]),
            "hq_packed_size": (sz, [dp]),
            "hq_pack_weights": (st, [dp, vp, vp, vp, ctypes.c_float, vp, sz]),
            "hq_workspace_size": (sz, [dp, i32, tp]),
            "hq_gemm_w4a16": (st, [dp, vp, vp, i32, vp, tp, vp, sz, vp]),
            "hq_gemm_mxfp4_a8": (st, [dp, vp, vp, vp, i32, vp, tp, vp, sz, vp]),
            "hq_gemm_nvfp4": (st, [dp, vp, vp, vp, ctypes.c_float, i32, vp, tp, vp, sz, vp]),
            "hq_quantize_fp8_rows": (st, [vp, i32, i32, vp, vp, vp]),
            "hq_quantize_nvfp4_workspace_size": (sz, [i32, i32]),
            "hq_quantize_nvfp4": (st, [vp, i32, i32, vp, vp, vp, vp, sz, vp]),
            "hq_moe_topk": (st, [vp, i32, i32, i32, vp, vp]),
            "hq_moe_topk_softmax": (st, [vp, i32, i32, i32, vp, vp, vp]),
            "hq_moe_swiglu": (st, [vp, i32, i32, vp, vp]),
            "hq_moe_combine_workspace_size": (sz, [i32, i32]),
            "hq_moe_combine": (st, [vp, vp, vp, i32, i32, i32, vp, vp, sz, vp]),
            "hq_moe_permute_workspace_size": (sz, [i32, i32, i32]),
            "hq_moe_permute": (st, [vp, i32, i32, i32, vp, vp, vp, i32, vp, vp, sz, vp]),
            "hq_grouped_gemm_moe": (st, [dp, vp, vp, vp, i32, vp, tp, vp, sz, vp]),
            "hq_check_device_status": (st, [vp, vp]),
            "hq_debug_timeout_probe": (st, [vp, ctypes.c_uint64, vp]),
            "hq_gemm_w4a16_static": (st, [dp, vp, vp, i32, vp, tp, vp]),
            "hq_static_check_device_status": (st, [vp]),
            "hq_pack_weights_gated": (st, [dp, vp, vp, vp, vp, sz]),
            "hq_grouped_gemm_moe_swiglu": (st, [dp, vp, vp, vp, i32, vp, tp, vp, sz, vp]),
            "hq_tuning_table_set": (st, [ctypes.POINTER(TuningEntry), i32]),
            "hq_plan_describe": (st, [dp, i32, tp, ctypes.POINTER(Plan)]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def status_string(status):
    try:
        return lib().hq_status_string(int(status)).decode()
    except RuntimeError:
        return f"status {status}"


def _check(status, where):
    if status != HQ_OK:
        raise HQError(status, where)


def _ptr(t):
    """Raw address of a torch tensor / numpy array (None -> NULL)."""
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return t.ctypes.data
    return t.data_ptr()


def _stream(stream):
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    return torch.cuda.current_stream().cuda_stream


def _tuning(t):
    if t is None:
        return None
    if isinstance(t, Tuning):
        return ctypes.byref(t)
    return ctypes.byref(Tuning(**t))


def _host(x):
    if x is None:
        return None
    if not isinstance(x, np.ndarray):
        x = x.contiguous().numpy()
    return np.ascontiguousarray(x)


# ---------------------------------------------------------------- C ABI mirror

def hq_layout_version():
    return lib().hq_layout_version()


def hq_quant_desc_init(fmt, n, k, group_size, has_zero_point=0, num_experts=1):
    d = QuantDesc()
    _check(lib().hq_quant_desc_init(ctypes.byref(d), fmt, n, k, group_size, int(has_zero_point), num_experts),
           "hq_quant_desc_init")
    return d


def hq_packed_size(desc):
    return lib().hq_packed_size(ctypes.byref(desc))


def hq_pack_weights(desc, codes, scales, zeros=None, global_scale=0.0):
    """Host packer: returns the packed blob as a numpy uint8 array."""
    codes, scales, zeros = _host(codes), _host(scales), _host(zeros)
    if scales.dtype == np.float16:
        scales = scales.view(np.uint16)
    out = np.empty(hq_packed_size(desc), dtype=np.uint8)
    _check(lib().hq_pack_weights(ctypes.byref(desc), _ptr(codes), _ptr(scales), _ptr(zeros),
                                 float(global_scale), _ptr(out), out.nbytes), "hq_pack_weights")
    return out


def hq_pack_weights_gated(desc, codes, scales, zeros=None):
    """Host packer of gate+up weights in the gated row order (for
    hq_grouped_gemm_moe_swiglu): returns the blob as a numpy uint8 array."""
    codes, scales, zeros = _host(codes), _host(scales), _host(zeros)
    if scales.dtype == np.float16:
        scales = scales.view(np.uint16)
    out = np.empty(hq_packed_size(desc), dtype=np.uint8)
    _check(lib().hq_pack_weights_gated(ctypes.byref(desc), _ptr(codes), _ptr(scales), _ptr(zeros), _ptr(out),
                                       out.nbytes), "hq_pack_weights_gated")
    return out


def hq_workspace_size(desc, m, tuning=None):
    return lib().hq_workspace_size(ctypes.byref(desc), int(m), _tuning(tuning))


def hq_gemm_w4a16(desc, packed_w, a, m, c, ws, tuning=None, stream=None):
    _check(lib().hq_gemm_w4a16(ctypes.byref(desc), _ptr(packed_w), _ptr(a), int(m), _ptr(c), _tuning(tuning),
                               _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)), "hq_gemm_w4a16")


def hq_gemm_mxfp4_a8(desc, packed_w, a_e4m3, a_scale, m, c, ws, tuning=None, stream=None):
    _check(lib().hq_gemm_mxfp4_a8(ctypes.byref(desc), _ptr(packed_w), _ptr(a_e4m3), _ptr(a_scale), int(m), _ptr(c),
                                  _tuning(tuning), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "hq_gemm_mxfp4_a8")


def hq_gemm_nvfp4(desc, packed_w, a_fp4, a_sf, a_global, m, c, ws, tuning=None, stream=None):
    _check(lib().hq_gemm_nvfp4(ctypes.byref(desc), _ptr(packed_w), _ptr(a_fp4), _ptr(a_sf), float(a_global), int(m),
                               _ptr(c), _tuning(tuning), _ptr(ws), ws.numel() * ws.element_size(),
                               _stream(stream)), "hq_gemm_nvfp4")


def hq_quantize_fp8_rows(x, rows, k, q, scale, stream=None):
    _check(lib().hq_quantize_fp8_rows(_ptr(x), int(rows), int(k), _ptr(q), _ptr(scale), _stream(stream)),
           "hq_quantize_fp8_rows")


def hq_quantize_nvfp4_workspace_size(rows, k):
    return lib().hq_quantize_nvfp4_workspace_size(int(rows), int(k))


def hq_quantize_nvfp4(x, rows, k, codes, sf, g, ws, stream=None):
    _check(lib().hq_quantize_nvfp4(_ptr(x), int(rows), int(k), _ptr(codes), _ptr(sf), _ptr(g), _ptr(ws),
                                   ws.numel() * ws.element_size(), _stream(stream)), "hq_quantize_nvfp4")


def hq_moe_topk(logits, t, e, k, topk_ids, stream=None):
    _check(lib().hq_moe_topk(_ptr(logits), int(t), int(e), int(k), _ptr(topk_ids), _stream(stream)), "hq_moe_topk")


def hq_moe_topk_softmax(logits, t, e, k, topk_ids, topk_weights, stream=None):
    _check(lib().hq_moe_topk_softmax(_ptr(logits), int(t), int(e), int(k), _ptr(topk_ids), _ptr(topk_weights),
                                     _stream(stream)), "hq_moe_topk_softmax")


def hq_moe_swiglu(gate_up, rows, inter, h, stream=None):
    _check(lib().hq_moe_swiglu(_ptr(gate_up), int(rows), int(inter), _ptr(h), _stream(stream)), "hq_moe_swiglu")


def hq_moe_combine_workspace_size(t, k):
    return lib().hq_moe_combine_workspace_size(int(t), int(k))


def hq_moe_combine(y_sorted, sorted_src, topk_weights, t, k, hidden, out, ws, stream=None):
    _check(lib().hq_moe_combine(_ptr(y_sorted), _ptr(sorted_src), _ptr(topk_weights), int(t), int(k), int(hidden),
                                _ptr(out), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "hq_moe_combine")


def hq_moe_permute_workspace_size(t, k, e):
    return lib().hq_moe_permute_workspace_size(int(t), int(k), int(e))


def hq_moe_permute(topk_ids, t, k, e, sorted_src, expert_offsets, ws, a=None, hidden=0, a_sorted=None,
                   stream=None):
    _check(lib().hq_moe_permute(_ptr(topk_ids), int(t), int(k), int(e), _ptr(sorted_src), _ptr(expert_offsets),
                                _ptr(a), int(hidden), _ptr(a_sorted), _ptr(ws), ws.numel() * ws.element_size(),
                                _stream(stream)), "hq_moe_permute")


def hq_grouped_gemm_moe(desc, packed_w, a_sorted, expert_offsets, total_rows, c_sorted, ws, tuning=None,
                        stream=None):
    _check(lib().hq_grouped_gemm_moe(ctypes.byref(desc), _ptr(packed_w), _ptr(a_sorted), _ptr(expert_offsets),
                                     int(total_rows), _ptr(c_sorted), _tuning(tuning), _ptr(ws),
                                     ws.numel() * ws.element_size(), _stream(stream)), "hq_grouped_gemm_moe")


def hq_grouped_gemm_moe_swiglu(desc, packed_w, a_sorted, expert_offsets, total_rows, h_sorted, ws, tuning=None,
                               stream=None):
    _check(lib().hq_grouped_gemm_moe_swiglu(ctypes.byref(desc), _ptr(packed_w), _ptr(a_sorted),
                                            _ptr(expert_offsets), int(total_rows), _ptr(h_sorted), _tuning(tuning),
                                            _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "hq_grouped_gemm_moe_swiglu")


def hq_check_device_status(ws, stream=None):
    """Returns the device-side status recorded in the workspace (and clears it)."""
    return lib().hq_check_device_status(_ptr(ws), _stream(stream))


def hq_debug_timeout_probe(ws, limit_ns, stream=None):
    _check(lib().hq_debug_timeout_probe(_ptr(ws), int(limit_ns), _stream(stream)), "hq_debug_timeout_probe")


def hq_gemm_w4a16_static(desc, packed_w, a, m, c, tuning=None, stream=None):
    """hq_gemm_w4a16 for callers that cannot allocate device memory: the
    split-K scratch lives in a fixed array inside the library (see
    include/hq.h for its size and sharing rules)."""
    _check(lib().hq_gemm_w4a16_static(ctypes.byref(desc), _ptr(packed_w), _ptr(a), int(m), _ptr(c),
                                      _tuning(tuning), _stream(stream)), "hq_gemm_w4a16_static")


def hq_static_check_device_status(stream=None):
    """First device-side error of the allocation-free calls since the last
    read (HQ_OK when none); synchronizes the stream."""
    return int(lib().hq_static_check_device_status(_stream(stream)))


def hq_tuning_table_set(entries):
    """Install a per-shape tuning table: a list of TuningEntry (or dicts with
    fmt, n, k, num_experts, m_min, m_max and tuning fields)."""
    ents = []
    for e in entries:
        if isinstance(e, dict):
            t = Tuning(**{f: int(e.get("tuning", {}).get(f, 0)) for f, _ in Tuning._fields_})
            e = TuningEntry(int(e["fmt"]), int(e["n"]), int(e["k"]), int(e.get("num_experts", 1)),
                            int(e["m_min"]), int(e["m_max"]), t)
        ents.append(e)
    arr = (TuningEntry * max(1, len(ents)))(*ents)
    _check(lib().hq_tuning_table_set(arr, len(ents)), "hq_tuning_table_set")


def hq_plan_describe(desc, m, tuning=None):
    """The launch plan a call with these arguments would run (a Plan)."""
    out = Plan()
    _check(lib().hq_plan_describe(ctypes.byref(desc), int(m), _tuning(tuning), ctypes.byref(out)), "hq_plan_describe")
    return out
