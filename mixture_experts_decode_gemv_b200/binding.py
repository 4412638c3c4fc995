"""ctypes binding of ``libmoedecode.so`` (declared in ``include/moe_decode.h``).

Every C entry point has a Python function of the same name. The Python side only marshals
arguments (ints or objects with ``data_ptr()`` for device pointers, numpy arrays for host
buffers); every step of the layer runs in the library. A non-zero status raises ``MoeError``.
Importing this module fails loudly when the shared library has not been built.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
# MOE_DECODE_LIBRARY may name another build of the same library (e.g. an instrumented one).
LIB_PATH = os.environ.get("MOE_DECODE_LIBRARY") or os.path.join(_PKG, "libmoedecode.so")

MOE_OK = 0
MOE_ERR_NULL_POINTER = -1
MOE_ERR_BAD_SHAPE = -2
MOE_ERR_BAD_FORMAT = -3
MOE_ERR_BAD_OPTION = -4
MOE_ERR_WORKSPACE = -5
MOE_ERR_MISALIGNED = -6
MOE_ERR_CUDA = -7
MOE_ERR_DEVICE_TIMEOUT = -8
MOE_ERR_UNSUPPORTED_DEVICE = -9
MOE_ERR_DEVICE_CHECK = -10

MOE_MAX_ROWS = 64
MOE_MAX_EXPERTS = 256
MOE_MAX_TOP_K = 8

(MOE_FMT_F32, MOE_FMT_BF16, MOE_FMT_Q4_AFFINE_G64, MOE_FMT_NVFP4, MOE_FMT_MXFP4,
 MOE_FMT_FP8_E4M3) = 0, 1, 2, 3, 4, 5
MOE_ROUTE_SOFTMAX, MOE_ROUTE_SIGMOID, MOE_ROUTE_SQRTSOFTPLUS = 0, 1, 2
MOE_ACT_SWIGLU, MOE_ACT_GEGLU = 0, 1
MOE_SHARED_NONE, MOE_SHARED_PLAIN, MOE_SHARED_SIGMOID_GATE = 0, 1, 2

FORMAT_CODES = {"f32": MOE_FMT_F32, "bf16": MOE_FMT_BF16, "q4_affine_g64": MOE_FMT_Q4_AFFINE_G64,
                "nvfp4": MOE_FMT_NVFP4, "mxfp4": MOE_FMT_MXFP4, "fp8_e4m3": MOE_FMT_FP8_E4M3}
ROUTING_CODES = {"softmax": MOE_ROUTE_SOFTMAX, "sigmoid": MOE_ROUTE_SIGMOID,
                 "sqrtsoftplus": MOE_ROUTE_SQRTSOFTPLUS}
ACTIVATION_CODES = {"swiglu": MOE_ACT_SWIGLU, "geglu": MOE_ACT_GEGLU}
SHARED_CODES = {"none": MOE_SHARED_NONE, "plain": MOE_SHARED_PLAIN,
                "sigmoid_gate": MOE_SHARED_SIGMOID_GATE}

# Every symbol the header declares (checked by a CPU test).
EXPORTS = (
    "moe_workspace_bytes", "moe_workspace_init", "moe_decode_forward", "moe_decode_read_routing",
    "moe_get_device_status", "moe_packed_bytes", "moe_pack_bf16", "moe_quantize_q4_affine",
    "moe_quantize_nvfp4", "moe_dequantize", "moe_status_string", "moe_last_cuda_error",
    "moe_version", "moe_decode_forward_no_alloc", "moe_decode_launches",
    "moe_debug_barrier_test", "moe_quantize_mxfp4", "moe_quantize_fp8_e4m3",
    "moe_debug_set_path", "moe_debug_set_split",
)

MOE_NO_ALLOC_SCRATCH_BYTES = 16 << 20


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = moe_status_string(status)
        if status == MOE_ERR_CUDA:
            msg += f" (cudaError {moe_last_cuda_error()})"
        super().__init__(f"{where}: {msg} [{status}]")


class moe_cfg(ctypes.Structure):
    _fields_ = [
        ("hidden", ctypes.c_int32), ("num_experts", ctypes.c_int32), ("top_k", ctypes.c_int32),
        ("moe_inter", ctypes.c_int32), ("shared_inter", ctypes.c_int32),
        ("routing", ctypes.c_int32), ("norm_topk_prob", ctypes.c_int32),
        ("select_on_raw_logits", ctypes.c_int32), ("has_expert_bias", ctypes.c_int32),
        ("routed_scaling_factor", ctypes.c_float), ("weight_before_ffn", ctypes.c_int32),
        ("shared_kind", ctypes.c_int32), ("x_dtype", ctypes.c_int32),
        ("out_dtype", ctypes.c_int32), ("activation", ctypes.c_int32),
    ]


class moe_matrix(ctypes.Structure):
    _fields_ = [
        ("format", ctypes.c_int32), ("reserved", ctypes.c_int32),
        ("packed", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("biases", ctypes.c_void_p),
        ("tensor_scale", ctypes.c_void_p), ("expert_stride", ctypes.c_int64),
        ("scale_stride", ctypes.c_int64),
    ]


class moe_expert_table(ctypes.Structure):
    _fields_ = [("gate", moe_matrix), ("up", moe_matrix), ("down", moe_matrix)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m mixture_experts_decode_gemv_b200.build`"
            " (there is no fallback implementation)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    P = ctypes.POINTER
    sig = {
        "moe_workspace_bytes": [P(moe_cfg), i32, P(sz)],
        "moe_workspace_init": [vp, sz, vp],
        "moe_decode_forward": [P(moe_cfg), i32, vp, vp, vp, P(moe_expert_table),
                               P(moe_expert_table), vp, vp, vp, sz, vp],
        "moe_decode_read_routing": [P(moe_cfg), i32, vp, sz, vp, vp, vp, vp, vp, vp, vp, vp, vp],
        "moe_get_device_status": [vp, sz, vp, P(ctypes.c_int32)],
        "moe_packed_bytes": [i32, i32, i32, P(sz), P(sz), P(sz)],
        "moe_pack_bf16": [vp, i64, vp],
        "moe_quantize_q4_affine": [vp, i32, i32, vp, vp, vp],
        "moe_quantize_nvfp4": [vp, i32, i32, vp, vp, vp],
        "moe_quantize_mxfp4": [vp, i32, i32, vp, vp],
        "moe_quantize_fp8_e4m3": [vp, i32, i32, vp, vp],
        "moe_dequantize": [i32, vp, vp, vp, vp, i32, i32, vp],
        "moe_decode_forward_no_alloc": [P(moe_cfg), i32, vp, vp, vp, P(moe_expert_table),
                                        P(moe_expert_table), vp, vp, vp],
        "moe_decode_launches": [P(moe_cfg), i32, P(moe_expert_table), P(moe_expert_table),
                                P(ctypes.c_int32)],
        "moe_debug_barrier_test": [i32, i64],
        "moe_debug_set_path": [i32],
        "moe_debug_set_split": [i32],
        "moe_status_string": [i32],
        "moe_last_cuda_error": [],
        "moe_version": [],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_char_p if name == "moe_status_string" else ctypes.c_int
    return lib


lib = _load()


def _ptr(a) -> Optional[int]:
    """Device or host address of ``a``: None, an int, a torch tensor or a numpy array."""
    if a is None:
        return None
    if isinstance(a, int):
        return a
    if hasattr(a, "data_ptr"):
        return a.data_ptr()
    if isinstance(a, np.ndarray):
        if not a.flags["C_CONTIGUOUS"]:
            raise ValueError("host arrays must be C-contiguous")
        return a.ctypes.data
    raise TypeError(f"cannot take the address of {type(a).__name__}")


def _check(rc: int, where: str) -> int:
    if rc != MOE_OK:
        raise MoeError(rc, where)
    return rc


def _stream(stream) -> Optional[int]:
    if stream is None:
        return None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream  # torch.cuda.Stream


# ---- the layer ---------------------------------------------------------------------------------

def moe_workspace_bytes(cfg: moe_cfg, m: int) -> int:
    out = ctypes.c_size_t(0)
    _check(lib.moe_workspace_bytes(ctypes.byref(cfg), m, ctypes.byref(out)), "moe_workspace_bytes")
    return out.value


def moe_workspace_init(workspace, workspace_bytes: int, stream=None) -> None:
    _check(lib.moe_workspace_init(_ptr(workspace), workspace_bytes, _stream(stream)),
           "moe_workspace_init")


def moe_decode_forward(cfg: moe_cfg, m: int, x, router_w, expert_bias, routed: moe_expert_table,
                       shared: Optional[moe_expert_table], shared_gate_w, out, workspace,
                       workspace_bytes: int, stream=None) -> None:
    rc = lib.moe_decode_forward(
        ctypes.byref(cfg), m, _ptr(x), _ptr(router_w), _ptr(expert_bias), ctypes.byref(routed),
        ctypes.byref(shared) if shared is not None else None, _ptr(shared_gate_w), _ptr(out),
        _ptr(workspace), workspace_bytes, _stream(stream))
    _check(rc, "moe_decode_forward")


def moe_decode_forward_no_alloc(cfg: moe_cfg, m: int, x, router_w, expert_bias,
                                routed: moe_expert_table, shared: Optional[moe_expert_table],
                                shared_gate_w, out, stream=None) -> None:
    """The layer with the library's fixed device scratch instead of a caller workspace."""
    rc = lib.moe_decode_forward_no_alloc(
        ctypes.byref(cfg), m, _ptr(x), _ptr(router_w), _ptr(expert_bias), ctypes.byref(routed),
        ctypes.byref(shared) if shared is not None else None, _ptr(shared_gate_w), _ptr(out),
        _stream(stream))
    _check(rc, "moe_decode_forward_no_alloc")


def moe_decode_launches(cfg: moe_cfg, m: int, routed: moe_expert_table,
                        shared: Optional[moe_expert_table]) -> int:
    """Kernel launches one moe_decode_forward call makes on the current device."""
    n = ctypes.c_int32(0)
    rc = lib.moe_decode_launches(ctypes.byref(cfg), m, ctypes.byref(routed),
                                 ctypes.byref(shared) if shared is not None else None,
                                 ctypes.byref(n))
    _check(rc, "moe_decode_launches")
    return int(n.value)


def moe_debug_barrier_test(extra_arrivals: int, spin_limit_cycles: int) -> None:
    """Failure-detection test aid: make the persistent kernel's grid-barrier waits run out."""
    _check(lib.moe_debug_barrier_test(extra_arrivals, spin_limit_cycles), "moe_debug_barrier_test")


def moe_debug_set_path(path: int) -> None:
    """Test aid: 0 automatic launch path, 1 the multi-kernel path at every m (process-wide)."""
    _check(lib.moe_debug_set_path(path), "moe_debug_set_path")


def moe_debug_set_split(mode: int) -> None:
    """Test aid: 0 automatic work split, 1 whole jobs per warp, 2 jobs split by chunk."""
    _check(lib.moe_debug_set_split(mode), "moe_debug_set_split")


def moe_decode_read_routing(cfg: moe_cfg, m: int, workspace, workspace_bytes: int, stream=None):
    """Host copies of the routing and grouping of the last call (dict of numpy arrays)."""
    te = m * cfg.top_k
    cap = min(te, cfg.num_experts)
    out = {
        "idx": np.zeros(te, np.int32), "w": np.zeros(te, np.float32),
        "sorted_pairs": np.zeros(te, np.int32),
        "expert_offsets": np.zeros(cfg.num_experts + 1, np.int32),
        "token_to_perm": np.zeros(te, np.int32), "active": np.zeros(cap, np.int32),
        "active_count": np.zeros(1, np.int32), "gamma": np.zeros(m, np.float32),
    }
    rc = lib.moe_decode_read_routing(
        ctypes.byref(cfg), m, _ptr(workspace), workspace_bytes, _stream(stream),
        *[out[k].ctypes.data for k in ("idx", "w", "sorted_pairs", "expert_offsets",
                                       "token_to_perm", "active", "active_count", "gamma")])
    _check(rc, "moe_decode_read_routing")
    out["active_count"] = int(out["active_count"][0])
    out["active"] = out["active"][: max(0, min(cap, out["active_count"]))]
    out["idx"] = out["idx"].reshape(m, cfg.top_k)
    out["w"] = out["w"].reshape(m, cfg.top_k)
    return out


def moe_get_device_status(workspace, workspace_bytes: int, stream=None) -> int:
    st = ctypes.c_int32(0)
    _check(lib.moe_get_device_status(_ptr(workspace), workspace_bytes, _stream(stream),
                                     ctypes.byref(st)), "moe_get_device_status")
    return st.value


# ---- pack / quantise helpers (host) --------------------------------------------------------------

def moe_packed_bytes(fmt: int, n: int, k: int):
    a, b, c = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib.moe_packed_bytes(fmt, n, k, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)),
           "moe_packed_bytes")
    return a.value, b.value, c.value


def moe_pack_bf16(w: np.ndarray) -> np.ndarray:
    w = np.ascontiguousarray(w, dtype=np.float32)
    out = np.empty(w.shape, dtype=np.uint16)
    _check(lib.moe_pack_bf16(w.ctypes.data, w.size, out.ctypes.data), "moe_pack_bf16")
    return out


def moe_quantize_q4_affine(w: np.ndarray):
    w = np.ascontiguousarray(w, dtype=np.float32)
    n, k = w.shape
    packed = np.empty((n, k // 2), np.uint8)
    scales = np.empty((n, k // 64), np.uint16)
    biases = np.empty((n, k // 64), np.uint16)
    _check(lib.moe_quantize_q4_affine(w.ctypes.data, n, k, packed.ctypes.data,
                                      scales.ctypes.data, biases.ctypes.data),
           "moe_quantize_q4_affine")
    return packed, scales, biases


def moe_quantize_nvfp4(w: np.ndarray):
    w = np.ascontiguousarray(w, dtype=np.float32)
    n, k = w.shape
    packed = np.empty((n, k // 2), np.uint8)
    scales = np.empty((n, k // 16), np.uint8)
    ts = np.zeros(1, np.float32)
    _check(lib.moe_quantize_nvfp4(w.ctypes.data, n, k, packed.ctypes.data, scales.ctypes.data,
                                  ts.ctypes.data), "moe_quantize_nvfp4")
    return packed, scales, ts


def moe_quantize_mxfp4(w: np.ndarray):
    w = np.ascontiguousarray(w, dtype=np.float32)
    n, k = w.shape
    packed = np.empty((n, k // 2), np.uint8)
    scales = np.empty((n, k // 32), np.uint8)
    _check(lib.moe_quantize_mxfp4(w.ctypes.data, n, k, packed.ctypes.data, scales.ctypes.data),
           "moe_quantize_mxfp4")
    return packed, scales


def moe_quantize_fp8_e4m3(w: np.ndarray):
    w = np.ascontiguousarray(w, dtype=np.float32)
    n, k = w.shape
    packed = np.empty((n, k), np.uint8)
    ts = np.zeros(1, np.float32)
    _check(lib.moe_quantize_fp8_e4m3(w.ctypes.data, n, k, packed.ctypes.data, ts.ctypes.data),
           "moe_quantize_fp8_e4m3")
    return packed, ts


def moe_dequantize(fmt: int, packed: np.ndarray, scales, biases, tensor_scale, n: int, k: int):
    out = np.empty((n, k), np.float32)
    keep = [np.ascontiguousarray(a) if a is not None else None
            for a in (packed, scales, biases, tensor_scale)]
    _check(lib.moe_dequantize(fmt, *[_ptr(a) for a in keep], n, k, out.ctypes.data),
           "moe_dequantize")
    return out


def moe_status_string(status: int) -> str:
    return lib.moe_status_string(status).decode()


def moe_last_cuda_error() -> int:
    return lib.moe_last_cuda_error()


def moe_version() -> int:
    return lib.moe_version()
