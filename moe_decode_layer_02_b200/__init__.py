"""Python binding of libmoe_decode.so (the C ABI in include/moe_decode.h).

Argument marshalling only: every step of the layer runs in the CUDA kernels of
the shared library; there is no Python or CPU implementation of the layer
here, and loading fails loudly if the library has not been built.  PyTorch
tensors are accepted for device (or host) buffers and streams; plain integer
addresses work as well.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_decode.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_UNSUPPORTED_CONFIG = -2
MOE_ERR_ALIGNMENT = -3
MOE_ERR_OOM = -4
MOE_ERR_CUDA = -5
MOE_ERR_DEVICE_TIMEOUT = -6
MOE_ERR_DEVICE_BOUNDS = -7
MOE_ERR_SCRATCH_LIMIT = -8
MOE_STATIC_SCRATCH_BYTES = 1536 * 1024

EXPORTED = ("moe_decode_create", "moe_decode_step", "moe_decode_step_host", "moe_decode_sync_status",
            "moe_decode_get_intermediate", "moe_decode_kernels_per_step", "moe_decode_profile_step",
            "moe_decode_step_static", "moe_decode_check_error_path", "moe_decode_destroy",
            "moe_decode_strerror")

KERNEL_NAMES = {1: "oproj_residual_rmsnorm", 2: "router_topk", 3: "experts_small_m", 4: "gateup_rows",
                5: "down_rows", 6: "layer_fused_small_m"}


class moe_decode_config(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int), ("d_o", ctypes.c_int), ("n_experts", ctypes.c_int),
                ("top_k", ctypes.c_int), ("inter", ctypes.c_int), ("max_batch", ctypes.c_int),
                ("n_layers", ctypes.c_int), ("rms_eps", ctypes.c_float),
                ("enable_prefetch", ctypes.c_int), ("force_variant", ctypes.c_int)]


class moe_decode_layer_weights(ctypes.Structure):
    _fields_ = [("w_o", ctypes.c_void_p), ("gamma", ctypes.c_void_p), ("w_router", ctypes.c_void_p),
                ("w_gate_up", ctypes.c_void_p), ("w_down", ctypes.c_void_p)]


class MoeError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {strerror(code)} ({code})")


_lib = None


def load(path: str = LIB_PATH):
    """Loads the library (once).  Raises if it is missing: there is no fallback."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with moe_decode_layer_02_b200.build.build()")
    lib = ctypes.CDLL(path)
    P, I = ctypes.c_void_p, ctypes.c_int
    lib.moe_decode_create.argtypes = [ctypes.POINTER(moe_decode_config),
                                      ctypes.POINTER(moe_decode_layer_weights), P,
                                      ctypes.POINTER(P)]
    lib.moe_decode_step.argtypes = [P, I, P, P, P, P, P, P]
    lib.moe_decode_step_host.argtypes = [P, I, P, P, P, P, P, P]
    lib.moe_decode_sync_status.argtypes = [P, P]
    lib.moe_decode_get_intermediate.argtypes = [P, I, P, ctypes.c_size_t, P]
    lib.moe_decode_kernels_per_step.argtypes = [P, I]
    lib.moe_decode_profile_step.argtypes = [P, I, P, P, P, P, P, P, P, P, I]
    lib.moe_decode_step_static.argtypes = [ctypes.POINTER(moe_decode_config),
                                           ctypes.POINTER(moe_decode_layer_weights), I, P, P, P, P, P, P, P]
    lib.moe_decode_check_error_path.argtypes = [P, I, ctypes.c_ulonglong, P]
    lib.moe_decode_destroy.argtypes = [P]
    lib.moe_decode_strerror.argtypes = [I]
    lib.moe_decode_strerror.restype = ctypes.c_char_p
    for n in EXPORTED[:-1]:
        getattr(lib, n).restype = I
    _lib = lib
    return lib


def strerror(code: int) -> str:
    return load().moe_decode_strerror(int(code)).decode()


def _addr(x) -> int | None:
    """Address of a tensor / buffer / int (None for None)."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if hasattr(x, "ctypes"):
        return x.ctypes.data
    raise TypeError(f"cannot take the address of {type(x)}")


def _stream(s) -> int | None:
    if s is None:
        return None
    if isinstance(s, int):
        return s
    if hasattr(s, "cuda_stream"):
        return s.cuda_stream
    raise TypeError(f"not a stream: {type(s)}")


def _check(rc: int, where: str) -> int:
    if rc < 0:
        raise MoeError(rc, where)
    return rc


def moe_decode_create(cfg: moe_decode_config, weights, stream=None) -> int:
    """weights: sequence of (w_o, gamma, w_router, w_gate_up, w_down) per layer."""
    lib = load()
    arr = (moe_decode_layer_weights * len(weights))()
    for i, w in enumerate(weights):
        arr[i] = moe_decode_layer_weights(*[_addr(t) for t in w])
    h = ctypes.c_void_p()
    _check(lib.moe_decode_create(ctypes.byref(cfg), arr, _stream(stream), ctypes.byref(h)),
           "moe_decode_create")
    return h.value


def moe_decode_step(h: int, batch: int, attn_out, residual_in, out, topk_idx=None, topk_gate=None,
                    stream=None) -> None:
    _check(load().moe_decode_step(h, batch, _addr(attn_out), _addr(residual_in), _addr(out),
                                  _addr(topk_idx), _addr(topk_gate), _stream(stream)), "moe_decode_step")


def moe_decode_step_host(h: int, batch: int, attn_out, residual_in, out, topk_idx=None,
                         topk_gate=None, stream=None) -> None:
    _check(load().moe_decode_step_host(h, batch, _addr(attn_out), _addr(residual_in), _addr(out),
                                       _addr(topk_idx), _addr(topk_gate), _stream(stream)),
           "moe_decode_step_host")


def moe_decode_sync_status(h: int, stream=None) -> int:
    return load().moe_decode_sync_status(h, _stream(stream))


def moe_decode_get_intermediate(h: int, which: int, dst, nbytes: int, stream=None) -> None:
    _check(load().moe_decode_get_intermediate(h, which, _addr(dst), nbytes, _stream(stream)),
           "moe_decode_get_intermediate")


def moe_decode_kernels_per_step(h: int, batch: int) -> int:
    return _check(load().moe_decode_kernels_per_step(h, batch), "moe_decode_kernels_per_step")


def moe_decode_profile_step(h: int, batch: int, attn_out, residual_in, out, topk_idx=None,
                            topk_gate=None, stream=None, max_kernels: int = 1024):
    """[(kernel name, milliseconds)] of one eagerly launched, event-bracketed step."""
    ms = (ctypes.c_float * max_kernels)()
    ids = (ctypes.c_int * max_kernels)()
    n = _check(load().moe_decode_profile_step(h, batch, _addr(attn_out), _addr(residual_in), _addr(out),
                                              _addr(topk_idx), _addr(topk_gate), _stream(stream), ms, ids,
                                              max_kernels), "moe_decode_profile_step")
    return [(KERNEL_NAMES.get(ids[i], str(ids[i])), ms[i]) for i in range(n)]


def moe_decode_step_static(cfg: moe_decode_config, weights, batch: int, attn_out, residual_in, out,
                           topk_idx=None, topk_gate=None, err_word=None, stream=None) -> None:
    """One layer step (batch 1 or 2) with its scratch in the library's static device array."""
    if isinstance(weights, moe_decode_layer_weights):
        w = weights
    elif isinstance(weights, dict):
        w = moe_decode_layer_weights(*[_addr(weights[k]) for k in ("w_o", "gamma", "w_router", "w_gate_up",
                                                                   "w_down")])
    else:  # (w_o, gamma, w_router, w_gate_up, w_down)
        w = moe_decode_layer_weights(*[_addr(t) for t in weights])
    _check(load().moe_decode_step_static(ctypes.byref(cfg), ctypes.byref(w), batch, _addr(attn_out),
                                         _addr(residual_in), _addr(out), _addr(topk_idx), _addr(topk_gate),
                                         _addr(err_word), _stream(stream)), "moe_decode_step_static")


def moe_decode_check_error_path(h: int, what: int, limit_ns: int = 1_000_000, stream=None) -> None:
    """Launches the error-path probe (1: bounded waits run out; 2: an out-of-range index)."""
    _check(load().moe_decode_check_error_path(h, what, limit_ns, _stream(stream)), "moe_decode_check_error_path")


def moe_decode_destroy(h: int) -> int:
    return load().moe_decode_destroy(h)


def config(d, d_o, n_experts, top_k, inter, max_batch, n_layers=1, rms_eps=1e-6, enable_prefetch=0,
           force_variant=0) -> moe_decode_config:
    return moe_decode_config(d, d_o, n_experts, top_k, inter, max_batch, n_layers, rms_eps,
                             enable_prefetch, force_variant)
