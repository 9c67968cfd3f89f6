"""Thin Python binding of libmoe.so (the routed MoE FFN layer for B200).

Argument marshalling only: every step of the layer runs in the CUDA library.  Functions
carry the C ABI's names (``include/moe.h``); tensors are torch CUDA tensors (device memory
and streams come from PyTorch), passed to the library as raw pointers.  If the shared
library is missing the import fails: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_CUDA, MOE_ERR_OOM, MOE_ERR_TIMEOUT, MOE_ERR_RANGE, MOE_ERR_UNSUPPORTED = range(7)
MOE_ROUTER_SOFTMAX_TOPK, MOE_ROUTER_SIGMOID_BIAS = 0, 1
MOE_W_INT4_ROWSCALE, MOE_W_BF16, MOE_W_INT8_ROWSCALE, MOE_W_INT2_ROWSCALE = 0, 1, 2, 3

# Every symbol that include/moe.h declares.
EXPORTS = (
    "moe_pack_int4", "moe_pack_int8", "moe_pack_int2", "moe_layer_create", "moe_route", "moe_forward", "moe_forward_host", "moe_forward_host_async",
    "moe_last_error",
    "moe_layer_destroy", "moe_layer_workspace_bytes", "moe_layer_last_launches", "moe_status_str",
    "moe_profile_enable", "moe_profile_read", "moe_kernel_name", "moe_route_noalloc",
    "moe_layer_set_option", "moe_layer_get_option", "moe_layer_debug_read", "moe_layer_set_expert",
    "moe_expert_cache_create", "moe_expert_cache_layer", "moe_expert_cache_prepare", "moe_expert_cache_pin",
    "moe_expert_cache_stats", "moe_expert_cache_slot_of", "moe_expert_cache_destroy",
)
(MOE_OPT_PREFILL_MIN_TOKENS, MOE_OPT_PREFILL_AVAILABLE, MOE_OPT_SINGLE_TOKEN_KERNELS, MOE_OPT_PROGRAMMATIC_LAUNCH,
 MOE_OPT_WAIT_LIMIT_US, MOE_OPT_TEST_SKIP_GEMM_B_COPIES, MOE_OPT_ROUTER_GROUPS, MOE_OPT_ROUTER_TOP_P,
 MOE_OPT_UNION_TENSOR_CORES, MOE_OPT_PHASE_TRACE) = range(10)
DEBUG_ITEMS = {"h": 0, "y": 1, "idx": 2, "w": 3, "asc": 4, "ulist": 5, "cnt": 6, "xsum": 7, "trace": 8}
KERNELS = ("router_logits", "topk", "bucket", "gateup", "down", "combine", "gather", "gemm_gateup", "gemm_down",
           "fused")


class MoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_str(status)} ({status})")


class moe_config(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int32), ("f", ctypes.c_int32), ("n_experts", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("n_shared", ctypes.c_int32), ("f_shared", ctypes.c_int32),
                ("max_tokens", ctypes.c_int32), ("router", ctypes.c_int32),
                ("routed_scaling_factor", ctypes.c_float), ("wkind", ctypes.c_int32), ("out_bf16", ctypes.c_int32)]


class moe_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "router_w", "router_bias", "gate_up", "gate_up_scale", "down", "down_scale",
        "shared_gate_up", "shared_gate_up_scale", "shared_down", "shared_down_scale")]


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libmoe.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise ImportError(f"{path} is missing: build it with `python -m quantized_expert_ffn_02_b200.build`")
        L = ctypes.CDLL(path)
        P, I32, I64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
        L.moe_pack_int4.argtypes = [P, I64, I64, P, P, P]
        L.moe_pack_int8.argtypes = [P, I64, I64, P, P, P]
        L.moe_pack_int2.argtypes = [P, I64, I64, P, P, P]
        L.moe_layer_create.argtypes = [ctypes.POINTER(moe_config), ctypes.POINTER(moe_weights), ctypes.POINTER(P)]
        L.moe_route.argtypes = [P, P, I32, P, P, P]
        L.moe_forward.argtypes = [P, P, I32, P, P]
        L.moe_forward_host.argtypes = [P, P, I32, P, P]
        L.moe_forward_host_async.argtypes = [P, P, I32, P, P]
        L.moe_last_error.argtypes = [P]
        L.moe_layer_destroy.argtypes = [P]
        L.moe_layer_destroy.restype = None
        L.moe_layer_workspace_bytes.argtypes = [P]
        L.moe_layer_workspace_bytes.restype = I64
        L.moe_layer_last_launches.argtypes = [P]
        L.moe_layer_last_launches.restype = I32
        L.moe_status_str.argtypes = [ctypes.c_int]
        L.moe_status_str.restype = ctypes.c_char_p
        L.moe_profile_enable.argtypes = [P, I32]
        L.moe_profile_read.argtypes = [P, I32, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(I64)]
        L.moe_kernel_name.argtypes = [I32]
        L.moe_kernel_name.restype = ctypes.c_char_p
        L.moe_route_noalloc.argtypes = [ctypes.POINTER(moe_config), P, P, P, I32, P, P, P]
        L.moe_layer_set_option.argtypes = [P, I32, I64]
        L.moe_layer_get_option.argtypes = [P, I32, ctypes.POINTER(I64)]
        L.moe_layer_debug_read.argtypes = [P, I32, P, I64]
        L.moe_layer_set_expert.argtypes = [P, I32, P, P, P, P, P]
        L.moe_expert_cache_create.argtypes = [ctypes.POINTER(moe_config), ctypes.POINTER(moe_weights),
                                              ctypes.POINTER(moe_weights), I32, ctypes.POINTER(P)]
        L.moe_expert_cache_layer.argtypes = [P]
        L.moe_expert_cache_layer.restype = P
        L.moe_expert_cache_prepare.argtypes = [P, P, I32, P]
        L.moe_expert_cache_pin.argtypes = [P, I32, I32]
        L.moe_expert_cache_stats.argtypes = [P, ctypes.POINTER(I64), ctypes.POINTER(I64), ctypes.POINTER(I64),
                                             ctypes.POINTER(I32)]
        L.moe_expert_cache_slot_of.argtypes = [P, I32]
        L.moe_expert_cache_slot_of.restype = I32
        L.moe_expert_cache_destroy.argtypes = [P]
        L.moe_expert_cache_destroy.restype = None
        for n in ("moe_pack_int4", "moe_pack_int8", "moe_pack_int2", "moe_layer_create", "moe_route", "moe_forward", "moe_forward_host",
                  "moe_forward_host_async", "moe_last_error", "moe_profile_enable", "moe_profile_read", "moe_route_noalloc",
                  "moe_layer_set_option", "moe_layer_get_option", "moe_layer_debug_read", "moe_layer_set_expert",
                  "moe_expert_cache_create", "moe_expert_cache_prepare", "moe_expert_cache_pin",
                  "moe_expert_cache_stats"):
            getattr(L, n).restype = ctypes.c_int
        _lib = L
    return _lib


def status_str(status: int) -> str:
    return load().moe_status_str(int(status)).decode()


def _check(rc: int, what: str):
    if rc != MOE_OK:
        raise MoeError(rc, what)


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


# ------------------------------------------------------------------------------------------
# entry points (same names as the C ABI)
# ------------------------------------------------------------------------------------------

def moe_pack_int4(w, packed, scales, stream=None):
    """w fp32 [rows][cols] (CUDA) -> packed uint8 [rows][cols/2], scales fp32 [rows] (written)."""
    rows, cols = w.shape
    _check(load().moe_pack_int4(_ptr(w), rows, cols, _ptr(packed), _ptr(scales), _stream(stream)),
           "moe_pack_int4")


def moe_pack_int8(w, q, scales, stream=None):
    """w fp32 [rows][cols] (CUDA) -> q int8 [rows][cols] (the 8-bit tier), scales fp32 [rows] (written)."""
    rows, cols = w.shape
    _check(load().moe_pack_int8(_ptr(w), rows, cols, _ptr(q), _ptr(scales), _stream(stream)), "moe_pack_int8")


def moe_pack_int2(w, packed, scales, stream=None):
    """w fp32 [rows][cols] (CUDA) -> packed uint8 [rows][cols/4] (the 2-bit tier), scales fp32 [rows]."""
    rows, cols = w.shape
    _check(load().moe_pack_int2(_ptr(w), rows, cols, _ptr(packed), _ptr(scales), _stream(stream)), "moe_pack_int2")


def moe_layer_create(cfg: moe_config, weights: moe_weights) -> int:
    h = ctypes.c_void_p()
    _check(load().moe_layer_create(ctypes.byref(cfg), ctypes.byref(weights), ctypes.byref(h)), "moe_layer_create")
    return h.value


def moe_route(layer: int, x, T: int, idx, w, stream=None):
    _check(load().moe_route(layer, _ptr(x), T, _ptr(idx), _ptr(w), _stream(stream)), "moe_route")


def moe_forward(layer: int, x, T: int, out, stream=None):
    _check(load().moe_forward(layer, _ptr(x), T, _ptr(out), _stream(stream)), "moe_forward")


def moe_forward_host(layer: int, x_host, T: int, out_host, stream=None):
    """x_host / out_host are CPU tensors (pinned for asynchronous copies)."""
    _check(load().moe_forward_host(layer, _ptr(x_host), T, _ptr(out_host), _stream(stream)), "moe_forward_host")


def moe_forward_host_async(layer: int, x_host, T: int, out_host, stream=None):
    """moe_forward_host without the final wait: the host buffers may be reused, and out_host read,
    once the stream has passed the call."""
    _check(load().moe_forward_host_async(layer, _ptr(x_host), T, _ptr(out_host), _stream(stream)),
           "moe_forward_host_async")


def moe_last_error(layer: int) -> int:
    return int(load().moe_last_error(layer))


def moe_layer_destroy(layer: int):
    load().moe_layer_destroy(layer)


def moe_layer_workspace_bytes(layer: int) -> int:
    return int(load().moe_layer_workspace_bytes(layer))


def moe_layer_last_launches(layer: int) -> int:
    return int(load().moe_layer_last_launches(layer))


def moe_profile_enable(layer: int, on: bool):
    _check(load().moe_profile_enable(layer, 1 if on else 0), "moe_profile_enable")


def moe_profile_read(layer: int, kernel: int):
    """(summed device milliseconds, launches) of one kernel since the last read; resets them."""
    ms, n = ctypes.c_double(), ctypes.c_int64()
    _check(load().moe_profile_read(layer, kernel, ctypes.byref(ms), ctypes.byref(n)), "moe_profile_read")
    return ms.value, n.value


def moe_kernel_name(kernel: int) -> str:
    return load().moe_kernel_name(kernel).decode()


def moe_layer_set_option(layer: int, option: int, value: int):
    _check(load().moe_layer_set_option(layer, option, int(value)), "moe_layer_set_option")


def moe_layer_get_option(layer: int, option: int) -> int:
    v = ctypes.c_int64()
    _check(load().moe_layer_get_option(layer, option, ctypes.byref(v)), "moe_layer_get_option")
    return v.value


def moe_layer_debug_read(layer: int, item: str, dst) -> None:
    """Copy an intermediate of the last forward into the numpy array ``dst`` (see moe.h)."""
    _check(load().moe_layer_debug_read(layer, DEBUG_ITEMS[item], dst.ctypes.data, dst.nbytes),
           "moe_layer_debug_read")


def moe_layer_set_expert(layer: int, e: int, gate_up, gate_up_scale, down, down_scale, stream=None):
    """Point routed expert e at one expert's device tensors (a ragged expert table; see moe.h)."""
    _check(load().moe_layer_set_expert(layer, int(e), _ptr(gate_up), _ptr(gate_up_scale), _ptr(down),
                                       _ptr(down_scale), _stream(stream)), "moe_layer_set_expert")


def moe_route_noalloc(cfg: moe_config, router_w, router_bias, x, T: int, idx, w, stream=None):
    """Routing without any device allocation (for callers that may not allocate; see moe.h)."""
    _check(load().moe_route_noalloc(ctypes.byref(cfg), _ptr(router_w), _ptr(router_bias), _ptr(x), T, _ptr(idx),
                                    _ptr(w), _stream(stream)), "moe_route_noalloc")


# ------------------------------------------------------------------------------------------
# convenience owner of a layer handle
# ------------------------------------------------------------------------------------------

class MoELayer:
    """Owns a moe_layer handle and keeps the borrowed weight tensors alive.

    ``weights`` maps the moe_weights field names to CUDA tensors (or None)."""

    def __init__(self, d, f, n_experts, top_k, max_tokens, router, wkind, weights: dict, n_shared=0, f_shared=0,
                 routed_scaling_factor=1.0, out_bf16=False):
        self.cfg = moe_config(d=d, f=f, n_experts=n_experts, top_k=top_k, n_shared=n_shared, f_shared=f_shared,
                              max_tokens=max_tokens, router=router, routed_scaling_factor=routed_scaling_factor,
                              wkind=wkind, out_bf16=1 if out_bf16 else 0)
        self._tensors = dict(weights)
        self.w = moe_weights(**{k: _ptr(v) for k, v in weights.items()})
        self.handle = moe_layer_create(self.cfg, self.w)

    def route(self, x, idx, w, stream=None):
        moe_route(self.handle, x, x.shape[0], idx, w, stream)

    def forward(self, x, out, stream=None):
        moe_forward(self.handle, x, x.shape[0], out, stream)

    def forward_host(self, x_host, out_host, stream=None):
        moe_forward_host(self.handle, x_host, x_host.shape[0], out_host, stream)

    def forward_host_async(self, x_host, out_host, stream=None):
        moe_forward_host_async(self.handle, x_host, x_host.shape[0], out_host, stream)

    def last_error(self) -> int:
        return moe_last_error(self.handle)

    def workspace_bytes(self) -> int:
        return moe_layer_workspace_bytes(self.handle)

    def last_launches(self) -> int:
        return moe_layer_last_launches(self.handle)

    def set_single_token_mode(self, mode: int) -> int:
        """T = 1 path: 2 one cooperative launch, 1 router + two single-token kernels, 0 general
        kernels.  A mode the shape does not allow falls back to the next lower one; returns the
        mode in use."""
        moe_layer_set_option(self.handle, MOE_OPT_SINGLE_TOKEN_KERNELS, int(mode))
        return self.single_token_mode

    @property
    def single_token_mode(self) -> int:
        return moe_layer_get_option(self.handle, MOE_OPT_SINGLE_TOKEN_KERNELS)

    def debug_read(self, item: str, dst):
        moe_layer_debug_read(self.handle, item, dst)

    def set_router_groups(self, n_group: int, topk_group: int):
        """Group-limited selection (n_group = 1: the plain router)."""
        moe_layer_set_option(self.handle, MOE_OPT_ROUTER_GROUPS, int(n_group) + (int(topk_group) << 16))

    def set_router_top_p(self, p: float):
        """Adaptive expert top-p (0 or 1: off)."""
        moe_layer_set_option(self.handle, MOE_OPT_ROUTER_TOP_P, int(round(p * 1e6)))

    def set_phase_trace(self, on: bool):
        """Single launch: record the phase times read back as debug item "trace"."""
        moe_layer_set_option(self.handle, MOE_OPT_PHASE_TRACE, 1 if on else 0)

    def set_union_tensor_cores(self, on: bool):
        """Small batches (T >= 2) on the tensor-core union kernels (default) or the general kernels."""
        moe_layer_set_option(self.handle, MOE_OPT_UNION_TENSOR_CORES, 1 if on else 0)

    def set_prefill_min_tokens(self, n: int):
        moe_layer_set_option(self.handle, MOE_OPT_PREFILL_MIN_TOKENS, n)

    @property
    def has_gemm_path(self) -> bool:
        return moe_layer_get_option(self.handle, MOE_OPT_PREFILL_AVAILABLE) == 1

    def profile(self, on: bool):
        moe_profile_enable(self.handle, on)

    def profile_read(self) -> dict:
        """{kernel name: (ms, launches)} for the kernels that ran since the last read."""
        out = {}
        for kid, name in enumerate(KERNELS):
            ms, n = moe_profile_read(self.handle, kid)
            if n:
                out[name] = (ms, n)
        return out

    def close(self):
        if self.handle:
            moe_layer_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class ExpertCache:
    """A device-memory tier of routed experts in front of host memory (moe_expert_cache_*, see moe.h).

    ``device`` holds the always-resident tensors (router_w, router_bias, shared_*; CUDA); ``host``
    the routed experts (gate_up, gate_up_scale, down, down_scale; CPU tensors, pinned for
    asynchronous copies).  ``layer`` is the layer to call forward on after ``prepare``."""

    def __init__(self, d, f, n_experts, top_k, max_tokens, router, wkind, device: dict, host: dict, n_slots,
                 n_shared=0, f_shared=0, routed_scaling_factor=1.0, out_bf16=False):
        self.cfg = moe_config(d=d, f=f, n_experts=n_experts, top_k=top_k, n_shared=n_shared, f_shared=f_shared,
                              max_tokens=max_tokens, router=router, routed_scaling_factor=routed_scaling_factor,
                              wkind=wkind, out_bf16=1 if out_bf16 else 0)
        self._tensors = (dict(device), dict(host))
        self.dw = moe_weights(**{k: _ptr(v) for k, v in device.items()})
        self.hw = moe_weights(**{k: _ptr(v) for k, v in host.items()})
        h = ctypes.c_void_p()
        _check(load().moe_expert_cache_create(ctypes.byref(self.cfg), ctypes.byref(self.dw), ctypes.byref(self.hw),
                                              int(n_slots), ctypes.byref(h)), "moe_expert_cache_create")
        self.handle = h.value
        self.layer = load().moe_expert_cache_layer(self.handle)

    def prepare(self, x, stream=None):
        _check(load().moe_expert_cache_prepare(self.handle, _ptr(x), x.shape[0], _stream(stream)),
               "moe_expert_cache_prepare")

    def forward(self, x, out, stream=None):
        moe_forward(self.layer, x, x.shape[0], out, stream)

    def pin(self, e: int, on: bool = True):
        _check(load().moe_expert_cache_pin(self.handle, int(e), 1 if on else 0), "moe_expert_cache_pin")

    def stats(self) -> dict:
        h, m, b, r = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int32()
        _check(load().moe_expert_cache_stats(self.handle, ctypes.byref(h), ctypes.byref(m), ctypes.byref(b),
                                             ctypes.byref(r)), "moe_expert_cache_stats")
        return {"hits": h.value, "misses": m.value, "bytes_in": b.value, "resident": r.value}

    def slot_of(self, e: int) -> int:
        return int(load().moe_expert_cache_slot_of(self.handle, int(e)))

    def last_error(self) -> int:
        return moe_last_error(self.layer)

    def close(self):
        if self.handle:
            load().moe_expert_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
