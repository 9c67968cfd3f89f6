"""fp64 CPU oracle of the routed MoE FFN layer -- test infrastructure only.

Only the tests, the smoke check and the benchmark's CPU-baseline leg import this
package.  The product library never does, and this package never imports the
product.  ``oracle.c`` holds the arithmetic; this file marshals numpy arrays into
it and builds the shared library on first use (gcc -O2 -fopenmp, no fast-math).

Parity pins: see ``tests/test_oracle_pins.py``; every function here is pinned there
except the readings that no page fixes (router precision, the tiny layer's softmax,
noaux_tc without groups, router weight dtype), which are "parity unpinned" beyond
the invariants that hold under any reading.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

ROUTER_SOFTMAX, ROUTER_SIGMOID = 0, 1
W_INT4, W_BF16, W_INT8, W_INT2 = 0, 1, 2, 3
MODE_PER_TOKEN, MODE_UNION, MODE_DENSE = 0, 1, 2
ERR = {0: "ok", 1: "range (non-finite input)", 2: "missing expert", 3: "bad argument", 4: "out of memory"}


def build(force: bool = False) -> str:
    """Compile liboracle.so next to its source if it is missing or stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
                               "-std=c11", "-Wall", "-fPIC", "-shared", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class _Layer(ctypes.Structure):
    _fields_ = [
        ("d", ctypes.c_int32), ("f", ctypes.c_int32), ("n_experts", ctypes.c_int32),
        ("top_k", ctypes.c_int32), ("n_shared", ctypes.c_int32), ("f_shared", ctypes.c_int32),
        ("router", ctypes.c_int32), ("wkind", ctypes.c_int32), ("scaling", ctypes.c_double),
        ("router_w", ctypes.c_void_p), ("router_bias", ctypes.c_void_p),
        ("gate_up", ctypes.c_void_p), ("gate_up_scale", ctypes.c_void_p),
        ("down", ctypes.c_void_p), ("down_scale", ctypes.c_void_p),
        ("shared_gate_up", ctypes.c_void_p), ("shared_gate_up_scale", ctypes.c_void_p),
        ("shared_down", ctypes.c_void_p), ("shared_down_scale", ctypes.c_void_p),
        ("n_group", ctypes.c_int32), ("topk_group", ctypes.c_int32), ("top_p", ctypes.c_double),
    ]


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P, I32, I64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
        L.oracle_quantize_int8.argtypes = [P, I64, I64, P, P]
        L.oracle_pack_int4.argtypes = [P, I64, I64, P, P]
        L.oracle_unpack_int4.argtypes = [P, I64, I64, P]
        L.oracle_unpack_int4.restype = None
        L.oracle_quantize_tier.argtypes = [P, I64, I64, I32, P, P]
        L.oracle_pack_int2.argtypes = [P, I64, I64, P, P]
        L.oracle_unpack_int2.argtypes = [P, I64, I64, P]
        L.oracle_unpack_int2.restype = None
        L.oracle_route.argtypes = [ctypes.POINTER(_Layer), P, I32, P, P, P, P]
        L.oracle_forward.argtypes = [ctypes.POINTER(_Layer), P, I32, I32, P, P, P, P]
        L.oracle_expert_ffn.argtypes = [ctypes.POINTER(_Layer), I32, P, P, P, P, P]
        L.oracle_num_threads.argtypes = []
        L.oracle_set_num_threads.argtypes = [ctypes.c_int]
        L.oracle_set_num_threads.restype = None
        _lib = L
    return _lib


def _p(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"oracle {what}: {ERR.get(rc, rc)}")


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def set_num_threads(n: int) -> None:
    """Threads of the following calls (results do not depend on it)."""
    lib().oracle_set_num_threads(int(n))


# ----------------------------------------------------------------------------------------
# quantiser / packer
# ----------------------------------------------------------------------------------------

def quantize_int8(w: np.ndarray):
    """int8 container: (q int8 [rows][cols], scales fp32 [rows]); raises on non-finite input."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    rows, cols = w.shape
    q = np.empty((rows, cols), np.int8)
    s = np.empty(rows, np.float32)
    _check(lib().oracle_quantize_int8(_p(w), rows, cols, _p(q), _p(s)), "quantize_int8")
    return q, s


def pack_int4(w: np.ndarray, allow_nonfinite: bool = False):
    """Packed int4: (bytes u8 [rows][cols/2], scales fp32 [rows])."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    rows, cols = w.shape
    p = np.empty((rows, cols // 2), np.uint8)
    s = np.empty(rows, np.float32)
    rc = lib().oracle_pack_int4(_p(w), rows, cols, _p(p), _p(s))
    if not (allow_nonfinite and rc == 1):
        _check(rc, "pack_int4")
    return p, s


def unpack_int4(packed: np.ndarray, cols: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    rows = packed.shape[0]
    q = np.empty((rows, cols), np.int8)
    lib().oracle_unpack_int4(_p(packed), rows, cols, _p(q))
    return q


def quantize_tier(w: np.ndarray, bits: int):
    """The b-bit tier (2, 4 or 8) in the int8 container: (q int8 [rows][cols], scales fp32 [rows])."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    rows, cols = w.shape
    q = np.empty((rows, cols), np.int8)
    s = np.empty(rows, np.float32)
    _check(lib().oracle_quantize_tier(_p(w), rows, cols, int(bits), _p(q), _p(s)), "quantize_tier")
    return q, s


def pack_int2(w: np.ndarray, allow_nonfinite: bool = False):
    """Packed int2: (bytes u8 [rows][cols/4], scales fp32 [rows])."""
    w = np.ascontiguousarray(w, dtype=np.float32)
    rows, cols = w.shape
    p = np.empty((rows, cols // 4), np.uint8)
    s = np.empty(rows, np.float32)
    rc = lib().oracle_pack_int2(_p(w), rows, cols, _p(p), _p(s))
    if not (allow_nonfinite and rc == 1):
        _check(rc, "pack_int2")
    return p, s


def unpack_int2(packed: np.ndarray, cols: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    rows = packed.shape[0]
    q = np.empty((rows, cols), np.int8)
    lib().oracle_unpack_int2(_p(packed), rows, cols, _p(q))
    return q


# ----------------------------------------------------------------------------------------
# layer
# ----------------------------------------------------------------------------------------

class Layer:
    """Host copy of a layer's weights for the oracle.

    ``experts`` maps an expert index to a dict with ``gate_up``, ``down`` (and, for int4 and
    int8, ``gate_up_scale`` and ``down_scale``); experts not present are unavailable and the
    oracle reports an error if a token routes to one.  ``shared`` is the same dict for the
    shared expert (or None).
    """

    def __init__(self, d, f, E, k, router, scaling, wkind, router_w, router_bias=None,
                 experts: Optional[Dict[int, dict]] = None, shared: Optional[dict] = None,
                 f_shared: Optional[int] = None, n_group: int = 1, topk_group: int = 1, top_p: float = 0.0):
        """n_group / topk_group: group-limited selection (n_group > 1); top_p in (0, 1): adaptive
        expert top-p (dropped experts come back as index -1 with weight 0)."""
        self.n_group, self.topk_group, self.top_p = int(n_group), int(topk_group), float(top_p)
        self.d, self.f, self.E, self.k = d, f, E, k
        self.router, self.scaling, self.wkind = router, float(scaling), wkind
        self.router_w = np.ascontiguousarray(router_w, dtype=np.float32)
        self.router_bias = None if router_bias is None else np.ascontiguousarray(router_bias, np.float32)
        self.experts = {int(e): {n: np.ascontiguousarray(a) for n, a in v.items()}
                        for e, v in (experts or {}).items()}
        self.shared = None if shared is None else {n: np.ascontiguousarray(a) for n, a in shared.items()}
        self.f_shared = f if f_shared is None else f_shared
        self._keep = []
        self._s = self._struct()

    def _struct(self) -> _Layer:
        E = self.E
        arrs = {}
        for name in ("gate_up", "gate_up_scale", "down", "down_scale"):
            a = (ctypes.c_void_p * E)()
            for e in range(E):
                ex = self.experts.get(e)
                a[e] = None if ex is None or name not in ex else ex[name].ctypes.data
            arrs[name] = a
            self._keep.append(a)
        sh = self.shared or {}
        return _Layer(
            d=self.d, f=self.f, n_experts=E, top_k=self.k, n_shared=1 if self.shared else 0,
            f_shared=self.f_shared, router=self.router, wkind=self.wkind, scaling=self.scaling,
            router_w=_p(self.router_w), router_bias=_p(self.router_bias),
            gate_up=ctypes.cast(arrs["gate_up"], ctypes.c_void_p),
            gate_up_scale=ctypes.cast(arrs["gate_up_scale"], ctypes.c_void_p),
            down=ctypes.cast(arrs["down"], ctypes.c_void_p),
            down_scale=ctypes.cast(arrs["down_scale"], ctypes.c_void_p),
            shared_gate_up=_p(sh.get("gate_up")), shared_gate_up_scale=_p(sh.get("gate_up_scale")),
            shared_down=_p(sh.get("down")), shared_down_scale=_p(sh.get("down_scale")),
            n_group=self.n_group, topk_group=self.topk_group, top_p=self.top_p)

    # ------------------------------------------------------------------------------
    def route(self, x_bits: np.ndarray):
        """Returns dict(idx int32 [T][k], w fp64 [T][k], logits fp64 [T][E], gap fp64 [T])."""
        x = np.ascontiguousarray(x_bits, dtype=np.uint16)
        T = x.shape[0]
        idx = np.empty((T, self.k), np.int32)
        w = np.empty((T, self.k), np.float64)
        logits = np.empty((T, self.E), np.float64)
        gap = np.empty(T, np.float64)
        _check(lib().oracle_route(ctypes.byref(self._s), _p(x), T, _p(idx), _p(w), _p(logits), _p(gap)),
               "route")
        return {"idx": idx, "w": w, "logits": logits, "gap": gap}

    def forward(self, x_bits: np.ndarray, mode: int = MODE_PER_TOKEN):
        """Returns dict(out fp64 [T][d], idx, w, gap)."""
        x = np.ascontiguousarray(x_bits, dtype=np.uint16)
        T = x.shape[0]
        out = np.empty((T, self.d), np.float64)
        idx = np.empty((T, self.k), np.int32)
        w = np.empty((T, self.k), np.float64)
        gap = np.empty(T, np.float64)
        _check(lib().oracle_forward(ctypes.byref(self._s), _p(x), T, mode, _p(out), _p(idx), _p(w),
                                    _p(gap)), "forward")
        return {"out": out, "idx": idx, "w": w, "gap": gap}

    def expert_ffn(self, e, x_row_bits: np.ndarray):
        """One expert on one token: dict(g, u, h [f], y [d]); ``e == "shared"`` for the shared one."""
        ei = self.E if e == "shared" else int(e)
        f = self.f_shared if e == "shared" else self.f
        x = np.ascontiguousarray(x_row_bits, dtype=np.uint16).reshape(-1)
        g, u, h = (np.empty(f, np.float64) for _ in range(3))
        y = np.empty(self.d, np.float64)
        _check(lib().oracle_expert_ffn(ctypes.byref(self._s), ei, _p(x), _p(g), _p(u), _p(h), _p(y)),
               "expert_ffn")
        return {"g": g, "u": u, "h": h, "y": y}


def tie_ambiguous(gap: np.ndarray, logits_or_keys_scale: np.ndarray, rel: float = 1e-12) -> np.ndarray:
    """Tokens whose k-th and (k+1)-th keys are closer than ``rel`` times the key scale."""
    return gap < rel * np.maximum(np.abs(logits_or_keys_scale), 1e-300)
