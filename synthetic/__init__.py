"""Seeded synthetic inputs for the routed MoE FFN layer.

This module only draws numbers; it holds none of the layer's arithmetic (no
routing, no quantisation, no FFN).  Both the oracle side and the CUDA side of
the tests receive the bytes produced here, so the two never disagree about
their inputs.

Generator (counter based, so any element can be drawn without drawing the ones
before it):

* every tensor has a name; its 64-bit stream key is
  ``splitmix64(seed) XOR fnv1a64(name)``;
* element ``i`` of a stream is ``splitmix64(key + i)`` (SplitMix64 as
  published by Steele, Lea and Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014: add the golden gamma, then the xor-shift-multiply
  finaliser);
* a uniform in (0, 1) is ``((z >> 11) + 0.5) * 2**-53``;
* normals come from the Box-Muller transform on the uniform pair
  ``(2j, 2j+1)``: ``r = sqrt(-2 ln u1)``, element ``2j`` is ``r cos(2 pi u2)`` and
  element ``2j+1`` is ``r sin(2 pi u2)``;
* a draw is made in float64, scaled, then rounded to float32 (round to
  nearest even); bf16 tensors are then rounded float32 -> bf16 (RNE), the cast
  convention that the open-1b-verify page states for its F32 -> F16 conversion
  ("Tensor mapping").

Workload shapes and distributions follow the five synthetic configurations of
the layer: x ~ N(0, 1) bf16, router weight fp32 N(0, 0.02), expert weights
N(0, 0.02) (quantised by the packer for int4 layers, rounded to bf16 for the
bf16 layer), selection bias U(-0.1, 0.1).

``torch_normal_fp32`` is the same generator written with torch int64 ops so a
GPU can draw a full-size layer in seconds.  Its integer part is bit-identical to
the numpy one; its log/cos/sin come from a different math library, so a value
can differ from the host draw in the last float64 bits (and, rarely, by one
float32 ulp after rounding).  Anything that the oracle consumes is drawn on the
host with numpy.
"""
from __future__ import annotations

import concurrent.futures
import dataclasses
import os
from typing import Dict, Optional

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_TWO_M53 = 2.0 ** -53


def _fnv1a64(name: str) -> int:
    h = 0xCBF29CE484222325
    for byte in name.encode("utf-8"):
        h ^= byte
        h = (h * 0x100000001B3) & 0xFFFFFFFFFFFFFFFF
    return h


def splitmix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output function applied to the counter array ``z`` (uint64)."""
    with np.errstate(over="ignore"):
        z = z + _GAMMA
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        return z ^ (z >> np.uint64(31))


def stream_key(seed: int, name: str) -> int:
    s = splitmix64(np.array([seed & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64))[0]
    return int(s) ^ _fnv1a64(name)


def raw_u64(seed: int, name: str, offset: int, n: int) -> np.ndarray:
    key = np.uint64(stream_key(seed, name))
    idx = np.arange(offset, offset + n, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return splitmix64(idx + key)


def uniform(seed: int, name: str, offset: int, n: int) -> np.ndarray:
    z = raw_u64(seed, name, offset, n)
    return ((z >> np.uint64(11)).astype(np.float64) + 0.5) * _TWO_M53


_THREADS = max(1, min(16, os.cpu_count() or 1))
_CHUNK = 1 << 21


def normal(seed: int, name: str, offset: int, n: int) -> np.ndarray:
    """Standard normals, elements ``[offset, offset + n)`` of stream ``name`` (float64).

    Large draws are split into even-aligned pieces drawn on a thread pool (numpy releases the
    GIL); the generator is counter based, so the pieces are exactly the serial draw."""
    if n > 2 * _CHUNK and _THREADS > 1:
        out = np.empty(n, dtype=np.float64)
        first = min(n, (_CHUNK - (offset % 2)))
        bounds = [(0, first)]
        while bounds[-1][1] < n:
            a = bounds[-1][1]
            bounds.append((a, min(n, a + _CHUNK)))

        def work(ab):
            a, b = ab
            out[a:b] = _normal_serial(seed, name, offset + a, b - a)

        with concurrent.futures.ThreadPoolExecutor(_THREADS) as ex:
            list(ex.map(work, bounds))
        return out
    return _normal_serial(seed, name, offset, n)


def _normal_serial(seed: int, name: str, offset: int, n: int) -> np.ndarray:
    if n == 0:
        return np.zeros(0, dtype=np.float64)
    j0 = offset // 2
    j1 = (offset + n + 1) // 2
    u = uniform(seed, name, 2 * j0, 2 * (j1 - j0)).reshape(-1, 2)
    r = np.sqrt(-2.0 * np.log(u[:, 0]))
    th = (2.0 * np.pi) * u[:, 1]
    out = np.empty(2 * (j1 - j0), dtype=np.float64)
    out[0::2] = r * np.cos(th)
    out[1::2] = r * np.sin(th)
    s = offset - 2 * j0
    return out[s:s + n]


def fp32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); returns the uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    bias = np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))
    return ((u + bias) >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_fp32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# --------------------------------------------------------------------------------------
# Layer configurations (the five synthetic workloads of the layer, plus the two batch
# sizes of the batch-union decode case).
# --------------------------------------------------------------------------------------

ROUTER_SOFTMAX = 0
ROUTER_SIGMOID = 1
W_INT4 = 0
W_BF16 = 1
W_INT8 = 2          # one code per byte, the int8 tier (scale max|w| / 127)
W_INT2 = 3          # four codes per byte, the int2 tier (scale max|w| / 1)


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    T: int
    d: int
    E: int
    k: int
    f: int
    n_shared: int
    f_shared: int
    router: int
    scaling: float
    wkind: int
    out_bf16: bool = False
    n_seq: int = 1          # independent T-token calls run one after another

    @property
    def rows_gate_up(self) -> int:
        return 2 * self.f


CONFIGS: Dict[str, LayerConfig] = {
    "tiny": LayerConfig("tiny", T=4, d=256, E=8, k=2, f=128, n_shared=0, f_shared=0,
                        router=ROUTER_SOFTMAX, scaling=1.0, wkind=W_INT4),
    "granite": LayerConfig("granite", T=1, d=1024, E=32, k=8, f=512, n_shared=0, f_shared=0,
                           router=ROUTER_SOFTMAX, scaling=1.0, wkind=W_BF16, n_seq=1000),
    "glm_decode": LayerConfig("glm_decode", T=1, d=6144, E=256, k=8, f=2048, n_shared=1,
                              f_shared=2048, router=ROUTER_SIGMOID, scaling=2.5, wkind=W_INT4),
    "glm_union2": LayerConfig("glm_union2", T=2, d=6144, E=256, k=8, f=2048, n_shared=1,
                              f_shared=2048, router=ROUTER_SIGMOID, scaling=2.5, wkind=W_INT4),
    "glm_union32": LayerConfig("glm_union32", T=32, d=6144, E=256, k=8, f=2048, n_shared=1,
                               f_shared=2048, router=ROUTER_SIGMOID, scaling=2.5, wkind=W_INT4),
    "glm_prefill": LayerConfig("glm_prefill", T=2048, d=6144, E=256, k=8, f=2048, n_shared=1,
                               f_shared=2048, router=ROUTER_SIGMOID, scaling=2.5, wkind=W_INT4,
                               out_bf16=True),
}

WEIGHT_STD = 0.02
BIAS_HALF_WIDTH = 0.1


def expert_tensor_name(e, which: str) -> str:
    """Stream name of an expert tensor; ``e`` is an int or ``"shared"``."""
    return f"expert.{e}.{which}"


def expert_shape(cfg: LayerConfig, e, which: str):
    f = cfg.f_shared if e == "shared" else cfg.f
    return (2 * f, cfg.d) if which == "gate_up" else (cfg.d, f)


def gen_x(cfg: LayerConfig, seed: int = 0, T: Optional[int] = None, token_offset: int = 0) -> np.ndarray:
    """Token activations, bf16 bit patterns [T][d]; token t is elements [t*d, (t+1)*d) of stream "x"."""
    T = cfg.T if T is None else T
    v = normal(seed, "x", token_offset * cfg.d, T * cfg.d).astype(np.float32)
    return fp32_to_bf16_bits(v).reshape(T, cfg.d)


def gen_router_w(cfg: LayerConfig, seed: int = 0) -> np.ndarray:
    v = (normal(seed, "router.w", 0, cfg.E * cfg.d) * WEIGHT_STD).astype(np.float32)
    return v.reshape(cfg.E, cfg.d)


def gen_router_bias(cfg: LayerConfig, seed: int = 0) -> Optional[np.ndarray]:
    if cfg.router != ROUTER_SIGMOID:
        return None
    u = uniform(seed, "router.bias", 0, cfg.E)
    return (-BIAS_HALF_WIDTH + (2.0 * BIAS_HALF_WIDTH) * u).astype(np.float32)


def gen_expert_fp32(cfg: LayerConfig, e, which: str, seed: int = 0) -> np.ndarray:
    rows, cols = expert_shape(cfg, e, which)
    v = normal(seed, expert_tensor_name(e, which), 0, rows * cols) * WEIGHT_STD
    return v.astype(np.float32).reshape(rows, cols)


def gen_expert_bf16(cfg: LayerConfig, e, which: str, seed: int = 0) -> np.ndarray:
    return fp32_to_bf16_bits(gen_expert_fp32(cfg, e, which, seed))


# --------------------------------------------------------------------------------------
# Device-side copy of the same generator (fast full-size layers for benchmarking).
# --------------------------------------------------------------------------------------

def _s64(v: int) -> int:
    v &= 0xFFFFFFFFFFFFFFFF
    return v - (1 << 64) if v >= (1 << 63) else v


def torch_normal_fp32(seed: int, name: str, n: int, std: float, device, offset: int = 0):
    """float32 tensor of ``std * N(0,1)`` draws, elements [offset, offset+n) of stream ``name``."""
    import torch

    def srl(z, s):  # logical shift right of int64 bit patterns
        return (z >> s) & ((1 << (64 - s)) - 1)

    def mix(z):
        z = z + _s64(0x9E3779B97F4A7C15)
        z = (z ^ srl(z, 30)) * _s64(0xBF58476D1CE4E5B9)
        z = (z ^ srl(z, 27)) * _s64(0x94D049BB133111EB)
        return z ^ srl(z, 31)

    key = _s64(stream_key(seed, name))
    j0 = offset // 2
    j1 = (offset + n + 1) // 2
    idx = torch.arange(2 * j0, 2 * j1, dtype=torch.int64, device=device)
    z = mix(idx + key)
    u = (srl(z, 11).to(torch.float64) + 0.5) * _TWO_M53
    u = u.view(-1, 2)
    r = torch.sqrt(-2.0 * torch.log(u[:, 0]))
    th = (2.0 * np.pi) * u[:, 1]
    out = torch.empty(2 * (j1 - j0), dtype=torch.float64, device=device)
    out[0::2] = r * torch.cos(th)
    out[1::2] = r * torch.sin(th)
    s = offset - 2 * j0
    return (out[s:s + n] * std).to(torch.float32)
