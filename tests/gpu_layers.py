"""Builds layers on the GPU (through the C ABI) from the same seeded draws the oracle sees.

Experts listed in ``host_experts`` (and the shared expert) are drawn on the host with the numpy
generator -- bit-identical to what ``layers.oracle_layer`` gives the oracle.  Other experts are
drawn on the device by the torch copy of the generator: full-size layers build in seconds, and
those experts are never compared against the oracle (no compared token routes to them).
"""
from __future__ import annotations

from typing import Iterable, Optional

import numpy as np
import torch

import quantized_expert_ffn_02_b200 as qe
import synthetic as syn


def check_close(gpu: np.ndarray, ref: np.ndarray, rel_l2: float = 2e-3, max_rms: float = 1e-2):
    """The layer's output tolerance: relative L2 <= 2e-3 and max-abs <= 1e-2 * RMS(ref)."""
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    assert gpu.shape == ref.shape
    assert np.isfinite(gpu).all()
    err = gpu - ref
    r = np.linalg.norm(err) / np.linalg.norm(ref)
    rms = np.sqrt(np.mean(ref ** 2))
    m = np.abs(err).max()
    assert r <= rel_l2, f"relative L2 {r:.3e} > {rel_l2}"
    assert m <= max_rms * rms, f"max abs {m:.3e} > {max_rms} * rms {rms:.3e}"
    return r, m / rms


def _fp32_dev(cfg, e, which, seed, host: bool, dev):
    rows, cols = syn.expert_shape(cfg, e, which)
    if host:
        return torch.from_numpy(syn.gen_expert_fp32(cfg, e, which, seed)).to(dev)
    return syn.torch_normal_fp32(seed, syn.expert_tensor_name(e, which), rows * cols, syn.WEIGHT_STD,
                                 dev).view(rows, cols)


def build_gpu_layer(cfg: syn.LayerConfig, seed: int = 0, host_experts: Optional[Iterable[int]] = None,
                    max_tokens: Optional[int] = None, out_bf16: Optional[bool] = None, device="cuda",
                    oracle_experts: Optional[dict] = None):
    """Returns (MoELayer, weights dict of device tensors).  host_experts=None draws every expert on the host.

    oracle_experts: if a dict is given, every host-drawn expert is also stored there in the
    oracle's storage format (packed on the host by the oracle's packer, or bf16 bits), keyed by
    expert id or "shared", so a full-size expert is drawn once for both sides."""
    dev = torch.device(device)
    E, d, f = cfg.E, cfg.d, cfg.f
    int4 = cfg.wkind != syn.W_BF16          # a packed container with per-row scales (int4, int8, int2)
    hset = None if host_experts is None else set(int(e) for e in host_experts)
    W = {}
    # bytes per row of n columns, storage dtype, the GPU packer and the oracle's packer per kind
    per = {syn.W_INT4: (2, torch.uint8), syn.W_INT8: (1, torch.int8), syn.W_INT2: (4, torch.uint8)}

    def cols(n):
        return n // per[cfg.wkind][0]

    def gpu_pack(w, dst, dst_s):
        {syn.W_INT4: qe.moe_pack_int4, syn.W_INT8: qe.moe_pack_int8, syn.W_INT2: qe.moe_pack_int2}[cfg.wkind](
            w, dst, dst_s)

    def oracle_pack(w):
        import oracle
        if cfg.wkind == syn.W_INT8:
            return oracle.quantize_tier(w, 8)
        if cfg.wkind == syn.W_INT2:
            return oracle.pack_int2(w)
        return oracle.pack_int4(w)

    if int4:
        dt = per[cfg.wkind][1]
        W["gate_up"] = torch.empty((E, 2 * f, cols(d)), dtype=dt, device=dev)
        W["gate_up_scale"] = torch.empty((E, 2 * f), dtype=torch.float32, device=dev)
        W["down"] = torch.empty((E, d, cols(f)), dtype=dt, device=dev)
        W["down_scale"] = torch.empty((E, d), dtype=torch.float32, device=dev)
    else:
        W["gate_up"] = torch.empty((E, 2 * f, d), dtype=torch.int16, device=dev)
        W["down"] = torch.empty((E, d, f), dtype=torch.int16, device=dev)

    def put(e, which, dst, dst_s):
        host = hset is None or e == "shared" or e in hset
        if not int4 and host:
            bits = syn.gen_expert_bf16(cfg, e, which, seed)
            if oracle_experts is not None:
                oracle_experts.setdefault(e, {})[which] = bits
            dst.copy_(torch.from_numpy(bits.view(np.int16)).to(dev))
            return
        if host and oracle_experts is not None:
            w_host = syn.gen_expert_fp32(cfg, e, which, seed)
            rec = oracle_experts.setdefault(e, {})
            rec[which], rec[which + "_scale"] = oracle_pack(w_host)
            w = torch.from_numpy(w_host).to(dev)
            del w_host
        else:
            w = _fp32_dev(cfg, e, which, seed, host, dev)
        if int4:
            gpu_pack(w, dst, dst_s)
        else:
            dst.copy_(w.to(torch.bfloat16).view(torch.int16))

    for e in range(E):
        for which in ("gate_up", "down"):
            put(e, which, W[which][e], W.get(which + "_scale", [None] * E)[e] if int4 else None)
    if cfg.n_shared:
        fs = cfg.f_shared
        if int4:
            dt = per[cfg.wkind][1]
            W["shared_gate_up"] = torch.empty((2 * fs, cols(d)), dtype=dt, device=dev)
            W["shared_gate_up_scale"] = torch.empty((2 * fs,), dtype=torch.float32, device=dev)
            W["shared_down"] = torch.empty((d, cols(fs)), dtype=dt, device=dev)
            W["shared_down_scale"] = torch.empty((d,), dtype=torch.float32, device=dev)
        else:
            W["shared_gate_up"] = torch.empty((2 * fs, d), dtype=torch.int16, device=dev)
            W["shared_down"] = torch.empty((d, fs), dtype=torch.int16, device=dev)
        put("shared", "gate_up", W["shared_gate_up"], W.get("shared_gate_up_scale"))
        put("shared", "down", W["shared_down"], W.get("shared_down_scale"))
    W["router_w"] = torch.from_numpy(syn.gen_router_w(cfg, seed)).to(dev)
    b = syn.gen_router_bias(cfg, seed)
    W["router_bias"] = None if b is None else torch.from_numpy(b).to(dev)
    torch.cuda.synchronize()
    layer = qe.MoELayer(d, f, E, cfg.k, max_tokens or cfg.T, cfg.router, cfg.wkind, W, n_shared=cfg.n_shared,
                        f_shared=cfg.f_shared, routed_scaling_factor=cfg.scaling,
                        out_bf16=cfg.out_bf16 if out_bf16 is None else out_bf16)
    return layer, W


def x_dev(x_bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x_bits).view(np.int16)).to(device)


def run_forward(layer, x_bits: np.ndarray, out_bf16: bool = False) -> np.ndarray:
    x = x_dev(x_bits)
    T, d = x.shape
    out = torch.empty((T, d), dtype=torch.int16 if out_bf16 else torch.float32, device="cuda")
    layer.forward(x, out)
    torch.cuda.synchronize()
    st = layer.last_error()
    assert st == qe.MOE_OK, qe.status_str(st)
    o = out.cpu().numpy()
    return syn.bf16_bits_to_fp32(o.view(np.uint16)) if out_bf16 else o


def run_route(layer, x_bits: np.ndarray, k: int):
    x = x_dev(x_bits)
    T = x.shape[0]
    idx = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    layer.route(x, idx, w)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), w.cpu().numpy()
