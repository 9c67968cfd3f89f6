"""Builds oracle layers from the synthetic configurations (host side only)."""
from __future__ import annotations

import dataclasses
from typing import Iterable, Optional

import numpy as np

import oracle
import synthetic as syn


def small_config(base: str = "glm_decode", **kw) -> syn.LayerConfig:
    """A scaled-down copy of a configuration (same router and weight kinds)."""
    return dataclasses.replace(syn.CONFIGS[base], **kw)


def host_expert(cfg: syn.LayerConfig, e, seed: int = 0, wkind: Optional[int] = None,
                bits: Optional[int] = None) -> dict:
    """One expert's weights in the layer's storage kind, drawn and packed on the host.

    For the int8 container, ``bits`` picks the tier of its codes: 4 (the default, the int4 tier
    the packed int4 container holds) or 8 (the int8 tier)."""
    wkind = cfg.wkind if wkind is None else wkind
    out = {}
    for which in ("gate_up", "down"):
        w = syn.gen_expert_fp32(cfg, e, which, seed)
        if wkind == syn.W_BF16:
            out[which] = syn.fp32_to_bf16_bits(w)
        elif wkind == oracle.W_INT8:
            q, s = oracle.quantize_int8(w) if bits in (None, 4) else oracle.quantize_tier(w, bits)
            out[which], out[which + "_scale"] = q, s
        elif wkind == oracle.W_INT2:
            p, s = oracle.pack_int2(w)
            out[which], out[which + "_scale"] = p, s
        else:
            p, s = oracle.pack_int4(w)
            out[which], out[which + "_scale"] = p, s
    return out


def oracle_layer(cfg: syn.LayerConfig, seed: int = 0, experts: Optional[Iterable[int]] = None,
                 wkind: Optional[int] = None, bits: Optional[int] = None) -> oracle.Layer:
    """Oracle layer with the given experts (all by default) drawn on the host."""
    wkind = cfg.wkind if wkind is None else wkind
    ids = range(cfg.E) if experts is None else sorted(set(int(e) for e in experts))
    ex = {e: host_expert(cfg, e, seed, wkind, bits) for e in ids}
    shared = host_expert(cfg, "shared", seed, wkind, bits) if cfg.n_shared else None
    return oracle.Layer(cfg.d, cfg.f, cfg.E, cfg.k, cfg.router, cfg.scaling, wkind,
                        syn.gen_router_w(cfg, seed), syn.gen_router_bias(cfg, seed),
                        experts=ex, shared=shared, f_shared=cfg.f_shared or cfg.f)


def router_only(cfg: syn.LayerConfig, seed: int = 0) -> oracle.Layer:
    return oracle.Layer(cfg.d, cfg.f, cfg.E, cfg.k, cfg.router, cfg.scaling, cfg.wkind,
                        syn.gen_router_w(cfg, seed), syn.gen_router_bias(cfg, seed),
                        f_shared=cfg.f_shared or cfg.f)


def oracle_layer_from(cfg: syn.LayerConfig, experts: dict, seed: int = 0) -> oracle.Layer:
    """Oracle layer over experts already drawn and stored in the oracle's format (``experts`` maps
    expert ids, and "shared" for the shared expert, to their weight dicts)."""
    ex = {e: v for e, v in experts.items() if e != "shared"}
    return oracle.Layer(cfg.d, cfg.f, cfg.E, cfg.k, cfg.router, cfg.scaling, cfg.wkind,
                        syn.gen_router_w(cfg, seed), syn.gen_router_bias(cfg, seed),
                        experts=ex, shared=experts.get("shared"), f_shared=cfg.f_shared or cfg.f)
