"""GPU tests of the device-memory expert tier (moe_expert_cache_*): routed experts in host memory,
a few expert slots in HBM, streamed in on demand with LRU eviction and an optional pinned set
(colibri README, "The idea": experts streamed on demand behind an LRU cache and a pinned hot set;
iliria page, "What's implemented": pinned/LRU slabs behind a ragged descriptor).

The layer over the tier must give the oracle's outputs within the layer's tolerance, and exactly
the outputs of the same layer with every expert resident (the same kernels read the same bytes).
"""
import numpy as np
import pytest
import torch

import quantized_expert_ffn_02_b200 as qe
import synthetic as syn
from gpu_layers import build_gpu_layer, check_close, run_forward, x_dev
from layers import oracle_layer, small_config

pytestmark = pytest.mark.gpu

CFG = small_config("glm_decode", T=2, d=256, E=16, k=4, f=128, f_shared=128)


def _tier(cfg, n_slots, max_tokens=2):
    resident, W = build_gpu_layer(cfg, max_tokens=max_tokens)
    resident.set_single_token_mode(0)            # the general kernels, as the tier's layer uses
    device = {n: W.get(n) for n in ("router_w", "router_bias", "shared_gate_up", "shared_gate_up_scale",
                                     "shared_down", "shared_down_scale")}
    host = {n: W[n].cpu().pin_memory() for n in ("gate_up", "gate_up_scale", "down", "down_scale")}
    cache = qe.ExpertCache(cfg.d, cfg.f, cfg.E, cfg.k, max_tokens, cfg.router, cfg.wkind, device, host, n_slots,
                           n_shared=cfg.n_shared, f_shared=cfg.f_shared, routed_scaling_factor=cfg.scaling)
    return cache, resident, W


def _run(cache, x_bits):
    x = x_dev(x_bits)
    out = torch.empty((x.shape[0], CFG.d), dtype=torch.float32, device="cuda")
    cache.prepare(x)
    cache.forward(x, out)
    torch.cuda.synchronize()
    assert cache.last_error() == qe.MOE_OK
    return out.cpu().numpy()


def test_tier_matches_oracle_and_resident_layer():
    cache, resident, _ = _tier(CFG, n_slots=9)
    try:
        ora = oracle_layer(CFG)
        seen = set()
        for b in range(8):
            x = syn.gen_x(CFG, 0, T=2, token_offset=7 * b)
            out = _run(cache, x)
            ref = ora.forward(x)
            check_close(out, ref["out"])
            assert np.array_equal(out, run_forward(resident, x))
            need = set(ref["idx"].reshape(-1).tolist())
            assert all(cache.slot_of(e) >= 0 for e in need)
            seen |= need
        st = cache.stats()
        assert st["misses"] >= min(len(seen), 9) and st["resident"] <= 9
        # the same batch again: every expert is resident, nothing is copied
        before = cache.stats()
        x = syn.gen_x(CFG, 0, T=2, token_offset=49)
        _run(cache, x)
        mid = cache.stats()
        _run(cache, x)
        after = cache.stats()
        assert after["misses"] == mid["misses"] and after["bytes_in"] == mid["bytes_in"]
        assert after["hits"] > mid["hits"] >= before["hits"]
    finally:
        cache.close()
        resident.close()


def test_pinned_expert_survives_eviction_and_lru_order():
    cache, resident, _ = _tier(CFG, n_slots=8)
    try:
        ora = oracle_layer(CFG)
        x0 = syn.gen_x(CFG, 0, T=2, token_offset=0)
        _run(cache, x0)
        pin = int(ora.route(x0)["idx"][0, 0])
        cache.pin(pin)
        for b in range(1, 12):
            x = syn.gen_x(CFG, 0, T=2, token_offset=13 * b)
            check_close(_run(cache, x), ora.forward(x)["out"])
            assert cache.slot_of(pin) >= 0, "a pinned expert was evicted"
        cache.pin(pin, False)
    finally:
        cache.close()
        resident.close()


def test_batch_needing_more_experts_than_slots_is_refused():
    cache, resident, _ = _tier(CFG, n_slots=3)
    try:
        x = syn.gen_x(CFG, 0, T=2, token_offset=3)
        n_need = len(set(oracle_layer(CFG).route(x)["idx"].reshape(-1).tolist()))
        assert n_need > 3
        with pytest.raises(qe.MoeError) as ei:
            cache.prepare(x_dev(x))
        assert ei.value.status == qe.MOE_ERR_UNSUPPORTED
        # one token (4 experts) still does not fit; the layer itself is untouched
        assert cache.stats()["misses"] == 0
    finally:
        cache.close()
        resident.close()


def test_set_expert_repoints_one_expert():
    """moe_layer_set_expert: point expert e at a copy of expert e2's weights; every token that routes
    to e then sees e2's FFN (the oracle with e2's weights under index e)."""
    layer, W = build_gpu_layer(CFG)
    try:
        ora = oracle_layer(CFG)
        x = syn.gen_x(CFG, 0, T=2, token_offset=5)
        idx = ora.route(x)["idx"]
        e = int(idx[0, 0])
        e2 = next(i for i in range(CFG.E) if i not in set(idx.reshape(-1).tolist()))
        copies = {n: W[n][e2].clone() for n in ("gate_up", "gate_up_scale", "down", "down_scale")}
        qe.moe_layer_set_expert(layer.handle, e, copies["gate_up"], copies["gate_up_scale"], copies["down"],
                                copies["down_scale"])
        assert not layer.has_gemm_path                  # the tensor maps cover only the contiguous arrays
        swapped = dict(ora.experts)
        swapped[e] = ora.experts[e2]
        import oracle
        ref = oracle.Layer(CFG.d, CFG.f, CFG.E, CFG.k, CFG.router, CFG.scaling, CFG.wkind, ora.router_w,
                           ora.router_bias, experts=swapped, shared=ora.shared, f_shared=CFG.f_shared).forward(x)
        check_close(run_forward(layer, x), ref["out"])
        for mode in (2, 1):                             # the single-token paths read the table too
            layer.set_single_token_mode(mode)
            check_close(run_forward(layer, x[:1]), ref["out"][:1])
        with pytest.raises(qe.MoeError):
            qe.moe_layer_set_expert(layer.handle, CFG.E, copies["gate_up"], copies["gate_up_scale"],
                                    copies["down"], copies["down_scale"])
    finally:
        layer.close()
