"""GPU parity of the router variants: group-limited selection (the DeepSeek-V3 router's noaux_tc,
n_group = 8, topk_group = 4 for 256 experts) and adaptive expert top-p (the colibri README's
--topp), against the oracle on the same seeded inputs.

Expert indices are compared bit for bit (dropped entries: -1 on both sides), gate weights within
1e-6 relative, outputs within the layer's tolerance.  Every routing path runs: T = 1 (the
general kernels, since the single-token paths take the plain router only), T <= 32 (the fused
small-batch router), T > 32 (the fp64 router GEMM and the top-k kernel), and the tcgen05
expert GEMMs, whose gather must skip the slots that top-p leaves unused.
"""
import numpy as np
import pytest

import oracle
import synthetic as syn
from gpu_layers import build_gpu_layer, check_close, run_forward, run_route
from layers import oracle_layer, small_config

pytestmark = pytest.mark.gpu


def _layers(cfg, n_group=1, topk_group=1, top_p=0.0, max_tokens=None):
    layer, _ = build_gpu_layer(cfg, max_tokens=max_tokens)
    if n_group > 1:
        layer.set_router_groups(n_group, topk_group)
    if top_p:
        layer.set_router_top_p(top_p)
    base = oracle_layer(cfg)
    ora = oracle.Layer(cfg.d, cfg.f, cfg.E, cfg.k, cfg.router, cfg.scaling, cfg.wkind, base.router_w,
                       base.router_bias, experts=base.experts, shared=base.shared, f_shared=cfg.f_shared or cfg.f,
                       n_group=n_group, topk_group=topk_group, top_p=top_p)
    return layer, ora


def _top_p_margin(ora, x, p):
    """Smallest distance between p and a running share of the plain router's weights (a token
    whose share sits within rounding of p could be decided either way)."""
    plain = oracle.Layer(ora.d, ora.f, ora.E, ora.k, ora.router, ora.scaling, ora.wkind, ora.router_w,
                         ora.router_bias).route(x)
    share = np.cumsum(plain["w"], axis=1) / plain["w"].sum(axis=1, keepdims=True)
    return np.abs(share - p).min()


CFG = small_config("glm_decode", T=1, d=256, E=64, k=6, f=128, f_shared=128)


@pytest.mark.parametrize("T", [1, 7, 40, 300])
def test_grouped_selection_matches_oracle(T):
    cfg = small_config("glm_decode", T=T, d=256, E=64, k=6, f=128, f_shared=128)
    layer, ora = _layers(cfg, n_group=8, topk_group=3)
    try:
        x = syn.gen_x(cfg, 0, token_offset=23)
        ref = ora.forward(x)
        idx, w = run_route(layer, x, cfg.k)
        assert np.array_equal(idx, ref["idx"])
        np.testing.assert_allclose(w, ref["w"], rtol=1e-6)
        check_close(run_forward(layer, x), ref["out"])
        # grouping changes the choice for some token (the test is not vacuous)
        plain = oracle_layer(cfg).route(x)["idx"]
        if T >= 40:
            assert not np.array_equal(np.sort(plain, 1), np.sort(ref["idx"], 1))
    finally:
        layer.close()


@pytest.mark.parametrize("T", [1, 7, 40, 300])
def test_top_p_matches_oracle_and_drops_experts(T):
    cfg = small_config("glm_decode", T=T, d=256, E=64, k=6, f=128, f_shared=128)
    p = 0.7
    layer, ora = _layers(cfg, top_p=p)
    try:
        x = syn.gen_x(cfg, 0, token_offset=31)
        assert _top_p_margin(ora, x, p) > 1e-9
        ref = ora.forward(x)
        idx, w = run_route(layer, x, cfg.k)
        assert np.array_equal(idx, ref["idx"])
        np.testing.assert_allclose(w, ref["w"], rtol=1e-6, atol=0)
        assert (idx == -1).any()
        check_close(run_forward(layer, x), ref["out"])
        if T >= 40:      # the same batch through the tcgen05 expert GEMMs
            layer.set_prefill_min_tokens(1)
            check_close(run_forward(layer, x), ref["out"])
    finally:
        layer.close()


def test_both_variants_with_the_deepseek_group_setting():
    # 256 experts in 8 groups of 32, 4 groups kept, top-8, adaptive top-p 0.7
    cfg = small_config("glm_decode", T=24, d=512, E=256, k=8, f=128, f_shared=128)
    layer, ora = _layers(cfg, n_group=8, topk_group=4, top_p=0.7)
    try:
        x = syn.gen_x(cfg, 0, token_offset=57)
        assert _top_p_margin(ora, x, 0.7) > 1e-9
        ref = ora.forward(x)
        idx, w = run_route(layer, x, cfg.k)
        assert np.array_equal(idx, ref["idx"])
        np.testing.assert_allclose(w, ref["w"], rtol=1e-6)
        check_close(run_forward(layer, x), ref["out"])
        # switching the variants off restores the plain router and the single-launch path
        layer.set_router_groups(1, 1)
        layer.set_router_top_p(0.0)
        plain = oracle_layer(cfg).forward(x[:1])
        check_close(run_forward(layer, x[:1]), plain["out"])
    finally:
        layer.close()


def test_variant_options_are_checked():
    import quantized_expert_ffn_02_b200 as qe
    layer, _ = build_gpu_layer(CFG)
    try:
        for G, TG in ((3, 1), (8, 0), (8, 9), (64, 1), (16, 1)):  # 64 % 3, topk_group 0 or > n_group,
            with pytest.raises(qe.MoeError):                       # n_group > 32, too few experts left
                layer.set_router_groups(G, TG)
        with pytest.raises(qe.MoeError):
            qe.moe_layer_set_option(layer.handle, qe.MOE_OPT_ROUTER_TOP_P, 1_000_001)
        layer.set_router_groups(4, 2)
        assert qe.moe_layer_get_option(layer.handle, qe.MOE_OPT_ROUTER_GROUPS) == 4 + (2 << 16)
    finally:
        layer.close()
