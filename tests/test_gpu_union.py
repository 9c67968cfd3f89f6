"""Batch-union decode on the tensor-core kernels (2 <= T < the grouped-GEMM threshold, int4).

Each chosen expert's tokens run in groups of up to 8 columns of one mma.sync product with 16
weight rows.  The shapes vary what that splits: one or several column groups per expert (a
batch where many tokens share the biased favourites), a shared expert with its own f or none,
d from 1024 to 8192, f of 1024 and 2048, batches that use the fp64 router GEMM (T >= 64), and
the adaptive top-p router (dropped experts leave buckets short).  Every token is compared with
the oracle; the general (FP32-pipe) kernels give the same outputs within a much tighter bound.
"""
import numpy as np
import pytest

import oracle
import synthetic as syn
from gpu_layers import build_gpu_layer, check_close, run_forward
from layers import oracle_layer, oracle_layer_from, small_config

pytestmark = pytest.mark.gpu

SHAPES = {
    # GLM-like routing (sigmoid + bias, top-8, shared expert) at a smaller E and d
    "d2048_E32_k8_f1024_shared": dict(base="glm_decode", d=2048, E=32, k=8, f=1024, f_shared=1024),
    # the shared expert wider than the routed ones, d = 8192
    "d8192_E8_k2_f1024_shared2048": dict(base="glm_decode", d=8192, E=8, k=2, f=1024, f_shared=2048),
    # no shared expert, softmax router, f = 2048
    "d1024_E32_k6_f2048_softmax": dict(base="tiny", d=1024, E=32, k=6, f=2048, f_shared=0, n_shared=0,
                                       wkind=syn.W_INT4),
}


def _cfg(name, T):
    kw = dict(SHAPES[name])
    return small_config(kw.pop("base"), T=T, **kw)


_BUILT = {}


@pytest.fixture(scope="module")
def built():
    yield _BUILT
    for layer, _ in _BUILT.values():
        layer.close()
    _BUILT.clear()


def _layer(built, name):
    if name not in built:
        cfg = _cfg(name, 100)
        drawn = {}
        layer, _ = build_gpu_layer(cfg, max_tokens=100, oracle_experts=drawn)
        layer.set_single_token_mode(1)     # T = 2 too goes to the batch kernels
        built[name] = (layer, oracle_layer_from(cfg, drawn))
    return built[name]


@pytest.mark.parametrize("name", list(SHAPES))
@pytest.mark.parametrize("T", [2, 9, 40, 100])
def test_union_tensor_cores_match_oracle(built, name, T):
    cfg = _cfg(name, T)
    layer, ora = _layer(built, name)
    x = syn.gen_x(cfg, 0, T=T, token_offset=17)
    ref = ora.forward(x)
    layer.set_union_tensor_cores(True)
    out = run_forward(layer, x)
    check_close(out, ref["out"])
    for t in range(T):
        check_close(out[t:t + 1], ref["out"][t:t + 1])
    # the general kernels: the same sums in another order (h may differ by an fp16 rounding)
    layer.set_union_tensor_cores(False)
    try:
        out_g = run_forward(layer, x)
    finally:
        layer.set_union_tensor_cores(True)
    check_close(out, out_g.astype(np.float64), rel_l2=1e-4, max_rms=1e-3)


def test_union_tensor_cores_with_top_p():
    cfg = _cfg("d2048_E32_k8_f1024_shared", 24)
    layer, _ = build_gpu_layer(cfg, max_tokens=24)
    try:
        p = 0.6
        layer.set_router_top_p(p)
        x = syn.gen_x(cfg, 0, T=24, token_offset=5)
        base = oracle_layer(cfg)
        ora = oracle.Layer(cfg.d, cfg.f, cfg.E, cfg.k, cfg.router, cfg.scaling, cfg.wkind, base.router_w,
                           base.router_bias, experts=base.experts, shared=base.shared,
                           f_shared=cfg.f_shared or cfg.f, top_p=p)
        plain = base.route(x)
        share = np.cumsum(plain["w"], axis=1) / plain["w"].sum(axis=1, keepdims=True)
        assert np.abs(share - p).min() > 1e-9, "no token's kept prefix is decided by rounding"
        ref = ora.forward(x)
        assert (ref["idx"] < 0).any(), "the case must drop some experts"
        check_close(run_forward(layer, x), ref["out"])
    finally:
        layer.close()


def test_union_option_round_trips():
    cfg = _cfg("d2048_E32_k8_f1024_shared", 2)
    layer, _ = build_gpu_layer(cfg, max_tokens=2)
    try:
        import quantized_expert_ffn_02_b200 as qe
        assert qe.moe_layer_get_option(layer.handle, qe.MOE_OPT_UNION_TENSOR_CORES) == 1
        layer.set_union_tensor_cores(False)
        assert qe.moe_layer_get_option(layer.handle, qe.MOE_OPT_UNION_TENSOR_CORES) == 0
        with pytest.raises(qe.MoeError):
            qe.moe_layer_set_option(layer.handle, qe.MOE_OPT_UNION_TENSOR_CORES, 2)
    finally:
        layer.close()
