"""GPU parity of the int8 and packed int2 containers (colibri README, "What's implemented":
int8 / packed int4 / packed int2 quantisation, per-row scales, dequant-on-use).

The packers must equal the oracle's bytes and scales bit for bit; the layer over either
container must match the oracle over the same codes within the layer's tolerance (relative L2
<= 2e-3, max-abs <= 1e-2 RMS), and its expert indices must be identical.
"""
import numpy as np
import pytest
import torch

import oracle
import quantized_expert_ffn_02_b200 as qe
import synthetic as syn
from gpu_layers import build_gpu_layer, check_close, run_forward, run_route
from layers import oracle_layer, oracle_layer_from, router_only, small_config

pytestmark = pytest.mark.gpu

TIERS = {"int8": (syn.W_INT8, 8), "int2": (syn.W_INT2, 2)}


def _gpu_pack(kind, w):
    wd = torch.from_numpy(np.ascontiguousarray(w, np.float32)).cuda()
    rows, cols = w.shape
    s = torch.empty((rows,), dtype=torch.float32, device="cuda")
    if kind == "int8":
        q = torch.empty((rows, cols), dtype=torch.int8, device="cuda")
        qe.moe_pack_int8(wd, q, s)
    else:
        q = torch.empty((rows, cols // 4), dtype=torch.uint8, device="cuda")
        qe.moe_pack_int2(wd, q, s)
    return q.cpu().numpy(), s.cpu().numpy()


def _oracle_pack(kind, w):
    return oracle.quantize_tier(w, 8) if kind == "int8" else oracle.pack_int2(w)


@pytest.mark.parametrize("kind", sorted(TIERS))
@pytest.mark.parametrize("shape", [(1, 4), (3, 12), (5, 20), (7, 64), (33, 132), (300, 4096)])
def test_tier_pack_bitexact_random(kind, shape):
    rng = np.random.default_rng(shape[0] * 131 + shape[1])
    w = (rng.standard_normal(shape) * 0.02).astype(np.float32)
    w[0] = 0.0
    q, s = _gpu_pack(kind, w)
    qo, so = _oracle_pack(kind, w)
    assert np.array_equal(s.view(np.uint32), so.view(np.uint32))
    assert np.array_equal(q.view(np.uint8), qo.view(np.uint8))


@pytest.mark.parametrize("kind", sorted(TIERS))
def test_tier_pack_bitexact_glm_expert_and_ties(kind):
    cfg = syn.CONFIGS["glm_decode"]
    for which in ("gate_up", "down"):
        w = syn.gen_expert_fp32(cfg, 5, which)
        q, s = _gpu_pack(kind, w)
        qo, so = _oracle_pack(kind, w)
        assert np.array_equal(q.view(np.uint8), qo.view(np.uint8)) and np.array_equal(s, so)
    ties = np.array([[127.0, -127.0, 63.5, 0.5, -0.5, 1.5, 2.5, 0.0],
                     [3.0, 1.5, -1.5, 0.5, -3.0, 0.75, 0.0, 0.0]], np.float32)
    q, s = _gpu_pack(kind, ties)
    qo, so = _oracle_pack(kind, ties)
    assert np.array_equal(q.view(np.uint8), qo.view(np.uint8)) and np.array_equal(s, so)


@pytest.mark.parametrize("kind", sorted(TIERS))
def test_tier_pack_nonfinite_reports_range(kind):
    w = (np.random.default_rng(1).standard_normal((4, 16)) * 0.02).astype(np.float32)
    w[1, 3] = np.inf
    with pytest.raises(qe.MoeError) as ei:
        _gpu_pack(kind, w)
    assert ei.value.status == qe.MOE_ERR_RANGE


@pytest.mark.parametrize("kind", sorted(TIERS))
@pytest.mark.parametrize("T", [1, 5, 40])
def test_tier_layer_matches_oracle(kind, T):
    wkind, bits = TIERS[kind]
    cfg = small_config("glm_decode", T=T, d=256, E=16, k=4, f=128, f_shared=64, wkind=wkind)
    layer, _ = build_gpu_layer(cfg)
    try:
        x = syn.gen_x(cfg, 0, token_offset=17)
        ref = oracle_layer(cfg, bits=bits).forward(x)
        check_close(run_forward(layer, x), ref["out"])
        idx, w = run_route(layer, x, cfg.k)
        assert np.array_equal(idx, ref["idx"])
        # the tcgen05 path takes packed int4 only: the forced-GEMM option changes nothing here
        layer.set_prefill_min_tokens(1)
        check_close(run_forward(layer, x), ref["out"])
    finally:
        layer.close()


@pytest.mark.parametrize("kind", sorted(TIERS))
def test_tier_softmax_layer_without_shared_expert(kind):
    wkind, bits = TIERS[kind]
    cfg = small_config("tiny", T=7, d=192, E=8, k=2, f=64, wkind=wkind)
    layer, _ = build_gpu_layer(cfg)
    try:
        x = syn.gen_x(cfg, 0)
        check_close(run_forward(layer, x), oracle_layer(cfg, bits=bits).forward(x)["out"])
    finally:
        layer.close()


@pytest.mark.parametrize("kind", sorted(TIERS))
def test_tier_glm_decode_full_size(kind):
    """The GLM-5.2-like layer (d = 6144, E = 256, top-8 + shared, f = 2048) in the int8 or int2
    container, one token at a time and two tokens in a batch, against the oracle."""
    wkind, bits = TIERS[kind]
    cfg = small_config("glm_decode", T=2, wkind=wkind)
    xs = syn.gen_x(cfg, 0, T=3, token_offset=40)
    touched = set(router_only(cfg).route(xs)["idx"].reshape(-1).tolist())
    drawn = {}
    layer, _ = build_gpu_layer(cfg, host_experts=touched, max_tokens=2, oracle_experts=drawn)
    try:
        ora = oracle_layer_from(cfg, drawn)
        ref = ora.forward(xs)["out"]
        for t in range(3):
            check_close(run_forward(layer, xs[t:t + 1]), ref[t:t + 1])
        check_close(run_forward(layer, xs[1:3]), ref[1:3])
    finally:
        layer.close()
