"""moe_route_noalloc: routing for callers that may not allocate device memory.

Such callers (code running under CUDA-graph capture, engines that serve all device memory from
their own arena, real-time loops with no allocation after start-up) cannot create a layer, so
this entry point takes the router weights directly and keeps its scratch in a fixed array inside
the library.  Its results must equal moe_route's -- expert indices bit for bit, gate weights
within 1e-6 relative -- on consecutive calls that reuse that array.

Kept in a file of its own, collected last, so a failure here never hides the other tests; it
passes alone in a fresh process (the first call does the per-device set-up) and after them.
"""
import numpy as np
import pytest
import torch

import quantized_expert_ffn_02_b200 as qe
import synthetic as syn
from gpu_layers import x_dev

pytestmark = pytest.mark.gpu


def _router_layer(cfg, seed=0):
    """A layer whose router weights are the seeded draws; its expert tensors are never read here."""
    dev = "cuda"
    W = {"router_w": torch.from_numpy(syn.gen_router_w(cfg, seed)).to(dev)}
    b = syn.gen_router_bias(cfg, seed)
    W["router_bias"] = None if b is None else torch.from_numpy(b).to(dev)
    W["gate_up"] = torch.zeros((cfg.E, 2 * cfg.f, cfg.d // 2), dtype=torch.uint8, device=dev)
    W["gate_up_scale"] = torch.zeros((cfg.E, 2 * cfg.f), dtype=torch.float32, device=dev)
    W["down"] = torch.zeros((cfg.E, cfg.d, cfg.f // 2), dtype=torch.uint8, device=dev)
    W["down_scale"] = torch.zeros((cfg.E, cfg.d), dtype=torch.float32, device=dev)
    layer = qe.MoELayer(cfg.d, cfg.f, cfg.E, cfg.k, 512, cfg.router, syn.W_INT4, W, routed_scaling_factor=cfg.scaling)
    return layer, W


def _both(layer, W, cfg, x_bits):
    x = x_dev(x_bits)
    T = x.shape[0]
    idx_a = torch.empty((T, cfg.k), dtype=torch.int32, device="cuda")
    w_a = torch.empty((T, cfg.k), dtype=torch.float32, device="cuda")
    layer.route(x, idx_a, w_a)
    idx_b = torch.full((T, cfg.k), -1, dtype=torch.int32, device="cuda")
    w_b = torch.full((T, cfg.k), -1.0, dtype=torch.float32, device="cuda")
    qe.moe_route_noalloc(layer.cfg, W["router_w"], W["router_bias"], x, T, idx_b, w_b)
    torch.cuda.synchronize()
    return idx_a.cpu().numpy(), w_a.cpu().numpy(), idx_b.cpu().numpy(), w_b.cpu().numpy()


@pytest.mark.parametrize("name", ["glm_decode", "tiny"])
def test_noalloc_route_matches_moe_route_on_consecutive_calls(name):
    cfg = syn.CONFIGS[name]
    cfg = syn.LayerConfig(**{**cfg.__dict__, "f": 64}) if name == "glm_decode" else cfg
    layer, W = _router_layer(cfg)
    # two calls in a row, different batches: the second reuses (and must not depend on) the
    # scratch contents the first one left behind
    for T, offset in ((32, 0), (5, 777)):
        ia, wa, ib, wb = _both(layer, W, cfg, syn.gen_x(cfg, 0, T=T, token_offset=offset))
        assert np.array_equal(ia, ib)
        np.testing.assert_allclose(wb, wa, rtol=1e-6)
    layer.close()


def test_noalloc_route_long_batches_match_moe_route():
    # T >= 64 with E = 256 takes the tiled fp64 router GEMM, whose logits and sums of x land in
    # the static array at its 256-byte aligned offsets; T = 200 is not a multiple of the 64-token
    # tile and T = 510 is the largest batch the array holds
    cfg = syn.LayerConfig(**{**syn.CONFIGS["glm_decode"].__dict__, "f": 64})
    layer, W = _router_layer(cfg)
    for T, offset in ((64, 40), (200, 1234), (510, 9), (64, 40)):
        ia, wa, ib, wb = _both(layer, W, cfg, syn.gen_x(cfg, 0, T=T, token_offset=offset))
        assert np.array_equal(ia, ib), T
        np.testing.assert_allclose(wb, wa, rtol=1e-6)
    layer.close()


def test_noalloc_route_rejects_batches_beyond_its_scratch():
    cfg = syn.CONFIGS["glm_decode"]
    c = qe.moe_config(d=cfg.d, f=cfg.f, n_experts=cfg.E, top_k=cfg.k, n_shared=0, f_shared=0, max_tokens=1,
                      router=cfg.router, routed_scaling_factor=cfg.scaling, wkind=0, out_bf16=0)
    T = 511                                   # 511 * (256 * 8 + 8) bytes > 1 MiB
    x = torch.zeros((T, cfg.d), dtype=torch.int16, device="cuda")
    wr = torch.zeros((cfg.E, cfg.d), dtype=torch.float32, device="cuda")
    idx = torch.empty((T, cfg.k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, cfg.k), dtype=torch.float32, device="cuda")
    with pytest.raises(qe.MoeError) as ei:
        qe.moe_route_noalloc(c, wr, None, x, T, idx, w)
    assert ei.value.status == qe.MOE_ERR_UNSUPPORTED
    qe.moe_route_noalloc(c, wr, None, x, 510, idx, w)      # the largest batch that fits
    torch.cuda.synchronize()
