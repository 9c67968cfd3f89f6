"""Error paths of the layer on the GPU, made on the host side: no kernel faults, traps or hangs.

* A bounded device wait that runs out.  The test hook MOE_OPT_TEST_SKIP_GEMM_B_COPIES makes the
  grouped-GEMM kernels' activation-tile producer issue nothing, so the MMA warp's wait for those
  tiles can only end at its time limit (shortened to 1 ms with MOE_OPT_WAIT_LIMIT_US).  Every other
  waiter of the CTA gives up through the CTA's abort flag within the same limit.  The forward must
  report MOE_ERR_TIMEOUT through moe_last_error, and the next normal forward must be correct.
* A workspace allocation that fails.  A layer whose max_tokens needs more device memory than the
  GPU has must return MOE_ERR_OOM, leave no device memory behind, and leave the device usable.
"""
import numpy as np
import pytest
import torch

import quantized_expert_ffn_02_b200 as qe
import synthetic as syn
from gpu_layers import build_gpu_layer, check_close, run_forward, x_dev
from layers import oracle_layer, small_config

pytestmark = pytest.mark.gpu


def test_gemm_wait_limit_reports_timeout_and_the_layer_recovers():
    cfg = small_config("glm_decode", T=40, d=256, E=16, k=4, f=128, f_shared=128)
    layer, _ = build_gpu_layer(cfg)
    try:
        assert layer.has_gemm_path
        layer.set_prefill_min_tokens(1)
        x = syn.gen_x(cfg, 0, token_offset=3)
        ref = oracle_layer(cfg).forward(x)["out"]
        check_close(run_forward(layer, x), ref)

        qe.moe_layer_set_option(layer.handle, qe.MOE_OPT_WAIT_LIMIT_US, 1000)
        assert qe.moe_layer_get_option(layer.handle, qe.MOE_OPT_WAIT_LIMIT_US) == 1000
        qe.moe_layer_set_option(layer.handle, qe.MOE_OPT_TEST_SKIP_GEMM_B_COPIES, 1)
        out = torch.empty((cfg.T, cfg.d), dtype=torch.float32, device="cuda")
        layer.forward(x_dev(x), out)
        assert layer.last_error() == qe.MOE_ERR_TIMEOUT
        assert layer.last_error() == qe.MOE_OK            # reading the status clears it

        qe.moe_layer_set_option(layer.handle, qe.MOE_OPT_TEST_SKIP_GEMM_B_COPIES, 0)
        qe.moe_layer_set_option(layer.handle, qe.MOE_OPT_WAIT_LIMIT_US, 2_000_000)
        again = run_forward(layer, x)                     # asserts MOE_OK itself
        check_close(again, ref)
    finally:
        layer.close()


def test_wait_limit_option_rejects_out_of_range_values():
    cfg = small_config("glm_decode", T=4, d=256, E=16, k=4, f=128, f_shared=128)
    layer, _ = build_gpu_layer(cfg)
    try:
        for bad in (0, 99, 10_000_001):
            with pytest.raises(qe.MoeError) as ei:
                qe.moe_layer_set_option(layer.handle, qe.MOE_OPT_WAIT_LIMIT_US, bad)
            assert ei.value.status == qe.MOE_ERR_INVALID_ARG
        with pytest.raises(qe.MoeError):
            qe.moe_layer_set_option(layer.handle, qe.MOE_OPT_TEST_SKIP_GEMM_B_COPIES, 2)
    finally:
        layer.close()


def test_workspace_allocation_failure_returns_oom_and_leaks_nothing():
    cfg = syn.CONFIGS["tiny"]
    layer, W = build_gpu_layer(cfg)
    try:
        torch.cuda.synchronize()
        free0, total = torch.cuda.mem_get_info()
        # 100 M tokens: the per-slot expert outputs alone are 100e6 * 2 * 256 * 4 B = 205 GB,
        # more than any B200 holds
        big = qe.moe_config(d=cfg.d, f=cfg.f, n_experts=cfg.E, top_k=cfg.k, n_shared=0, f_shared=0,
                            max_tokens=100_000_000, router=cfg.router, routed_scaling_factor=1.0,
                            wkind=cfg.wkind, out_bf16=0)
        assert 100_000_000 * 2 * cfg.d * 4 > total
        for _ in range(3):
            with pytest.raises(qe.MoeError) as ei:
                qe.moe_layer_create(big, layer.w)
            assert ei.value.status == qe.MOE_ERR_OOM
        torch.cuda.synchronize()
        free1, _ = torch.cuda.mem_get_info()
        assert abs(free1 - free0) < (64 << 20), (free0, free1)
        # the device is still usable and the existing layer still correct
        x = syn.gen_x(cfg, 0)
        check_close(run_forward(layer, x), oracle_layer(cfg).forward(x)["out"])
    finally:
        layer.close()
