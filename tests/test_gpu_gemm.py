"""GPU parity of the tcgen05 grouped-GEMM path (the expert FFN for large batches).

The path is forced on (or off) with MOE_OPT_PREFILL_MIN_TOKENS so that small layers, which the
oracle evaluates in a moment, cover ragged groups, experts with more than 128 tokens, a shared
expert of a different width, and batches smaller than one MMA column block.
"""
import numpy as np
import pytest

import synthetic as syn
from gpu_layers import build_gpu_layer, check_close, run_forward
from layers import oracle_layer, small_config

pytestmark = pytest.mark.gpu

ALWAYS, NEVER = 1, 1 << 30


def _both_paths(cfg, x, max_tokens=None):
    layer, _ = build_gpu_layer(cfg, max_tokens=max_tokens or x.shape[0])
    assert layer.has_gemm_path
    layer.set_prefill_min_tokens(ALWAYS)
    gemm = run_forward(layer, x)
    gemm2 = run_forward(layer, x)
    layer.set_prefill_min_tokens(NEVER)
    dec = run_forward(layer, x)
    layer.close()
    assert np.array_equal(gemm, gemm2), "grouped-GEMM path is not deterministic"
    return gemm, dec


@pytest.mark.parametrize("T", [300, 17, 1])
def test_gemm_sigmoid_shared(T):
    cfg = small_config("glm_decode", T=T, d=256, E=16, k=4, f=128, f_shared=128)
    x = syn.gen_x(cfg, 0, token_offset=5)
    gemm, dec = _both_paths(cfg, x)
    ref = oracle_layer(cfg).forward(x)["out"]
    check_close(gemm, ref)
    check_close(dec, ref)


def test_gemm_softmax_no_shared():
    cfg = small_config("tiny", T=200, d=256, E=8, k=2, f=128)
    x = syn.gen_x(cfg, 0)
    gemm, _ = _both_paths(cfg, x)
    check_close(gemm, oracle_layer(cfg).forward(x)["out"])


def test_gemm_experts_with_more_than_128_tokens():
    # identical tokens: the chosen experts' buckets hold every token (3 groups of <= 128)
    cfg = small_config("glm_decode", T=300, d=256, E=16, k=4, f=128, f_shared=128)
    x = np.repeat(syn.gen_x(cfg, 0, T=1, token_offset=9), cfg.T, axis=0)
    gemm, dec = _both_paths(cfg, x)
    check_close(gemm, oracle_layer(cfg).forward(x[:1])["out"].repeat(cfg.T, axis=0))
    assert (gemm == gemm[0]).all()


def test_gemm_wider_layer_shared_expert_of_other_width():
    cfg = small_config("glm_decode", T=500, d=1024, E=16, k=4, f=256, f_shared=384)
    x = syn.gen_x(cfg, 0)
    gemm, dec = _both_paths(cfg, x)
    ref = oracle_layer(cfg).forward(x)["out"]
    check_close(gemm, ref)
    check_close(dec, ref)


def test_gemm_bf16_output():
    cfg = small_config("glm_decode", T=260, d=256, E=16, k=4, f=128, f_shared=128)
    x = syn.gen_x(cfg, 0)
    l32, _ = build_gpu_layer(cfg)
    l16, _ = build_gpu_layer(cfg, out_bf16=True)
    for L in (l32, l16):
        L.set_prefill_min_tokens(ALWAYS)
    o32 = run_forward(l32, x)
    o16 = run_forward(l16, x, out_bf16=True)
    assert np.array_equal(syn.fp32_to_bf16_bits(o16), syn.fp32_to_bf16_bits(o32))
    check_close(o32, oracle_layer(cfg).forward(x)["out"])
    l32.close()
    l16.close()
