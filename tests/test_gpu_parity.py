"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the same seeded inputs.

Bars: packed bytes, scales and expert indices bit-exact (indices outside tie-ambiguous tokens,
which are counted); gate weights within 1e-6 relative; outputs (fp32 accumulation) within
relative L2 <= 2e-3 and max-abs <= 1e-2 * RMS of the oracle output.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import quantized_expert_ffn_02_b200 as qe
import synthetic as syn
from gpu_layers import build_gpu_layer, check_close, run_forward, run_route, x_dev
from layers import oracle_layer, oracle_layer_from, router_only, small_config

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------------------------------------
# K1 packer: bit-exact
# ------------------------------------------------------------------------------------------

def _gpu_pack(w: np.ndarray):
    wd = torch.from_numpy(np.ascontiguousarray(w, np.float32)).cuda()
    rows, cols = w.shape
    p = torch.empty((rows, cols // 2), dtype=torch.uint8, device="cuda")
    s = torch.empty((rows,), dtype=torch.float32, device="cuda")
    qe.moe_pack_int4(wd, p, s)
    return p.cpu().numpy(), s.cpu().numpy()


@pytest.mark.parametrize("shape", [(1, 2), (3, 6), (5, 10), (7, 64), (33, 130), (128, 1024), (300, 4096)])
def test_pack_bitexact_random(shape):
    rng = np.random.default_rng(shape[0] * 7919 + shape[1])
    w = (rng.standard_normal(shape) * 0.02).astype(np.float32)
    w[0] = 0.0                                              # a zero row
    p, s = _gpu_pack(w)
    po, so = oracle.pack_int4(w)
    assert np.array_equal(s.view(np.uint32), so.view(np.uint32))
    assert np.array_equal(p, po)


def test_pack_bitexact_ties_and_exact_multiples():
    rows = np.array([[7.0, 0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 3.5],
                     [-1.75, 1.25, 0.25, -0.5, 0, 0, 0, 0],
                     [3.0, 1.5, 0, 0, 0, 0, 0, 0],
                     [1.0, 0.5, 0, 0, 0, 0, 0, 0]], np.float32)
    p, s = _gpu_pack(rows)
    po, so = oracle.pack_int4(rows)
    assert np.array_equal(p, po) and np.array_equal(s, so)


def test_pack_bitexact_glm_expert():
    cfg = syn.CONFIGS["glm_decode"]
    for which in ("gate_up", "down"):
        w = syn.gen_expert_fp32(cfg, 3, which)
        p, s = _gpu_pack(w)
        po, so = oracle.pack_int4(w)
        assert np.array_equal(p, po) and np.array_equal(s.view(np.uint32), so.view(np.uint32))


def test_pack_nonfinite_reports_range():
    w = (np.random.default_rng(0).standard_normal((4, 16)) * 0.02).astype(np.float32)
    w[2, 5] = np.nan
    with pytest.raises(qe.MoeError) as ei:
        _gpu_pack(w)
    assert ei.value.status == qe.MOE_ERR_RANGE
    wd = torch.from_numpy(w).cuda()
    p = torch.empty((4, 8), dtype=torch.uint8, device="cuda")
    s = torch.empty((4,), dtype=torch.float32, device="cuda")
    with pytest.raises(qe.MoeError):
        qe.moe_pack_int4(wd, p, s)
    po, so = oracle.pack_int4(w, allow_nonfinite=True)
    assert np.array_equal(p.cpu().numpy(), po) and np.array_equal(s.cpu().numpy(), so)


# ------------------------------------------------------------------------------------------
# full GLM-5.2-like layer, built once; only experts that compared tokens reach are host-drawn
# ------------------------------------------------------------------------------------------

GLM = syn.CONFIGS["glm_decode"]
DECODE_TOKENS = [0, 1]                     # T = 1 calls on tokens 0 and 1 of stream x
UNION2_OFFSET = 100                        # T = 2: tokens 100, 101
UNION32_OFFSET = 200                       # T = 32: tokens 200 .. 231, every one compared
PREFILL_OFFSET = 1000                      # T = 2048: tokens 1000 .. 3047, a sample compared


def _glm_x(T, offset):
    return syn.gen_x(GLM, 0, T=T, token_offset=offset)


def prefill_sample(idx: np.ndarray, group: int = 128) -> list:
    """Tokens of the 2048-token batch that the oracle checks.

    * Two tokens of every 128-token block of the batch: the shared expert runs over the whole
      batch in blocks of 128 tokens (one GEMM column block each), so every block is checked.
    * The largest routed bucket: its first and last token and the first token of each further
      128-token block of that bucket (the routed GEMMs also split a bucket into blocks of 128).
    * Every token of the smallest non-empty routed bucket.
    """
    T = idx.shape[0]
    pick = set()
    for b in range(0, T, group):
        pick.add(b + 3)
        pick.add(min(T - 1, b + group - 5))
    cnt = np.bincount(idx.reshape(-1), minlength=GLM.E)
    big = int(np.argmax(cnt))
    toks = np.nonzero((idx == big).any(axis=1))[0]
    pick.update(int(t) for t in toks[::group])
    pick.add(int(toks[-1]))
    small = int(np.argmin(np.where(cnt > 0, cnt, np.iinfo(np.int64).max)))
    pick.update(int(t) for t in np.nonzero((idx == small).any(axis=1))[0])
    return sorted(pick)


@pytest.fixture(scope="module")
def glm():
    router = router_only(GLM)
    x32 = _glm_x(32, UNION32_OFFSET)
    xp = _glm_x(2048, PREFILL_OFFSET)
    psample = prefill_sample(router.route(xp)["idx"])
    sample_rows = [_glm_x(1, t) for t in DECODE_TOKENS] + [_glm_x(2, UNION2_OFFSET), x32, xp[psample]]
    touched = set()
    for xr in sample_rows:
        touched |= set(router.route(xr)["idx"].reshape(-1).tolist())
    drawn = {}
    layer, W = build_gpu_layer(GLM, host_experts=touched, max_tokens=2048, oracle_experts=drawn)
    ora = oracle_layer_from(GLM, drawn)
    yield {"layer": layer, "W": W, "oracle": ora, "router": router, "x32": x32, "xp": xp,
           "psample": psample, "touched": touched}
    layer.close()


@pytest.mark.parametrize("mode", [2, 1, 0])
def test_glm_decode_t1(glm, mode):
    layer = glm["layer"]
    assert layer.set_single_token_mode(mode) == mode
    try:
        for t in DECODE_TOKENS:
            x = _glm_x(1, t)
            ref = glm["oracle"].forward(x)
            out = run_forward(layer, x)
            check_close(out, ref["out"])
            if mode == 2:
                # the single launch also leaves the routing tables of its one token
                idx = np.zeros(layer.cfg.top_k, np.int32)
                layer.debug_read("idx", idx)
                assert np.array_equal(idx, ref["idx"][0])
    finally:
        layer.set_single_token_mode(2)


def test_glm_union_t2(glm):
    x = _glm_x(2, UNION2_OFFSET)
    ref = glm["oracle"].forward(x)
    check_close(run_forward(glm["layer"], x), ref["out"])


def test_glm_union_t32_every_token(glm):
    out = run_forward(glm["layer"], glm["x32"])
    ref = glm["oracle"].forward(glm["x32"])
    check_close(out, ref["out"])
    for t in range(32):                   # and token by token
        check_close(out[t:t + 1], ref["out"][t:t + 1])


def test_glm_prefill_sample_covers_every_block(glm):
    ps = glm["psample"]
    blocks = {t // 128 for t in ps}
    assert blocks == set(range(16)), "every 128-token block of the batch is sampled"
    assert len(ps) >= 32


def test_glm_prefill_t2048_sampled_and_properties(glm):
    layer = glm["layer"]
    assert layer.has_gemm_path
    out = run_forward(layer, glm["xp"])
    ps = glm["psample"]
    ref = glm["oracle"].forward(glm["xp"][ps])
    check_close(out[ps], ref["out"])
    worst = max(np.linalg.norm(out[t] - ref["out"][i]) / np.linalg.norm(ref["out"][i]) for i, t in enumerate(ps))
    assert worst <= 2e-3, worst
    # properties at full size: finite, deterministic run to run
    assert np.isfinite(out).all()
    out2 = run_forward(layer, glm["xp"])
    assert np.array_equal(out, out2)


@pytest.mark.parametrize("T,offset", [(1, 0), (2, UNION2_OFFSET), (32, UNION32_OFFSET), (2048, PREFILL_OFFSET)])
def test_glm_route_bitexact(glm, T, offset):
    x = _glm_x(T, offset)
    ref = glm["router"].route(x)
    idx, w = run_route(glm["layer"], x, GLM.k)
    keys = 1.0 / (1.0 + np.exp(-ref["logits"])) + glm["router"].router_bias.astype(np.float64)
    amb = oracle.tie_ambiguous(ref["gap"], np.abs(keys).max(axis=1))
    assert amb.sum() == 0, f"{amb.sum()} tie-ambiguous tokens"
    assert np.array_equal(idx, ref["idx"])
    np.testing.assert_allclose(w, ref["w"], rtol=1e-6)


def test_glm_batch_union_reads_each_expert_once_per_call(glm):
    # the union result of a batch equals the per-token results (same token, same output)
    x = glm["x32"]
    layer = glm["layer"]
    out_b = run_forward(layer, x)
    for mode, tol in ((0, 1e-4), (1, 1e-4), (2, 1e-4)):
        # every T = 1 path adds the same products in another order than the batch's tensor-core
        # kernels, and an fp16 rounding of h can flip, so the bound is 1e-4 (far inside the spec)
        assert layer.set_single_token_mode(mode) == mode
        for i in (0, 7, 31):
            out_1 = run_forward(layer, x[i:i + 1])
            check_close(out_1, out_b[i:i + 1].astype(np.float64), rel_l2=tol, max_rms=10 * tol)
    layer.set_single_token_mode(2)


# ------------------------------------------------------------------------------------------
# tiny and Granite-like layers: every token compared
# ------------------------------------------------------------------------------------------

def test_tiny_full():
    cfg = syn.CONFIGS["tiny"]
    layer, _ = build_gpu_layer(cfg)
    x = syn.gen_x(cfg, 0)
    ref = oracle_layer(cfg).forward(x)
    check_close(run_forward(layer, x), ref["out"])
    idx, w = run_route(layer, x, cfg.k)
    assert np.array_equal(idx, ref["idx"])
    np.testing.assert_allclose(w, ref["w"], rtol=1e-6)
    layer.close()


@pytest.mark.parametrize("T", [1, 2, 3])
def test_tiny_ragged_batches(T):
    cfg = syn.CONFIGS["tiny"]
    layer, _ = build_gpu_layer(cfg, max_tokens=4)
    x = syn.gen_x(cfg, 0, T=T, token_offset=11)
    check_close(run_forward(layer, x), oracle_layer(cfg).forward(x)["out"])
    layer.close()


def test_granite_1000_sequential_tokens():
    cfg = syn.CONFIGS["granite"]
    layer, _ = build_gpu_layer(cfg, max_tokens=1)
    x = syn.gen_x(cfg, 0, T=cfg.n_seq)
    xd = x_dev(x)
    out = torch.empty((cfg.n_seq, cfg.d), dtype=torch.float32, device="cuda")
    for t in range(cfg.n_seq):
        layer.forward(xd[t:t + 1], out[t:t + 1])
    torch.cuda.synchronize()
    assert layer.last_error() == qe.MOE_OK
    ref = oracle_layer(cfg).forward(x)
    check_close(out.cpu().numpy(), ref["out"])
    worst = max(np.linalg.norm(out.cpu().numpy()[t] - ref["out"][t]) / np.linalg.norm(ref["out"][t])
                for t in range(cfg.n_seq))
    assert worst < 2e-3
    layer.close()


# ------------------------------------------------------------------------------------------
# degenerate cases
# ------------------------------------------------------------------------------------------

def test_identical_tokens_share_every_bucket():
    cfg = small_config("glm_decode", T=16, d=256, E=16, k=4, f=128, f_shared=64)
    layer, _ = build_gpu_layer(cfg)
    x = np.repeat(syn.gen_x(cfg, 0, T=1), 16, axis=0)
    out = run_forward(layer, x)
    check_close(out, oracle_layer(cfg).forward(x)["out"])
    assert (out == out[0]).all()
    layer.close()


@pytest.mark.parametrize("E,k", [(4, 4), (8, 1), (1, 1), (64, 32)])
def test_extreme_topk(E, k):
    cfg = small_config("tiny", T=5, d=128, E=E, k=k, f=64)
    layer, _ = build_gpu_layer(cfg)
    x = syn.gen_x(cfg, 0)
    ref = oracle_layer(cfg).forward(x)
    check_close(run_forward(layer, x), ref["out"])
    layer.close()


def test_bf16_weights_with_shared_expert_and_sigmoid():
    cfg = small_config("glm_decode", T=9, d=192, E=12, k=3, f=64, f_shared=128, wkind=syn.W_BF16)
    layer, _ = build_gpu_layer(cfg)
    x = syn.gen_x(cfg, 0)
    check_close(run_forward(layer, x), oracle_layer(cfg).forward(x)["out"])
    layer.close()


def test_bf16_output_is_the_rounded_fp32_output():
    cfg = small_config("glm_decode", T=40, d=256, E=16, k=4, f=128, f_shared=64)
    l32, _ = build_gpu_layer(cfg)
    l16, _ = build_gpu_layer(cfg, out_bf16=True)
    x = syn.gen_x(cfg, 0)
    o32 = run_forward(l32, x)
    xd = x_dev(x)
    o16 = torch.empty((cfg.T, cfg.d), dtype=torch.int16, device="cuda")
    l16.forward(xd, o16)
    torch.cuda.synchronize()
    assert np.array_equal(o16.cpu().numpy().view(np.uint16), syn.fp32_to_bf16_bits(o32))
    l32.close()
    l16.close()


def test_zero_tokens_is_a_no_op():
    cfg = syn.CONFIGS["tiny"]
    layer, _ = build_gpu_layer(cfg)
    out = torch.full((1, cfg.d), 7.0, device="cuda")
    layer.forward(torch.empty((0, cfg.d), dtype=torch.int16, device="cuda"), out)
    torch.cuda.synchronize()
    assert (out == 7.0).all()
    layer.close()


def test_forward_host_matches_device():
    cfg = small_config("glm_decode", T=8, d=256, E=16, k=4, f=128, f_shared=64)
    layer, _ = build_gpu_layer(cfg)
    x = syn.gen_x(cfg, 0)
    dev_out = run_forward(layer, x)
    xh = torch.from_numpy(x.view(np.int16)).pin_memory()
    oh = torch.empty((cfg.T, cfg.d), dtype=torch.float32).pin_memory()
    layer.forward_host(xh, oh)
    assert np.array_equal(oh.numpy(), dev_out)
    # the asynchronous form: several calls in a row on one stream, one wait at the end; each
    # call's output lands in its own pinned buffer, in stream order
    outs = [torch.empty((cfg.T, cfg.d), dtype=torch.float32).pin_memory() for _ in range(3)]
    xs = [xh, torch.from_numpy(x[::-1].copy().view(np.int16)).pin_memory(), xh]
    for xi, oi in zip(xs, outs):
        layer.forward_host_async(xi, oi)
    torch.cuda.synchronize()
    assert layer.last_error() == 0
    assert np.array_equal(outs[0].numpy(), dev_out)
    assert np.array_equal(outs[2].numpy(), dev_out)
    assert np.array_equal(outs[1].numpy(), run_forward(layer, x[::-1].copy()))
    # an output in ordinary (pageable) host memory goes through the staging buffer and a copy;
    # a pinned one is written in place by the kernels: the same values either way
    op = torch.empty((cfg.T, cfg.d), dtype=torch.float32)
    assert not op.is_pinned()
    layer.forward_host(xh, op)
    assert np.array_equal(op.numpy(), dev_out)
    layer.close()


def test_argument_errors():
    cfg = syn.CONFIGS["tiny"]
    layer, W = build_gpu_layer(cfg)
    x = x_dev(syn.gen_x(cfg, 0))
    out = torch.empty((cfg.T, cfg.d), device="cuda")
    with pytest.raises(qe.MoeError) as ei:
        qe.moe_forward(layer.handle, x, cfg.T + 1, out)           # T > max_tokens
    assert ei.value.status == qe.MOE_ERR_INVALID_ARG
    with pytest.raises(qe.MoeError):
        qe.moe_forward(layer.handle, x, -1, out)
    big = torch.empty(2 * cfg.T * cfg.d + 8, dtype=torch.int16, device="cuda")
    rc = qe.load().moe_forward(layer.handle, big.data_ptr() + 2, cfg.T, out.data_ptr(), None)
    assert rc == qe.MOE_ERR_INVALID_ARG                           # misaligned activations
    c = qe.moe_config(d=100, f=128, n_experts=8, top_k=2, n_shared=0, f_shared=0, max_tokens=4, router=0,
                      routed_scaling_factor=1.0, wkind=0, out_bf16=0)
    with pytest.raises(qe.MoeError) as ei:
        qe.moe_layer_create(c, layer.w)                           # d not a multiple of 64
    assert ei.value.status == qe.MOE_ERR_INVALID_ARG
    assert layer.last_error() == qe.MOE_OK
    layer.close()
