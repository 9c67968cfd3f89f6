"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each test names the passage (page and section) or the mathematical fact that fixes the
expected value.  A plausible slip anywhere in the oracle -- a swapped nibble, a transposed
matrix, the gate and up halves exchanged, a dropped shared expert, the bias leaking into the
gate weights, a wrong tie-break -- fails at least one of these.
"""
import itertools
import json
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle
import synthetic as syn
from layers import oracle_layer, router_only, small_config

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as fh:
        return json.load(fh)


# ------------------------------------------------------------------------------------------
# P1 / P2: the packed int4 container (colibri README, "What's implemented")
# ------------------------------------------------------------------------------------------

def test_nibble_layout_golden():
    g = _golden("int4_container.json")["nibble_bytes"]["cases"]
    packed = np.array([[c["byte"]] for c in g], np.uint8)
    q = oracle.unpack_int4(packed, 2)
    assert q[:, 0].tolist() == [c["lo"] for c in g]
    assert q[:, 1].tolist() == [c["hi"] for c in g]


def test_unpack_is_exhaustive_and_pack_inverts_it():
    # every byte value: unpack gives two codes in [-8, 7]; re-quantising a row whose largest
    # magnitude is 7 (scale 1) reproduces the byte whenever neither code is -8
    packed = np.arange(256, dtype=np.uint8).reshape(256, 1)
    q = oracle.unpack_int4(packed, 2)
    assert q.min() == -8 and q.max() == 7
    assert len({(a, b) for a, b in q.tolist()}) == 256
    keep = (q != -8).all(axis=1)
    rows = np.concatenate([q[keep].astype(np.float32), np.full((keep.sum(), 2), [7.0, 0.0], np.float32)], 1)
    p, s = oracle.pack_int4(rows)
    assert (s == 1.0).all()
    assert (p[:, 0] == packed[keep, 0]).all()


def test_quantiser_golden_rows():
    for case in _golden("int4_container.json")["quantiser_rows"]["cases"]:
        w = np.array([case["w"]], np.float32)
        if w.shape[1] % 2:
            w = np.concatenate([w, np.zeros((1, 1), np.float32)], 1)
        q, s = oracle.quantize_int8(w)
        assert s[0] == np.float32(case["scale"]), case
        assert q[0, :len(case["q"])].tolist() == case["q"], case
        p, s4 = oracle.pack_int4(w)
        assert s4[0] == s[0]
        assert (oracle.unpack_int4(p, w.shape[1]) == q).all()


def test_nonfinite_is_rejected():
    w = np.array([[1.0, np.nan, 0.5, 0.25]], np.float32)
    with pytest.raises(RuntimeError):
        oracle.pack_int4(w)
    w = np.array([[1.0, np.inf, 0.5, 0.25]], np.float32)
    with pytest.raises(RuntimeError):
        oracle.quantize_int8(w)


@pytest.mark.parametrize("shape", [(1, 2), (7, 64), (33, 130), (128, 1024)])
def test_int4_packing_bit_identical_to_int8_container(shape):
    rng = np.random.default_rng(sum(shape))
    w = (rng.standard_normal(shape) * 0.02).astype(np.float32)
    q8, s8 = oracle.quantize_int8(w)
    p, s4 = oracle.pack_int4(w)
    assert (s4 == s8).all()
    assert (oracle.unpack_int4(p, shape[1]) == q8).all()
    assert q8.min() >= -7 and q8.max() <= 7        # |w/s| <= 7 up to rounding: -8 is never produced
    # a row's scale is the fp32 quotient max|w| / 7
    m = np.abs(w).max(axis=1)
    assert (s8 == (m / np.float32(7.0)).astype(np.float32)).all()


def test_int8_container_forward_equals_int4_forward_bitwise():
    cfg = small_config("glm_decode", T=6, d=128, E=8, k=3, f=64, f_shared=32)
    x = syn.gen_x(cfg, 0)
    a = oracle_layer(cfg, wkind=oracle.W_INT4).forward(x)["out"]
    b = oracle_layer(cfg, wkind=oracle.W_INT8).forward(x)["out"]
    assert np.array_equal(a, b)


def test_page_sizes_pin_the_container_layout():
    """fp32 per-row scales and two nibbles per byte reproduce the sizes the pages print."""
    g = _golden("page_sizes.json")
    d, f = 6144, 2048
    gu, gu_s = oracle.pack_int4(np.zeros((2 * f, d), np.float32))
    dn, dn_s = oracle.pack_int4(np.zeros((d, f), np.float32))
    nibble_bytes = gu.nbytes + dn.nbytes
    scale_bytes = gu_s.nbytes + dn_s.nbytes
    total = nibble_bytes + scale_bytes
    assert nibble_bytes == 18_874_368 and scale_bytes == 40_960 and total == 18_915_328
    assert abs(total / 1e6 - g["expert_mb_approx"]["value"]) <= g["expert_mb_approx"]["rel_tol"] * 19.0
    assert abs(100.0 * scale_bytes / nibble_bytes - g["scale_share_pct"]["value"]) <= g["scale_share_pct"]["abs_tol"]
    c = g["cold_token_gb"]
    assert abs(c["layers"] * c["experts_per_token"] * total / 1e9 - c["value"]) <= c["rel_tol"] * c["value"]
    h = g["hot_store"]
    assert abs(h["experts"] * total / 1e9 - h["gb"]) <= h["rel_tol"] * h["gb"]
    dk = g["disk_gb_approx"]
    assert abs(dk["experts"] * total / 1e9 - dk["value"]) <= dk["rel_tol"] * dk["value"]


# ------------------------------------------------------------------------------------------
# Router (Glacial "What works"; colibri README "What's implemented")
# ------------------------------------------------------------------------------------------

def test_logits_equal_library_matmul():
    cfg = syn.CONFIGS["tiny"]
    L = router_only(cfg)
    x = syn.gen_x(cfg, 0)
    r = L.route(x)
    ref = syn.bf16_bits_to_fp32(x).astype(np.float64) @ L.router_w.astype(np.float64).T
    np.testing.assert_allclose(r["logits"], ref, rtol=1e-13, atol=1e-15)


def _brute_topk(keys, k):
    """Largest-sum subset of size k; equal sums go to the lexicographically smallest index set."""
    best = None
    for sub in itertools.combinations(range(len(keys)), k):
        s = sum(keys[i] for i in sub)
        if best is None or s > best[0]:
            best = (s, sub)
    return set(best[1])


def _rank_order(keys, chosen):
    return sorted(chosen, key=lambda e: (-keys[e], e))


@pytest.mark.parametrize("cfg_name,T", [("tiny", 4), ("tiny", 64)])
def test_topk_brute_force_tiny(cfg_name, T):
    cfg = syn.CONFIGS[cfg_name]
    L = router_only(cfg)
    x = syn.gen_x(cfg, 0, T=T)
    r = L.route(x)
    for t in range(T):
        keys = r["logits"][t].tolist()
        chosen = _brute_topk(keys, cfg.k)
        assert set(r["idx"][t].tolist()) == chosen
        assert r["idx"][t].tolist() == _rank_order(keys, chosen)
        # rank-count formulation: rank_e = #{j : key_j > key_e or (key_j == key_e and j < e)}
        rank = [sum(1 for j in range(cfg.E) if keys[j] > keys[e] or (keys[j] == keys[e] and j < e))
                for e in range(cfg.E)]
        assert {e for e in range(cfg.E) if rank[e] < cfg.k} == chosen


def test_topk_sigmoid_brute_force_with_bias():
    cfg = small_config("glm_decode", d=64, E=10, k=3)
    L = router_only(cfg)
    x = syn.gen_x(cfg, 0, T=40)
    r = L.route(x)
    bias = L.router_bias.astype(np.float64)
    for t in range(40):
        keys = (scipy.special.expit(r["logits"][t]) + bias).tolist()
        chosen = _brute_topk(keys, cfg.k)
        assert r["idx"][t].tolist() == _rank_order(keys, chosen)


def test_exact_ties_go_to_lower_index():
    # two identical router rows give bit-identical logits; the lower index must win
    d, E, k = 16, 6, 3
    wr = np.zeros((E, d), np.float32)
    wr[:, 0] = [0.5, 2.0, 1.0, 2.0, 1.0, -1.0]      # experts 1 and 3 tie; 2 and 4 tie
    x = syn.fp32_to_bf16_bits(np.ones((1, d), np.float32))
    L = oracle.Layer(d, 8, E, k, oracle.ROUTER_SOFTMAX, 1.0, oracle.W_BF16, wr)
    r = L.route(x)
    assert r["idx"][0].tolist() == [1, 3, 2]
    assert r["gap"][0] == 0.0                        # expert 4 ties with the last chosen one


def test_gate_weights_closed_forms():
    cfg = small_config("glm_decode", d=64, E=12, k=4)
    x = syn.gen_x(cfg, 0, T=16)
    r = router_only(cfg).route(x)
    np.testing.assert_allclose(r["w"].sum(1), 2.5, rtol=1e-13)
    # weights are 2.5 * sigmoid / sum(sigmoid) of the chosen logits: the bias does not enter
    sig = scipy.special.expit(np.take_along_axis(r["logits"], r["idx"], 1))
    np.testing.assert_allclose(r["w"], 2.5 * sig / sig.sum(1, keepdims=True), rtol=1e-13)

    tiny = syn.CONFIGS["tiny"]                                    # k < E: softmax over the chosen k
    rt = router_only(tiny).route(syn.gen_x(tiny, 0, T=32))
    np.testing.assert_allclose(rt["w"].sum(1), 1.0, rtol=1e-13)
    chosen = np.take_along_axis(rt["logits"], rt["idx"], 1)
    np.testing.assert_allclose(rt["w"], scipy.special.softmax(chosen, axis=1), rtol=1e-12)

    soft = small_config("tiny", E=8, k=8)
    rs = router_only(soft).route(syn.gen_x(soft, 0, T=8))
    np.testing.assert_allclose(rs["w"].sum(1), 1.0, rtol=1e-13)
    full = scipy.special.softmax(rs["logits"], axis=1)          # k == E: a full softmax
    np.testing.assert_allclose(rs["w"], np.take_along_axis(full, rs["idx"], 1), rtol=1e-12)


def test_bias_changes_selection_not_weights():
    d, E, k = 8, 4, 2
    wr = np.zeros((E, d), np.float32)
    wr[:, 0] = [0.4, 0.3, 0.2, 0.1]
    x = syn.fp32_to_bf16_bits(np.ones((1, d), np.float32))
    bias = np.array([0.0, 0.0, 0.0, 0.5], np.float32)
    L = oracle.Layer(d, 8, E, k, oracle.ROUTER_SIGMOID, 2.5, oracle.W_BF16, wr, bias)
    r = L.route(x)
    assert r["idx"][0].tolist() == [3, 0]
    s = scipy.special.expit(np.array([0.1, 0.4], np.float64) * np.float64(1.0))
    s = scipy.special.expit(np.array([np.float32(0.1), np.float32(0.4)], np.float64))
    np.testing.assert_allclose(r["w"][0], 2.5 * s / s.sum(), rtol=1e-14)


# ------------------------------------------------------------------------------------------
# Expert FFN: textbook SwiGLU reduction and exact-arithmetic case
# ------------------------------------------------------------------------------------------

def _dense(layer, e, which, f):
    ex = layer.shared if e == "shared" else layer.experts[e]
    a = ex[which]
    if layer.wkind == oracle.W_BF16:
        return syn.bf16_bits_to_fp32(a).astype(np.float64)
    cols = layer.d if which == "gate_up" else f
    q = oracle.unpack_int4(a, cols) if layer.wkind == oracle.W_INT4 else a
    return q.astype(np.float64) * ex[which + "_scale"].astype(np.float64)[:, None]


@pytest.mark.parametrize("wkind", [oracle.W_INT4, oracle.W_BF16])
def test_single_expert_layer_is_textbook_swiglu(wkind):
    """E = 1, k = 1, no shared expert, softmax (weight 1): the layer is one SwiGLU MLP,
    down(silu(gate(x)) * up(x)), evaluated here with torch's fp64 matmul and silu."""
    cfg = small_config("tiny", T=5, d=96, E=1, k=1, f=40, wkind=wkind)
    L = oracle_layer(cfg)
    x = syn.gen_x(cfg, 0)
    out = L.forward(x)["out"]
    wgu = torch.from_numpy(_dense(L, 0, "gate_up", cfg.f))
    wd = torch.from_numpy(_dense(L, 0, "down", cfg.f))
    xt = torch.from_numpy(syn.bf16_bits_to_fp32(x).astype(np.float64))
    gate, up = wgu[:cfg.f], wgu[cfg.f:]
    ref = (torch.nn.functional.silu(xt @ gate.T) * (xt @ up.T)) @ wd.T
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-11, atol=1e-13)


def test_shared_expert_adds_with_weight_one():
    cfg = small_config("glm_decode", T=3, d=64, E=6, k=2, f=32, f_shared=48)
    L = oracle_layer(cfg)
    x = syn.gen_x(cfg, 0)
    fw = L.forward(x)
    for t in range(cfg.T):
        ys = L.expert_ffn("shared", x[t])["y"]
        routed = sum(w * L.expert_ffn(int(e), x[t])["y"] for e, w in sorted(zip(fw["idx"][t], fw["w"][t])))
        np.testing.assert_allclose(fw["out"][t], routed + ys, rtol=1e-13, atol=1e-15)
        # the shared expert is a SwiGLU with its own width
        wgu = _dense(L, "shared", "gate_up", cfg.f_shared)
        wd = _dense(L, "shared", "down", cfg.f_shared)
        xv = syn.bf16_bits_to_fp32(x[t]).astype(np.float64)
        g, u = wgu[:cfg.f_shared] @ xv, wgu[cfg.f_shared:] @ xv
        np.testing.assert_allclose(ys, wd @ (scipy.special.expit(g) * g * u), rtol=1e-11, atol=1e-13)


def test_exact_integer_case():
    """Small-integer x, power-of-two scales and small-integer codes: g and u are exact integers
    (checked against exact int64 arithmetic); doubling every down scale doubles y exactly."""
    d, f = 32, 8
    rng = np.random.default_rng(7)
    xq = rng.integers(-3, 4, size=d)
    x = syn.fp32_to_bf16_bits(xq.astype(np.float32)).reshape(1, d)
    qgu = rng.integers(-7, 8, size=(2 * f, d)).astype(np.float32)
    qgu[:, 0] = 7                                    # every row's max |w| is 7 * scale
    qd = rng.integers(-7, 8, size=(d, f)).astype(np.float32)
    qd[:, 0] = -7
    sg, sd = 0.25, 0.125
    gu_p, gu_s = oracle.pack_int4(qgu * sg)
    dn_p, dn_s = oracle.pack_int4(qd * sd)
    assert (gu_s == sg).all() and (dn_s == sd).all()
    ex = {"gate_up": gu_p, "gate_up_scale": gu_s, "down": dn_p, "down_scale": dn_s}
    L = oracle.Layer(d, f, 1, 1, oracle.ROUTER_SOFTMAX, 1.0, oracle.W_INT4, np.zeros((1, d), np.float32),
                     experts={0: ex})
    r = L.expert_ffn(0, x[0])
    gu_exact = (qgu.astype(np.int64) @ xq.astype(np.int64))
    assert np.array_equal(r["g"], gu_exact[:f] * sg)
    assert np.array_equal(r["u"], gu_exact[f:] * sg)
    ex2 = dict(ex, down_scale=(dn_s * 2).astype(np.float32))
    L2 = oracle.Layer(d, f, 1, 1, oracle.ROUTER_SOFTMAX, 1.0, oracle.W_INT4, np.zeros((1, d), np.float32),
                      experts={0: ex2})
    assert np.array_equal(L2.expert_ffn(0, x[0])["y"], 2.0 * r["y"])


# ------------------------------------------------------------------------------------------
# Batch-union and the dense identity (colibri README, "What's implemented": batch-union MoE)
# ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("T", [2, 32, 2048])
def test_batch_union_equals_per_token_bitwise(T):
    cfg = small_config("glm_decode", T=T, d=64, E=16, k=4, f=32, f_shared=32)
    L = oracle_layer(cfg)
    x = syn.gen_x(cfg, 0)
    a = L.forward(x, oracle.MODE_PER_TOKEN)
    b = L.forward(x, oracle.MODE_UNION)
    assert np.array_equal(a["out"], b["out"])
    assert np.array_equal(a["idx"], b["idx"])


def test_batch_union_bf16_softmax_bitwise():
    cfg = small_config("granite", T=24, d=64, E=8, k=3, f=16)
    L = oracle_layer(cfg)
    x = syn.gen_x(cfg, 0)
    assert np.array_equal(L.forward(x, oracle.MODE_PER_TOKEN)["out"], L.forward(x, oracle.MODE_UNION)["out"])


@pytest.mark.parametrize("base", ["glm_decode", "tiny", "granite"])
def test_dense_sum_with_zero_gates_equals_routed_bitwise(base):
    """T = 1: summing all E experts in ascending order with the unchosen gates set to 0 gives the
    routed output exactly (adding +0 * y changes nothing)."""
    cfg = small_config(base, T=1, d=64, E=8, k=2, f=16, f_shared=16 if base == "glm_decode" else 0)
    L = oracle_layer(cfg)
    for seed_tok in range(3):
        x = syn.gen_x(cfg, 0, T=1, token_offset=seed_tok)
        assert np.array_equal(L.forward(x, oracle.MODE_PER_TOKEN)["out"], L.forward(x, oracle.MODE_DENSE)["out"])


def test_missing_shared_expert_changes_the_output():
    cfg = small_config("glm_decode", T=2, d=64, E=6, k=2, f=16, f_shared=16)
    L = oracle_layer(cfg)
    x = syn.gen_x(cfg, 0)
    no_shared = oracle.Layer(cfg.d, cfg.f, cfg.E, cfg.k, cfg.router, cfg.scaling, cfg.wkind, L.router_w,
                             L.router_bias, experts=L.experts)
    assert not np.allclose(L.forward(x)["out"], no_shared.forward(x)["out"])


# ------------------------------------------------------------------------------------------
# Symmetries
# ------------------------------------------------------------------------------------------

def test_token_permutation_permutes_outputs():
    cfg = small_config("glm_decode", T=9, d=64, E=8, k=2, f=16, f_shared=16)
    L = oracle_layer(cfg)
    x = syn.gen_x(cfg, 0)
    perm = np.random.default_rng(1).permutation(cfg.T)
    a = L.forward(x)["out"]
    b = L.forward(x[perm])["out"]
    assert np.array_equal(a[perm], b)


def test_expert_relabelling_permutes_indices_only():
    cfg = small_config("glm_decode", T=7, d=64, E=8, k=3, f=16, f_shared=16)
    L = oracle_layer(cfg)
    x = syn.gen_x(cfg, 0)
    pi = np.random.default_rng(3).permutation(cfg.E)      # new label of old expert e is pi[e]
    inv = np.argsort(pi)
    L2 = oracle.Layer(cfg.d, cfg.f, cfg.E, cfg.k, cfg.router, cfg.scaling, cfg.wkind,
                      L.router_w[inv], L.router_bias[inv],
                      experts={int(pi[e]): L.experts[e] for e in range(cfg.E)}, shared=L.shared,
                      f_shared=cfg.f_shared)
    a, b = L.forward(x), L2.forward(x)
    np.testing.assert_allclose(a["out"], b["out"], rtol=1e-12, atol=1e-14)
    assert np.array_equal(pi[a["idx"]], b["idx"])


def test_missing_expert_is_reported():
    cfg = small_config("glm_decode", T=4, d=64, E=8, k=2, f=16, f_shared=16)
    L = oracle_layer(cfg, experts=[0])
    with pytest.raises(RuntimeError):
        L.forward(syn.gen_x(cfg, 0))


# ------------------------------------------------------------------------------------------
# The int8 and packed int2 containers (colibri README, "What's implemented": int8 / packed
# int4 / packed int2 quantisation, per-row scales, bit-identical to the int8 container)
# ------------------------------------------------------------------------------------------

def _crumbs(byte_values):
    """2-bit two's-complement codes of each byte, lowest bits first (the golden layout rule)."""
    b = np.asarray(byte_values, np.int64)
    c = np.stack([(b >> (2 * i)) & 3 for i in range(4)], axis=-1)
    return np.where(c >= 2, c - 4, c)


def test_int2_crumb_layout_golden():
    cases = _golden("int2_int8_tiers.json")["crumb_bytes"]["cases"]
    packed = np.array([[c["byte"]] for c in cases], np.uint8)
    q = oracle.unpack_int2(packed, 4)
    assert q.tolist() == [c["codes"] for c in cases]


def test_int2_unpack_is_exhaustive_and_pack_inverts_it():
    packed = np.arange(256, dtype=np.uint8).reshape(256, 1)
    q = oracle.unpack_int2(packed, 4)
    assert np.array_equal(q, _crumbs(np.arange(256)))
    assert q.min() == -2 and q.max() == 1 and len({tuple(r) for r in q.tolist()}) == 256
    # re-quantising a row whose largest magnitude is 1 (scale 1) reproduces the byte whenever
    # no code is -2 (the tier's rule never produces -2: |w / s| <= 1)
    keep = (q != -2).all(axis=1)
    rows = np.concatenate([q[keep].astype(np.float32), np.full((keep.sum(), 4), [1.0, 0, 0, 0], np.float32)], 1)
    p, s = oracle.pack_int2(rows)
    assert (s == 1.0).all()
    assert (p[:, 0] == packed[keep, 0]).all() and (p[:, 1] == 1).all()


@pytest.mark.parametrize("tier", ["int2_rows", "int8_rows"])
def test_tier_quantiser_golden_rows(tier):
    g = _golden("int2_int8_tiers.json")[tier]
    bits = 2 if tier == "int2_rows" else 8
    for case in g["cases"]:
        w = np.array([case["w"]], np.float32)
        q, s = oracle.quantize_tier(w, bits)
        assert s[0] == np.float32(case["scale"]), case
        assert q[0].tolist() == case["q"], case
    for pk in g.get("packed", []):
        w = np.array([g["cases"][pk["row"]]["w"]], np.float32)
        p, _ = oracle.pack_int2(w)
        assert p[0].tolist() == pk["bytes"], pk


@pytest.mark.parametrize("shape", [(1, 4), (7, 64), (33, 132), (128, 1024)])
def test_int2_packing_bit_identical_to_int8_container(shape):
    rng = np.random.default_rng(sum(shape) + 2)
    w = (rng.standard_normal(shape) * 0.02).astype(np.float32)
    q8, s8 = oracle.quantize_tier(w, 2)
    p, s2 = oracle.pack_int2(w)
    assert (s2 == s8).all()
    assert np.array_equal(oracle.unpack_int2(p, shape[1]), q8)
    assert np.array_equal(_crumbs(p).reshape(shape), q8)         # the layout rule, decoded independently
    assert q8.min() >= -1 and q8.max() <= 1
    assert (s8 == np.abs(w).max(axis=1)).all()                     # scale = max|w| / 1


def test_int4_tier_of_the_general_quantiser_is_the_int4_container_rule():
    rng = np.random.default_rng(5)
    w = (rng.standard_normal((40, 96)) * 0.02).astype(np.float32)
    q4, s4 = oracle.quantize_int8(w)
    q, s = oracle.quantize_tier(w, 4)
    assert np.array_equal(q, q4) and np.array_equal(s, s4)


def test_int8_tier_scale_and_range():
    rng = np.random.default_rng(6)
    w = (rng.standard_normal((40, 96)) * 0.02).astype(np.float32)
    q, s = oracle.quantize_tier(w, 8)
    assert (s == (np.abs(w).max(axis=1) / np.float32(127.0)).astype(np.float32)).all()
    assert q.min() >= -127 and q.max() <= 127
    assert (np.abs(q).max(axis=1) == 127).all()                   # the largest magnitude reaches qmax
    # codes times scales reproduce w to within half a scale step
    assert (np.abs(q * s[:, None].astype(np.float64) - w) <= 0.5 * s[:, None] * (1 + 1e-6)).all()


def test_int2_container_forward_equals_int8_container_forward_bitwise():
    """The packed int2 container and the int8 container holding the same int2-tier codes and
    scales give the same layer output bit for bit (only the storage differs)."""
    cfg = small_config("glm_decode", T=6, d=128, E=8, k=3, f=64, f_shared=32)
    x = syn.gen_x(cfg, 0)
    a = oracle_layer(cfg, wkind=oracle.W_INT2).forward(x)["out"]
    b = oracle_layer(cfg, wkind=oracle.W_INT8, bits=2).forward(x)["out"]
    assert np.array_equal(a, b)


def _dense_tier(layer, e, which, f):
    """Dense fp64 weights of the int8 or packed int2 container, decoded without the oracle."""
    ex = layer.shared if e == "shared" else layer.experts[e]
    a = ex[which]
    q = _crumbs(a).reshape(a.shape[0], -1) if layer.wkind == oracle.W_INT2 else a
    return q.astype(np.float64) * ex[which + "_scale"].astype(np.float64)[:, None]


@pytest.mark.parametrize("wkind,bits", [(oracle.W_INT2, 2), (oracle.W_INT8, 8)])
def test_single_expert_layer_is_textbook_swiglu_other_tiers(wkind, bits):
    cfg = small_config("tiny", T=5, d=96, E=1, k=1, f=40, wkind=wkind)
    L = oracle_layer(cfg, bits=bits)
    x = syn.gen_x(cfg, 0)
    out = L.forward(x)["out"]
    wgu = torch.from_numpy(_dense_tier(L, 0, "gate_up", cfg.f))
    wd = torch.from_numpy(_dense_tier(L, 0, "down", cfg.f))
    xt = torch.from_numpy(syn.bf16_bits_to_fp32(x).astype(np.float64))
    gate, up = wgu[:cfg.f], wgu[cfg.f:]
    ref = (torch.nn.functional.silu(xt @ gate.T) * (xt @ up.T)) @ wd.T
    np.testing.assert_allclose(out, ref.numpy(), rtol=1e-11, atol=1e-13)


# ------------------------------------------------------------------------------------------
# Router variants (colibri README: "noaux_tc" and the "--topp" adaptive expert top-p knob)
# ------------------------------------------------------------------------------------------

def _router_with_logits(logits, k, router=oracle.ROUTER_SOFTMAX, **kw):
    """An oracle router whose logits for x = (1, 0) are exactly `logits` (fp32 values)."""
    E = len(logits)
    wr = np.zeros((E, 2), np.float32)
    wr[:, 0] = np.asarray(logits, np.float32)
    x = syn.fp32_to_bf16_bits(np.array([[1.0, 0.0]], np.float32))
    L = oracle.Layer(2, 4, E, k, router, 1.0, oracle.W_INT4, wr, **kw)
    return L, x


def test_grouped_selection_golden():
    g = _golden("router_variants.json")["grouped"]
    L, x = _router_with_logits(g["logits"], g["k"], n_group=g["n_group"], topk_group=g["topk_group"])
    r = L.route(x)
    assert r["idx"][0].tolist() == g["idx"]
    L0, _ = _router_with_logits(g["logits"], g["k"])
    assert L0.route(x)["idx"][0].tolist() == g["ungrouped_idx"]
    tie = _golden("router_variants.json")["grouped_tie"]
    Lt, xt = _router_with_logits(tie["logits"], tie["k"], n_group=tie["n_group"], topk_group=tie["topk_group"])
    assert Lt.route(xt)["idx"][0].tolist() == tie["idx"]
    # the weights are the softmax over the chosen logits, as without groups
    lg = np.array(g["logits"], np.float64)[g["idx"]]
    np.testing.assert_allclose(r["w"][0], np.exp(lg - lg.max()) / np.exp(lg - lg.max()).sum(), rtol=1e-15)


@pytest.mark.parametrize("router", [oracle.ROUTER_SOFTMAX, oracle.ROUTER_SIGMOID])
def test_grouped_selection_brute_force(router):
    """The kept groups maximise the summed group score over every topk_group-subset of groups, and
    the chosen experts maximise the summed key over every k-subset of the kept groups' experts."""
    E, G, TG, k = 16, 4, 2, 3
    base = "tiny" if router == oracle.ROUTER_SOFTMAX else "glm_decode"
    cfg = small_config(base, T=64, d=64, E=E, k=k, f=32, f_shared=32)
    L = oracle.Layer(cfg.d, cfg.f, E, k, router, cfg.scaling, cfg.wkind, syn.gen_router_w(cfg),
                     syn.gen_router_bias(cfg), n_group=G, topk_group=TG)
    x = syn.gen_x(cfg, 0)
    r = L.route(x)
    per = E // G
    for t in range(cfg.T):
        lg = r["logits"][t]
        key = lg if router == oracle.ROUTER_SOFTMAX else 1.0 / (1.0 + np.exp(-lg)) + L.router_bias.astype(np.float64)
        gscore = [sum(sorted(key[g * per:(g + 1) * per])[-2:]) for g in range(G)]
        best_groups = max(itertools.combinations(range(G), TG), key=lambda c: (sum(gscore[i] for i in c),
                                                                              [-i for i in c]))
        allowed = [e for g in best_groups for e in range(g * per, (g + 1) * per)]
        best = max(itertools.combinations(allowed, k), key=lambda c: (sum(key[i] for i in c), [-i for i in c]))
        assert sorted(r["idx"][t].tolist()) == sorted(best)
        assert set(r["idx"][t].tolist()) <= set(allowed)


def test_grouped_selection_reduces_to_plain_top_k():
    cfg = small_config("glm_decode", T=20, d=64, E=32, k=4, f=32, f_shared=32)
    args = (cfg.d, cfg.f, cfg.E, cfg.k, cfg.router, cfg.scaling, cfg.wkind, syn.gen_router_w(cfg),
            syn.gen_router_bias(cfg))
    x = syn.gen_x(cfg, 0)
    plain = oracle.Layer(*args).route(x)
    for G, TG in ((1, 1), (4, 4), (8, 8)):                 # one group, or every group kept
        v = oracle.Layer(*args, n_group=G, topk_group=TG).route(x)
        assert np.array_equal(v["idx"], plain["idx"]) and np.array_equal(v["w"], plain["w"])


def test_top_p_golden():
    g = _golden("router_variants.json")["top_p"]
    for case in g["cases"]:
        L, x = _router_with_logits(g["logits"], g["k"], top_p=case["p"])
        r = L.route(x)
        assert (r["idx"][0] >= 0).sum() == case["kept"], case
        assert (r["idx"][0][case["kept"]:] == -1).all()
        if "w" in case:
            np.testing.assert_allclose(r["w"][0], case["w"], rtol=1e-15, atol=1e-300)
        else:
            L0, _ = _router_with_logits(g["logits"], g["k"])
            assert np.array_equal(r["w"], L0.route(x)["w"])
    tie = g["exact_tie"]
    L, x = _router_with_logits(tie["logits"], tie["k"], top_p=tie["p"])
    r = L.route(x)
    assert (r["idx"][0] >= 0).sum() == tie["kept"] and r["w"][0].tolist() == tie["w"]


@pytest.mark.parametrize("p", [0.3, 0.7, 0.9])
def test_top_p_keeps_the_shortest_prefix_and_the_total(p):
    cfg = small_config("glm_decode", T=40, d=64, E=32, k=8, f=32, f_shared=32)
    args = (cfg.d, cfg.f, cfg.E, cfg.k, cfg.router, cfg.scaling, cfg.wkind, syn.gen_router_w(cfg),
            syn.gen_router_bias(cfg))
    x = syn.gen_x(cfg, 0)
    plain = oracle.Layer(*args).route(x)
    v = oracle.Layer(*args, top_p=p).route(x)
    for t in range(cfg.T):
        w0, i0 = plain["w"][t], plain["idx"][t]
        m = int((v["idx"][t] >= 0).sum())
        share = np.cumsum(w0) / w0.sum()
        assert share[m - 1] >= p and (m == 1 or share[m - 2] < p)       # the shortest prefix
        assert np.array_equal(v["idx"][t][:m], i0[:m]) and (v["idx"][t][m:] == -1).all()
        np.testing.assert_allclose(v["w"][t][:m].sum(), cfg.scaling, rtol=1e-14)
        np.testing.assert_allclose(v["w"][t][:m] / v["w"][t][0], w0[:m] / w0[0], rtol=1e-14)


def test_top_p_forward_applies_only_the_kept_experts():
    cfg = small_config("glm_decode", T=4, d=64, E=12, k=4, f=32, f_shared=48)
    base = oracle_layer(cfg)
    L = oracle.Layer(cfg.d, cfg.f, cfg.E, cfg.k, cfg.router, cfg.scaling, cfg.wkind, base.router_w,
                     base.router_bias, experts=base.experts, shared=base.shared, f_shared=cfg.f_shared, top_p=0.5)
    x = syn.gen_x(cfg, 0)
    fw = L.forward(x)
    assert (fw["idx"] < 0).any()                                          # some experts are dropped
    for t in range(cfg.T):
        kept = [(int(e), w) for e, w in zip(fw["idx"][t], fw["w"][t]) if e >= 0]
        routed = sum(w * L.expert_ffn(e, x[t])["y"] for e, w in sorted(kept))
        np.testing.assert_allclose(fw["out"][t], routed + L.expert_ffn("shared", x[t])["y"], rtol=1e-12, atol=1e-14)
    u = L.forward(x, mode=oracle.MODE_UNION)
    assert np.array_equal(u["out"], fw["out"])
