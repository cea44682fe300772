"""Pins for the oracle's router, top-k, activations and MoE layer (CPU only)."""
import itertools
import json
import math
import os

import numpy as np
import pytest

import synth
from oracle import moe as om
from oracle import qgemv as oq


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- top-k
def test_topk_golden(golden_dir):
    g = _load(golden_dir, "topk_hand.json")
    for case in g["cases"]:
        lg = np.array([case["logits"]], dtype=np.float32)
        idx, w = om.router_topk(lg, case["k"])
        assert idx[0].tolist() == case["idx"], case["derivation"]
        if case["w"] is not None:
            np.testing.assert_allclose(w[0], case["w"], rtol=0, atol=case.get("w_tol", 1e-15))


def _rank_by_counting(l, e):
    """Rank of expert e: how many experts come before it (larger logit, or equal and lower index)."""
    return sum(1 for f in range(len(l)) if l[f] > l[e] or (l[f] == l[e] and f < e))


def test_topk_exhaustive_small_with_ties():
    """Every logit vector over {0,1,2}^E for E <= 6, every k: the oracle's sort agrees with
    selection by counting ranks (an independent definition of the same order)."""
    for E in range(1, 7):
        for vals in itertools.product([0.0, 1.0, 2.0], repeat=E):
            lg = np.array([vals], dtype=np.float32)
            for k in range(1, E + 1):
                idx = om.topk_select(lg, k)[0].tolist()
                want = [None] * k
                for e in range(E):
                    r = _rank_by_counting(vals, e)
                    if r < k:
                        want[r] = e
                assert idx == want, (vals, k)


def test_topk_random_against_subset_brute_force():
    """Tiny E with random logits: the selected set maximises the sum of logits over all
    k-subsets (unique when logits are distinct)."""
    rng = np.random.default_rng(1)
    for _ in range(200):
        E = int(rng.integers(2, 9))
        k = int(rng.integers(1, E + 1))
        lg = rng.standard_normal(E).astype(np.float32)
        best = max(itertools.combinations(range(E), k), key=lambda S: sum(float(lg[e]) for e in S))
        idx = om.topk_select(lg[None], k)[0]
        assert sorted(idx.tolist()) == sorted(best)
        assert all(lg[idx[i]] >= lg[idx[i + 1]] for i in range(k - 1))


def test_topk_weights_invariants():
    rng = np.random.default_rng(2)
    lg = (rng.standard_normal((50, 128)) * 3).astype(np.float32)
    idx, w = om.router_topk(lg, 8)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    assert np.all(np.diff(w, axis=1) <= 0)
    # closed form: softmax over the selected logits only (identical in exact arithmetic)
    for t in range(50):
        sel = lg[t, idx[t]].astype(np.float64)
        z = np.exp(sel - sel.max())
        np.testing.assert_allclose(w[t], z / z.sum(), rtol=1e-12)


def test_topk_k_equals_e_identical_logits_uniform():
    lg = np.full((3, 16), 0.25, dtype=np.float32)
    idx, w = om.router_topk(lg, 16)
    assert (idx == np.arange(16)).all()
    np.testing.assert_allclose(w, 1.0 / 16, rtol=0, atol=1e-15)


def test_softmax_shift_invariance():
    rng = np.random.default_rng(4)
    l = rng.standard_normal((4, 32))
    np.testing.assert_allclose(om.softmax(l), om.softmax(l + 100.0), rtol=1e-12)
    np.testing.assert_allclose(om.softmax(l).sum(axis=1), 1.0, rtol=1e-14)


def test_router_logits_small_integer_case():
    R = np.array([[1, 2, 3], [-1, 0, 4]], dtype=np.float32)
    x = np.array([[1, 1, 1], [2, -1, 0.5]], dtype=np.float32)
    assert om.router_logits(R, x).tolist() == [[6.0, 3.0], [1.5, 0.0]]


# ---------------------------------------------------------------- activations
def test_gelu_tanh_properties():
    g = np.linspace(-8, 8, 2001)
    y = om.gelu_tanh(g)
    assert om.gelu_tanh(0.0) == 0.0
    # odd-part identity: gelu(g) - gelu(-g) = g for the tanh form
    np.testing.assert_allclose(y - om.gelu_tanh(-g), g, rtol=0, atol=1e-12)
    # close to the exact erf-based GELU (different formula; known deviation below 1e-3)
    erf_gelu = np.array([0.5 * v * (1 + math.erf(v / math.sqrt(2))) for v in g])
    assert np.max(np.abs(y - erf_gelu)) < 1e-3
    assert abs(om.gelu_tanh(20.0) - 20.0) < 1e-12 and abs(om.gelu_tanh(-20.0)) < 1e-12


def test_gelu_tanh_matches_library_routine():
    """The tanh form against an independent implementation of the same formula: PyTorch's
    gelu(approximate="tanh") evaluated in float64.  A slip in the cubic coefficient or in
    sqrt(2/pi) (which the properties above cannot see) moves the values by far more than 1e-12."""
    import torch
    g = np.concatenate([np.linspace(-8, 8, 4001), [-3.3, -1e-3, 1e-3, 0.7, 2.5]])
    ref = torch.nn.functional.gelu(torch.from_numpy(g), approximate="tanh").numpy()
    np.testing.assert_allclose(om.gelu_tanh(g), ref, rtol=0, atol=1e-12)
    # a plausible typo of the coefficient is caught at this tolerance
    bad = 0.5 * g * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (g + 0.0447 * g ** 3)))
    assert np.max(np.abs(bad - ref)) > 1e-6


def test_silu_properties():
    g = np.linspace(-10, 10, 1001)
    s = om.silu(g)
    np.testing.assert_allclose(s - om.silu(-g), g, rtol=0, atol=1e-12)
    np.testing.assert_allclose(s + om.silu(-g), g * np.tanh(g / 2), rtol=0, atol=1e-12)
    assert om.silu(0.0) == 0.0


# ---------------------------------------------------------------- MoE layer
def _tiny_layer(E=6, k=3, H=64, I=32, fmt=oq.FMT_Q4_0, act=om.ACT_GELU_TANH, shared=True,
                identical=False, seed=3):
    def mk(e):
        tag = "same" if identical else f"e{e}"
        return om.Expert(fmt,
                         synth.matrix(fmt, I, H, seed, f"{tag}/g").numpy(),
                         synth.matrix(fmt, I, H, seed, f"{tag}/u").numpy(),
                         synth.matrix(fmt, H, I, seed, f"{tag}/d").numpy())
    experts = {e: mk(e) for e in range(E)}
    sh = None
    if shared:
        sh = om.Expert(oq.FMT_Q8_0, synth.matrix(oq.FMT_Q8_0, 64, H, seed, "s/g").numpy(),
                       synth.matrix(oq.FMT_Q8_0, 64, H, seed, "s/u").numpy(),
                       synth.matrix(oq.FMT_Q8_0, H, 64, seed, "s/d").numpy())
    return om.Layer(E, k, H, I, act, lambda e: experts[e], sh, 64 if shared else 0)


def _ffn_via_gemv(ex, I, H, act, x):
    """Dense FFN built from the oracle's block-formula GEMVs (not from dequantize())."""
    g = oq.qgemv(ex.fmt, ex.gate, x, I, H)
    u = oq.qgemv(ex.fmt, ex.up, x, I, H)
    return oq.qgemv(ex.fmt, ex.down, om.activation(act)(g) * u, H, I)


def test_moe_single_expert_weight_one_is_dense_ffn():
    L = _tiny_layer(k=1, shared=False)
    x = synth.normal(0, 1, 2 * 64).numpy().reshape(2, 64)
    idx = np.array([[4], [1]], dtype=np.int32)
    w = np.ones((2, 1))
    y = om.moe_layer(L, x, idx, w)
    for t in range(2):
        np.testing.assert_allclose(y[t], _ffn_via_gemv(L.expert(int(idx[t, 0])), 32, 64, L.act, x[t]),
                                   rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("act", [om.ACT_GELU_TANH, om.ACT_SILU])
def test_moe_identical_experts_any_routing(act):
    L = _tiny_layer(identical=True, act=act)
    T = 4
    x = synth.normal(0, 2, T * 64).numpy().reshape(T, 64)
    lg = synth.normal(0, 3, T * 6).numpy().reshape(T, 6).astype(np.float32)
    idx, w = om.router_topk(lg, 3)
    y = om.moe_layer(L, x, idx, w)
    for t in range(T):
        want = _ffn_via_gemv(L.expert(0), 32, 64, act, x[t]) + _ffn_via_gemv(L.shared, 64, 64, act, x[t])
        np.testing.assert_allclose(y[t], want, rtol=1e-10, atol=1e-10)


def test_moe_k_equals_e_uniform_is_mean_of_experts():
    L = _tiny_layer(E=4, k=4, shared=False)
    x = synth.normal(0, 5, 64).numpy().reshape(1, 64)
    idx, w = om.router_topk(np.zeros((1, 4), np.float32), 4)
    y = om.moe_layer(L, x, idx, w)
    want = sum(_ffn_via_gemv(L.expert(e), 32, 64, L.act, x[0]) for e in range(4)) / 4
    np.testing.assert_allclose(y[0], want, rtol=1e-10, atol=1e-12)


def test_moe_shared_added_unweighted_and_slot_linearity():
    L = _tiny_layer()
    T = 3
    x = synth.normal(0, 6, T * 64).numpy().reshape(T, 64)
    lg = synth.normal(0, 7, T * 6).numpy().reshape(T, 6).astype(np.float32)
    idx, w = om.router_topk(lg, 3)
    y_all = om.moe_layer(L, x, idx, w)
    y_routed = om.moe_layer(L, x, idx, w, with_shared=False)
    for t in range(T):
        np.testing.assert_allclose(y_all[t] - y_routed[t], _ffn_via_gemv(L.shared, 64, 64, L.act, x[t]),
                                   rtol=1e-9, atol=1e-9)
        want = sum(w[t, j] * _ffn_via_gemv(L.expert(int(idx[t, j])), 32, 64, L.act, x[t]) for j in range(3))
        np.testing.assert_allclose(y_routed[t], want, rtol=1e-10, atol=1e-12)


def test_moe_stack_chains_layers():
    L1 = _tiny_layer(shared=False, fmt=oq.FMT_I4_ROW, act=om.ACT_SILU, seed=5)
    L2 = _tiny_layer(shared=False, fmt=oq.FMT_I4_ROW, act=om.ACT_SILU, seed=6)
    x = synth.normal(0, 8, 2 * 64).numpy().reshape(2, 64)
    lg = [synth.normal(0, 9 + i, 2 * 6).numpy().reshape(2, 6).astype(np.float32) for i in range(2)]
    y = om.moe_stack([L1, L2], x, lg)
    i1, w1 = om.router_topk(lg[0], 3)
    h = om.moe_layer(L1, x, i1, w1)
    i2, w2 = om.router_topk(lg[1], 3)
    np.testing.assert_allclose(y, om.moe_layer(L2, h, i2, w2), rtol=1e-12, atol=1e-12)


def test_glm_expert_size_matches_page_figure():
    """One int4 expert (gate, up 2048x6144 and down 6144x2048 with fp32 row scales) is
    18,915,328 bytes, about the 19 MB per expert the colibri summary gives."""
    b = 2 * synth.weight_bytes(synth.FMT_I4_ROW, 2048, 6144) + synth.weight_bytes(synth.FMT_I4_ROW, 6144, 2048)
    assert b == 18_915_328
    assert abs(b / 1e6 - 19) < 0.5
    assert abs(8 * 256 * b / 1e9 - 38.7) < 0.1
