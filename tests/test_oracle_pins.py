"""Pins for the CPU oracle: checks against what the pages and the mathematics fix.

Each test compares the oracle with something other than itself: brute-force
enumeration, hand-written examples, closed forms and invariants the pages
state, or library routines (torch float64) for special cases.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from sparse_moe_transformer_fp32_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _sigmoid32(x):
    return (1.0 / (1.0 + np.exp(-x.astype(np.float64)))).astype(np.float32)


def _brute_force_route(logits, bias, G, Gk, k, S):
    """Selection by exhaustive search over group subsets and expert subsets."""
    E = logits.shape[0]
    per = E // G
    s = _sigmoid32(logits)
    sb = (s + bias.astype(np.float32)).astype(np.float32)
    gs = []
    for g in range(G):
        top = sorted(sb[g * per:(g + 1) * per].tolist(), reverse=True)
        gs.append(np.float32(top[0]) + np.float32(top[1]) if per >= 2 else np.float32(top[0]))
    best_groups, best_val = None, -math.inf
    for sub in itertools.combinations(range(G), Gk):
        v = sum(float(gs[g]) for g in sub)
        if v > best_val:
            best_groups, best_val = sub, v
    cand = [e for e in range(E) if e // per in best_groups]
    best_set, best_val = None, -math.inf
    for sub in itertools.combinations(cand, k):
        v = sum(float(sb[e]) for e in sub)
        if v > best_val:
            best_set, best_val = sub, v
    chosen = sorted(best_set)
    ssum = sum(float(s[e]) for e in chosen)
    w = [np.float32(S * float(s[e]) / ssum) for e in chosen]
    return chosen, w, best_groups


@pytest.mark.parametrize("E,G,Gk,k", [(8, 2, 1, 2), (12, 3, 2, 3), (16, 4, 2, 4), (16, 4, 3, 5),
                                      (16, 8, 4, 4), (8, 4, 2, 3)])
def test_route_matches_brute_force(E, G, Gk, k):
    rng = np.random.default_rng(1000 + E * 31 + G * 7 + Gk * 3 + k)
    T = 40
    logits = rng.normal(0, 1, size=(T, E)).astype(np.float32)
    bias = rng.uniform(-0.1, 0.1, size=E).astype(np.float32)
    idx, w, _, _ = oracle.route(logits, bias, G, Gk, k, 2.5, True)
    for t in range(T):
        chosen, wbf, groups = _brute_force_route(logits[t], bias, G, Gk, k, 2.5)
        assert idx[t].tolist() == chosen, (t, idx[t], chosen)
        np.testing.assert_allclose(w[t], wbf, rtol=3e-7, atol=0)
        assert len({e // (E // G) for e in idx[t]}) <= Gk


def test_group_score_hand_examples():
    with open(os.path.join(GOLDEN, "group_score_examples.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        target = np.asarray(c["biased_scores"], np.float32)
        bias = (target - np.float32(0.5)).astype(np.float32)
        logits = np.zeros((1, c["E"]), np.float32)  # sigmoid(0) = 0.5 exactly
        idx, w, _, _ = oracle.route(logits, bias, c["n_group"], c["topk_group"], c["top_k"],
                                    c["scale"], True)
        assert idx[0].tolist() == c["expected_idx"], c["name"]
        np.testing.assert_allclose(w[0], c["expected_weights"], rtol=2e-7, err_msg=c["name"])


def test_bias_is_selection_only():
    wl = W.WORKLOADS["tiny"]
    h, Wr, b = W.hidden(wl), W.router_weight(wl), W.router_bias(wl)
    logits = oracle.router_logits(h, Wr)
    idx0, w0, me, mg = oracle.route(logits, b, wl.n_group, wl.topk_group, wl.top_k)
    # the same constant on every bias: same choice, bit-identical weights
    idx1, w1, _, _ = oracle.route(logits, b + 0.25, wl.n_group, wl.topk_group, wl.top_k)
    ok = (me > 1e-5) & (mg > 1e-5)
    assert ok.sum() > 40
    assert np.array_equal(idx0[ok], idx1[ok])
    assert np.array_equal(w0[ok].view(np.uint32), w1[ok].view(np.uint32))
    # raising one unchosen expert of a kept group above the rest switches exactly it in
    t = int(np.nonzero(ok)[0][0])
    s = _sigmoid32(logits[t])
    per = wl.E // wl.n_group
    kept_groups = {e // per for e in idx0[t]}
    outsider = next(e for e in range(wl.E) if e // per in kept_groups and e not in idx0[t])
    b2 = b.clone()
    b2[outsider] = 5.0
    idx2, w2, _, _ = oracle.route(logits[t:t + 1], b2, wl.n_group, wl.topk_group, wl.top_k)
    sb = s + b.numpy()
    dropped = min(idx0[t], key=lambda e: (sb[e], -e))
    expect = sorted([e for e in idx0[t] if e != dropped] + [outsider])
    assert idx2[0].tolist() == expect
    ssum = sum(float(s[e]) for e in expect)
    np.testing.assert_allclose(w2[0], [2.5 * float(s[e]) / ssum for e in expect], rtol=3e-7)


@pytest.mark.parametrize("name", ["tiny"])
def test_weights_sum_to_scaling_factor(name):
    wl = W.WORKLOADS[name]
    h, Wr, b = W.hidden(wl), W.router_weight(wl), W.router_bias(wl)
    _, idx, w, _, _ = oracle.layer_routing(h, Wr, b, wl)
    tot = w.astype(np.float64).sum(axis=1)
    ulp = np.spacing(np.float32(2.5))
    assert np.all(np.abs(tot - 2.5) <= 4 * ulp)
    # Beam shapes on random logits too
    rng = np.random.default_rng(7)
    L = rng.normal(0, 0.7, size=(512, 256)).astype(np.float32)
    bb = rng.uniform(-0.05, 0.05, size=256).astype(np.float32)
    idx, w, _, _ = oracle.route(L, bb, 8, 4, 8, 2.5, True)
    assert np.all(np.abs(w.astype(np.float64).sum(1) - 2.5) <= 4 * ulp)
    assert np.all(np.diff(idx, axis=1) > 0)  # ascending, distinct
    groups = idx // 32
    assert all(len(set(r)) <= 4 for r in groups.tolist())


def test_unnormalised_weights_are_scaled_scores():
    rng = np.random.default_rng(3)
    L = rng.normal(0, 1, size=(64, 16)).astype(np.float32)
    L[0, :] = 0.0
    bb = rng.uniform(-0.1, 0.1, size=16).astype(np.float32)
    idx, w, _, _ = oracle.route(L, bb, 4, 2, 4, 2.5, False)
    s = _sigmoid32(L)
    expect = (2.5 * np.take_along_axis(s, idx, axis=1).astype(np.float64)).astype(np.float32)
    assert np.array_equal(w, expect)
    assert np.all(w[0] == np.float32(1.25))  # sigmoid(0) = 1/2


def test_illustrated_routing_violates_group_limit():
    # The review page's routing illustration (experts 12, 41, 67, 103, 140, 171, 203, 238) is
    # labelled random; it spans 8 groups of 32, so group-limited routing cannot produce it.
    illus = [12, 41, 67, 103, 140, 171, 203, 238]
    assert len({e // 32 for e in illus}) == 8 > 4
    rng = np.random.default_rng(11)
    L = rng.normal(0, 0.7, size=(2048, 256)).astype(np.float32)
    bb = rng.uniform(-0.05, 0.05, size=256).astype(np.float32)
    idx, _, _, _ = oracle.route(L, bb, 8, 4, 8, 2.5, True)
    assert not any(r == illus for r in idx.tolist())
    assert max(len({e // 32 for e in r}) for r in idx.tolist()) <= 4


def test_router_logits_match_float64_matmul():
    wl = W.WORKLOADS["tiny"]
    h, Wr = W.hidden(wl), W.router_weight(wl)
    got = oracle.router_logits(h, Wr)
    ref = (h.double() @ Wr.double().T).float().numpy()
    diff = np.abs(got.view(np.int32).astype(np.int64) - ref.view(np.int32).astype(np.int64))
    assert diff.max() <= 1 and (diff == 0).mean() > 0.99


def _torch_swiglu_f64(x, wg, wu, wd):
    """Dense SwiGLU with float64 matmuls and the same rounding points."""
    g = (x.double() @ wg.double().T).float()
    u = (x.double() @ wu.double().T).float()
    act = torch.nn.functional.silu(g.double()).float()
    a = (act * u).to(torch.bfloat16)
    return (a.double() @ wd.double().T).float()


def test_expert_mlp_matches_torch_float64():
    wl = W.WORKLOADS["tiny"]
    x = W.hidden(wl)[:5]
    wg, wu, wd = (W.expert_weight(wl, m, 3) for m in ("gate", "up", "down"))
    ref = _torch_swiglu_f64(x, wg, wu, wd).numpy()
    for t in range(5):
        y = oracle.expert_mlp(x[t], wg, wu, wd)
        np.testing.assert_allclose(y, ref[t], rtol=1e-5, atol=1e-6)


def test_identical_experts_equal_scaled_dense_swiglu():
    wl = W.WORKLOADS["tiny"]
    h, Wr, b = W.hidden(wl), W.router_weight(wl), W.router_bias(wl)
    _, idx, w, _, _ = oracle.layer_routing(h, Wr, b, wl)
    shared = tuple(W.expert_weight(wl, m, 0) for m in ("gate", "up", "down"))
    experts = {e: shared for e in range(wl.E)}
    out = oracle.moe_tokens(np.arange(wl.T), h, idx, w, experts)
    dense = _torch_swiglu_f64(h, *shared).numpy().astype(np.float64)
    ref = 2.5 * dense
    err = np.abs(out - ref).max() / np.abs(ref).max()
    assert err < 1e-5, err


def test_combine_is_weighted_sum_of_expert_outputs():
    wl = W.WORKLOADS["tiny"]
    h, Wr, b = W.hidden(wl), W.router_weight(wl), W.router_bias(wl)
    _, idx, w, _, _ = oracle.layer_routing(h, Wr, b, wl)
    experts = {e: tuple(W.expert_weight(wl, m, e) for m in ("gate", "up", "down"))
               for e in range(wl.E)}
    toks = [0, 7, 63]
    out = oracle.moe_tokens(toks, h, idx, w, experts)
    for n, t in enumerate(toks):
        ref = np.zeros(wl.d)
        for j in range(wl.top_k):
            e = int(idx[t, j])
            ref += float(w[t, j]) * _torch_swiglu_f64(h[t:t + 1], *experts[e]).numpy()[0]
        np.testing.assert_allclose(out[n], ref, rtol=1e-5, atol=1e-6)


def test_residual_coefficients_square_sum_is_one():
    for k in range(1, 105):
        cx, cf = oracle.residual_coefficients(k)
        assert abs(cx * cx + cf * cf - 1.0) < 4e-16
    cx, cf = oracle.residual_coefficients(1)
    assert cx == 0.0 and cf == 1.0       # the embedding is the first contribution
    cx, cf = oracle.residual_coefficients(10)
    assert abs(np.float32(cx) ** 2 + np.float32(cf) ** 2 - 1.0) <= np.spacing(np.float32(1.0))


def test_residual_after_104_contributions_weighs_each_equally():
    # After k contributions the stream is their sum divided by sqrt(k): run the recursion
    # with one-hot contributions and read each one's final weight.
    n = 104
    x = np.zeros(n, np.float32)
    for k in range(1, n + 1):
        f = np.zeros(n, np.float32)
        f[k - 1] = 1.0
        x = oracle.residual(x, f, k)
    np.testing.assert_allclose(x, np.full(n, 1.0 / math.sqrt(n)), rtol=2e-5)


def test_rmsnorm_matches_torch_and_closed_form():
    rng = np.random.default_rng(5)
    x = rng.normal(0, 1, size=(16, 512)).astype(np.float32)
    g = rng.uniform(0.9, 1.1, size=512).astype(np.float32)
    y = oracle.rmsnorm(x, g, 1e-6)
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x).double(), (512,),
                                       weight=torch.from_numpy(g).double(), eps=1e-6).float()
    np.testing.assert_allclose(y, ref.numpy(), rtol=3e-7, atol=1e-7)
    ones = np.ones(512, np.float32)
    y1 = oracle.rmsnorm(x, ones, 1e-6).astype(np.float64)
    ms = (x.astype(np.float64) ** 2).mean(1)
    np.testing.assert_allclose((y1 ** 2).mean(1), ms / (ms + 1e-6), rtol=1e-6)


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(9)
    v = np.concatenate([rng.normal(0, 1, 10000), rng.normal(0, 1e-38, 100),
                        [0.0, -0.0, np.inf, -np.inf, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8,
                         3.0e38, -1.00390625]]).astype(np.float32)
    got = oracle.f32_to_bf16(v)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)
    assert np.isnan(oracle.bf16_to_f32(oracle.f32_to_bf16(np.array([np.nan], np.float32))))[0]


def test_beam_config_accounting():
    with open(os.path.join(GOLDEN, "beam_config.json")) as f:
        c = json.load(f)
    per_expert = 3 * c["hidden_size"] * c["moe_intermediate_size"]
    assert abs(per_expert - c["params_per_expert_approx"]) / c["params_per_expert_approx"] < 0.01
    experts = per_expert * c["num_experts"] * c["moe_layers"]
    assert abs(100 * experts / c["total_params"] - c["expert_weight_share_percent"]) < 0.05
    beam = W.WORKLOADS["prefill"]
    assert (beam.d, beam.I, beam.E, beam.top_k, beam.n_group, beam.topk_group, beam.scale) == (
        c["hidden_size"], c["moe_intermediate_size"], c["num_experts"], c["num_experts_per_tok"],
        c["n_group"], c["topk_group"], c["routed_scaling_factor"])


def test_bias_update_hand_example_and_invariants():
    with open(os.path.join(GOLDEN, "bias_update_example.json")) as f:
        c = json.load(f)
    got = oracle.bias_update(np.array(c["counts"]), np.array(c["bias"], np.float32), c["gamma"],
                             c["slots"])
    assert got.tolist() == c["expected"]
    # repeated updates move an always-overloaded expert's bias down and an idle one's up,
    # by exactly gamma per step, and leave the total unchanged when loads are symmetric
    counts = np.array([10, 0, 5, 5])
    b = np.zeros(4, np.float32)
    for _ in range(8):
        b = oracle.bias_update(counts, b, 0.25, 20)
    assert b.tolist() == [-2.0, 2.0, 0.0, 0.0]


def test_dense_mlp_is_one_expert_with_unit_weight():
    wl = W.WORKLOADS["tiny"]
    h = W.hidden(wl)[:6]
    mats = tuple(W.expert_weight(wl, m, 5) for m in ("gate", "up", "down"))
    out = oracle.dense_mlp(range(6), h, *mats)
    ref = _torch_swiglu_f64(h, *mats).numpy()
    np.testing.assert_allclose(out, ref, rtol=1e-5, atol=1e-6)
