"""Pins of the oracle's router, top-k and permutation.

* logits against numpy's float64 matmul of the bf16 values (library);
* top-k against brute-force sorting on tiny inputs, and the weights against
  scipy's softmax over all E renormalised over the selected k;
* invariants: k distinct experts, weights in (0, 1], non-increasing, sum 1;
  k = E is the full softmax; equal logits give 0..k-1 and 1/k;
* the permutation against numpy's stable argsort and bincount; bijection;
  stability; rejection of out-of-range experts; empty input.
"""
import math

import numpy as np
import pytest
from scipy.special import softmax

from quantized_expert_ffn_top_b200 import synth


def _bits_to_f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_logits_match_numpy(orc):
    w = synth.workload("tiny")
    x = synth.x_bits(w)
    wr = synth.router_bits(w)
    b = np.linspace(-1, 1, w.E).astype(np.float32)
    L = orc.router_logits(x, wr, b)
    ref = _bits_to_f64(x) @ _bits_to_f64(wr).T + b.astype(np.float64)
    assert np.allclose(L, ref, rtol=0, atol=1e-12)
    L0 = orc.router_logits(x, wr, None)
    assert np.allclose(L0, _bits_to_f64(x) @ _bits_to_f64(wr).T, rtol=0, atol=1e-12)


@pytest.mark.parametrize("T,E,k", [(5, 8, 2), (7, 16, 5), (3, 6, 6), (4, 32, 1)])
def test_topk_matches_brute_force(orc, T, E, k):
    rng = np.random.default_rng(T * 100 + E)
    L = rng.standard_normal((T, E))
    L[0, 1] = L[0, 3]                       # an exact tie
    idx, w, st = orc.topk(L, k)
    assert st == 0
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-L[t, e], e))[:k]
        assert list(idx[t]) == order
        p = softmax(L[t])
        ref = p[order] / p[order].sum()
        assert np.allclose(w[t], ref, rtol=1e-12, atol=0)


def test_topk_invariants(orc):
    L = synth.random_logits(64, 128, kind="normal").astype(np.float64)
    idx, w, st = orc.topk(L, 8)
    assert st == 0
    for t in range(64):
        assert len(set(idx[t])) == 8
        assert np.all(w[t] > 0) and np.all(w[t] <= 1)
        assert np.all(np.diff(w[t]) <= 0)
        assert abs(w[t].sum() - 1) < 1e-12


def test_full_softmax_when_k_equals_E(orc):
    L = synth.random_logits(3, 10, kind="normal").astype(np.float64)
    idx, w, _ = orc.topk(L, 10)
    for t in range(3):
        p = softmax(L[t])
        assert np.allclose(w[t], p[idx[t]], rtol=1e-12)
        assert sorted(idx[t]) == list(range(10))


def test_equal_logits_and_minus_inf(orc):
    idx, w, st = orc.topk(np.zeros((2, 6)), 3)
    assert st == 0 and idx.tolist() == [[0, 1, 2]] * 2 and np.allclose(w, 1 / 3)
    L = np.array([[0.0, -np.inf, -np.inf, 1.0]])
    idx, w, st = orc.topk(L, 3)
    assert st == 0 and idx.tolist() == [[3, 0, 1]]
    e = math.e
    assert np.allclose(w[0], [e / (e + 1), 1 / (e + 1), 0.0])


def test_invalid_logits_flagged(orc):
    _, _, st = orc.topk(np.array([[0.0, np.nan, 1.0]]), 1)
    assert st == -1
    _, _, st = orc.topk(np.full((1, 4), -np.inf), 2)
    assert st == -1


@pytest.mark.parametrize("T,k,E,skew", [(8, 2, 8, 0.0), (300, 8, 64, 1.1), (33, 4, 5, 0.5), (1, 1, 1, 0.0)])
def test_permute_matches_stable_argsort(orc, T, k, E, skew):
    idx = synth.random_topk_idx(T, k, E, skew=skew)
    off, perm, inv, st = orc.permute(idx, E)
    assert st == 0
    flat = idx.reshape(-1)
    ref_order = np.argsort(flat, kind="stable")
    assert np.array_equal(perm, (ref_order // k).astype(np.int32))
    ref_off = np.concatenate([[0], np.cumsum(np.bincount(flat, minlength=E))])
    assert np.array_equal(off, ref_off)
    assert off[-1] == T * k
    # bijection and inverse
    assert np.array_equal(np.sort(inv), np.arange(T * k))
    assert np.array_equal(inv[ref_order], np.arange(T * k))
    # every slot lies inside its expert's segment
    for i in range(T * k):
        e = flat[i]
        assert off[e] <= inv[i] < off[e + 1]


def test_permute_rejects_bad_expert_and_handles_empty(orc):
    _, _, _, st = orc.permute(np.array([[0, 9]], np.int32), 4)
    assert st == -1
    off, perm, inv, st = orc.permute(np.zeros((0, 4), np.int32), 6)
    assert st == 0 and not off.any() and perm.size == 0


def test_permute_then_unpermute_is_identity(orc):
    # combine with w = 1/k over k copies of each token row: exact for k = 2^m
    T, k, E, H = 40, 4, 16, 24
    idx = synth.random_topk_idx(T, k, E, skew=0.7)
    off, perm, inv, st = orc.permute(idx, E)
    rng = np.random.default_rng(7)
    x = rng.standard_normal((T, H))
    y_perm = x[perm]
    out = orc.combine(y_perm, inv, np.full((T, k), 1.0 / k), k)
    assert np.array_equal(out, x)


# ------------------------------------------------ fixed-order fp32 logits ----
def _f32_to_bits(a):
    a = np.asarray(a, np.float32)
    assert np.array_equal(_bits_to_f64(synth.to_bf16_bits(a)), a.astype(np.float64)), "values must be bf16-exact"
    return synth.to_bf16_bits(a)


@pytest.mark.parametrize("order", [1, 2])
@pytest.mark.parametrize("H", [8, 2048, 2304, 4096])
def test_ordered_logits_exact_on_small_integers(orc, order, H):
    """Small-integer products: every partial sum is an integer below 2^24, so
    any summation order gives the exact dot product (integer arithmetic)."""
    rng = np.random.default_rng(H + order)
    xi = rng.integers(-4, 5, (5, H))
    wi = rng.integers(-4, 5, (7, H))
    bias = rng.integers(-8, 9, 7).astype(np.float32)
    L = orc.router_logits_ordered(_f32_to_bits(xi), _f32_to_bits(wi), bias, order=order)
    assert np.array_equal(L.astype(np.int64), xi @ wi.T + bias.astype(np.int64))


def _one_hot_products(H, cols_vals):
    """x = 1 everywhere on the given columns, w = the wanted product there."""
    x = np.zeros((1, H), np.float32)
    w = np.zeros((1, H), np.float32)
    for c, v in cols_vals:
        x[0, c] = 1.0
        w[0, c] = v
    return _f32_to_bits(x), _f32_to_bits(w)


def test_ordered_logits_follow_the_stated_order(orc):
    """Hand-derived sums where fp32 rounding reveals the order.  2^24 + 1 is a
    tie that rounds to the even 2^24; 2^24 + 2 is exact."""
    big = float(2 ** 24)
    # products 2^24 at column 0, 1 at columns 8 and 9 (partial 1 of the small
    # batch order): sequentially 2^24 + 1 + 1 = 2^24; partial 0 = 2^24, partial
    # 1 = 2, joined by the exchange step d = 1: 2^24 + 2
    x, w = _one_hot_products(2048, [(0, big), (8, 1.0), (9, 1.0)])
    assert orc.router_logits_ordered(x, w, order=2)[0, 0] == big
    assert orc.router_logits_ordered(x, w, order=1)[0, 0] == big + 2
    # partials 1 and 3 (columns 8 and 24) each hold 1: the exchange adds them
    # at d = 2 before partial 0 joins at d = 1 -> 2^24 + 2; sequentially 2^24
    x, w = _one_hot_products(2048, [(0, big), (8, 1.0), (24, 1.0)])
    assert orc.router_logits_ordered(x, w, order=1)[0, 0] == big + 2
    assert orc.router_logits_ordered(x, w, order=2)[0, 0] == big
    # partials 1 and 2 (columns 8 and 16): partial 2 meets partial 0 at d = 2
    # (2^24 + 1 -> 2^24), partial 1 meets partial 3 (0) there, and at d = 1
    # 2^24 + 1 -> 2^24 again
    x, w = _one_hot_products(2048, [(0, big), (8, 1.0), (16, 1.0)])
    assert orc.router_logits_ordered(x, w, order=1)[0, 0] == big
    # group sums in order g = 0..7 onto 0: group 0 = 1, group 1 = 2^24
    # (partial 32, column 256), group 2 = 1 (partial 64, column 512):
    # 1 + 2^24 -> 2^24 (tie to even), + 1 -> 2^24
    x, w = _one_hot_products(2048, [(0, 1.0), (256, big), (512, 1.0)])
    assert orc.router_logits_ordered(x, w, order=1)[0, 0] == big
    # a partial's second stretch starts 2048 columns on: columns 2048 and 2049
    # belong to partial 0, which already holds 2^24 (each + 1 rounds away) ...
    x, w = _one_hot_products(4096, [(0, big), (2048, 1.0), (2049, 1.0)])
    assert orc.router_logits_ordered(x, w, order=1)[0, 0] == big
    # ... while columns 2056 and 2057 belong to partial 1, which sums them to 2
    x, w = _one_hot_products(4096, [(0, big), (2056, 1.0), (2057, 1.0)])
    assert orc.router_logits_ordered(x, w, order=1)[0, 0] == big + 2
    assert orc.router_logits_ordered(x, w, order=2)[0, 0] == big


@pytest.mark.parametrize("order", [1, 2])
def test_ordered_logits_within_the_fp32_summation_bound(orc, order):
    """Any summation order of n terms in fp32 is within (n - 1) u sum|terms|
    (u = 2^-24, first order) of the exact sum, here the fp64 definition."""
    w = synth.workload("decode")
    x = synth.x_bits(w)
    wr = synth.router_bits(w)
    b = np.linspace(-1, 1, w.E).astype(np.float32)
    L = orc.router_logits_ordered(x, wr, b, order=order).astype(np.float64)
    ref = orc.router_logits(x, wr, b)
    absum = np.abs(_bits_to_f64(x)) @ np.abs(_bits_to_f64(wr)).T + np.abs(b.astype(np.float64))
    bound = (w.H + 1) * 2.0 ** -24 * absum * 1.01
    assert np.all(np.abs(L - ref) <= bound)
    assert np.any(L != ref.astype(np.float32))   # fp32 rounding really happened


def test_ordered_logits_reject_ragged_small_batch_order(orc):
    x = synth.to_bf16_bits(np.ones((1, 12), np.float32))
    with pytest.raises(ValueError):
        orc.router_logits_ordered(x, x, order=1)
    assert orc.router_logits_ordered(x, x, order=2)[0, 0] == 12.0


def test_forward_routes_on_the_ordered_logits(orc):
    """orc_moe_forward with a fixed router order selects on exactly the fp32
    logits of router_logits_ordered (converted to double)."""
    w = synth.workload("tiny")
    x = synth.x_bits(w)
    wr = synth.router_bits(w)
    W = orc.quantize_expert_weights(orc.FMT_NVFP4, synth.all_w13(w), synth.all_w2(w))
    r = orc.moe_forward(x, wr, None, w.k, W, act=orc.ACT_MATCH, router_order=1)
    L = orc.router_logits_ordered(x, wr, None, order=1).astype(np.float64)
    assert np.array_equal(r["logits"], L)
    idx, wt, _ = orc.topk(L, w.k)
    assert np.array_equal(r["idx"], idx)
    assert np.array_equal(r["w"], wt)
