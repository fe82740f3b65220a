"""Pins of the oracle's expert FFN and whole-layer forward.

* E = 1, k = 1 reduces to one dense SwiGLU FFN, computed here with numpy's
  float64 matmul on independently decoded weights;
* all experts identical reduces to that dense FFN for any routing (the
  renormalised weights sum to 1);
* weights that are exactly representable (so quantisation is lossless) give
  the dense FFN of the original fp32 weights;
* MATCH mode equals the dense FFN of the quantised-then-dequantised
  activations (quantisers pinned separately);
* the grouped (permuted) FFN followed by the combine equals the per-token
  forward; a token subset equals the same rows of the full forward.
"""
import numpy as np
import pytest
import torch

from quantized_expert_ffn_top_b200 import synth

E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, -0.0, -0.5, -1.0, -1.5, -2.0, -3.0, -4.0, -6.0])


def _bf(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _indep_dequant(fmt, codes, sf, gs, K):
    """Decode without the oracle: golden e2m1 table, torch's e4m3, 2^(c-127)."""
    rows = codes.shape[0]
    if fmt == 4:  # bf16 bit patterns, decoded by torch
        b = np.ascontiguousarray(codes).view(np.uint16).copy()
        return torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).double().numpy().reshape(rows, K)
    if fmt == 3:
        v = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).double().numpy()
        return v * gs
    lo = codes & 15
    hi = codes >> 4
    el = np.empty((rows, K))
    el[:, 0::2] = E2M1[lo]
    el[:, 1::2] = E2M1[hi]
    if fmt == 1:
        s = torch.from_numpy(sf.copy()).view(torch.float8_e4m3fn).double().numpy()
        return el * np.repeat(s, 16, axis=1) * gs
    return el * np.repeat(np.ldexp(1.0, sf.astype(np.int64) - 127), 32, axis=1)


def _dense_swiglu(a, W13, W2):
    I = W13.shape[0] // 2
    gu = a @ W13.T
    g, u = gu[:, :I], gu[:, I:]
    h = g / (1 + np.exp(-g)) * u
    return h, h @ W2.T


def _expert_dense(orc, W, e):
    fmt, H, I = W.fmt, W.H, W.I
    gs13 = W.w13_gs[e] if W.w13_gs is not None else np.ones(2, np.float32)
    sf13 = W.w13_sf[e] if W.w13_sf is not None else None
    W13 = np.concatenate([
        _indep_dequant(fmt, W.w13[e, :I], None if sf13 is None else sf13[:I], float(gs13[0]), H),
        _indep_dequant(fmt, W.w13[e, I:], None if sf13 is None else sf13[I:], float(gs13[1]), H)])
    gs2 = float(W.w2_gs[e]) if W.w2_gs is not None else 1.0
    W2 = _indep_dequant(fmt, W.w2[e], None if W.w2_sf is None else W.w2_sf[e], gs2, I)
    return W13, W2


def _layer(orc, fmt, E, H, I, seed=0, identical=False):
    w = synth.workload("tiny", E=E, H=H, I=I)
    w13 = synth.all_w13(w, seed)
    w2 = synth.all_w2(w, seed)
    if identical:
        w13[:] = w13[0]
        w2[:] = w2[0]
    return orc.quantize_expert_weights(fmt, w13, w2)


@pytest.mark.parametrize("fmt", [1, 2, 3, 4])
def test_single_expert_is_dense_swiglu(orc, fmt):
    T, H, I = 6, 64, 64
    W = _layer(orc, fmt, 1, H, I)
    x = synth.x_bits(synth.workload("tiny", H=H), T=T)
    wr = synth.router_bits(synth.workload("tiny", E=1, H=H))
    r = orc.moe_forward(x, wr, None, 1, W, act=orc.ACT_BF16)
    W13, W2 = _expert_dense(orc, W, 0)
    _, y = _dense_swiglu(_bf(x), W13, W2)
    assert np.allclose(r["out"], y, rtol=1e-12, atol=1e-12)
    assert np.all(r["w"] == 1.0) and np.all(r["idx"] == 0)


@pytest.mark.parametrize("fmt", [1, 2, 3, 4])
def test_identical_experts_reduce_to_dense(orc, fmt):
    T, H, I, E, k = 9, 64, 64, 6, 3
    W = _layer(orc, fmt, E, H, I, identical=True)
    wk = synth.workload("tiny", E=E, H=H, k=k)
    x = synth.x_bits(wk, T=T)
    r = orc.moe_forward(x, synth.router_bits(wk), None, k, W, act=orc.ACT_BF16)
    W13, W2 = _expert_dense(orc, W, 0)
    _, y = _dense_swiglu(_bf(x), W13, W2)
    assert np.allclose(r["out"], y, rtol=1e-10, atol=1e-12)


def test_exactly_representable_weights(orc):
    # weights drawn from the e2m1 grid times powers of two: NVFP4 with g = 1
    # holds them exactly, so the layer equals the dense FFN of the originals.
    rng = np.random.default_rng(8)
    E, H, I, T = 2, 32, 32, 5
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])

    def draw(shape, K):
        v = rng.choice(grid, size=shape) * rng.choice([-1, 1], size=shape)
        # each 16-block holds a 6 so its scale lands on 2^j exactly
        v.reshape(-1, 16)[:, 0] = 6.0
        scale = 2.0 ** rng.integers(-6, 2, size=(shape[0], K // 16))
        return (v * np.repeat(scale, 16, axis=1)).astype(np.float32)

    w13 = np.stack([draw((2 * I, H), H) for _ in range(E)])
    w2 = np.stack([draw((H, I), I) for _ in range(E)])
    W = orc.quantize_expert_weights(1, w13, w2)
    W.w13_gs[:] = 1.0
    W.w2_gs[:] = 1.0
    for e in range(E):
        for part in range(2):
            c, s = orc.quant_nvfp4(w13[e, part * I:(part + 1) * I], 1.0)
            W.w13[e, part * I:(part + 1) * I], W.w13_sf[e, part * I:(part + 1) * I] = c, s
        W.w2[e], W.w2_sf[e] = orc.quant_nvfp4(w2[e], 1.0)
    for e in range(E):
        W13, W2 = _expert_dense(orc, W, e)
        assert np.array_equal(W13, w13[e].astype(np.float64))
        assert np.array_equal(W2, w2[e].astype(np.float64))
    wk = synth.workload("tiny", E=E, H=H, k=2)
    x = synth.x_bits(wk, T=T)
    r = orc.moe_forward(x, synth.router_bits(wk), None, 2, W, act=orc.ACT_BF16)
    a = _bf(x)
    ref = np.zeros((T, H))
    for t in range(T):
        for j in range(2):
            e = r["idx"][t, j]
            _, y = _dense_swiglu(a[t:t + 1], w13[e].astype(np.float64), w2[e].astype(np.float64))
            ref[t] += r["w"][t, j] * y[0]
    assert np.allclose(r["out"], ref, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("fmt", [1, 2, 3])
def test_match_mode_is_dense_ffn_of_quantised_activations(orc, fmt):
    T, H, I = 4, 64, 64
    W = _layer(orc, fmt, 1, H, I, seed=3)
    wk = synth.workload("tiny", E=1, H=H)
    x = synth.x_bits(wk, T=T)
    r = orc.moe_forward(x, synth.router_bits(wk), None, 1, W, act=orc.ACT_MATCH)
    xf = _bf(x).astype(np.float32)

    def act(v):
        v = v.astype(np.float32)
        if fmt == 1:
            g = orc.nvfp4_global_scale(orc.amax(v))
            c, s = orc.quant_nvfp4(v, g)
            return _indep_dequant(1, c, s, g, v.shape[1])
        if fmt == 2:
            c, s = orc.quant_mxfp4(v)
            return _indep_dequant(2, c, s, 1.0, v.shape[1])
        sc = orc.fp8_scale(orc.amax(v))
        return _indep_dequant(3, orc.quant_fp8(v, sc), None, sc, v.shape[1])

    W13, W2 = _expert_dense(orc, W, 0)
    I_ = W.I
    gu = act(xf) @ W13.T
    h = gu[:, :I_] / (1 + np.exp(-gu[:, :I_])) * gu[:, I_:]
    y = act(h) @ W2.T
    assert np.allclose(r["out"], y, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("act", [0, 1])
def test_grouped_ffn_and_combine_equal_forward(orc, act):
    wk = synth.workload("tiny")
    W = orc.quantize_expert_weights(1, synth.all_w13(wk), synth.all_w2(wk))
    x = synth.x_bits(wk)
    wr = synth.router_bits(wk)
    r = orc.moe_forward(x, wr, None, wk.k, W, act=act)
    off, perm, inv, st = orc.permute(r["idx"], wk.E)
    y, _ = orc.grouped_ffn(x, perm, off, W, act)
    out = orc.combine(y, inv, r["w"], wk.k)
    assert np.allclose(out, r["out"], rtol=1e-12, atol=1e-14)


def test_subset_equals_full_rows_and_shared_expert(orc):
    wk = synth.workload("fp8_shared", T=12, H=64, E=8, k=2, I=64, shared_I=64)
    W = orc.quantize_expert_weights(3, synth.all_w13(wk), synth.all_w2(wk))
    Ws = orc.quantize_expert_weights(3, synth.shared_w13(wk), synth.shared_w2(wk))
    x = synth.x_bits(wk)
    wr = synth.router_bits(wk)
    full = orc.moe_forward(x, wr, None, 2, W, shared=Ws, act=orc.ACT_MATCH)
    sub = orc.moe_forward(x, wr, None, 2, W, shared=Ws, act=orc.ACT_MATCH, tokens=np.array([7, 2, 11]))
    assert np.array_equal(sub["out"], full["out"][[7, 2, 11]])
    noshared = orc.moe_forward(x, wr, None, 2, W, act=orc.ACT_MATCH)
    # the shared expert adds its own dense FFN with weight 1
    W13s, W2s = _expert_dense(orc, Ws, 0)
    xf = _bf(x).astype(np.float32)
    sc = orc.fp8_scale(orc.amax(xf))
    xq = _indep_dequant(3, orc.quant_fp8(xf, sc), None, sc, wk.H)
    gu = xq @ W13s.T
    h = gu[:, :64] / (1 + np.exp(-gu[:, :64])) * gu[:, 64:]
    hs = orc.fp8_scale(orc.amax(h.astype(np.float32)))
    ysh = _indep_dequant(3, orc.quant_fp8(h.astype(np.float32), hs), None, hs, 64) @ W2s.T
    assert np.allclose(full["out"] - noshared["out"], ysh, rtol=1e-9, atol=1e-12)


def test_static_scales_make_tokens_independent(orc):
    wk = synth.workload("tiny")
    W = orc.quantize_expert_weights(1, synth.all_w13(wk), synth.all_w2(wk))
    x = synth.x_bits(wk)
    wr = synth.router_bits(wk)
    a13, a2 = synth.static_act_scales()
    full = orc.moe_forward(x, wr, None, wk.k, W, act=1, a13_static=a13, a2_static=a2)
    one = orc.moe_forward(x[3:4], wr, None, wk.k, W, act=1, a13_static=a13, a2_static=a2)
    assert np.array_equal(one["out"][0], full["out"][3])


def test_bf16_weights_match_mode_rounds_h_to_bf16(orc):
    """BF16 expert weights in MATCH mode: x is bf16 already and h is rounded to
    bf16 (torch's rounding here) before the down projection."""
    T, H, I = 5, 64, 128
    W = _layer(orc, 4, 1, H, I)
    x = synth.x_bits(synth.workload("tiny", H=H), T=T)
    wr = synth.router_bits(synth.workload("tiny", E=1, H=H))
    r = orc.moe_forward(x, wr, None, 1, W, act=orc.ACT_MATCH)
    W13, W2 = _expert_dense(orc, W, 0)
    h, _ = _dense_swiglu(_bf(x), W13, W2)
    hb = torch.from_numpy(h.astype(np.float32)).to(torch.bfloat16).double().numpy()
    assert np.allclose(r["out"], hb @ W2.T, rtol=1e-12, atol=1e-12)
    # and it differs from A16 (h kept in double) by at most bf16's rounding of h
    a16 = orc.moe_forward(x, wr, None, 1, W, act=orc.ACT_BF16)["out"]
    bound = (np.abs(h) * 2.0 ** -8) @ np.abs(W2).T + 1e-12
    assert np.all(np.abs(r["out"] - a16) <= bound)


def test_bf16_weights_equal_nvfp4_weights_when_exact(orc):
    """NVFP4 weights with g = 1 and 2-significant-bit scales decode to values
    bf16 holds exactly; stored as BF16 weights they give the same layer."""
    rng = np.random.default_rng(5)
    E, H, I, T, k = 3, 64, 64, 7, 2
    c13 = rng.integers(0, 256, (E, 2 * I, H // 2), dtype=np.uint8)
    c2 = rng.integers(0, 256, (E, H, I // 2), dtype=np.uint8)
    # e4m3 codes with mantissa 0 or 4 (1.0 or 1.5 times a power of two)
    def scales(shape):
        ex = rng.integers(4, 10, shape)
        return ((ex << 3) | (rng.integers(0, 2, shape) * 4)).astype(np.uint8)
    s13, s2 = scales((E, 2 * I, H // 16)), scales((E, H, I // 16))
    g13, g2 = np.ones((E, 2), np.float32), np.ones(E, np.float32)
    Wn = orc.Weights(1, E, H, I, c13, s13, g13, c2, s2, g2)
    d13 = np.stack([orc.dequant(1, c13[e], s13[e], 1.0, 2 * I, H) for e in range(E)])
    d2 = np.stack([orc.dequant(1, c2[e], s2[e], 1.0, H, I) for e in range(E)])
    # exact in bf16: the low 16 bits of the fp32 encoding are zero
    f13, f2 = d13.astype(np.float32), d2.astype(np.float32)
    assert np.all(f13.view(np.uint32) & 0xFFFF == 0) and np.all(f2.view(np.uint32) & 0xFFFF == 0)
    Wb = orc.quantize_expert_weights(4, f13, f2)
    wk = synth.workload("tiny", E=E, H=H, k=k)
    x = synth.x_bits(wk, T=T)
    wr = synth.router_bits(wk)
    a = orc.moe_forward(x, wr, None, k, Wn, act=orc.ACT_BF16)["out"]
    b = orc.moe_forward(x, wr, None, k, Wb, act=orc.ACT_BF16)["out"]
    assert np.array_equal(a, b)


def test_bank_by_expert_equals_whole_bank(orc):
    """The per-expert, threaded bank builder gives the bytes of the
    whole-array one (NVFP4 with its per-part scales, MXFP4)."""
    for fmt, name in ((orc.FMT_NVFP4, "nvfp4"), (orc.FMT_MXFP4, "mxfp4"), (orc.FMT_FP8, "fp8")):
        w = synth.workload("tiny", fmt=name, E=5, H=256, I=256)
        A = orc.quantize_expert_weights(fmt, synth.all_w13(w), synth.all_w2(w))
        B = orc.quantize_expert_weights_by_expert(fmt, w.E, lambda e: synth.expert_w13(w, e),
                                                  lambda e: synth.expert_w2(w, e), threads=3)
        for f in ("w13", "w13_sf", "w13_gs", "w2", "w2_sf", "w2_gs"):
            a, b = getattr(A, f), getattr(B, f)
            assert (a is None and b is None) or np.array_equal(a, b), (name, f)
