"""Tensor-core grouped GEMM path against the oracle (and against the GEMV
path), through the C ABI: ragged and skewed expert segments, every format,
static and dynamic activation scales, and the full-size workloads on sampled
tokens in the configuration the benchmark times."""
import numpy as np
import pytest
import torch

import oracle
from quantized_expert_ffn_top_b200 import ops, synth
from tests.gpu_helpers import (TOL, bits_to_dev_bf16, dev_to_f64, device_bank, forward_reference, max_abs_rel,
                               oracle_bank, routed_inputs)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _path():
    assert torch.cuda.is_available()
    ops.moe_set_option(ops.OPT_FFN_PATH, 0)
    yield
    ops.moe_set_option(ops.OPT_FFN_PATH, 0)


GEMM_CASES = [
    # name, overrides, static scales, routing skew
    ("nvfp4-static", dict(fmt="nvfp4", T=200, H=512, E=8, k=2, I=256), True, 1.2),
    ("nvfp4-dynamic", dict(fmt="nvfp4", T=200, H=512, E=8, k=2, I=256), False, 1.2),
    ("mxfp4", dict(fmt="mxfp4", T=160, H=512, E=6, k=2, I=256), False, 0.8),
    ("fp8", dict(fmt="fp8", T=150, H=256, E=10, k=3, I=256), False, 1.0),
    ("nvfp4-big-expert", dict(fmt="nvfp4", T=400, H=256, E=4, k=1, I=512), True, 3.0),
    ("nvfp4-some-empty", dict(fmt="nvfp4", T=64, H=256, E=32, k=2, I=256), True, 2.5),
]


def _run(over, static, skew, path):
    w = synth.workload("tiny", **over)
    W, _ = oracle_bank(w)
    a13, a2 = synth.static_act_scales() if static else (None, None)
    bank = device_bank(W, a13, a2)
    idx = synth.random_topk_idx(w.T, w.k, w.E, skew=skew)
    off, perm, inv, _ = oracle.permute(idx, w.E)
    x = synth.x_bits(w)
    ws = ops.new_workspace(ops.workspace_size(w.T, w.k, bank, None, 1))
    ops.moe_set_option(ops.OPT_FFN_PATH, path)
    y = ops.moe_grouped_ffn(bits_to_dev_bf16(x), w.k, torch.from_numpy(perm).cuda(), torch.from_numpy(off).cuda(),
                            bank, 1, ws)
    torch.cuda.synchronize()
    st = ops.moe_get_device_status(ws)
    return w, W, x, perm, off, a13, a2, dev_to_f64(y), st


@pytest.mark.parametrize("tile_n,pair", [(64, 1), (128, 1), (192, 0), (192, 1), (256, 0), (256, 1)])
@pytest.mark.parametrize("name,over,static,skew", GEMM_CASES)
def test_gemm_path_matches_oracle(name, over, static, skew, tile_n, pair):
    """Every token-tile width; 192- and 256-token tiles on one CTA and on CTA
    pairs (cta_group::2, 256 weight rows per tile; 64 and 128 ignore pairs)."""
    ops.moe_set_option(ops.OPT_GEMM_TILE_N, tile_n)
    ops.moe_set_option(ops.OPT_GEMM_PAIR, pair)
    try:
        w, W, x, perm, off, a13, a2, y, st = _run(over, static, skew, 2)
    finally:
        ops.moe_set_option(ops.OPT_GEMM_TILE_N, 0)
        ops.moe_set_option(ops.OPT_GEMM_PAIR, 2)
    assert st == 0
    ry, _ = oracle.grouped_ffn(x, perm, off, W, 1, a13 or 0.0, a2 or 0.0)
    err = max_abs_rel(y, ry)
    assert err < TOL, err
    # per expert too: a wrong tile or a dropped segment shows up here
    for e in range(w.E):
        a, b = off[e], off[e + 1]
        if b > a:
            assert max_abs_rel(y[a:b], ry[a:b]) < 5 * TOL, e


@pytest.mark.parametrize("tile_n", [64, 192])
@pytest.mark.parametrize("name,over,static,skew", [GEMM_CASES[0], GEMM_CASES[3], GEMM_CASES[5]])
def test_early_weight_loads_change_nothing(name, over, static, skew, tile_n):
    """Weight tiles loaded before the wait on the previous kernel (the expert
    named by the offsets, or by the tile list) or prefetched to L2 give the
    same bits as loading every stage after it."""
    ops.moe_set_option(ops.OPT_GEMM_TILE_N, tile_n)
    ys = []
    try:
        for mode in (0, 1, 2):
            ops.moe_set_option(ops.OPT_EARLY_WEIGHTS, mode)
            *_, y, st = _run(over, static, skew, 2)
            assert st == 0, mode
            ys.append(y)
    finally:
        ops.moe_set_option(ops.OPT_EARLY_WEIGHTS, 1)
        ops.moe_set_option(ops.OPT_GEMM_TILE_N, 0)
    assert np.array_equal(ys[0], ys[1]) and np.array_equal(ys[0], ys[2])


@pytest.mark.parametrize("name,over,static,skew", [GEMM_CASES[0], GEMM_CASES[2], GEMM_CASES[4], GEMM_CASES[5]])
def test_fused_ffn_kernel_matches_two_kernels(name, over, static, skew):
    """64-token tiles: the one-kernel FFN (down tiles waiting on their token
    tile's gate|up slices) gives the bits of the two separate projections."""
    ops.moe_set_option(ops.OPT_GEMM_TILE_N, 64)
    ys = []
    try:
        for fused in (0, 1):
            ops.moe_set_option(ops.OPT_FUSED_FFN, fused)
            w, W, x, perm, off, a13, a2, y, st = _run(over, static, skew, 2)
            assert st == 0, fused
            ys.append(y)
    finally:
        ops.moe_set_option(ops.OPT_FUSED_FFN, 1)
        ops.moe_set_option(ops.OPT_GEMM_TILE_N, 0)
    assert np.array_equal(ys[0], ys[1])
    ry, _ = oracle.grouped_ffn(x, perm, off, W, 1, a13 or 0.0, a2 or 0.0)
    assert max_abs_rel(ys[1], ry) < TOL


BF16_CASES = [
    ("bf16-ragged", dict(fmt="bf16", T=200, H=512, E=8, k=2, I=256), 1.2),
    ("bf16-small-batch", dict(fmt="bf16", T=4, H=256, E=16, k=4, I=256), 0.0),
    ("bf16-some-empty", dict(fmt="bf16", T=64, H=256, E=32, k=2, I=256), 2.5),
    ("bf16-long-k", dict(fmt="bf16", T=96, H=1024, E=4, k=2, I=384), 1.0),
]


@pytest.mark.parametrize("tile_n", [0, 64, 192, 256])
@pytest.mark.parametrize("act", [0, 1])
@pytest.mark.parametrize("name,over,skew", BF16_CASES)
def test_bf16_weights_match_oracle(name, over, skew, act, tile_n):
    """BF16 expert weights on the tensor cores (kind::f16): x gathered into
    padded bf16 rows, h stored in bf16 by the gate|up epilogue."""
    ops.moe_set_option(ops.OPT_GEMM_TILE_N, tile_n)
    try:
        w = synth.workload("tiny", **over)
        W, _ = oracle_bank(w)
        bank = device_bank(W)
        idx = synth.random_topk_idx(w.T, w.k, w.E, skew=skew)
        off, perm, inv, _ = oracle.permute(idx, w.E)
        x = synth.x_bits(w)
        ws = ops.new_workspace(ops.workspace_size(w.T, w.k, bank, None, act))
        y = ops.moe_grouped_ffn(bits_to_dev_bf16(x), w.k, torch.from_numpy(perm).cuda(),
                                torch.from_numpy(off).cuda(), bank, act, ws)
        torch.cuda.synchronize()
        st = ops.moe_get_device_status(ws)
    finally:
        ops.moe_set_option(ops.OPT_GEMM_TILE_N, 0)
    assert st == 0
    ry, _ = oracle.grouped_ffn(x, perm, off, W, act)
    assert max_abs_rel(dev_to_f64(y), ry) < TOL


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4", "fp8"])
def test_dequantized_bank_and_a16_layer(fmt):
    """moe_dequantize_weights: every bf16 weight equals the oracle's decode
    rounded to bf16 (torch); the bf16-activation layer on the expanded bank
    (bf16 tensor cores) matches the oracle's A16 layer on the quantised bank."""
    from tests.gpu_helpers import routed_inputs
    w = synth.workload("tiny", fmt=fmt, T=96, H=256, E=8, k=2, I=256)
    W, _ = oracle_bank(w)
    bf = ops.moe_dequantize_weights(device_bank(W, prepare=False))
    torch.cuda.synchronize()
    E, H, I = W.E, W.H, W.I

    def ref_bits(codes, sf, gs, rows, K):
        d = oracle.dequant(W.fmt, codes, sf, gs, rows, K).astype(np.float32)
        return torch.from_numpy(d).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)

    got13 = bf.w13.cpu().numpy().view(np.uint16).reshape(E, 2 * I, H)
    got2 = bf.w2.cpu().numpy().view(np.uint16).reshape(E, H, I)
    for e in range(E):
        for part in range(2):
            rows = slice(part * I, (part + 1) * I)
            sf = None if W.w13_sf is None else W.w13_sf[e, rows]
            gs = 1.0 if W.w13_gs is None else float(W.w13_gs[e, part])
            assert np.array_equal(got13[e, rows], ref_bits(W.w13[e, rows], sf, gs, I, H)), (e, part)
        sf = None if W.w2_sf is None else W.w2_sf[e]
        gs = 1.0 if W.w2_gs is None else float(W.w2_gs[e])
        assert np.array_equal(got2[e], ref_bits(W.w2[e], sf, gs, H, I)), e
    bank = ops.moe_prepare_weights(bf)
    x, wr, b = routed_inputs(w)
    ws = ops.new_workspace(ops.workspace_size(w.T, w.k, bank, None, 0))
    out = ops.moe_forward(bits_to_dev_bf16(x), bits_to_dev_bf16(wr), None if b is None else torch.from_numpy(b).cuda(),
                          w.k, bank, None, 0, ws)
    assert ops.moe_get_device_status(ws) == 0
    r, keep = forward_reference(w, x, wr, b, W, act=oracle.ACT_BF16)
    assert max_abs_rel(dev_to_f64(out)[keep], r["out"][keep]) < TOL


@pytest.mark.parametrize("name,over,static,skew", GEMM_CASES[:4])
def test_gemm_and_gemv_paths_agree(name, over, static, skew):
    *_, yg, st1 = _run(over, static, skew, 2)
    *_, yv, st2 = _run(over, static, skew, 1)
    assert st1 == 0 and st2 == 0
    assert max_abs_rel(yg, yv) < TOL


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
def test_long_k_loop_default_options_match_oracle(fmt):
    """The large prefill's K (H = 4096: 16 stages a tile) with the default
    options, so the gate|up projection runs on CTA pairs and the down
    projection on single CTAs, Zipf-like skew, ragged tiles."""
    w = synth.workload("tiny", fmt=fmt, T=300, H=4096, E=8, k=2, I=512)
    W, _ = oracle_bank(w)
    a13, a2 = (None, None) if fmt == "mxfp4" else synth.static_act_scales()
    bank = device_bank(W, a13, a2)
    idx = synth.random_topk_idx(w.T, w.k, w.E, skew=1.5)
    off, perm, inv, _ = oracle.permute(idx, w.E)
    x = synth.x_bits(w)
    ws = ops.new_workspace(ops.workspace_size(w.T, w.k, bank, None, 1))
    y = ops.moe_grouped_ffn(bits_to_dev_bf16(x), w.k, torch.from_numpy(perm).cuda(), torch.from_numpy(off).cuda(),
                            bank, 1, ws)
    torch.cuda.synchronize()
    assert ops.moe_get_device_status(ws) == 0
    ry, _ = oracle.grouped_ffn(x, perm, off, W, 1, a13 or 0.0, a2 or 0.0)
    assert max_abs_rel(dev_to_f64(y), ry) < TOL


@pytest.fixture(scope="module")
def prefill_layer():
    w = synth.workload("prefill")
    W, _ = oracle_bank(w)
    return w, W


def test_prefill_forward_full_size_sampled(prefill_layer):
    """T=4096 prefill through moe_forward in the benchmark's configuration
    (tensor-core path, static activation scales): 512 evenly spaced tokens
    (static scales leave tokens independent, so a subset is exact)."""
    w, W = prefill_layer
    a13, a2 = synth.static_act_scales()
    bank = device_bank(W, a13, a2)
    x, wr, b = routed_inputs(w)
    ws = ops.new_workspace(ops.workspace_size(w.T, w.k, bank, None, 1))
    out = ops.moe_forward(bits_to_dev_bf16(x), bits_to_dev_bf16(wr), torch.from_numpy(b).cuda(), w.k, bank, None, 1,
                          ws)
    assert ops.moe_get_device_status(ws) == 0
    toks = np.linspace(0, w.T - 1, 512).astype(np.int32)
    r, keep = forward_reference(w, x, wr, b, W, act=1, a13=a13, a2=a2, tokens=toks, what="prefill static")
    got = dev_to_f64(out)[toks]
    err = max_abs_rel(got[keep], r["out"][keep])
    print(f"prefill static, 512 tokens: max-abs-rel {err:.3e}")
    assert err < TOL, err


def test_prefill_forward_full_size_dynamic_scales(prefill_layer):
    """The prefill layer with the default activation scales: x's and h's
    NVFP4 global scales from their tensor amax (h over all 32768 slots), so
    every token is evaluated by the oracle and compared."""
    w, W = prefill_layer
    bank = device_bank(W)
    x, wr, b = routed_inputs(w)
    ws = ops.new_workspace(ops.workspace_size(w.T, w.k, bank, None, 1))
    out = ops.moe_forward(bits_to_dev_bf16(x), bits_to_dev_bf16(wr), torch.from_numpy(b).cuda(), w.k, bank, None, 1,
                          ws)
    assert ops.moe_get_device_status(ws) == 0
    r, keep = forward_reference(w, x, wr, b, W, act=1, what="prefill dynamic")
    err = max_abs_rel(dev_to_f64(out)[keep], r["out"][keep])
    print(f"prefill dynamic scales, {int(keep.sum())} tokens: max-abs-rel {err:.3e}")
    assert err < TOL, err


def test_decode_forward_full_size(prefill_layer):
    """The decode workload shares the prefill layer's weights (T=4)."""
    _, W = prefill_layer
    w = synth.workload("decode")
    bank = device_bank(W)
    x, wr, b = routed_inputs(w)
    ws = ops.new_workspace(ops.workspace_size(w.T, w.k, bank, None, 1))
    out = ops.moe_forward(bits_to_dev_bf16(x), bits_to_dev_bf16(wr), None, w.k, bank, None, 1, ws)
    assert ops.moe_get_device_status(ws) == 0
    r, keep = forward_reference(w, x, wr, b, W, act=1)
    assert keep.all()      # the small-batch router: routing replayed exactly
    assert max_abs_rel(dev_to_f64(out), r["out"]) < TOL


def test_fp8_shared_forward_full_size():
    """T=512, E=256 routed top-8 + one shared expert, FP8 W8A8 with dynamic
    per-tensor activation scales (all tokens: the h scale couples them)."""
    w = synth.workload("fp8_shared")
    W, Ws = oracle_bank(w)
    bank = device_bank(W)
    sbank = device_bank(Ws)
    x, wr, b = routed_inputs(w)
    ws = ops.new_workspace(ops.workspace_size(w.T, w.k, bank, sbank, 1))
    out = ops.moe_forward(bits_to_dev_bf16(x), bits_to_dev_bf16(wr), None, w.k, bank, sbank, 1, ws)
    assert ops.moe_get_device_status(ws) == 0
    r, keep = forward_reference(w, x, wr, b, W, Ws, act=1, what="fp8_shared")
    err = max_abs_rel(dev_to_f64(out)[keep], r["out"][keep])
    assert err < TOL, err


GATHER_CASES = [
    ("nvfp4-decode", dict(fmt="nvfp4", T=4, H=2048, E=128, k=8, I=768), True, 0.0),
    ("nvfp4-32", dict(fmt="nvfp4", T=32, H=512, E=32, k=4, I=256), True, 1.2),
    ("mxfp4-7", dict(fmt="mxfp4", T=7, H=512, E=6, k=2, I=256), False, 0.8),
]


@pytest.mark.parametrize("name,over,static,skew", GATHER_CASES)
def test_gathered_token_rows_change_nothing(name, over, static, skew):
    """Small batches (T <= 32): the one-kernel FFN copies each tile's token
    rows from the gather layout of x instead of loading quantised padded rows;
    y_perm is bit-identical to the two separate projections' and within the
    tolerance of the oracle."""
    ys = []
    try:
        ops.moe_set_option(ops.OPT_GATHER_X, 1)
        for fused in (0, 1):
            ops.moe_set_option(ops.OPT_FUSED_FFN, fused)
            w, W, x, perm, off, a13, a2, y, st = _run(over, static, skew, 2)
            assert st == 0, fused
            ys.append(y)
    finally:
        ops.moe_set_option(ops.OPT_FUSED_FFN, 1)
        ops.moe_set_option(ops.OPT_GATHER_X, 0)
    assert np.array_equal(ys[0], ys[1])
    ry, _ = oracle.grouped_ffn(x, perm, off, W, 1, a13 or 0.0, a2 or 0.0)
    assert max_abs_rel(ys[1], ry) < TOL
