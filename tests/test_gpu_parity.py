"""CUDA path against the oracle, through the C ABI, on seeded inputs.

Integer and byte results (quantised codes and scales, routing indices,
offsets and permutations) must match bit for bit; floating-point outputs must
be within the layer's max-abs-relative bound of 2e-2 of the fp64 oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_expert_ffn_top_b200 import ops, synth
from tests.gpu_helpers import (TOL, ambiguous_tokens, bits_to_dev_bf16, dev_to_f64, device_bank,
                               forward_reference, max_abs_rel, oracle_bank, report_ambiguous, routed_inputs,
                               router_order, routing_tol)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    ops.lib()
    ops.moe_set_option(ops.OPT_FFN_PATH, 0)
    yield
    ops.moe_set_option(ops.OPT_FFN_PATH, 0)


def ws(nbytes=1 << 24):
    return ops.new_workspace(nbytes)


def route_ws_bytes(w) -> int:
    # moe_route's partial logits (up to 4 parts of T x E fp32) and the status words
    return max(1 << 24, 16 * w.T * w.E + (1 << 20))


# ----------------------------------------------------------- quantisers ----
def _all_finite_bf16_as_f32(limit=None):
    bits = np.arange(1 << 16, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    f = f[np.isfinite(f)]
    if limit is not None:
        f = f[np.abs(f) < limit]
    return f


def test_e4m3_conversion_matches_oracle_on_every_bf16():
    f = _all_finite_bf16_as_f32()
    n = (f.size // 16) * 16
    x = torch.from_numpy(f[:n].reshape(-1, 16)).cuda()
    codes, _, _ = ops.moe_quantize(ops.FMT_FP8, x, scale_in=torch.ones(1, device="cuda"))
    got = codes.cpu().numpy().reshape(-1)
    ref = np.array([oracle.e4m3_encode(float(v)) for v in f[:n]], np.uint8)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, f"{bad.size} mismatches, first: {f[bad[:5]]} got {got[bad[:5]]} ref {ref[bad[:5]]}"


def test_e2m1_conversion_matches_oracle_on_every_bf16_below_8():
    # blocks of 32 led by 4.0 have MXFP4 scale 2^0, so every element goes
    # through e2m1 rounding with multiplier 1
    f = _all_finite_bf16_as_f32(limit=8.0)
    per = 31
    nb = f.size // per
    blocks = np.zeros((nb, 32), np.float32)
    blocks[:, 0] = 4.0
    blocks[:, 1:] = f[:nb * per].reshape(nb, per)
    x = torch.from_numpy(blocks).cuda()
    codes, sf, _ = ops.moe_quantize(ops.FMT_MXFP4, x)
    assert np.all(sf.cpu().numpy() == 127)
    c = codes.cpu().numpy()
    nib = np.empty((nb, 32), np.uint8)
    nib[:, 0::2] = c & 15
    nib[:, 1::2] = c >> 4
    ref = np.array([oracle.e2m1_encode(float(v)) for v in blocks[:, 1:].reshape(-1)], np.uint8).reshape(nb, per)
    bad = np.nonzero(nib[:, 1:] != ref)
    assert bad[0].size == 0, f"{bad[0].size} mismatches: {blocks[:, 1:][bad][:5]} got {nib[:, 1:][bad][:5]}"


@pytest.mark.parametrize("fmt", ["nvfp4", "mxfp4", "fp8", "bf16"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("static", [False, True])
def test_quantize_matches_oracle(fmt, dtype, static):
    rng = np.random.default_rng(11)
    rows, K = 96, 512
    xf = (rng.standard_normal((rows, K)) * rng.uniform(1e-3, 30, (rows, 1))).astype(np.float32)
    xf[7, 64:96] = 0.0
    xf[9, :] = 0.0
    if dtype == "bf16":
        bits = synth.to_bf16_bits(xf)
        xf = (bits.astype(np.uint32) << 16).view(np.float32)
        xd = bits_to_dev_bf16(bits)
    else:
        xd = torch.from_numpy(xf).cuda()
    f = {"nvfp4": 1, "mxfp4": 2, "fp8": 3, "bf16": 4}[fmt]
    scale = 0.0123 if static else None
    sd = torch.tensor([scale], dtype=torch.float32, device="cuda") if static else None
    codes, sf, s_used = ops.moe_quantize(f, xd, scale_in=sd)
    if f == 1:
        g = scale if static else oracle.nvfp4_global_scale(oracle.amax(xf))
        rc, rs = oracle.quant_nvfp4(xf, g)
    elif f == 2:
        g = 1.0
        rc, rs = oracle.quant_mxfp4(xf)
    elif f == 4:
        g = 1.0
        rc, rs = oracle.quant_bf16(xf), None
    else:
        g = scale if static else oracle.fp8_scale(oracle.amax(xf))
        rc, rs = oracle.quant_fp8(xf, g), None
    assert np.array_equal(codes.cpu().numpy(), rc)
    if rs is not None:
        assert np.array_equal(sf.cpu().numpy(), rs)
    if f != 2:
        assert float(s_used.item()) == np.float32(g)
    if f == 4:
        assert sf is None


# --------------------------------------------------------------- routing ----
@pytest.mark.parametrize("T,E,k", [(1, 8, 2), (37, 128, 8), (300, 256, 8), (5, 1024, 16), (9, 7, 7), (64, 40, 1)])
def test_route_logits_bit_exact(T, E, k):
    L = synth.random_logits(T, E, kind="uniform" if E != 40 else "normal")
    L[0, :] = L[0, 0]  # a row of equal logits
    idx, w = ops.moe_route_logits(torch.from_numpy(L).cuda(), k, ws())
    ridx, rw, st = oracle.topk(L.astype(np.float64), k)
    assert st == 0
    assert np.array_equal(idx.cpu().numpy(), ridx)
    assert np.allclose(w.cpu().numpy(), rw, rtol=2e-6, atol=1e-7)


def test_route_logits_flags_invalid_rows():
    L = np.zeros((4, 16), np.float32)
    L[1, 3] = np.nan
    L[2, :] = -np.inf
    L[3, 5] = -np.inf
    W = ws()
    idx, w = ops.moe_route_logits(torch.from_numpy(L).cuda(), 4, W)
    assert ops.moe_get_device_status(W) == ops.MoeError(5, "").status
    assert ops.moe_get_device_status(W) == 0  # cleared
    wn = w.cpu().numpy()
    assert np.all(wn[1] == 0) and np.all(wn[2] == 0)
    assert np.allclose(wn[3], 0.25)


ROUTE_CASES = [("tiny", {}), ("decode", {}), ("prefill", {}), ("large", dict(T=300)), ("fp8_shared", dict(T=130)),
               # small batches: the fixed small-batch order, Zipf bias, H = 4096 (two stretches),
               # H = 2304 (a ragged second stretch), one token
               ("prefill", dict(T=64)), ("large", dict(T=37)), ("decode", dict(T=9, H=2304, E=60, k=4)),
               ("large", dict(T=1)),
               # the sequential order: 64 < T < 128, or E off the tensor-core grid
               ("decode", dict(T=100)), ("prefill", dict(T=300, E=60, k=4)), ("tiny", dict(T=200)),
               ("prefill", dict(T=129, E=48, k=6)), ("prefill", dict(T=1000, E=32, k=16)),
               ("prefill", dict(T=257, E=16, k=1)),
               # the router GEMM: E = 256 with a ragged tile; k = 17
               ("large", dict(T=700)), ("prefill", dict(T=300, E=128, k=17)),
               # the one-kernel router with top-k (128-token tiles for half the
               # SMs and more): ragged last tile with small E, k = 16 (the most
               # it takes)
               ("prefill", dict(T=9600, k=4)), ("prefill", dict(T=9601, E=48, k=6)),
               ("prefill", dict(T=9500, E=32, k=16))]


@pytest.mark.parametrize("name,over", ROUTE_CASES)
def test_route_matches_oracle(name, over):
    """Small batches and shapes off the tensor-core grid sum the logits in a
    fixed fp32 order that the oracle replays: logits, indices and the
    selection are then bit-exact on every token.  Larger batches use the
    tcgen05 bf16 GEMM: its logits are within rounding of the fp64 ones, and
    the indices match on every token whose k/k+1 gap exceeds twice the
    largest logit difference seen (those left out are counted and bounded)."""
    w = synth.workload(name, **over)
    x, wr, b = routed_inputs(w)
    logits = torch.empty((w.T, w.E), dtype=torch.float32, device="cuda")
    idx, wt = ops.moe_route(bits_to_dev_bf16(x), bits_to_dev_bf16(wr),
                            None if b is None else torch.from_numpy(b).cuda(), w.k, ws(route_ws_bytes(w)),
                            logits=logits)
    gl = logits.cpu().numpy()
    gi = idx.cpu().numpy()
    order = router_order(w.T, w.E, w.H, w.k)
    RL = oracle.router_logits(x, wr, b)
    assert max_abs_rel(gl.astype(np.float64), RL) < 1e-5
    if order:
        OL = oracle.router_logits_ordered(x, wr, b, order=order)
        assert np.array_equal(gl, OL), f"order {order}: {np.sum(gl != OL)} logits differ"
        ridx, rw, st = oracle.topk(OL.astype(np.float64), w.k)
        assert st == 0
        assert np.array_equal(gi, ridx)
        assert np.allclose(wt.cpu().numpy(), rw, rtol=2e-6, atol=1e-7)
        return
    ridx, rw, _ = oracle.topk(RL, w.k)
    amb = ambiguous_tokens(RL, w.k, routing_tol(RL, gl))
    report_ambiguous(amb, f"route {name} {over}")
    assert np.array_equal(gi[~amb], ridx[~amb])
    assert np.allclose(wt.cpu().numpy()[~amb], rw[~amb], rtol=1e-4, atol=1e-6)
    # ambiguous tokens: still k distinct experts, ordered by the GPU's logits
    for t in np.nonzero(amb)[0]:
        assert len(set(gi[t])) == w.k
        assert np.all(np.diff(gl[t, gi[t]].astype(np.float64)) <= 0)


ROUTER_TOPK_CASES = [("prefill", dict(T=9600)), ("large", dict(T=10240)), ("prefill", dict(T=9601, E=48, k=6)),
                     ("prefill", dict(T=9500, E=32, k=16))]


@pytest.mark.parametrize("name,over", ROUTER_TOPK_CASES)
def test_router_topk_kernel_agrees_with_router_gemm(name, over):
    """The one-kernel router (all of H in one accumulator, top-k in the
    epilogue) against the two-kernel router (logits, then the top-k kernel):
    logits within fp32 rounding of each other; indices and weights equal on
    every token whose top-k order the difference cannot flip."""
    w = synth.workload(name, **over)
    x, wr, b = routed_inputs(w)
    xd, wrd = bits_to_dev_bf16(x), bits_to_dev_bf16(wr)
    bd = None if b is None else torch.from_numpy(b).cuda()
    res = []
    try:
        for opt in (0, 1):
            ops.moe_set_option(ops.OPT_ROUTER_TOPK, opt)
            logits = torch.empty((w.T, w.E), dtype=torch.float32, device="cuda")
            W = ws(route_ws_bytes(w))
            n0 = ops.moe_kernel_launch_count()
            idx, wt = ops.moe_route(xd, wrd, bd, w.k, W, logits=logits)
            n = ops.moe_kernel_launch_count() - n0
            assert ops.moe_get_device_status(W) == 0
            res.append((logits.cpu().numpy().astype(np.float64), idx.cpu().numpy(), wt.cpu().numpy(), n))
    finally:
        ops.moe_set_option(ops.OPT_ROUTER_TOPK, 1)
    (l0, i0, w0, n0_), (l1, i1, w1, n1_) = res
    assert n1_ == 1 and n0_ == 2, (n0_, n1_)
    RL = oracle.router_logits(x, wr, b)
    assert max_abs_rel(l1, RL) < 1e-5 and max_abs_rel(l0, RL) < 1e-5
    amb = ambiguous_tokens(l0, w.k, 2.0 * float(np.max(np.abs(l1 - l0))) + 1e-7)
    report_ambiguous(amb, f"router_topk {name} {over}")
    assert np.array_equal(i1[~amb], i0[~amb])
    assert np.allclose(w1[~amb], w0[~amb], rtol=1e-4, atol=1e-6)
    # every token: k distinct experts, descending in the kernel's own logits
    assert all(len(set(r)) == w.k for r in i1)
    assert np.all(np.diff(np.take_along_axis(l1, i1.astype(np.int64), 1), axis=1) <= 0)


# ----------------------------------------------------------- permutation ----
@pytest.mark.parametrize("T,k,E,skew", [(8, 2, 8, 0.0), (4, 8, 128, 0.0), (4096, 8, 128, 1.1), (16384, 8, 256, 1.1),
                                        (777, 1, 1, 0.0), (50, 16, 1024, 0.3), (3000, 5, 37, 2.0),
                                        # one-block path up to 8192 slots, then the three-pass path
                                        (1000, 8, 256, 1.1), (1024, 8, 256, 0.0), (1025, 8, 256, 0.0)])
def test_permute_bit_exact(T, k, E, skew):
    if k > E:
        pytest.skip("k > E")
    idx = synth.random_topk_idx(T, k, E, skew=skew) if E > 1 else np.zeros((T, k), np.int32)
    off, perm, inv = ops.moe_permute(torch.from_numpy(idx).cuda(), E, ws(1 << 26))
    roff, rperm, rinv, st = oracle.permute(idx, E)
    assert st == 0
    assert np.array_equal(off.cpu().numpy(), roff)
    assert np.array_equal(perm.cpu().numpy(), rperm)
    assert np.array_equal(inv.cpu().numpy(), rinv)


def test_permute_empty_and_bad_index():
    W = ws()
    off, _, _ = ops.moe_permute(torch.zeros((0, 4), dtype=torch.int32, device="cuda"), 6, W)
    assert not off.cpu().numpy().any()
    idx = np.array([[0, 1], [2, 9]], np.int32)
    off, perm, inv = ops.moe_permute(torch.from_numpy(idx).cuda(), 4, W)
    assert ops.moe_get_device_status(W) == 5
    assert inv.cpu().numpy()[3] == -1
    assert off.cpu().numpy()[-1] == 3


# ------------------------------------------------------------ grouped FFN ----
FFN_CASES = [
    ("tiny", {}, 0), ("tiny", {}, 1), ("tiny", {}, 2),
    ("decode", {}, 0), ("decode", {}, 1),
    ("tiny", dict(fmt="mxfp4", H=256, I=256, E=4, k=2, T=6), 0),
    ("tiny", dict(fmt="mxfp4", H=256, I=256, E=4, k=2, T=6), 1),
    ("tiny", dict(fmt="fp8", H=256, I=128, E=8, k=2, T=10), 0),
    ("tiny", dict(fmt="fp8", H=256, I=128, E=8, k=2, T=10), 1),
    ("tiny", dict(T=40, E=4, k=2, H=128, I=128), 1),       # > 8 tokens per expert
    # K = 128 mod 256: the streamed FP4 rows end on half a 128-byte chunk
    ("tiny", dict(fmt="mxfp4", H=384, I=384, E=6, k=2, T=20), 1),
    ("tiny", dict(H=384, I=640, E=5, k=3, T=33), 1),
    ("tiny", dict(fmt="fp8", H=384, I=640, E=5, k=3, T=33), 1),
]


@pytest.mark.parametrize("name,over,mode", FFN_CASES)
def test_grouped_ffn_matches_oracle(name, over, mode):
    """mode 0 = BF16 activations, 1 = MATCH dynamic scales, 2 = MATCH static."""
    w = synth.workload(name, **over)
    W, _ = oracle_bank(w)
    a13, a2 = synth.static_act_scales() if mode == 2 else (None, None)
    bank = device_bank(W, a13, a2)
    idx = synth.random_topk_idx(w.T, w.k, w.E, skew=0.5)
    off, perm, inv, _ = oracle.permute(idx, w.E)
    x = synth.x_bits(w)
    act = 0 if mode == 0 else 1
    y = ops.moe_grouped_ffn(bits_to_dev_bf16(x), w.k, torch.from_numpy(perm).cuda(), torch.from_numpy(off).cuda(),
                            bank, act, ws(ops.workspace_size(w.T, w.k, bank, None, act)))
    ry, _ = oracle.grouped_ffn(x, perm, off, W, act, a13 or 0.0, a2 or 0.0)
    err = max_abs_rel(dev_to_f64(y), ry)
    assert err < TOL, err


def test_combine_matches_oracle():
    T, k, H = 33, 4, 256
    rng = np.random.default_rng(12)
    S = T * k
    y = synth.to_bf16_bits(rng.standard_normal((S, H)).astype(np.float32))
    sh = synth.to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    inv = rng.permutation(S).astype(np.int32)
    w = rng.dirichlet(np.ones(k), size=T).astype(np.float32)
    W = ws()
    out = ops.moe_combine(bits_to_dev_bf16(y), torch.from_numpy(inv).cuda(), torch.from_numpy(w).cuda(), W,
                          shared_y=bits_to_dev_bf16(sh))
    yf = (y.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    shf = (sh.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ref = oracle.combine(yf, inv, w.astype(np.float64), k, shf)
    got = dev_to_f64(out)
    # one bf16 rounding of the fp32 sum
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2 ** -8 + 1e-6)
    assert ops.moe_get_device_status(W) == 0


# --------------------------------------------------------------- forward ----
FWD_CASES = [
    ("tiny", {}, 1, False), ("tiny", {}, 0, False), ("tiny", {}, 1, True),
    ("decode", {}, 1, False), ("decode", {}, 0, False), ("decode", {}, 1, True),
    ("fp8_shared", dict(T=24, H=256, E=16, k=4, I=128, shared_I=128), 1, False),
    ("tiny", dict(fmt="mxfp4", T=12, H=256, E=8, k=2, I=256), 1, False),
    # H = 2048 + 256: the per-token x quantiser's second stretch is ragged
    ("tiny", dict(T=40, H=2304, E=8, k=3, I=256), 1, False),
    ("tiny", dict(fmt="fp8", T=40, H=2176, E=8, k=3, I=256), 1, False),
    # BF16 expert weights (tensor cores, kind::f16) in both activation modes,
    # a shared expert, and a prefill-sized batch with Zipf routing
    ("tiny", dict(fmt="bf16"), 1, False), ("tiny", dict(fmt="bf16"), 0, False),
    ("tiny", dict(fmt="bf16", T=24, H=256, E=16, k=4, I=128, shared_I=128), 1, False),
    ("prefill", dict(fmt="bf16", T=512, H=512, E=32, k=4, I=256), 1, False),
    # degenerate layers: one expert (k = 1), every expert picked (k = E), one token
    ("tiny", dict(E=1, k=1, T=16), 1, False), ("tiny", dict(E=4, k=4, T=33), 1, False),
    ("tiny", dict(T=1), 1, False),
    # a shared expert beside the one-kernel FFN at small batches: two
    # persistent FFN kernels (routed, shared) run at once on two streams, so
    # neither has every SM to itself
    ("decode", dict(shared_I=768), 1, True),
    ("tiny", dict(fmt="mxfp4", T=6, H=256, E=8, k=2, I=256, shared_I=256), 1, False),
]


@pytest.mark.parametrize("name,over,act,static", FWD_CASES)
def test_forward_matches_oracle(name, over, act, static):
    w = synth.workload(name, **over)
    W, Ws = oracle_bank(w)
    a13, a2 = synth.static_act_scales() if static else (None, None)
    bank = device_bank(W, a13, a2)
    sbank = device_bank(Ws, None, a2) if Ws is not None else None
    x, wr, b = routed_inputs(w)
    W_ = ws(ops.workspace_size(w.T, w.k, bank, sbank, act))
    out = ops.moe_forward(bits_to_dev_bf16(x), bits_to_dev_bf16(wr), None if b is None else torch.from_numpy(b).cuda(),
                          w.k, bank, sbank, act, W_)
    assert ops.moe_get_device_status(W_) == 0
    r, keep = forward_reference(w, x, wr, b, W, Ws, act=act, a13=a13, a2=a2, sh_a2=a2, what=f"{name} {over}")
    err = max_abs_rel(dev_to_f64(out)[keep], r["out"][keep])
    assert err < TOL, err


# small batches (T <= 8) on the one-kernel FFN (tensor-core shapes: H and I
# multiples of 256): x quantised inside the permutation kernel (NVFP4 static
# and dynamic x scales; MXFP4 with a ragged second 2048-value stretch and at
# E = 256; a single slot)
PERM_QUANT_CASES = [
    ("decode", {}, "static"),
    ("tiny", dict(H=256), "h-static"),
    ("tiny", dict(fmt="mxfp4", T=7, H=256, E=8, k=2, I=256), "none"),
    ("tiny", dict(fmt="mxfp4", T=8, H=2304, E=32, k=2, I=256), "none"),
    ("tiny", dict(fmt="mxfp4", T=8, H=256, E=256, k=8, I=256), "none"),
    ("tiny", dict(T=1, k=1, E=8, H=256), "static"),
]


@pytest.mark.parametrize("name,over,scales", PERM_QUANT_CASES)
def test_permutation_with_x_quantisation_changes_nothing(name, over, scales):
    """The permutation kernel that also quantises x (and the FFN kernel that
    then takes its tile list from the top-k ids) gives the bits of the
    separate x quantiser, with one kernel launch fewer."""
    w = synth.workload(name, **over)
    W, _ = oracle_bank(w)
    a13, a2 = synth.static_act_scales()
    if scales == "h-static":
        a13 = None
    elif scales == "none":
        a13 = a2 = None
    bank = device_bank(W, a13, a2)
    x, wr, b = routed_inputs(w)
    xd, wrd = bits_to_dev_bf16(x), bits_to_dev_bf16(wr)
    bd = None if b is None else torch.from_numpy(b).cuda()
    W_ = ws(ops.workspace_size(w.T, w.k, bank, None, 1))
    outs, launches = [], []
    try:
        ops.moe_set_option(ops.OPT_SMALL_BATCH_FORWARD, 0)   # the permutation path
        for opt in (0, 1):
            ops.moe_set_option(ops.OPT_PERMUTE_QUANT, opt)
            n0 = ops.moe_kernel_launch_count()
            out = ops.moe_forward(xd, wrd, bd, w.k, bank, None, 1, W_)
            launches.append(ops.moe_kernel_launch_count() - n0)
            assert ops.moe_get_device_status(W_) == 0, opt
            outs.append(out.view(torch.int16).cpu().numpy())
    finally:
        ops.moe_set_option(ops.OPT_PERMUTE_QUANT, 1)
    assert np.array_equal(outs[0], outs[1])
    assert launches[1] == launches[0] - 1, launches
    r, keep = forward_reference(w, x, wr, b, W, act=1, a13=a13, a2=a2)
    assert keep.all()
    got = outs[1].view(np.uint16).astype(np.uint32) << 16
    err = max_abs_rel(got.view(np.float32).astype(np.float64)[keep], r["out"][keep])
    assert err < TOL, err


# the layer on host buffers: token slices (static scales; a ragged last
# slice), and one slice when the x scale depends on the batch
HOST_CASES = [
    ("tiny", dict(T=40, H=256, E=8, k=2, I=256), "static", 4),
    ("tiny", dict(T=37, H=256, E=16, k=4, I=256), "static", 5),
    ("tiny", dict(T=24, H=256, E=8, k=2, I=256), "none", 3),
]


@pytest.mark.parametrize("name,over,scales,n_slices", HOST_CASES)
def test_forward_on_host_buffers_matches_oracle(name, over, scales, n_slices):
    """moe_forward_host: slices copied in, run and copied out on three
    streams give the oracle's layer output, with a workspace sized for one
    slice."""
    w = synth.workload(name, **over)
    W, _ = oracle_bank(w)
    a13, a2 = synth.static_act_scales() if scales == "static" else (None, None)
    bank = device_bank(W, a13, a2)
    x, wr, b = routed_inputs(w)
    Ts = -(-w.T // n_slices) if scales == "static" else w.T
    W_ = ws(ops.workspace_size(Ts, w.k, bank, None, 1))
    x_host = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).pin_memory()
    x_dev = torch.empty((w.T, w.H), dtype=torch.bfloat16, device="cuda")
    out_dev = torch.empty_like(x_dev)
    bd = None if b is None else torch.from_numpy(b).cuda()
    out = ops.moe_forward_host(x_host, bits_to_dev_bf16(wr), bd, w.k, bank, None, 1, W_, x_dev, out_dev,
                               n_slices=n_slices)
    torch.cuda.synchronize()
    assert ops.moe_get_device_status(W_) == 0
    assert torch.equal(out_dev.cpu(), out)
    r, keep = forward_reference(w, x, wr, b, W, act=1, a13=a13, a2=a2, route_T=Ts)
    err = max_abs_rel(out.float().numpy().astype(np.float64)[keep], r["out"][keep])
    assert err < TOL, err


def test_forward_and_ffn_with_no_tokens():
    """T = 0: every entry point returns success and writes nothing."""
    w = synth.workload("tiny")
    W, _ = oracle_bank(w)
    bank = device_bank(W)
    x = torch.zeros((0, w.H), dtype=torch.bfloat16, device="cuda")
    wr = bits_to_dev_bf16(synth.router_bits(w))
    W_ = ws(ops.workspace_size(0, w.k, bank, None, 1))
    out = ops.moe_forward(x, wr, None, w.k, bank, None, 1, W_)
    assert out.shape == (0, w.H)
    off = torch.zeros(w.E + 1, dtype=torch.int32, device="cuda")
    perm = torch.zeros(0, dtype=torch.int32, device="cuda")
    y = ops.moe_grouped_ffn(x, w.k, perm, off, bank, 1, W_)
    assert y.shape == (0, w.H)
    torch.cuda.synchronize()
    assert ops.moe_get_device_status(W_) == 0


# the weighted combine in the down projection's epilogue (fp32 reductions)
# against the ordered combine of bf16 y_perm, and both against the oracle:
# NVFP4 prefill-shaped batches (192-token tiles, single CTAs and CTA pairs),
# MXFP4, and FP8 with a shared expert adding into the same rows
FUSED_COMBINE_CASES = [
    ("prefill", dict(T=600, E=32), True),
    ("tiny", dict(T=300, H=4096, E=8, k=2, I=512), True),
    ("tiny", dict(fmt="mxfp4", T=200, H=512, E=8, k=2, I=256), False),
    ("fp8_shared", dict(T=160, H=256, E=16, k=4, I=128, shared_I=128), False),
]


@pytest.mark.parametrize("name,over,static", FUSED_COMBINE_CASES)
def test_combine_in_down_epilogue_matches_ordered_combine(name, over, static):
    w = synth.workload(name, **over)
    W, Ws = oracle_bank(w)
    a13, a2 = synth.static_act_scales() if static else (None, None)
    bank = device_bank(W, a13, a2)
    sbank = device_bank(Ws, None, a2) if Ws is not None else None
    x, wr, b = routed_inputs(w)
    xd, wrd = bits_to_dev_bf16(x), bits_to_dev_bf16(wr)
    bd = None if b is None else torch.from_numpy(b).cuda()
    W_ = ws(ops.workspace_size(w.T, w.k, bank, sbank, 1))
    outs = []
    try:
        for fused in (0, 1):
            ops.moe_set_option(ops.OPT_FUSED_COMBINE, fused)
            n0 = ops.moe_kernel_launch_count()
            o = ops.moe_forward(xd, wrd, bd, w.k, bank, sbank, 1, W_)
            assert ops.moe_get_device_status(W_) == 0, fused
            outs.append(dev_to_f64(o))
    finally:
        ops.moe_set_option(ops.OPT_FUSED_COMBINE, 0)   # the default
    # apart by the bf16 rounding of y_perm and of each output (a few bf16
    # ulps of the largest output), half the layer tolerance at most
    assert max_abs_rel(outs[1], outs[0]) < 1e-2
    r, keep = forward_reference(w, x, wr, b, W, Ws, act=1, a13=a13, a2=a2, sh_a2=a2, what=f"{name} {over}")
    for o in outs:
        assert max_abs_rel(o[keep], r["out"][keep]) < TOL


# small batches in two kernels (router with x quantisation and top-k; the
# FFN gathering token rows, combining in its down epilogue and rounding in
# its last CTA) against the permutation path, and both against the oracle on
# every token (the small-batch router's order is replayed exactly)
SMALL_FORWARD_CASES = [
    ("decode", {}, "static"), ("decode", dict(T=1), "static"), ("decode", dict(T=32), "static"),
    ("decode", dict(T=9, E=256), "h-static"),
    ("tiny", dict(fmt="mxfp4", T=16, H=512, E=8, k=2, I=256), "none"),
    ("tiny", dict(fmt="mxfp4", T=5, H=2304, E=64, k=4, I=512), "none"),
]


@pytest.mark.parametrize("name,over,scales", SMALL_FORWARD_CASES)
def test_small_batch_forward_in_two_kernels(name, over, scales):
    w = synth.workload(name, **over)
    W, _ = oracle_bank(w)
    a13, a2 = synth.static_act_scales()
    if scales == "h-static":
        a13 = None
    elif scales == "none":
        a13 = a2 = None
    bank = device_bank(W, a13, a2)
    x, wr, b = routed_inputs(w)
    xd, wrd = bits_to_dev_bf16(x), bits_to_dev_bf16(wr)
    bd = None if b is None else torch.from_numpy(b).cuda()
    W_ = ws(ops.workspace_size(w.T, w.k, bank, None, 1))
    outs, launches = [], []
    try:
        ops.moe_set_option(ops.OPT_GATHER_X, 1)
        for opt in (0, 1):
            ops.moe_set_option(ops.OPT_SMALL_BATCH_FORWARD, opt)
            n0 = ops.moe_kernel_launch_count()
            o = ops.moe_forward(xd, wrd, bd, w.k, bank, None, 1, W_)
            launches.append(ops.moe_kernel_launch_count() - n0)
            assert ops.moe_get_device_status(W_) == 0, opt
            outs.append(dev_to_f64(o))
    finally:
        ops.moe_set_option(ops.OPT_SMALL_BATCH_FORWARD, 0)
        ops.moe_set_option(ops.OPT_GATHER_X, 0)
    assert launches[1] == (3 if a13 is None and w.fmt == "nvfp4" else 2), launches
    assert max_abs_rel(outs[1], outs[0]) < 1e-2
    r, keep = forward_reference(w, x, wr, b, W, act=1, a13=a13, a2=a2)
    assert keep.all()
    for o in outs:
        assert max_abs_rel(o, r["out"]) < TOL
