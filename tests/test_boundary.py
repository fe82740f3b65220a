"""The C-ABI library without a GPU: it loads, exports every function the
headers declare, and rejects bad arguments on the host before touching the
device.  (No compute call runs here.)"""
import ctypes
import glob
import os
import re

import pytest

from quantized_expert_ffn_top_b200 import build, ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return ops.lib()


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"\b(moe_[a-z0-9_]+)\s*\(", src):
            names.add(m.group(1))
    return names


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert {"moe_route", "moe_permute", "moe_grouped_ffn", "moe_combine", "moe_forward"} <= names
    for n in names:
        assert hasattr(L, n), n
    assert names == set(ops.EXPORTED)


def test_status_strings_and_version(L):
    for s in range(7):
        assert ops.status_string(s).startswith("MOE_")
    assert L.moe_version() >= 100


def _bank(fmt=1, E=8, H=128, I=256, layout=0, ptr=256):
    return ops.MoeWeightsC(fmt, E, H, I, layout, ptr, ptr, ptr, ptr, ptr, ptr, None, None)


def test_workspace_and_prepared_sizes(L):
    b = _bank()
    n = L.moe_workspace_size(8, 2, ctypes.byref(b), None, 1)
    assert n > 0 and n % 256 == 0
    assert L.moe_workspace_size(4096, 8, ctypes.byref(_bank(E=128, H=2048, I=768)), None, 1) > n
    assert L.moe_workspace_size(8, 2, ctypes.byref(_bank(fmt=7)), None, 1) == 0
    assert L.moe_workspace_size(8, 2, ctypes.byref(_bank(H=100)), None, 1) == 0
    p = L.moe_prepared_weights_size(ctypes.byref(b))
    # w13 8*512*64 + w2 8*128*128 + sf13 8*512*8 + sf2 8*128*16 bytes, 256-aligned pieces
    assert p >= 8 * 512 * 64 + 8 * 128 * 128 + 8 * 512 * 8 + 8 * 128 * 16
    # BF16 weights: no scales, two bytes an element
    bb = ops.MoeWeightsC(4, 8, 128, 256, 0, 256, None, None, 256, None, None, None, None)
    assert L.moe_workspace_size(8, 2, ctypes.byref(bb), None, 0) > 0
    assert L.moe_workspace_size(8, 2, ctypes.byref(bb), None, 1) > 0
    pb = L.moe_prepared_weights_size(ctypes.byref(bb))
    assert 8 * 512 * 256 + 8 * 128 * 512 <= pb < 8 * 512 * 256 + 8 * 128 * 512 + 4096
    # FP4 -> BF16 expansion: two bytes per weight; none for a BF16 bank
    d = L.moe_dequantized_weights_size(ctypes.byref(b))
    assert 2 * (8 * 512 * 128 + 8 * 128 * 256) <= d < 2 * (8 * 512 * 128 + 8 * 128 * 256) + 4096
    assert L.moe_dequantized_weights_size(ctypes.byref(bb)) == 0


def test_host_side_argument_errors(L):
    P = ctypes.c_void_p
    one = P(256)
    # k > E
    assert L.moe_route(one, 4, 128, one, None, 8, 9, None, one, one, one, 1 << 20, None) == ops.MoeError(1, "").status
    assert L.moe_route_logits(one, 4, 8, 0, one, one, one, 1 << 20, None) == 1
    # workspace too small
    assert L.moe_route_logits(one, 4, 8, 2, one, one, one, 16, None) == 3
    # unknown format / canonical bank where a prepared one is required
    b = _bank(fmt=9)
    assert L.moe_grouped_ffn(one, 4, 2, one, one, ctypes.byref(b), 1, one, one, 1 << 20, None) == 2
    c = _bank(layout=0)
    assert L.moe_forward(one, 4, one, None, 2, ctypes.byref(c), None, 1, one, one, 1 << 30, None) == 2
    # shape not a multiple of 128
    d = _bank(H=96, layout=1)
    assert L.moe_forward(one, 4, one, None, 2, ctypes.byref(d), None, 1, one, one, 1 << 30, None) == 2
    # quantize: K not a multiple of the block, unknown format
    assert L.moe_quantize(1, one, 0, 2, 24, None, one, one, None, one, 1 << 20, None) == 2
    assert L.moe_quantize(5, one, 0, 2, 32, None, one, one, None, one, 1 << 20, None) == 2
    assert L.moe_quantize(4, one, 0, 2, 24, None, one, None, None, one, 1 << 20, None) == 2  # BF16, K % 16
    # permute: E out of range
    assert L.moe_permute(one, 4, 2, 2000, one, one, one, one, 1 << 20, None) == 1
    assert L.moe_set_option(1, 5) == 1 and L.moe_set_option(99, 0) == 1
    assert L.moe_set_option(1, 0) == 0
    # token tile: 0 (by batch size), 64, 128, 192 or 256
    assert L.moe_set_option(2, 32) == 1 and L.moe_set_option(2, 96) == 1
    for v in (64, 128, 256, 0):
        assert L.moe_set_option(2, v) == 0
    # CTA pairs: off, on, for long K loops
    assert L.moe_set_option(3, 3) == 1 and L.moe_set_option(3, -1) == 1
    for v in (0, 1, 2):
        assert L.moe_set_option(3, v) == 0
    # early weight loads: 0, 1 or 2
    assert L.moe_set_option(5, 3) == 1 and L.moe_set_option(5, -1) == 1
    for v in (0, 2, 1):
        assert L.moe_set_option(5, v) == 0
    # fused FFN on or off
    assert L.moe_set_option(6, 2) == 1
    assert L.moe_set_option(6, 0) == 0 and L.moe_set_option(6, 1) == 0
    assert L.moe_set_option(7, 2) == 1 and L.moe_set_option(7, -1) == 1
    assert L.moe_set_option(7, 0) == 0 and L.moe_set_option(7, 1) == 0
    # combine: k beyond the 1024 the kernel stages
    assert L.moe_combine(one, one, one, 1, 1025, 8, None, one, one, 1 << 20, None) == 1
    # forward on host buffers: slice count, staging alignment, workspace for
    # one slice -- all rejected before anything is enqueued
    g = _bank(layout=1)
    host = ctypes.create_string_buffer(64 * 128 * 2)
    hp = ctypes.cast(host, P)

    def fh(T=64, n=4, xd=one, ws_bytes=1 << 30):
        return L.moe_forward_host(hp, T, one, None, 2, ctypes.byref(g), None, 1, hp, xd, one, n, one, ws_bytes,
                                  None)
    hdr = open(os.path.join(ROOT, "include", "moe_b200.h")).read()
    assert int(re.search(r"#define MOE_MAX_HOST_SLICES (\d+)", hdr).group(1)) == ops.MAX_HOST_SLICES
    assert fh(n=0) == 1 and fh(n=ops.MAX_HOST_SLICES + 1) == 1 and fh(T=-1) == 1
    assert fh(xd=P(258)) == 1
    one_slice = L.moe_workspace_size(16, 2, ctypes.byref(g), None, 1)
    assert fh(ws_bytes=one_slice - 1) == 3
    assert fh(T=0, ws_bytes=one_slice) == 0


def test_wait_bound_option(L):
    """MOE_OPT_WAIT_CYCLES: any positive cycle count, 0 restores the default,
    a negative count is rejected."""
    assert L.moe_set_option(ops.OPT_WAIT_CYCLES, -1) == 1
    assert L.moe_set_option(ops.OPT_WAIT_CYCLES, 1) == 0
    assert L.moe_set_option(ops.OPT_WAIT_CYCLES, 2 ** 31 - 1) == 0
    assert L.moe_set_option(ops.OPT_WAIT_CYCLES, 0) == 0
    hdr = open(os.path.join(ROOT, "include", "moe_b200.h")).read()
    assert re.search(r"MOE_OPT_WAIT_CYCLES = (\d+)", hdr).group(1) == str(ops.OPT_WAIT_CYCLES)


def test_switch_options_take_0_or_1_and_match_the_header(L):
    """The on/off switches added with the routing and small-batch paths
    accept 0 and 1, reject anything else, and carry the header's numbers;
    each is put back to its default."""
    hdr = open(os.path.join(ROOT, "include", "moe_b200.h")).read()
    defaults = {"FUSED_COMBINE": 0, "SMALL_BATCH_FORWARD": 0, "GATHER_X": 0, "FFN_SCHEDULE": 0, "ROUTER_TOPK": 1}
    for name, default in defaults.items():
        opt = getattr(ops, "OPT_" + name)
        assert re.search(r"^\s+MOE_OPT_%s = (\d+),?\s*$" % name, hdr, re.M).group(1) == str(opt), name
        assert L.moe_set_option(opt, 2) == 1 and L.moe_set_option(opt, -1) == 1, name
        assert L.moe_set_option(opt, 1 - default) == 0, name
        assert L.moe_set_option(opt, default) == 0, name


@pytest.mark.parametrize("E,H,I,k", [(128, 128, 256, 2), (256, 4096, 2048, 8), (8, 256, 256, 2)])
def test_workspace_size_never_decreases_with_T(L, E, H, I, k):
    """A workspace sized for T serves every smaller batch: moe_forward_host
    sizes one for its first slice and runs a shorter last slice in it.  The
    sweep crosses the batch sizes where the router's split of H changes."""
    b = _bank(E=E, H=H, I=I, layout=1)
    prev = 0
    for T in sorted(set(range(0, 300)) | set(range(300, 9000, 37)) | {4036, 4037, 4096, 4100, 16384, 16385}):
        n = L.moe_workspace_size(T, k, ctypes.byref(b), None, 1)
        assert n >= prev, (T, n, prev)
        prev = n


def test_host_slices_with_a_shorter_last_slice(L):
    """An uneven last slice that falls where the router's split is deeper than
    at the first slice's size: the workspace for ceil(T / n) tokens is
    accepted, and no slice needs more (checked by the host-side sizing
    before anything is enqueued)."""
    g = _bank(E=128, H=128, I=256, layout=1)
    T, n = 63 * 4100 + 4037, 64
    Ts = -(-T // n)
    ws_bytes = L.moe_workspace_size(Ts, 2, ctypes.byref(g), None, 1)
    assert ws_bytes >= L.moe_workspace_size(T - (n - 1) * Ts, 2, ctypes.byref(g), None, 1)
    P = ctypes.c_void_p
    one = P(256)
    host = P(4096)
    # one byte short is rejected on the host, before any CUDA call
    assert L.moe_forward_host(host, T, one, None, 2, ctypes.byref(g), None, 1, host, one, one, n, one,
                              ws_bytes - 1, None) == 3


def test_expert_cache_sizing(L):
    """moe_expert_cache_bytes: 0 for a canonical bank or a slot count outside
    1 .. min(E, 1024); otherwise at least the PREPARED bytes of n_slots
    experts, growing with n_slots."""
    prep = _bank(E=64, H=256, I=256, layout=1)
    assert L.moe_expert_cache_bytes(ctypes.byref(_bank(E=64, H=256, I=256, layout=0)), 8) == 0
    assert L.moe_expert_cache_bytes(ctypes.byref(prep), 0) == 0
    assert L.moe_expert_cache_bytes(ctypes.byref(prep), 65) == 0
    sizes = [L.moe_expert_cache_bytes(ctypes.byref(prep), n) for n in (1, 8, 32, 64)]
    assert all(s > 0 for s in sizes) and sizes == sorted(sizes) and len(set(sizes)) == 4
    for n, s in zip((1, 8, 32, 64), sizes):
        one = _bank(E=n, H=256, I=256, layout=1)
        assert s >= L.moe_prepared_weights_size(ctypes.byref(one))
