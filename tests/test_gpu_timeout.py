"""Bounded device waits run out into a status code, not a hang.

Every wait in the tensor-core kernels (the TMA ring, the accumulator
hand-offs, the one-kernel FFN's wait for a token tile's gate|up slices) gives
up after MOE_OPT_WAIT_CYCLES SM clocks.  With the bound set to one cycle,
ordinary waits for memory run out: the call must still return, the device
status word must read MOE_ERR_TIMEOUT, the timed-out call's output must be
all zeros, and the next call on the same workspace, with the default bound,
must be clean and give the same bits as before.  Covered: the one-kernel
decode FFN, the 192-token grouped GEMMs on single CTAs, the CTA-pair
(cta_group::2) gate|up GEMM of a long K loop and the one-kernel router.
Nothing here faults or hangs the GPU: a wait that runs out sets a flag that
the kernel's other warps see, they leave their loops, the copies in flight
land and the tensor memory is freed before the kernel returns."""
import numpy as np
import pytest
import torch

from quantized_expert_ffn_top_b200 import ops, synth
from tests.gpu_helpers import bits_to_dev_bf16, device_bank, oracle_bank, routed_inputs

pytestmark = pytest.mark.gpu

MOE_ERR_TIMEOUT = 6

CASES = [
    # decode: T*k < 8E, the one-kernel FFN (NVFP4, static scales)
    ("decode-one-kernel", "decode", {}),
    # 192-token tiles, K = 2048 (8 stages): single-CTA GEMMs
    ("prefill-single-cta", "prefill", dict(T=512, E=16)),
    # K = 4096 (16 stages): the gate|up projection on CTA pairs
    ("prefill-cta-pairs", "tiny", dict(T=300, H=4096, E=8, k=2, I=512)),
    # 128-token tiles for half the SMs and more: the one-kernel router with top-k
    ("router-topk", "prefill", dict(T=9600)),
]


@pytest.mark.parametrize("name,base,over", CASES)
def test_wait_that_runs_out_sets_timeout_and_the_next_call_is_clean(name, base, over):
    assert torch.cuda.is_available()
    w = synth.workload(base, **over)
    W, _ = oracle_bank(w)
    a13, a2 = synth.static_act_scales()
    bank = device_bank(W, a13, a2)
    x, wr, b = routed_inputs(w)
    xd, wrd = bits_to_dev_bf16(x), bits_to_dev_bf16(wr)
    bd = None if b is None else torch.from_numpy(b).cuda()
    ws = ops.new_workspace(ops.workspace_size(w.T, w.k, bank, None, ops.ACT_MATCH))
    try:
        ops.moe_set_option(ops.OPT_FUSED_COMBINE, 0)   # the ordered combine (the default): bit-reproducible
        ref = ops.moe_forward(xd, wrd, bd, w.k, bank, None, ops.ACT_MATCH, ws)
        assert ops.moe_get_device_status(ws) == 0
        try:
            ops.moe_set_option(ops.OPT_WAIT_CYCLES, 1)
            bad = ops.moe_forward(xd, wrd, bd, w.k, bank, None, ops.ACT_MATCH, ws)
            torch.cuda.synchronize()            # the call returned and the kernels ended
            st = ops.moe_get_device_status(ws)
        finally:
            ops.moe_set_option(ops.OPT_WAIT_CYCLES, 0)
        assert st == MOE_ERR_TIMEOUT, st
        # the layer's output after a timeout: zeros, not whatever the
        # kernels that gave up left behind
        assert not bad.view(torch.int16).any()
        assert ops.moe_get_device_status(ws) == 0       # read and cleared
        out = ops.moe_forward(xd, wrd, bd, w.k, bank, None, ops.ACT_MATCH, ws)
        assert ops.moe_get_device_status(ws) == 0
    finally:
        ops.moe_set_option(ops.OPT_FUSED_COMBINE, 0)   # the default
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
