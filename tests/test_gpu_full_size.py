"""The large prefill layer at its full size against the oracle, through the
C ABI, in the configuration the benchmark times: T=16384 tokens, hidden 4096,
256 experts, top-8, intermediate 2048, MXFP4 weights and activations (W4A4),
Zipf(1.1) routing -- about 3.4 GB of expert weights and an E=256, 16384-token
tile schedule with CTA-pair gate|up tiles and 28x expert skew.

* every one of the 16384 x 8 routing indices, against the fp64 oracle's
  top-k (tokens whose k/k+1 logit gap lies within the router's own rounding
  are counted, bounded below 1 % and checked for validity instead);
* the layer output of 512 evenly spaced tokens, element by element within
  the 2e-2 max-abs-relative bound.  MXFP4 has no tensor-wide scale, so the
  tokens are independent and a subset is exact.

The bank is drawn and quantised by the oracle on the host, one expert per
thread, then uploaded and prepared by the library."""
import os

import numpy as np
import pytest
import torch

import oracle
from quantized_expert_ffn_top_b200 import ops, synth
from tests.gpu_helpers import (TOL, ambiguous_tokens, bits_to_dev_bf16, dev_to_f64, device_bank, max_abs_rel,
                               report_ambiguous, routed_inputs, routing_tol)

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def large_layer():
    assert torch.cuda.is_available()
    w = synth.workload("large")
    threads = max(1, os.cpu_count() or 1)
    W = oracle.quantize_expert_weights_by_expert(oracle.FMT_MXFP4, w.E, lambda e: synth.expert_w13(w, e),
                                                 lambda e: synth.expert_w2(w, e), threads=threads)
    bank = device_bank(W)
    torch.cuda.synchronize()
    yield w, W, bank
    del bank
    torch.cuda.empty_cache()


def test_large_layer_full_size(large_layer):
    w, W, bank = large_layer
    ops.moe_set_option(ops.OPT_FFN_PATH, 0)
    x, wr, b = routed_inputs(w)
    xd, wrd, bd = bits_to_dev_bf16(x), bits_to_dev_bf16(wr), torch.from_numpy(b).cuda()
    # routing of every token
    logits = torch.empty((w.T, w.E), dtype=torch.float32, device="cuda")
    idx, _ = ops.moe_route(xd, wrd, bd, w.k, ops.new_workspace(w.T * w.E * 16 + (1 << 20)), logits=logits)
    gl = logits.cpu().numpy()
    gi = idx.cpu().numpy()
    RL = oracle.router_logits(x, wr, b)
    assert max_abs_rel(gl.astype(np.float64), RL) < 1e-5
    ridx, _, st = oracle.topk(RL, w.k)
    assert st == 0
    amb = ambiguous_tokens(RL, w.k, routing_tol(RL, gl))
    report_ambiguous(amb, "large layer routing (all 16384 tokens)")
    assert np.array_equal(gi[~amb], ridx[~amb])
    for t in np.nonzero(amb)[0]:
        assert len(set(gi[t])) == w.k
        assert np.all(np.diff(gl[t, gi[t]].astype(np.float64)) <= 0)
    counts = np.bincount(gi.reshape(-1), minlength=w.E)
    print(f"large layer routing: max/mean {counts.max() / counts.mean():.1f}, min {counts.min()}")
    # the layer
    ws = ops.new_workspace(ops.workspace_size(w.T, w.k, bank, None, ops.ACT_MATCH))
    out = ops.moe_forward(xd, wrd, bd, w.k, bank, None, ops.ACT_MATCH, ws)
    assert ops.moe_get_device_status(ws) == 0
    toks = np.linspace(0, w.T - 1, 512).astype(np.int32)
    r = oracle.moe_forward(x, wr, b, w.k, W, act=oracle.ACT_MATCH, tokens=toks)
    keep = ~ambiguous_tokens(r["logits"], w.k, routing_tol(r["logits"], gl[toks]), boundary_only=True)
    got = dev_to_f64(out)[toks]
    err = max_abs_rel(got[keep], r["out"][keep])
    print(f"large layer output, {int(keep.sum())} of 512 tokens: max-abs-rel {err:.3e}")
    assert err < TOL, err
    # per token too: no token's row may be far off (a wrong tile would show here)
    for i in np.nonzero(keep)[0]:
        assert max_abs_rel(got[i], r["out"][i]) < 5 * TOL, int(toks[i])
