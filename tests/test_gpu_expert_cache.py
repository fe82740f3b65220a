"""Host -> HBM expert streaming: the layer through an LRU pool of expert slots
in HBM smaller than the bank, whose experts live in page-locked host memory.

* every batch's output equals the whole-bank forward's (within rounding of
  the combine) and the oracle's (routing replayed exactly at small batches);
* the counters (experts fetched per call, hits) equal those of the pool's
  stated policy replayed on the host by the oracle's model
  (oracle/slot_pool.py): the batch's resident experts are hits,
  every other one takes, in expert order, the next slot of the ordering
  "empty slots, then least recently used, ties to the lower slot", among the
  slots no expert of this batch holds;
* batches that route to more distinct experts than the pool holds in all
  evict and re-fetch."""
import numpy as np
import pytest
import torch

import oracle
from oracle.slot_pool import SlotPool
from quantized_expert_ffn_top_b200 import ops, synth
from tests.gpu_helpers import (TOL, bits_to_dev_bf16, dev_to_f64, device_bank, forward_reference, max_abs_rel,
                               oracle_bank)

pytestmark = pytest.mark.gpu


CASES = [
    # name, layer, slots, static scales, batches
    ("nvfp4-decode", dict(fmt="nvfp4", T=4, H=256, E=64, k=4, I=256), 24, True, 6),
    ("mxfp4-small", dict(fmt="mxfp4", T=6, H=512, E=40, k=2, I=256), 16, False, 6),
    ("nvfp4-64tok", dict(fmt="nvfp4", T=40, H=256, E=96, k=2, I=256), 80, True, 4),
    ("fp8-gemm", dict(fmt="fp8", T=128, H=256, E=16, k=2, I=128), 16, False, 2),
]


@pytest.mark.parametrize("name,over,n_slots,static,batches", CASES)
def test_forward_through_the_slot_pool(name, over, n_slots, static, batches):
    assert torch.cuda.is_available()
    w = synth.workload("tiny", **over)
    W, _ = oracle_bank(w)
    a13, a2 = synth.static_act_scales() if static else (None, None)
    dbank = device_bank(W, a13, a2)
    hbank = ops.bank_to_host(dbank)
    cache = ops.moe_expert_cache_init(hbank, n_slots)
    wr = synth.router_bits(w)
    wrd = bits_to_dev_bf16(wr)
    ws_c = ops.new_workspace(ops.workspace_size(w.T, w.k, hbank, None, 1))
    ws_d = ops.new_workspace(ops.workspace_size(w.T, w.k, dbank, None, 1))
    mirror = SlotPool(w.E, n_slots)
    fetched_total = 0
    seen = set()
    for b in range(batches):
        x = synth.x_bits(w, seed=100 + b)
        xd = bits_to_dev_bf16(x)
        out = ops.moe_forward_cached(xd, wrd, None, w.k, cache, 1, ws_c)
        assert ops.moe_get_device_status(ws_c) == 0, b
        idx, _ = ops.moe_route(xd, wrd, None, w.k, ops.new_workspace(1 << 22))
        experts = np.unique(idx.cpu().numpy())
        seen |= set(experts.tolist())
        m, hits = mirror.admit(experts)
        st = ops.moe_expert_cache_stats(cache)
        assert st["calls"] == b + 1
        assert st["fetched_last"] == m, (b, st, m)
        fetched_total += m
        assert st["fetched"] == fetched_total
        ref = ops.moe_forward(xd, wrd, None, w.k, dbank, None, 1, ws_d)
        assert ops.moe_get_device_status(ws_d) == 0
        got = dev_to_f64(out)
        assert max_abs_rel(got, dev_to_f64(ref)) < 1e-2, b
        r, keep = forward_reference(w, x, wr, None, W, act=1, a13=a13, a2=a2)
        assert max_abs_rel(got[keep], r["out"][keep]) < TOL, b
    if len(seen) > n_slots:
        assert fetched_total > n_slots      # experts were evicted and fetched again


def test_pool_too_small_for_a_batch_is_rejected():
    w = synth.workload("tiny", T=8, H=256, E=32, k=4, I=256)
    W, _ = oracle_bank(w)
    dbank = device_bank(W, *synth.static_act_scales())
    cache = ops.moe_expert_cache_init(ops.bank_to_host(dbank), 16)
    xd = bits_to_dev_bf16(synth.x_bits(w))
    wrd = bits_to_dev_bf16(synth.router_bits(w))
    ws = ops.new_workspace(ops.workspace_size(w.T, w.k, cache.host, None, 1))
    with pytest.raises(ops.MoeError):
        ops.moe_forward_cached(xd, wrd, None, w.k, cache, 1, ws)   # 32 slots of routing, 16 slots of pool
