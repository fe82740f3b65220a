"""moe_permute_fixed_scratch: the permutation for callers that cannot give the
library a workspace (their device memory is already handed out, or they run
during stream capture, where cudaMalloc is not allowed).  Its scratch is a
fixed array inside the library.  Checked through the C ABI against
moe_permute, which takes a caller workspace, on two calls in a row; the
second call reuses the array the first one left behind.

This file is collected last on purpose, and passes alone in a fresh process
as well as after the other tests."""
import ctypes

import numpy as np
import pytest
import torch

from quantized_expert_ffn_top_b200 import ops, synth

pytestmark = pytest.mark.gpu


def _fixed(idx: torch.Tensor, E: int):
    T, k = idx.shape
    S = T * k
    off = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    perm = torch.full((S,), -7, dtype=torch.int32, device="cuda")
    inv = torch.full((S,), -7, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    st = ops.lib().moe_permute_fixed_scratch(p(idx), T, k, E, p(off), p(perm), p(inv), p(status),
                                             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == ops.MOE_OK, ops.status_string(st)
    torch.cuda.synchronize()
    return off.cpu().numpy(), perm.cpu().numpy(), inv.cpu().numpy(), int(status.item())


def test_fixed_scratch_permute_matches_workspace_permute_twice():
    assert torch.cuda.is_available()
    ws = ops.new_workspace(1 << 22)
    # both calls take the multi-block path (more than 8192 slots), which is the
    # one that uses the fixed array: 16 chunks x 128 experts, then 6 chunks x
    # 60 experts in the same array
    cases = [(4096, 8, 128, 1.1, 0), (3000, 4, 60, 0.3, 1)]
    for T, k, E, skew, seed in cases:
        idx = torch.from_numpy(synth.random_topk_idx(T, k, E, seed=seed, skew=skew)).cuda()
        ref = [t.cpu().numpy() for t in ops.moe_permute(idx, E, ws)]
        off, perm, inv, status = _fixed(idx, E)
        assert status == 0
        assert np.array_equal(off, ref[0])
        assert np.array_equal(perm, ref[1])
        assert np.array_equal(inv, ref[2])


def test_fixed_scratch_rejects_sizes_beyond_its_capacity():
    big_T = 70000                       # ceil(70000 * 8 / 2048) * 256 > 65536
    dummy = torch.zeros(16, dtype=torch.int32, device="cuda")
    p = ctypes.c_void_p(dummy.data_ptr())
    st = ops.lib().moe_permute_fixed_scratch(p, big_T, 8, 256, p, p, p, None, None)
    assert st == 3   # MOE_ERR_WORKSPACE: nothing enqueued
