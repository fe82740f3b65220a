"""Helpers shared by the GPU parity tests: layers built from the seeded
generators, quantised by the oracle, uploaded to the device and prepared by
the library; error measures; routing-ambiguity detection."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from quantized_expert_ffn_top_b200 import ops, synth

FMT = {"nvfp4": oracle.FMT_NVFP4, "mxfp4": oracle.FMT_MXFP4, "fp8": oracle.FMT_FP8, "bf16": oracle.FMT_BF16}

# max-abs-relative error bound of the layer's outputs against the fp64 oracle
TOL = 2e-2


def max_abs_rel(y, r) -> float:
    y = np.asarray(y, np.float64)
    r = np.asarray(r, np.float64)
    den = float(np.max(np.abs(r)))
    return float(np.max(np.abs(y - r))) / (den if den > 0 else 1.0)


def bits_to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def dev_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def oracle_bank(w: synth.Workload, seed: int = synth.SEED):
    fmt = FMT[w.fmt]
    W = oracle.quantize_expert_weights(fmt, synth.all_w13(w, seed), synth.all_w2(w, seed))
    Ws = None
    if w.shared_I:
        Ws = oracle.quantize_expert_weights(fmt, synth.shared_w13(w, seed), synth.shared_w2(w, seed))
    return W, Ws


def device_bank(W: oracle.Weights, a13=None, a2=None, prepare=True) -> ops.WeightBank:
    b = ops.bank_from_host(W.fmt, W.E, W.H, W.I, W.w13, W.w13_sf, W.w13_gs, W.w2, W.w2_sf, W.w2_gs, a13, a2)
    return ops.moe_prepare_weights(b) if prepare else b


def ambiguous_tokens(L: np.ndarray, k: int, tol: float, boundary_only: bool = False) -> np.ndarray:
    """Tokens whose top-k selection (boundary_only) or order could flip under
    logit perturbations of size tol."""
    s = -np.sort(-L, axis=1)
    if boundary_only:
        if k >= L.shape[1]:
            return np.zeros(L.shape[0], bool)
        return (s[:, k - 1] - s[:, k]) < tol
    m = min(k + 1, L.shape[1])
    gaps = s[:, :m - 1] - s[:, 1:m]
    return np.any(gaps < tol, axis=1)


def routed_inputs(w: synth.Workload, seed: int = synth.SEED):
    x = synth.x_bits(w, seed)
    wr = synth.router_bits(w, seed)
    b = synth.router_bias(w, seed)
    return x, wr, b
