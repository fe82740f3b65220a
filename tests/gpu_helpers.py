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


def router_order(T: int, E: int, H: int, k: int) -> int:
    """Which fixed fp32 summation order moe_route's logits follow (the header
    documents it): 1 = the small-batch order (T <= 64, H % 8 == 0), 2 = one
    sequential sum, 0 = the tensor cores' own order (T >= 128, H % 64 == 0
    and either E % 128 == 0, or the one-kernel router: 128-token tiles for at
    least half the SMs, 16 <= E <= 256 with E % 16 == 0, k <= 16), which the
    oracle cannot replay."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    one_kernel = (T + 127) // 128 >= sms // 2 and 16 <= E <= 256 and E % 16 == 0 and k <= 16
    if T >= 128 and H % 64 == 0 and (one_kernel or E % 128 == 0):
        return 0
    if T <= 64 and H % 8 == 0:
        return 1
    return 2


def routing_tol(L_ref: np.ndarray, L_gpu: np.ndarray, floor: float = 1e-6) -> float:
    """Half-width of the band in which a top-k choice taken on the GPU's fp32
    logits may differ from one taken on the oracle's: twice the largest
    logit difference actually seen (a gap wider than that cannot flip)."""
    return max(2.0 * float(np.max(np.abs(np.asarray(L_gpu, np.float64) - L_ref))), floor)


def report_ambiguous(amb: np.ndarray, what: str, limit: float = 0.01) -> float:
    """Prints and bounds the fraction of tokens left out as ambiguous."""
    frac = float(np.mean(amb)) if amb.size else 0.0
    print(f"{what}: {int(np.sum(amb))} of {amb.size} tokens ambiguous ({100 * frac:.3f} %)")
    assert frac < limit, f"{what}: {100 * frac:.3f} % of tokens ambiguous"
    return frac


def forward_reference(w: synth.Workload, x, wr, b, W, Ws=None, act: int = 1, a13=None, a2=None, sh_a2=None,
                      tokens=None, route_T: int | None = None, what: str = ""):
    """The oracle's layer output for moe_forward's inputs, and the tokens whose
    routing both sides decide alike.  Where the library's router sums in a
    fixed order (router_order) the oracle routes on the same fp32 logits and
    every token is kept; behind the tensor-core router, tokens whose k/k+1
    logit gap lies within routing_tol of the GPU's own logits (moe_route on
    the same batch) are left out, counted and bounded.  route_T: the batch
    size the router sees (a slice of moe_forward_host)."""
    order = router_order(route_T or w.T, w.E, w.H, w.k)
    r = oracle.moe_forward(x, wr, b, w.k, W, Ws, act=act, a13_static=a13 or 0.0, a2_static=a2 or 0.0,
                           sh_a2_static=sh_a2 or 0.0, tokens=tokens, router_order=order)
    if order:
        return r, np.ones(r["out"].shape[0], bool)
    logits = torch.empty((w.T, w.E), dtype=torch.float32, device="cuda")
    ws = ops.new_workspace(w.T * w.E * 16 + (1 << 20))
    ops.moe_route(bits_to_dev_bf16(x), bits_to_dev_bf16(wr), None if b is None else torch.from_numpy(b).cuda(),
                  w.k, ws, logits=logits)
    gl = logits.cpu().numpy()
    if tokens is not None:
        gl = gl[np.asarray(tokens)]
    amb = ambiguous_tokens(r["logits"], w.k, routing_tol(r["logits"], gl), boundary_only=True)
    report_ambiguous(amb, what or f"forward {w.name}")
    return r, ~amb
