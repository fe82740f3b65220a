"""Seeded synthetic inputs for the routed MoE layer.

This module draws numbers and nothing else: it holds none of the layer's
arithmetic (no routing, no quantisation, no FFN).  Both the CPU oracle (through
the tests) and the CUDA library (through the tests and the benchmark) take
their inputs from here, so both sides see identical bytes.

Streams are counter-based: every tensor has its own Philox4x32-10 stream keyed
by (seed, tensor id) (Salmon et al., "Parallel random numbers: as easy as
1, 2, 3", SC'11), drawn through numpy's ``Philox`` bit generator.  A CUDA
variant (``device="cuda"``) draws the same distributions with torch's CUDA
Philox generator for full-size benchmark layers; its numbers differ from the
CPU stream but follow the same recipe.

Workloads (the layer shapes of the five configurations):
  tiny       T=8     H=128  E=8   k=2 I=256  NVFP4, uniform router
  decode     T=4     H=2048 E=128 k=8 I=768  NVFP4, uniform router
  prefill    T=4096  H=2048 E=128 k=8 I=768  NVFP4, Zipf(1.1) router
  fp8_shared T=512   H=2048 E=256 k=8 I=512  FP8 W8A8 + one shared expert (I=512)
  large      T=16384 H=4096 E=256 k=8 I=2048 MXFP4, Zipf(1.1) router

Recipe: activations x ~ N(0,1) rounded to bf16; router weights Wr ~ N(0,0.02)
rounded to bf16; expert weights ~ N(0,0.02) in fp32 (quantised later by the
side under test).  "Uniform" routing has no router bias: logits x.Wr^T are
i.i.d. across experts, so expert popularity is uniform.  "Zipf" routing adds a
bias b[e] = -s * ln(r_e), r a seeded random permutation of 1..E and s = 1.1,
the log of a Zipf(s) popularity weight, which leaves some experts with more
than ten times the mean load and some with none.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

SEED = 0

# tensor ids of the streams
TID_X, TID_WR, TID_ZIPF, TID_LOGITS, TID_IDX = 1, 2, 3, 4, 5
TID_W13, TID_W2 = 1_000, 100_000            # + expert index
TID_SH_W13, TID_SH_W2 = 900_000, 900_001


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    E: int
    k: int
    I: int
    fmt: str                  # "nvfp4" | "mxfp4" | "fp8"
    router: str               # "uniform" | "zipf"
    shared_I: int = 0         # 0 = no shared expert
    zipf_s: float = 1.1
    w_std: float = 0.02
    wr_std: float = 0.02
    extra: dict = field(default_factory=dict)


WORKLOADS = {
    "tiny": Workload("tiny", 8, 128, 8, 2, 256, "nvfp4", "uniform"),
    "decode": Workload("decode", 4, 2048, 128, 8, 768, "nvfp4", "uniform"),
    "prefill": Workload("prefill", 4096, 2048, 128, 8, 768, "nvfp4", "zipf"),
    "fp8_shared": Workload("fp8_shared", 512, 2048, 256, 8, 512, "fp8", "uniform", shared_I=512),
    "large": Workload("large", 16384, 4096, 256, 8, 2048, "mxfp4", "zipf"),
    # the prefill layer with BF16 expert weights (bf16 activations throughout)
    "bf16_prefill": Workload("bf16_prefill", 4096, 2048, 128, 8, 768, "bf16", "zipf"),
}


def workload(name: str, **over) -> Workload:
    """A named workload, optionally with fields overridden (smaller cases)."""
    w = WORKLOADS[name]
    if not over:
        return w
    d = dict(w.__dict__)
    d.update(over)
    return Workload(**d)


# Static activation global scales for NVFP4 layers (the calibrated per-tensor
# input scales an NVFP4 checkpoint carries): the nominal amax the scale spans,
# divided by 448 * 6.  x ~ N(0,1); h = SiLU(g)*u stays well inside 16 here.
STATIC_X_AMAX = 8.0
STATIC_H_AMAX = 16.0


def static_act_scales() -> tuple[float, float]:
    return (float(np.float32(STATIC_X_AMAX) / np.float32(2688.0)),
            float(np.float32(STATIC_H_AMAX) / np.float32(2688.0)))


# ------------------------------------------------------------------ streams --
def stream(tid: int, seed: int = SEED) -> np.random.Generator:
    return np.random.Generator(np.random.Philox(key=(int(seed) << 32) | int(tid)))


def normal_f32(shape, std: float, tid: int, seed: int = SEED) -> np.ndarray:
    g = stream(tid, seed)
    a = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return a


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even (torch)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


# ------------------------------------------------------------------- layers --
def x_bits(w: Workload, seed: int = SEED, T: int | None = None) -> np.ndarray:
    return to_bf16_bits(normal_f32((T or w.T, w.H), 1.0, TID_X, seed))


def router_bits(w: Workload, seed: int = SEED) -> np.ndarray:
    return to_bf16_bits(normal_f32((w.E, w.H), w.wr_std, TID_WR, seed))


def router_bias(w: Workload, seed: int = SEED):
    """None for uniform routing; the Zipf log-popularity bias otherwise."""
    if w.router != "zipf":
        return None
    ranks = stream(TID_ZIPF, seed).permutation(w.E) + 1
    return (-w.zipf_s * np.log(ranks.astype(np.float64))).astype(np.float32)


def expert_w13(w: Workload, e: int, seed: int = SEED) -> np.ndarray:
    """fp32 [2I][H]: gate rows 0..I-1, up rows I..2I-1."""
    return normal_f32((2 * w.I, w.H), w.w_std, TID_W13 + e, seed)


def expert_w2(w: Workload, e: int, seed: int = SEED) -> np.ndarray:
    """fp32 [H][I]."""
    return normal_f32((w.H, w.I), w.w_std, TID_W2 + e, seed)


def all_w13(w: Workload, seed: int = SEED, experts=None) -> np.ndarray:
    ex = range(w.E) if experts is None else experts
    return np.stack([expert_w13(w, e, seed) for e in ex])


def all_w2(w: Workload, seed: int = SEED, experts=None) -> np.ndarray:
    ex = range(w.E) if experts is None else experts
    return np.stack([expert_w2(w, e, seed) for e in ex])


def shared_w13(w: Workload, seed: int = SEED) -> np.ndarray:
    return normal_f32((1, 2 * w.shared_I, w.H), w.w_std, TID_SH_W13, seed)


def shared_w2(w: Workload, seed: int = SEED) -> np.ndarray:
    return normal_f32((1, w.H, w.shared_I), w.w_std, TID_SH_W2, seed)


def random_logits(T: int, E: int, seed: int = SEED, kind: str = "uniform") -> np.ndarray:
    """fp32 router logits for testing top-k alone: U(0,1) or N(0,1)."""
    g = stream(TID_LOGITS, seed)
    if kind == "uniform":
        return g.random(size=(T, E), dtype=np.float32)
    return g.standard_normal(size=(T, E), dtype=np.float32)


def random_topk_idx(T: int, k: int, E: int, seed: int = SEED, skew: float = 0.0) -> np.ndarray:
    """int32 [T][k]: k distinct experts per token, popularity ~ rank^-skew."""
    g = stream(TID_IDX, seed)
    p = np.arange(1, E + 1, dtype=np.float64) ** (-skew)
    p /= p.sum()
    out = np.empty((T, k), np.int32)
    for t in range(T):
        out[t] = g.choice(E, size=k, replace=False, p=p)
    return out


# --------------------------------------------------------- CUDA-side draws --
def cuda_normal(shape, std: float, tid: int, seed: int = SEED, dtype=None):
    """Same distribution on the GPU (torch CUDA Philox), for full-size layers."""
    import torch
    g = torch.Generator(device="cuda")
    g.manual_seed(int(seed) * 1_000_003 + int(tid))
    t = torch.randn(shape, generator=g, device="cuda", dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t if dtype is None else t.to(dtype)


def cuda_router_bias(w: Workload, seed: int = SEED):
    b = router_bias(w, seed)
    if b is None:
        return None
    import torch
    return torch.from_numpy(b).cuda()


def zipf_expected_histogram(w: Workload) -> dict:
    """Descriptive helper: nothing of the layer is computed here."""
    return {"E": w.E, "k": w.k, "s": w.zipf_s, "mean_load": w.T * w.k / w.E,
            "cap_ratio": w.E / w.k, "log_bias_span": w.zipf_s * math.log(w.E)}
