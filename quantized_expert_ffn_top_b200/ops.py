"""Thin ctypes binding of ``libmoe_b200.so`` (C ABI in include/moe_b200.h).

Argument marshalling only: every function passes raw device pointers, sizes
and torch's current CUDA stream to the library entry point of the same name
and raises ``MoeError`` on a non-OK status.  There is no CPU fallback: if the
library is missing or no CUDA device is present, the call fails.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field, replace

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmoe_b200.so")

MOE_OK = 0
FMT_NVFP4, FMT_MXFP4, FMT_FP8, FMT_BF16 = 1, 2, 3, 4
ACT_BF16, ACT_MATCH = 0, 1
LAYOUT_CANONICAL, LAYOUT_PREPARED = 0, 1
OPT_FFN_PATH = 1
OPT_GEMM_TILE_N = 2
OPT_GEMM_PAIR = 3
OPT_PDL = 4
OPT_EARLY_WEIGHTS = 5
OPT_FUSED_FFN = 6
OPT_PERMUTE_QUANT = 7
OPT_WAIT_CYCLES = 8
OPT_FUSED_COMBINE = 9
OPT_SMALL_BATCH_FORWARD = 10
OPT_GATHER_X = 11
OPT_FFN_SCHEDULE = 12
OPT_ROUTER_TOPK = 13
FMT_BY_NAME = {"nvfp4": FMT_NVFP4, "mxfp4": FMT_MXFP4, "fp8": FMT_FP8, "bf16": FMT_BF16}


def row_bytes(fmt: int, K: int) -> int:
    """Bytes of one row of K weight elements in a format."""
    return K if fmt == FMT_FP8 else (2 * K if fmt == FMT_BF16 else K // 2)

EXPORTED = (
    "moe_status_string", "moe_version", "moe_set_option", "moe_workspace_size", "moe_prepared_weights_size",
    "moe_prepare_weights", "moe_dequantize_weights", "moe_dequantized_weights_size", "moe_quantize", "moe_route", "moe_route_logits", "moe_permute", "moe_grouped_ffn",
    "moe_combine", "moe_forward", "moe_get_device_status", "moe_set_stage_events", "moe_kernel_launch_count",
    "moe_permute_fixed_scratch", "moe_forward_host", "moe_stage_mask", "moe_expert_cache_bytes",
    "moe_expert_cache_init", "moe_forward_cached", "moe_expert_cache_stats",
)
MAX_HOST_SLICES = 64
STAGES = ("route", "permute", "act_quant", "ffn_up", "ffn_down", "shared", "combine")


class MoeError(RuntimeError):
    """A moe_status other than MOE_OK, with the call that returned it."""
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_string(status)}")
        self.status = status


class MoeWeightsC(ctypes.Structure):
    """The C struct moe_weights: format, sizes, layout and device (or host) pointers."""
    _fields_ = [
        ("fmt", ctypes.c_int32), ("E", ctypes.c_int32), ("H", ctypes.c_int32), ("I", ctypes.c_int32),
        ("layout", ctypes.c_int32),
        ("w13", ctypes.c_void_p), ("w13_sf", ctypes.c_void_p), ("w13_gs", ctypes.c_void_p),
        ("w2", ctypes.c_void_p), ("w2_sf", ctypes.c_void_p), ("w2_gs", ctypes.c_void_p),
        ("a13_gs", ctypes.c_void_p), ("a2_gs", ctypes.c_void_p),
    ]


class MoeExpertCacheC(ctypes.Structure):
    """The C struct moe_expert_cache, filled by moe_expert_cache_init."""
    _fields_ = [
        ("bank", MoeWeightsC), ("pool", MoeWeightsC), ("bank_dev", ctypes.c_void_p * 6),
        ("state", ctypes.c_void_p), ("n_slots", ctypes.c_int32),
    ]


_lib = None


def lib():
    """Load the library (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m quantized_expert_ffn_top_b200.build` "
                               "(the layer has no CPU fallback)")
        L = ctypes.CDLL(LIB_PATH)
        _declare(L)
        _lib = L
    return _lib


def _declare(L):
    P, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    W = ctypes.POINTER(MoeWeightsC)
    sig = {
        "moe_status_string": ([ctypes.c_int], ctypes.c_char_p),
        "moe_version": ([], i32),
        "moe_set_option": ([i32, i32], ctypes.c_int),
        "moe_workspace_size": ([i64, i32, W, W, i32], sz),
        "moe_prepared_weights_size": ([W], sz),
        "moe_prepare_weights": ([W, P, sz, W, P], ctypes.c_int),
        "moe_dequantized_weights_size": ([W], sz),
        "moe_dequantize_weights": ([W, P, sz, W, P], ctypes.c_int),
        "moe_quantize": ([i32, P, i32, i64, i64, P, P, P, P, P, sz, P], ctypes.c_int),
        "moe_route": ([P, i64, i32, P, P, i32, i32, P, P, P, P, sz, P], ctypes.c_int),
        "moe_route_logits": ([P, i64, i32, i32, P, P, P, sz, P], ctypes.c_int),
        "moe_permute": ([P, i64, i32, i32, P, P, P, P, sz, P], ctypes.c_int),
        "moe_grouped_ffn": ([P, i64, i32, P, P, W, i32, P, P, sz, P], ctypes.c_int),
        "moe_combine": ([P, P, P, i64, i32, i32, P, P, P, sz, P], ctypes.c_int),
        "moe_forward": ([P, i64, P, P, i32, W, W, i32, P, P, sz, P], ctypes.c_int),
        "moe_get_device_status": ([P, P, ctypes.POINTER(ctypes.c_int32)], ctypes.c_int),
        "moe_set_stage_events": ([ctypes.POINTER(ctypes.c_void_p), i32], ctypes.c_int),
        "moe_kernel_launch_count": ([], ctypes.c_uint64),
        "moe_stage_mask": ([], ctypes.c_uint32),
        "moe_expert_cache_bytes": ([W, i32], sz),
        "moe_expert_cache_init": ([W, i32, P, sz, ctypes.POINTER(MoeExpertCacheC), P], ctypes.c_int),
        "moe_forward_cached": ([P, i64, P, P, i32, ctypes.POINTER(MoeExpertCacheC), i32, P, P, sz, P], ctypes.c_int),
        "moe_expert_cache_stats": ([ctypes.POINTER(MoeExpertCacheC), P, ctypes.POINTER(ctypes.c_int64)],
                                   ctypes.c_int),
        "moe_permute_fixed_scratch": ([P, i64, i32, i32, P, P, P, P, P], ctypes.c_int),
        "moe_forward_host": ([P, i64, P, P, i32, W, W, i32, P, P, P, i32, P, sz, P], ctypes.c_int),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res


def status_string(st: int) -> str:
    """moe_status_string: the name and meaning of a status code."""
    return lib().moe_status_string(int(st)).decode()


def _check(st: int, where: str):
    if st != MOE_OK:
        raise MoeError(st, where)


def _p(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("device tensor expected")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


# ------------------------------------------------------------ weight bank --
@dataclass
class WeightBank:
    """Device tensors of one expert bank (see moe_weights in the header)."""
    fmt: int
    E: int
    H: int
    I: int
    w13: torch.Tensor
    w13_sf: torch.Tensor | None
    w13_gs: torch.Tensor | None
    w2: torch.Tensor
    w2_sf: torch.Tensor | None
    w2_gs: torch.Tensor | None
    a13_gs: torch.Tensor | None = None
    a2_gs: torch.Tensor | None = None
    layout: int = LAYOUT_CANONICAL
    keep: list = field(default_factory=list)   # owners of memory the pointers reference

    def struct(self) -> MoeWeightsC:
        v = lambda t: None if t is None else t.data_ptr()
        return MoeWeightsC(self.fmt, self.E, self.H, self.I, self.layout, v(self.w13), v(self.w13_sf),
                           v(self.w13_gs), v(self.w2), v(self.w2_sf), v(self.w2_gs), v(self.a13_gs), v(self.a2_gs))

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in (self.w13, self.w13_sf, self.w2, self.w2_sf) if t is not None)


def _ref(b: WeightBank | None):
    return None if b is None else ctypes.byref(b.struct())


def workspace_size(T: int, k: int, routed: WeightBank, shared: WeightBank | None = None, act: int = ACT_MATCH) -> int:
    """moe_workspace_size: bytes of workspace moe_forward (and the stages) need for T tokens."""
    r = routed.struct()
    s = shared.struct() if shared is not None else None
    n = lib().moe_workspace_size(int(T), int(k), ctypes.byref(r), ctypes.byref(s) if s is not None else None,
                                 int(act))
    if n == 0:
        raise MoeError(1, "moe_workspace_size")
    return int(n)


def new_workspace(nbytes: int, device=None) -> torch.Tensor:
    """A zeroed workspace (the status word must start at zero)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")


def moe_prepare_weights(bank: WeightBank, stream=None) -> WeightBank:
    """moe_prepare_weights: a bank in the PREPARED layout (interleaved W13 rows, blocked scales), new device memory."""
    c = bank.struct()
    n = lib().moe_prepared_weights_size(ctypes.byref(c))
    if n == 0:
        raise MoeError(2, "moe_prepared_weights_size")
    dst = torch.empty(int(n), dtype=torch.uint8, device=bank.w13.device)
    out = MoeWeightsC()
    _check(lib().moe_prepare_weights(ctypes.byref(c), _p(dst), n, ctypes.byref(out), _stream(stream)),
           "moe_prepare_weights")

    def view(ptr, numel):
        if not ptr:
            return None
        off = ptr - dst.data_ptr()
        return dst[off:off + numel]

    rb13 = row_bytes(bank.fmt, bank.H)
    rb2 = row_bytes(bank.fmt, bank.I)
    bs = {FMT_NVFP4: 16, FMT_MXFP4: 32}.get(bank.fmt, 0)
    return replace(bank, layout=LAYOUT_PREPARED,
                   w13=view(out.w13, bank.E * 2 * bank.I * rb13),
                   w2=view(out.w2, bank.E * bank.H * rb2),
                   w13_sf=view(out.w13_sf, bank.E * 2 * bank.I * bank.H // bs) if bs else None,
                   w2_sf=view(out.w2_sf, bank.E * bank.H * bank.I // bs) if bs else None,
                   keep=[dst])


def moe_dequantize_weights(bank: WeightBank, stream=None) -> WeightBank:
    """CANONICAL NVFP4 / MXFP4 / FP8 bank -> CANONICAL BF16 bank (device), for
    bf16-activation prefill on the bf16 tensor cores."""
    c = bank.struct()
    n = lib().moe_dequantized_weights_size(ctypes.byref(c))
    if n == 0:
        raise MoeError(2, "moe_dequantized_weights_size")
    dst = torch.empty(int(n), dtype=torch.uint8, device=bank.w13.device)
    out = MoeWeightsC()
    _check(lib().moe_dequantize_weights(ctypes.byref(c), _p(dst), n, ctypes.byref(out), _stream(stream)),
           "moe_dequantize_weights")
    E, H, I = bank.E, bank.H, bank.I
    return WeightBank(FMT_BF16, E, H, I, dst[:E * 2 * I * H * 2], None, None,
                      dst[out.w2 - dst.data_ptr():out.w2 - dst.data_ptr() + E * H * I * 2], None, None,
                      keep=[dst])


# ------------------------------------------------------------ entry points --
def moe_quantize(fmt: int, x: torch.Tensor, scale_in: torch.Tensor | None = None, ws: torch.Tensor | None = None,
                 stream=None):
    """x: [rows][K] fp32 or bf16 (device).  Returns (codes, sf, scale_used)."""
    rows, K = x.shape
    dt = {torch.float32: 0, torch.bfloat16: 1}[x.dtype]
    codes = torch.empty((rows, row_bytes(fmt, K)), dtype=torch.uint8, device=x.device)
    bs = {FMT_NVFP4: 16, FMT_MXFP4: 32}.get(fmt, 0)
    sf = torch.empty((rows, K // bs), dtype=torch.uint8, device=x.device) if bs else None
    scale_out = torch.ones(1, dtype=torch.float32, device=x.device)
    ws = ws if ws is not None else new_workspace(4096, x.device)
    _check(lib().moe_quantize(fmt, _p(x.contiguous()), dt, rows, K, _p(scale_in), _p(codes), _p(sf), _p(scale_out),
                              _p(ws), ws.numel(), _stream(stream)), "moe_quantize")
    return codes, sf, scale_out


def moe_route(x: torch.Tensor, wr: torch.Tensor, bias: torch.Tensor | None, k: int, ws: torch.Tensor,
              logits: torch.Tensor | None = None, stream=None):
    """x [T][H] bf16, wr [E][H] bf16 -> (topk_idx int32 [T][k], topk_w fp32 [T][k])."""
    T, H = x.shape
    E = wr.shape[0]
    idx = torch.empty((T, k), dtype=torch.int32, device=x.device)
    w = torch.empty((T, k), dtype=torch.float32, device=x.device)
    _check(lib().moe_route(_p(x), T, H, _p(wr), _p(bias), E, k, _p(logits), _p(idx), _p(w), _p(ws), ws.numel(),
                           _stream(stream)), "moe_route")
    return idx, w


def moe_route_logits(logits: torch.Tensor, k: int, ws: torch.Tensor, stream=None):
    """moe_route_logits: top-k indices and renormalised weights from fp32 logits [T][E]."""
    T, E = logits.shape
    idx = torch.empty((T, k), dtype=torch.int32, device=logits.device)
    w = torch.empty((T, k), dtype=torch.float32, device=logits.device)
    _check(lib().moe_route_logits(_p(logits), T, E, k, _p(idx), _p(w), _p(ws), ws.numel(), _stream(stream)),
           "moe_route_logits")
    return idx, w


def moe_permute(topk_idx: torch.Tensor, E: int, ws: torch.Tensor, stream=None):
    """moe_permute: offsets [E+1], perm_token [S] and inv_perm [S] of the top-k ids [T][k]."""
    T, k = topk_idx.shape
    S = T * k
    offsets = torch.empty(E + 1, dtype=torch.int32, device=topk_idx.device)
    perm = torch.empty(S, dtype=torch.int32, device=topk_idx.device)
    inv = torch.empty(S, dtype=torch.int32, device=topk_idx.device)
    _check(lib().moe_permute(_p(topk_idx), T, k, E, _p(offsets), _p(perm), _p(inv), _p(ws), ws.numel(),
                             _stream(stream)), "moe_permute")
    return offsets, perm, inv


def moe_grouped_ffn(x: torch.Tensor, k: int, perm_token: torch.Tensor, offsets: torch.Tensor, w: WeightBank,
                    act: int, ws: torch.Tensor, y_perm: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """moe_grouped_ffn: the experts' SwiGLU FFN over the permuted slots, y_perm [T*k][H] bf16."""
    T, H = x.shape
    y = y_perm if y_perm is not None else torch.empty((T * k, H), dtype=torch.bfloat16, device=x.device)
    ws_ = w.struct()
    _check(lib().moe_grouped_ffn(_p(x), T, k, _p(perm_token), _p(offsets), ctypes.byref(ws_), act, _p(y), _p(ws),
                                 ws.numel(), _stream(stream)), "moe_grouped_ffn")
    return y


def moe_combine(y_perm: torch.Tensor, inv_perm: torch.Tensor, topk_w: torch.Tensor, ws: torch.Tensor,
                shared_y: torch.Tensor | None = None, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """moe_combine: out[t] = sum_j w[t,j] y_perm[inv_perm[t*k+j]] (+ shared_y[t]), bf16."""
    T, k = topk_w.shape
    H = y_perm.shape[1]
    o = out if out is not None else torch.empty((T, H), dtype=torch.bfloat16, device=y_perm.device)
    _check(lib().moe_combine(_p(y_perm), _p(inv_perm), _p(topk_w), T, k, H, _p(shared_y), _p(o), _p(ws),
                             ws.numel(), _stream(stream)), "moe_combine")
    return o


def moe_forward(x: torch.Tensor, wr: torch.Tensor, bias: torch.Tensor | None, k: int, routed: WeightBank,
                shared: WeightBank | None, act: int, ws: torch.Tensor, out: torch.Tensor | None = None,
                stream=None) -> torch.Tensor:
    """moe_forward: the whole layer, x [T][H] bf16 -> out [T][H] bf16, on the current stream."""
    T, H = x.shape
    o = out if out is not None else torch.empty((T, H), dtype=torch.bfloat16, device=x.device)
    r = routed.struct()
    s = shared.struct() if shared is not None else None
    _check(lib().moe_forward(_p(x), T, _p(wr), _p(bias), k, ctypes.byref(r),
                             ctypes.byref(s) if s is not None else None, act, _p(o), _p(ws), ws.numel(),
                             _stream(stream)), "moe_forward")
    return o


def _hp(t):
    if t.is_cuda or not t.is_contiguous():
        raise ValueError("contiguous host tensor expected")
    return ctypes.c_void_p(t.data_ptr())


def moe_forward_host(x_host: torch.Tensor, wr: torch.Tensor, bias: torch.Tensor | None, k: int,
                     routed: WeightBank, shared: WeightBank | None, act: int, ws: torch.Tensor,
                     x_dev: torch.Tensor, out_dev: torch.Tensor, out_host: torch.Tensor | None = None,
                     n_slices: int = 4, stream=None) -> torch.Tensor:
    """The layer on host buffers: x_host [T][H] bf16 (host; pinned for the
    copies to overlap) -> out_host [T][H] bf16 (host), through the device
    staging buffers x_dev and out_dev, in n_slices token slices whose copies
    overlap each other's forwards.  Only enqueues: synchronise the stream
    before reading out_host."""
    T, H = x_host.shape
    o = out_host if out_host is not None else torch.empty((T, H), dtype=torch.bfloat16, pin_memory=True)
    r = routed.struct()
    s = shared.struct() if shared is not None else None
    _check(lib().moe_forward_host(_hp(x_host), T, _p(wr), _p(bias), k, ctypes.byref(r),
                                  ctypes.byref(s) if s is not None else None, act, _hp(o), _p(x_dev), _p(out_dev),
                                  int(n_slices), _p(ws), ws.numel(), _stream(stream)), "moe_forward_host")
    return o


# ------------------------------------------------------------ expert cache --
@dataclass
class ExpertCache:
    """An HBM pool of n_slots expert slots in front of a host-memory bank."""
    c: MoeExpertCacheC
    dev: torch.Tensor
    host: WeightBank


def bank_to_host(bank: WeightBank) -> WeightBank:
    """A PREPARED device bank copied to page-locked host memory (the activation
    scales stay on the device)."""
    if bank.layout != LAYOUT_PREPARED:
        raise ValueError("a PREPARED bank is expected")
    h = lambda t: None if t is None else t.cpu().pin_memory()
    return replace(bank, w13=h(bank.w13), w13_sf=h(bank.w13_sf), w13_gs=h(bank.w13_gs), w2=h(bank.w2),
                   w2_sf=h(bank.w2_sf), w2_gs=h(bank.w2_gs), keep=[])


def moe_expert_cache_init(host_bank: WeightBank, n_slots: int, stream=None) -> ExpertCache:
    """moe_expert_cache_init: an HBM pool of n_slots experts in front of a PREPARED bank in pinned host memory."""
    b = host_bank.struct()
    n = lib().moe_expert_cache_bytes(ctypes.byref(b), int(n_slots))
    if n == 0:
        raise MoeError(1, "moe_expert_cache_bytes")
    dev = torch.empty(int(n), dtype=torch.uint8, device="cuda")
    c = MoeExpertCacheC()
    _check(lib().moe_expert_cache_init(ctypes.byref(b), int(n_slots), _p(dev), n, ctypes.byref(c), _stream(stream)),
           "moe_expert_cache_init")
    return ExpertCache(c, dev, host_bank)


def moe_forward_cached(x: torch.Tensor, wr: torch.Tensor, bias: torch.Tensor | None, k: int, cache: ExpertCache,
                       act: int, ws: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """moe_forward_cached: the layer through the slot pool (misses fetched from host memory)."""
    T, H = x.shape
    o = out if out is not None else torch.empty((T, H), dtype=torch.bfloat16, device=x.device)
    _check(lib().moe_forward_cached(_p(x), T, _p(wr), _p(bias), k, ctypes.byref(cache.c), act, _p(o), _p(ws),
                                    ws.numel(), _stream(stream)), "moe_forward_cached")
    return o


def moe_expert_cache_stats(cache: ExpertCache, stream=None) -> dict:
    """moe_expert_cache_stats: calls, experts fetched (last call and in total) and hits."""
    v = (ctypes.c_int64 * 4)()
    _check(lib().moe_expert_cache_stats(ctypes.byref(cache.c), _stream(stream), v), "moe_expert_cache_stats")
    return {"calls": int(v[0]), "fetched_last": int(v[1]), "fetched": int(v[2]), "hits": int(v[3])}


def moe_get_device_status(ws: torch.Tensor, stream=None) -> int:
    """moe_get_device_status: the workspace's device status word (synchronises; clears it)."""
    v = ctypes.c_int32(0)
    _check(lib().moe_get_device_status(_p(ws), _stream(stream), ctypes.byref(v)), "moe_get_device_status")
    return int(v.value)


def moe_set_option(option: int, value: int):
    """moe_set_option: a process-wide switch (OPT_*; the header documents values and defaults)."""
    _check(lib().moe_set_option(int(option), int(value)), "moe_set_option")


# ----------------------------------------------------- device-side banks --
def quantize_bank(fmt: int, w13: torch.Tensor, w2: torch.Tensor, ws: torch.Tensor | None = None) -> WeightBank:
    """fp32 expert weights on the device -> CANONICAL bank, quantised by the
    library (one amax-derived scale per part for NVFP4 / FP8).
    w13 [E][2I][H] (gate rows first), w2 [E][H][I]."""
    E, twoI, H = w13.shape
    I = twoI // 2
    dev = w13.device
    bs = {FMT_NVFP4: 16, FMT_MXFP4: 32}.get(fmt, 0)
    cb13 = row_bytes(fmt, H)
    cb2 = row_bytes(fmt, I)
    c13 = torch.empty((E, twoI, cb13), dtype=torch.uint8, device=dev)
    c2 = torch.empty((E, H, cb2), dtype=torch.uint8, device=dev)
    s13 = torch.empty((E, twoI, H // bs), dtype=torch.uint8, device=dev) if bs else None
    s2 = torch.empty((E, H, I // bs), dtype=torch.uint8, device=dev) if bs else None
    scaled = fmt in (FMT_NVFP4, FMT_FP8)
    g13 = torch.ones((E, 2), dtype=torch.float32, device=dev) if scaled else None
    g2 = torch.ones(E, dtype=torch.float32, device=dev) if scaled else None
    ws = ws if ws is not None else new_workspace(4096, dev)
    L = lib()
    st = _stream()
    for e in range(E):
        parts = [(w13[e, :I], c13[e, :I], None if s13 is None else s13[e, :I], None if g13 is None else g13[e, 0:1]),
                 (w13[e, I:], c13[e, I:], None if s13 is None else s13[e, I:], None if g13 is None else g13[e, 1:2]),
                 (w2[e], c2[e], None if s2 is None else s2[e], None if g2 is None else g2[e:e + 1])]
        for src, codes, sf, gs in parts:
            rows, K = src.shape
            _check(L.moe_quantize(fmt, _p(src), 0, rows, K, None, _p(codes), _p(sf), _p(gs), _p(ws), ws.numel(),
                                  st), "moe_quantize")
    return WeightBank(fmt, E, H, I, c13, s13, g13, c2, s2, g2)


def bank_from_host(fmt: int, E: int, H: int, I: int, w13, w13_sf, w13_gs, w2, w2_sf, w2_gs, a13_gs=None,
                   a2_gs=None, device="cuda") -> WeightBank:
    """A CANONICAL bank from host arrays (numpy or torch); scalars as floats."""
    def dev(a, dtype):
        if a is None:
            return None
        t = torch.as_tensor(a)
        return t.to(device=device, dtype=dtype).contiguous()

    def scal(v):
        return None if v is None else torch.tensor([float(v)], dtype=torch.float32, device=device)

    return WeightBank(fmt, E, H, I, dev(w13, torch.uint8), dev(w13_sf, torch.uint8), dev(w13_gs, torch.float32),
                      dev(w2, torch.uint8), dev(w2_sf, torch.uint8), dev(w2_gs, torch.float32), scal(a13_gs),
                      scal(a2_gs))


def moe_set_stage_events(events):
    """events: list of 2 * len(STAGES) torch.cuda.Event(enable_timing=True), or None."""
    if events is None:
        _check(lib().moe_set_stage_events(None, 0), "moe_set_stage_events")
        return
    for e in events:
        if not e.cuda_event:     # torch creates the CUDA event on first record
            e.record()
    arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    _check(lib().moe_set_stage_events(arr, len(events)), "moe_set_stage_events")


def moe_stage_mask() -> int:
    """Bit s: stage STAGES[s] was recorded since events were last installed."""
    return int(lib().moe_stage_mask())


def moe_kernel_launch_count() -> int:
    """Kernels this process has launched through the library so far."""
    return int(lib().moe_kernel_launch_count())
