"""Python front end of the plain CPU oracle (``moe_oracle.cpp``).

TEST INFRASTRUCTURE ONLY.  The test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are the only users.  The CUDA library does not
import, link or call anything here, and this module imports nothing from the
library: the two sides share only the seeded input generators.

Every function is argument marshalling (numpy <-> ctypes) around the C++
oracle; the arithmetic, with its citations, lives in ``moe_oracle.cpp``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.cpp")
_LIB = os.path.join(_HERE, "libmoe_oracle.so")

FMT_NVFP4, FMT_MXFP4, FMT_FP8, FMT_BF16 = 1, 2, 3, 4
ACT_BF16, ACT_MATCH = 0, 1


def build(force: bool = False) -> str:
    """Compile the oracle with g++ (-O2, OpenMP over tokens) into oracle/."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["g++", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c++17", "-Wall", "-o", _LIB, _SRC]
        subprocess.run(cmd, check=True)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _declare(_lib)
    return _lib


class OrcWeights(ctypes.Structure):
    _fields_ = [
        ("fmt", ctypes.c_int32), ("E", ctypes.c_int32), ("H", ctypes.c_int32), ("I", ctypes.c_int32),
        ("w13", ctypes.c_void_p), ("w13_sf", ctypes.c_void_p), ("w13_gs", ctypes.c_void_p),
        ("w2", ctypes.c_void_p), ("w2_sf", ctypes.c_void_p), ("w2_gs", ctypes.c_void_p),
    ]


def _declare(L):
    P = ctypes.c_void_p
    i64, i32, f32 = ctypes.c_int64, ctypes.c_int32, ctypes.c_float
    L.orc_e2m1_decode.argtypes = [ctypes.c_int]; L.orc_e2m1_decode.restype = ctypes.c_double
    L.orc_e4m3_decode.argtypes = [ctypes.c_int]; L.orc_e4m3_decode.restype = ctypes.c_double
    L.orc_e8m0_decode.argtypes = [ctypes.c_int]; L.orc_e8m0_decode.restype = ctypes.c_double
    L.orc_e2m1_encode.argtypes = [f32]; L.orc_e2m1_encode.restype = ctypes.c_int
    L.orc_e4m3_encode.argtypes = [f32]; L.orc_e4m3_encode.restype = ctypes.c_int
    L.orc_amax.argtypes = [P, i64]; L.orc_amax.restype = f32
    L.orc_nvfp4_global_scale.argtypes = [f32]; L.orc_nvfp4_global_scale.restype = f32
    L.orc_fp8_scale.argtypes = [f32]; L.orc_fp8_scale.restype = f32
    L.orc_quant_nvfp4.argtypes = [P, i64, i64, f32, P, P]; L.orc_quant_nvfp4.restype = None
    L.orc_quant_mxfp4.argtypes = [P, i64, i64, P, P]; L.orc_quant_mxfp4.restype = None
    L.orc_quant_fp8.argtypes = [P, i64, f32, P]; L.orc_quant_fp8.restype = None
    L.orc_bf16_encode.argtypes = [f32]; L.orc_bf16_encode.restype = ctypes.c_int
    L.orc_quant_bf16.argtypes = [P, i64, P]; L.orc_quant_bf16.restype = None
    L.orc_dequant.argtypes = [ctypes.c_int, P, P, ctypes.c_double, i64, i64, P]; L.orc_dequant.restype = None
    L.orc_router_logits.argtypes = [P, i64, i32, P, i32, P, P]; L.orc_router_logits.restype = None
    L.orc_topk.argtypes = [P, i64, i32, i32, P, P]; L.orc_topk.restype = ctypes.c_int
    L.orc_permute.argtypes = [P, i64, i32, i32, P, P, P]; L.orc_permute.restype = ctypes.c_int
    L.orc_grouped_ffn.argtypes = [P, i64, P, P, ctypes.POINTER(OrcWeights), i32, f32, f32, P, i32, P]
    L.orc_grouped_ffn.restype = ctypes.c_int
    L.orc_combine.argtypes = [P, P, P, i64, i32, i32, P, P]; L.orc_combine.restype = None
    L.orc_router_logits_ordered.argtypes = [P, i64, i32, P, i32, P, i32, P]
    L.orc_router_logits_ordered.restype = ctypes.c_int
    L.orc_moe_forward.argtypes = [P, i64, i32, P, P, i32, i32, ctypes.POINTER(OrcWeights),
                                  ctypes.POINTER(OrcWeights), i32, f32, f32, f32, P, i64, P, P, P, P, i32, i32]
    L.orc_moe_forward.restype = ctypes.c_int
    L.orc_num_threads_available.argtypes = []; L.orc_num_threads_available.restype = ctypes.c_int


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------- codecs ----
def e2m1_decode(code: int) -> float:
    return lib().orc_e2m1_decode(int(code))


def e4m3_decode(code: int) -> float:
    return lib().orc_e4m3_decode(int(code))


def e8m0_decode(code: int) -> float:
    return lib().orc_e8m0_decode(int(code))


def e2m1_encode(v: float) -> int:
    return lib().orc_e2m1_encode(float(np.float32(v)))


def e4m3_encode(v: float) -> int:
    return lib().orc_e4m3_encode(float(np.float32(v)))


# ------------------------------------------------------------ quantisers ----
def amax(x: np.ndarray) -> float:
    x = _c(x, np.float32)
    return float(np.float32(lib().orc_amax(_p(x), x.size)))


def nvfp4_global_scale(a: float) -> float:
    return float(np.float32(lib().orc_nvfp4_global_scale(float(a))))


def fp8_scale(a: float) -> float:
    return float(np.float32(lib().orc_fp8_scale(float(a))))


def quant_nvfp4(x: np.ndarray, g: float):
    """rows x K fp32 -> (codes uint8 [rows][K/2], sf e4m3 uint8 [rows][K/16])."""
    x = _c(x, np.float32)
    rows, K = x.shape
    codes = np.zeros((rows, K // 2), np.uint8)
    sf = np.zeros((rows, K // 16), np.uint8)
    lib().orc_quant_nvfp4(_p(x), rows, K, float(np.float32(g)), _p(codes), _p(sf))
    return codes, sf


def quant_mxfp4(x: np.ndarray):
    """rows x K fp32 -> (codes uint8 [rows][K/2], sf e8m0 uint8 [rows][K/32])."""
    x = _c(x, np.float32)
    rows, K = x.shape
    codes = np.zeros((rows, K // 2), np.uint8)
    sf = np.zeros((rows, K // 32), np.uint8)
    lib().orc_quant_mxfp4(_p(x), rows, K, _p(codes), _p(sf))
    return codes, sf


def quant_fp8(x: np.ndarray, s: float):
    x = _c(x, np.float32)
    codes = np.zeros(x.shape, np.uint8)
    lib().orc_quant_fp8(_p(x), x.size, float(np.float32(s)), _p(codes))
    return codes


def bf16_encode(v: float) -> int:
    return int(lib().orc_bf16_encode(float(np.float32(v))))


def quant_bf16(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 codes (little-endian uint16 bytes), the oracle's own rounding."""
    x = _c(x, np.float32)
    codes = np.zeros(x.shape[:-1] + (2 * x.shape[-1],), np.uint8)
    lib().orc_quant_bf16(_p(x), x.size, _p(codes))
    return codes


def dequant(fmt: int, codes: np.ndarray, sf, gs: float, rows: int, K: int) -> np.ndarray:
    codes = _c(codes, np.uint8)
    sf = None if sf is None else _c(sf, np.uint8)
    out = np.zeros((rows, K), np.float64)
    lib().orc_dequant(fmt, _p(codes), _p(sf), float(gs), rows, K, _p(out))
    return out


# ---------------------------------------------------------------- router ----
def router_logits(x_bf16_bits: np.ndarray, wr_bf16_bits: np.ndarray, bias=None) -> np.ndarray:
    x = _c(x_bf16_bits, np.uint16)
    wr = _c(wr_bf16_bits, np.uint16)
    T, H = x.shape
    E = wr.shape[0]
    b = None if bias is None else _c(bias, np.float32)
    out = np.zeros((T, E), np.float64)
    lib().orc_router_logits(_p(x), T, H, _p(wr), E, _p(b), _p(out))
    return out


ROUTER_ORDER_SMALL_BATCH = 1   # 256 partial sums, exchange within groups of 32, groups in order
ROUTER_ORDER_SEQUENTIAL = 2


def router_logits_ordered(x_bf16_bits: np.ndarray, wr_bf16_bits: np.ndarray, bias=None,
                          order: int = ROUTER_ORDER_SMALL_BATCH) -> np.ndarray:
    """fp32 logits [T][E] in one of the fixed summation orders (see moe_oracle.cpp)."""
    x = _c(x_bf16_bits, np.uint16)
    wr = _c(wr_bf16_bits, np.uint16)
    T, H = x.shape
    E = wr.shape[0]
    b = None if bias is None else _c(bias, np.float32)
    out = np.zeros((T, E), np.float32)
    if lib().orc_router_logits_ordered(_p(x), T, H, _p(wr), E, _p(b), int(order), _p(out)) != 0:
        raise ValueError("oracle router_logits_ordered rejected its arguments")
    return out


def topk(logits: np.ndarray, k: int):
    """-> (idx int32 [T,k], w float64 [T,k], status)."""
    L = _c(logits, np.float64)
    T, E = L.shape
    idx = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float64)
    st = lib().orc_topk(_p(L), T, E, k, _p(idx), _p(w))
    return idx, w, st


def permute(idx: np.ndarray, E: int):
    """-> (offsets [E+1], perm_token [S], inv_perm [S], status)."""
    idx = _c(idx, np.int32)
    T, k = idx.shape
    offsets = np.zeros(E + 1, np.int32)
    perm = np.zeros(T * k, np.int32)
    inv = np.zeros(T * k, np.int32)
    st = lib().orc_permute(_p(idx), T, k, E, _p(offsets), _p(perm), _p(inv))
    return offsets, perm, inv, st


# ------------------------------------------------------------- expert FFN ----
class Weights:
    """Canonical quantised expert weights held as numpy arrays (see moe_oracle.cpp)."""

    def __init__(self, fmt, E, H, I, w13, w13_sf, w13_gs, w2, w2_sf, w2_gs):
        self.fmt, self.E, self.H, self.I = fmt, E, H, I
        self.w13 = _c(w13, np.uint8)
        self.w13_sf = None if w13_sf is None else _c(w13_sf, np.uint8)
        self.w13_gs = None if w13_gs is None else _c(w13_gs, np.float32)
        self.w2 = _c(w2, np.uint8)
        self.w2_sf = None if w2_sf is None else _c(w2_sf, np.uint8)
        self.w2_gs = None if w2_gs is None else _c(w2_gs, np.float32)

    def struct(self) -> OrcWeights:
        return OrcWeights(self.fmt, self.E, self.H, self.I, _p(self.w13), _p(self.w13_sf), _p(self.w13_gs),
                          _p(self.w2), _p(self.w2_sf), _p(self.w2_gs))


def quantize_expert_weights_by_expert(fmt: int, E: int, w13_of, w2_of, threads: int = 1) -> Weights:
    """quantize_expert_weights for banks too large to hold in fp32 at once:
    w13_of(e) and w2_of(e) return expert e's fp32 [2I][H] and [H][I]; experts
    are drawn and quantised `threads` at a time (the quantisers release the
    interpreter lock)."""
    from concurrent.futures import ThreadPoolExecutor
    first = quantize_expert_weights(fmt, w13_of(0)[None], w2_of(0)[None])
    H, I = first.H, first.I
    parts = [None] * E
    parts[0] = first

    def one(e):
        parts[e] = quantize_expert_weights(fmt, w13_of(e)[None], w2_of(e)[None])

    with ThreadPoolExecutor(max(1, threads)) as ex:
        list(ex.map(one, range(1, E)))

    def cat(name):
        a = [getattr(p, name) for p in parts]
        return None if a[0] is None else np.concatenate(a)

    return Weights(fmt, E, H, I, cat("w13"), cat("w13_sf"), cat("w13_gs"), cat("w2"), cat("w2_sf"), cat("w2_gs"))


def quantize_expert_weights(fmt: int, w13: np.ndarray, w2: np.ndarray) -> Weights:
    """fp32 expert weights -> canonical quantised Weights, by the oracle's own
    quantisers.  w13 is [E][2I][H] (gate rows first), w2 is [E][H][I].  NVFP4
    and FP8 take one amax-derived scale per part (gate, up, down) per expert;
    MXFP4 has block scales only."""
    E, twoI, H = w13.shape
    I = twoI // 2
    if fmt == FMT_BF16:
        return Weights(fmt, E, H, I, quant_bf16(w13), None, None, quant_bf16(w2), None, None)
    if fmt == FMT_FP8:
        c13 = np.zeros((E, twoI, H), np.uint8)
        c2 = np.zeros((E, H, I), np.uint8)
        g13 = np.zeros((E, 2), np.float32)
        g2 = np.zeros(E, np.float32)
        for e in range(E):
            for part in range(2):
                blk = w13[e, part * I:(part + 1) * I]
                s = fp8_scale(amax(blk))
                g13[e, part] = s
                c13[e, part * I:(part + 1) * I] = quant_fp8(blk, s)
            s = fp8_scale(amax(w2[e]))
            g2[e] = s
            c2[e] = quant_fp8(w2[e], s)
        return Weights(fmt, E, H, I, c13, None, g13, c2, None, g2)
    bs = 16 if fmt == FMT_NVFP4 else 32
    c13 = np.zeros((E, twoI, H // 2), np.uint8)
    s13 = np.zeros((E, twoI, H // bs), np.uint8)
    c2 = np.zeros((E, H, I // 2), np.uint8)
    s2 = np.zeros((E, H, I // bs), np.uint8)
    g13 = np.ones((E, 2), np.float32) if fmt == FMT_NVFP4 else None
    g2 = np.ones(E, np.float32) if fmt == FMT_NVFP4 else None
    for e in range(E):
        for part in range(2):
            blk = w13[e, part * I:(part + 1) * I]
            if fmt == FMT_NVFP4:
                g = nvfp4_global_scale(amax(blk))
                g13[e, part] = g
                c, s = quant_nvfp4(blk, g)
            else:
                c, s = quant_mxfp4(blk)
            c13[e, part * I:(part + 1) * I] = c
            s13[e, part * I:(part + 1) * I] = s
        if fmt == FMT_NVFP4:
            g = nvfp4_global_scale(amax(w2[e]))
            g2[e] = g
            c, s = quant_nvfp4(w2[e], g)
        else:
            c, s = quant_mxfp4(w2[e])
        c2[e], s2[e] = c, s
    return Weights(fmt, E, H, I, c13, s13, g13, c2, s2, g2)


def grouped_ffn(x_bf16_bits, perm_token, offsets, W: Weights, act: int, a13_static=0.0, a2_static=0.0,
                nthreads: int = 0):
    """y_perm float64 [S][H] for the permuted slots; returns (y, (x_scale, h_scale))."""
    x = _c(x_bf16_bits, np.uint16)
    T = x.shape[0]
    perm = _c(perm_token, np.int32)
    off = _c(offsets, np.int32)
    S = int(off[-1])
    y = np.zeros((S, W.H), np.float64)
    scales = np.zeros(2, np.float32)
    ws = W.struct()
    st = lib().orc_grouped_ffn(_p(x), T, _p(perm), _p(off), ctypes.byref(ws), act, float(a13_static),
                               float(a2_static), _p(y), nthreads or default_threads(), _p(scales))
    if st != 0:
        raise ValueError("oracle grouped_ffn rejected its arguments")
    return y, (float(scales[0]), float(scales[1]))


def combine(y_perm, inv_perm, w, k: int, shared_y=None) -> np.ndarray:
    y = _c(y_perm, np.float64)
    inv = _c(inv_perm, np.int32)
    wt = _c(w, np.float64)
    T = wt.size // k
    H = y.shape[1]
    sh = None if shared_y is None else _c(shared_y, np.float64)
    out = np.zeros((T, H), np.float64)
    lib().orc_combine(_p(y), _p(inv), _p(wt), T, k, H, _p(sh), _p(out))
    return out


def moe_forward(x_bf16_bits, wr_bf16_bits, bias, k: int, routed: Weights, shared: Weights | None = None,
                act: int = ACT_MATCH, a13_static=0.0, a2_static=0.0, sh_a2_static=0.0, tokens=None,
                nthreads: int = 0, router_order: int = 0):
    """The whole layer.  Returns dict(out [n][H], logits [n][E], idx [n][k], w [n][k], status).
    router_order 0 routes on fp64 logits; 1 or 2 on fp32 logits in that fixed order."""
    x = _c(x_bf16_bits, np.uint16)
    wr = _c(wr_bf16_bits, np.uint16)
    T, H = x.shape
    E = wr.shape[0]
    b = None if bias is None else _c(bias, np.float32)
    tok = None if tokens is None else _c(tokens, np.int32)
    n = T if tok is None else tok.size
    out = np.zeros((n, H), np.float64)
    logits = np.zeros((n, E), np.float64)
    idx = np.zeros((n, k), np.int32)
    w = np.zeros((n, k), np.float64)
    rs = routed.struct()
    ss = shared.struct() if shared is not None else None
    st = lib().orc_moe_forward(_p(x), T, H, _p(wr), _p(b), E, k, ctypes.byref(rs),
                               ctypes.byref(ss) if ss is not None else None, act, float(a13_static),
                               float(a2_static), float(sh_a2_static), _p(tok), n, _p(out), _p(logits), _p(idx),
                               _p(w), nthreads or default_threads(), int(router_order))
    return dict(out=out, logits=logits, idx=idx, w=w, status=st)


def default_threads() -> int:
    return max(1, int(lib().orc_num_threads_available()))
