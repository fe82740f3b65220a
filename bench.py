#!/usr/bin/env python
"""Benchmark of the routed MoE expert-FFN layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one moe_forward (router -> top-k -> histogram/permutation ->
activation quantisation -> gate|up projection + SwiGLU -> down projection ->
combine) over one batch of the prefill workload: T=4096 tokens, hidden 2048,
128 experts, top-8, intermediate 768, NVFP4 weights and activations (W4A4,
static activation scales), Zipf(1.1)-skewed routing.  Inputs are seeded and
synthetic and resident in HBM; L2 is flushed (a 256 MiB write) between timed
steps, outside the timed events.  Time is taken with CUDA events on the
launching stream, max over ranks.  With N > 1 every rank runs an independent
replica (the layer needs no collective: tokens are independent given the
weights), so scaling is weak and `value` is the tokens of all ranks divided
by the slowest rank's time.

Rank 0 prints one JSON line.  Besides the contract keys it carries:
  stages       per-stage device time (ms) from the library's stage events
  roofline     the dominant stage against the measured peak
  e2e          the same metric with the input copied from pinned host memory
               and the output copied back inside the timed region, through
               moe_forward_host (token slices whose copies overlap the other
               slices' forwards; checked against the device-resident output)
  decode       the decode workload (T=4, static activation scales): step time
               and the expert-weight streaming rate of moe_grouped_ffn (GB/s)
  configs      the FP8 W8A8 + shared-expert and the large MXFP4 workloads:
               tokens/s (median, p10/p90), GEMM TFLOP/s against the format's
               tensor peak, active-expert weight GB/s against HBM, routing
  cpu_baseline the CPU oracle on a bounded token sample (rank 0, N = 1)
  clocks       nvidia-smi samples taken during the timed region
`--impl reference` times the CPU oracle instead (the only other arm).
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s at T=4096 prefill; decode weight GB/s (% of HBM peak)"
FP4_PER_BF16 = 4.0      # nominal dense FP4 : BF16 tensor rate on B200 (9 : 2.25 PFLOP/s)
FP8_PER_BF16 = 2.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="prefill")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-config report (fp8_shared, large)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target CPU time of the oracle sample")
    ap.add_argument("--e2e-slices", type=int, default=4, help="token slices of the end-to-end leg")
    ap.add_argument("--profile-range", action="store_true",
                    help="bracket the timed prefill replays with cudaProfilerStart/Stop (for ncu --profile-from-start off)")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks --
class ClockSampler:
    """nvidia-smi clocks and throttle reasons during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.2)
        self.proc.terminate()
        self.proc.wait()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        load = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": float(np.median(load)), "sm_max_mhz": float(max(smax)), "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------- layers -----
def build_layer(ops, synth, torch, w, static: bool):
    """Weights drawn on the GPU (CUDA Philox), quantised and prepared by the library."""
    fmt = ops.FMT_BY_NAME[w.fmt]
    ws = ops.new_workspace(4096)
    banks = []
    chunks13, chunks2 = [], []
    for e in range(w.E):
        chunks13.append(synth.cuda_normal((1, 2 * w.I, w.H), w.w_std, synth.TID_W13 + e))
        chunks2.append(synth.cuda_normal((1, w.H, w.I), w.w_std, synth.TID_W2 + e))
    w13 = torch.cat(chunks13)
    w2 = torch.cat(chunks2)
    del chunks13, chunks2
    bank = ops.quantize_bank(fmt, w13, w2, ws)
    del w13, w2
    if static and fmt in (ops.FMT_NVFP4, ops.FMT_FP8):
        a13, a2 = synth.static_act_scales()
        bank.a13_gs = torch.tensor([a13], dtype=torch.float32, device="cuda")
        bank.a2_gs = torch.tensor([a2], dtype=torch.float32, device="cuda")
    prepared = ops.moe_prepare_weights(bank)
    torch.cuda.synchronize()
    del bank
    shared = None
    if w.shared_I:
        s13 = synth.cuda_normal((1, 2 * w.shared_I, w.H), w.w_std, synth.TID_SH_W13)
        s2 = synth.cuda_normal((1, w.H, w.shared_I), w.w_std, synth.TID_SH_W2)
        sbank = ops.quantize_bank(fmt, s13, s2, ws)
        if static and fmt in (ops.FMT_NVFP4, ops.FMT_FP8):
            # the shared expert reads the routed layer's x scale; its own h scale
            sbank.a2_gs = torch.tensor([synth.static_act_scales()[1]], dtype=torch.float32, device="cuda")
        shared = ops.moe_prepare_weights(sbank)
        del s13, s2, sbank
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    x = synth.cuda_normal((w.T, w.H), 1.0, synth.TID_X, dtype=torch.bfloat16)
    wr = synth.cuda_normal((w.E, w.H), w.wr_std, synth.TID_WR, dtype=torch.bfloat16)
    bias = synth.cuda_router_bias(w)
    return prepared, x, wr, bias, shared


def algorithmic(w, bank_fmt: str, offsets: np.ndarray):
    """FLOPs and bytes of one forward by definition (routed slots only;
    weights of experts with at least one slot; x, out, Wr)."""
    T, H, E, k, I = w.T, w.H, w.E, w.k, w.I
    S = T * k
    flops_up = 2.0 * S * H * 2 * I
    flops_down = 2.0 * S * I * H
    counts = np.diff(offsets)
    active = int((counts > 0).sum())
    if bank_fmt == "fp8":
        per13, per2 = 2 * I * H, H * I
    elif bank_fmt == "bf16":
        per13, per2 = 2 * I * H * 2, H * I * 2
    else:
        bs = 16 if bank_fmt == "nvfp4" else 32
        per13 = 2 * I * H // 2 + 2 * I * H // bs
        per2 = H * I // 2 + H * I // bs
    wbytes_up = active * per13
    wbytes_down = active * per2
    io = T * H * 2 * 2 + E * H * 2
    return dict(flops_up=flops_up, flops_down=flops_down, wbytes_up=wbytes_up, wbytes_down=wbytes_down,
                io_bytes=io, active_experts=active, max_over_mean=float(counts.max() / max(counts.mean(), 1e-9)),
                zero_experts=int((counts == 0).sum()))


PROFILE_RANGE = False

# Sources the grouped GEMM is built from; a stored ncu traffic figure counts
# only while they are unchanged.
GEMM_SOURCES = ("gemm_tc.cu", "gemm_tc.cuh", "tc_ptx.cuh", "common.cuh", "kernels.cuh", "token_quant.cuh",
                "topk_warp.cuh")


def gemm_sources_sha256() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in GEMM_SOURCES:
        with open(os.path.join(ROOT, "quantized_expert_ffn_top_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def measured_traffic(kernel: str, workload: str):
    """DRAM bytes per launch (read + write) from profiles/traffic.json, or
    None when none was captured for this kernel and workload or the sources
    changed since."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(f"{workload}/{kernel}")
    if not d or d.get("sources_sha256") != gemm_sources_sha256():
        return None
    return d["dram_bytes_per_launch"]


def time_forward(ops, torch, layer, w, act, steps, warmup, flush, stage=True, host_io=False):
    """Times `steps` forwards.  Device-resident runs replay a CUDA graph of
    moe_forward (one graph launch per step, L2 flushed before each, CUDA
    events around each replay); the per-stage split comes from a second graph
    that records the library's stage events.  host_io runs time the eager
    user call with the host<->device copies inside the events."""
    prepared, x, wr, bias, shared = layer
    ws = ops.new_workspace(ops.workspace_size(w.T, w.k, prepared, shared, act))
    out = torch.empty_like(x)
    stream = torch.cuda.current_stream()

    def fwd():
        ops.moe_forward(x, wr, bias, w.k, prepared, shared, act, ws, out=out)

    l0 = ops.moe_kernel_launch_count()
    for _ in range(max(warmup, 1)):
        fwd()
    torch.cuda.synchronize()
    per_step_launches = (ops.moe_kernel_launch_count() - l0) // max(warmup, 1)
    if ops.moe_get_device_status(ws) != 0:
        raise RuntimeError("device status reported a fault during warm-up")
    step_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    stages = {}
    if host_io:
        x_host = x.cpu().pin_memory()
        out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        torch.cuda.synchronize()
        for i in range(steps):
            flush.zero_()
            step_evs[i][0].record(stream)
            x.copy_(x_host, non_blocking=True)
            fwd()
            out_host.copy_(out, non_blocking=True)
            step_evs[i][1].record(stream)
        torch.cuda.synchronize()
    else:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            fwd()
        torch.cuda.synchronize()
        if PROFILE_RANGE:
            torch.cuda.profiler.start()
        for i in range(steps):
            flush.zero_()
            step_evs[i][0].record(stream)
            graph.replay()
            step_evs[i][1].record(stream)
        torch.cuda.synchronize()
        if PROFILE_RANGE:
            torch.cuda.profiler.stop()
        if stage:
            evs = [torch.cuda.Event(enable_timing=True) for _ in range(2 * len(ops.STAGES))]
            ops.moe_set_stage_events(evs)
            g2 = torch.cuda.CUDAGraph()
            try:
                with torch.cuda.graph(g2):
                    fwd()
            finally:
                ops.moe_set_stage_events(None)
            # only the stages this forward records (the others' events hold
            # nothing but the binding's set-up records)
            mask = ops.moe_stage_mask()
            ran = [(si, n) for si, n in enumerate(ops.STAGES) if mask >> si & 1]
            acc = {n: [] for _, n in ran}
            for i in range(steps):
                flush.zero_()
                g2.replay()
                torch.cuda.synchronize()
                for si, name in ran:
                    acc[name].append(evs[2 * si].elapsed_time(evs[2 * si + 1]))
            stages = {n: float(np.mean(v)) for n, v in acc.items() if v}
            del g2
        del graph
    per_step = [a.elapsed_time(b) for a, b in step_evs]
    idx, _ = ops.moe_route(x, wr, bias, w.k, ops.new_workspace(ops.workspace_size(w.T, w.k, prepared, None, act)))
    off, _, _ = ops.moe_permute(idx, w.E, ops.new_workspace(1 << 24))
    return dict(ms=per_step, stages=stages, launches=per_step_launches * steps, offsets=off.cpu().numpy(),
                status=ops.moe_get_device_status(ws))


def time_forward_host(ops, torch, layer, w, act, steps, warmup, flush, n_slices):
    """Times `steps` calls of moe_forward_host (pinned host x in, host out
    back, n_slices token slices) with CUDA events on the caller's stream,
    which the call joins after its last copy-out.  Returns the step times
    and the number of tokens whose output differs from the device-resident
    forward's by more than the layer tolerance (a slice may route a token
    whose top-k logits tie within rounding differently)."""
    prepared, x, wr, bias, shared = layer
    Ts = -(-w.T // n_slices)
    ws = ops.new_workspace(ops.workspace_size(Ts, w.k, prepared, shared, act))
    ref = ops.moe_forward(x, wr, bias, w.k, prepared, shared, act,
                          ops.new_workspace(ops.workspace_size(w.T, w.k, prepared, shared, act)))
    x_host = x.cpu().pin_memory()
    out_host = torch.empty(x.shape, dtype=x.dtype).pin_memory()
    x_dev, out_dev = torch.empty_like(x), torch.empty_like(x)
    stream = torch.cuda.current_stream()

    def fwd():
        ops.moe_forward_host(x_host, wr, bias, w.k, prepared, shared, act, ws, x_dev, out_dev, out_host,
                             n_slices=n_slices)

    for _ in range(max(warmup, 1)):
        fwd()
    torch.cuda.synchronize()
    if ops.moe_get_device_status(ws) != 0:
        raise RuntimeError("device status reported a fault in moe_forward_host")
    r = ref.float().cpu()
    err = ((out_host.float() - r).abs().amax(dim=1) / r.abs().max().clamp_min(1e-30)).numpy()
    off = np.nonzero(err > 2e-2)[0]
    if off.size:
        ties = routing_near_ties(ops, torch, x, wr, bias, w.k, n_slices, off)
        if not ties.all():
            raise RuntimeError(f"{int((~ties).sum())} tokens differ from the device-resident forward "
                               "without a routing near-tie")
    bad = int(off.size)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        evs[i][0].record(stream)
        fwd()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    return dict(ms=[a.elapsed_time(b) for a, b in evs], bad_tokens=bad)


def routing_near_ties(ops, torch, x, wr, bias, k, n_slices, tokens):
    """For each token listed: whether its top-k choice may legitimately differ
    between a forward of its slice and of the whole batch -- the gap between
    its k-th and (k+1)-th whole-batch logits is within twice the largest
    difference between the two routers' logits (the router splits its sums
    differently at another batch size)."""
    T, E = x.shape[0], wr.shape[0]
    ws = ops.new_workspace(T * E * 16 + (1 << 20))
    Lw = torch.empty((T, E), dtype=torch.float32, device=x.device)
    ops.moe_route(x, wr, bias, k, ws, logits=Lw)
    Ls = torch.empty_like(Lw)
    Ts = -(-T // n_slices)
    for t0 in range(0, T, Ts):
        ops.moe_route(x[t0:t0 + Ts], wr, bias, k, ws, logits=Ls[t0:t0 + Ts])
    torch.cuda.synchronize()
    band = 2.0 * float((Ls - Lw).abs().max().item())
    srt = torch.sort(Lw[torch.as_tensor(tokens, device=x.device)], dim=1, descending=True).values
    gap = (srt[:, k - 1] - srt[:, k]) if k < E else torch.full((len(tokens),), float("inf"), device=x.device)
    return (gap <= band).cpu().numpy()


def time_grouped_ffn(ops, torch, layer, w, act, steps, warmup, flush):
    """Device time of the grouped expert FFN alone (moe_grouped_ffn: tile
    plan, activation quantisation, gate|up + SwiGLU, down) on the layer's
    routed slots, one CUDA-graph replay per step, L2 flushed before each."""
    prepared, x, wr, bias, _ = layer
    ws = ops.new_workspace(ops.workspace_size(w.T, w.k, prepared, None, act))
    idx, _ = ops.moe_route(x, wr, bias, w.k, ws)
    off, perm, _ = ops.moe_permute(idx, w.E, ops.new_workspace(1 << 24))
    y = torch.empty((w.T * w.k, w.H), dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream()

    def ffn():
        ops.moe_grouped_ffn(x, w.k, perm, off, prepared, act, ws, y_perm=y)

    for _ in range(max(warmup, 1)):
        ffn()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        ffn()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush.zero_()
        evs[i][0].record(stream)
        graph.replay()
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    del graph
    if ops.moe_get_device_status(ws) != 0:
        raise RuntimeError("device status reported a fault in the grouped FFN")
    return [a.elapsed_time(b) for a, b in evs], off.cpu().numpy()


def config_report(ops, torch, synth, name, act, steps, warmup, flush, pk, static=None):
    """Per-config figures: tokens/s, the GEMMs' TFLOP/s against the format's
    tensor peak, the active experts' weight GB/s against HBM, and the routing
    histogram.  Stage times come from the library's stage events.  static:
    static activation scales (default: for NVFP4 layers)."""
    w = synth.workload(name)
    static = (w.fmt == "nvfp4") if static is None else static
    layer = build_layer(ops, synth, torch, w, static=static)
    r = time_forward(ops, torch, layer, w, act, steps, warmup, flush)
    del layer
    torch.cuda.empty_cache()
    alg = algorithmic(w, w.fmt, r["offsets"])
    st = r["stages"]
    ms = np.array(r["ms"])
    peak = pk["bf16_tflops"] * {"fp8": FP8_PER_BF16, "bf16": 1.0}.get(w.fmt, FP4_PER_BF16)
    up, down = st.get("ffn_up", 0.0), st.get("ffn_down", 0.0)
    scales = "none" if w.fmt == "bf16" else ("static" if static and w.fmt in ("nvfp4", "fp8") else
                                               ("dynamic" if w.fmt in ("nvfp4", "fp8") else "none (block scales only)"))
    rep_ = {"workload": workload_name(w), "act_scales": scales,
            "ms_median": float(np.median(ms)), "ms_p10": float(np.percentile(ms, 10)),
            "ms_p90": float(np.percentile(ms, 90)), "tokens_per_s": w.T / (float(np.median(ms)) * 1e-3),
            "stages_ms": st, "routing": {"active_experts": alg["active_experts"],
                                         "max_over_mean": alg["max_over_mean"], "zero_experts": alg["zero_experts"]}}
    if up > 0 and down > 0:
        tf_up = alg["flops_up"] / (up * 1e-3) / 1e12
        tf_down = alg["flops_down"] / (down * 1e-3) / 1e12
        gbs = (alg["wbytes_up"] + alg["wbytes_down"]) / ((up + down) * 1e-3) / 1e9
        rep_.update({"gemm_up_tflops": tf_up, "gemm_up_frac": tf_up / peak, "gemm_down_tflops": tf_down,
                     "gemm_down_frac": tf_down / peak, "tensor_peak_tflops": peak,
                     "weight_gbs": gbs, "weight_hbm_frac": gbs / pk["hbm_gbs"]})
    return rep_


# ------------------------------------------------------------ CPU oracle ----
def cpu_oracle_sample(w, target_s: float, static: bool, max_tokens: int | None = None):
    """The oracle as it stands, on a bounded token sample of the workload."""
    import oracle
    from quantized_expert_ffn_top_b200 import synth
    fmt = {"nvfp4": 1, "mxfp4": 2, "fp8": 3}[w.fmt]
    t0 = time.time()
    W = oracle.quantize_expert_weights(fmt, synth.all_w13(w), synth.all_w2(w))
    x = synth.x_bits(w)
    wr = synth.router_bits(w)
    b = synth.router_bias(w)
    a13, a2 = synth.static_act_scales() if static else (0.0, 0.0)
    setup_s = time.time() - t0
    threads = oracle.default_threads()
    n = 4
    tok_s = None
    used = 0
    spent = 0.0
    while True:
        toks = np.arange(n, dtype=np.int32) * (w.T // max(n, 1))
        t1 = time.time()
        oracle.moe_forward(x, wr, b, w.k, W, act=1, a13_static=a13, a2_static=a2, tokens=toks, nthreads=threads)
        dt = time.time() - t1
        spent += dt
        used = n
        tok_s = n / dt
        if dt * 2 > target_s or spent > target_s or (max_tokens and n >= max_tokens):
            break
        n = int(min(max(n * 2, n * target_s / max(dt, 1e-3) * 0.5), max_tokens or 1 << 30))
    return {"value": tok_s, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{used} evenly spaced tokens of the {w.name} workload (T={w.T}), fp64 oracle, "
                      f"{threads} OpenMP threads; weights drawn and quantised on the host in {setup_s:.0f} s"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from quantized_expert_ffn_top_b200 import synth
    import oracle
    w = synth.workload(args.workload)
    fmt = {"nvfp4": 1, "mxfp4": 2, "fp8": 3}[w.fmt]
    W = oracle.quantize_expert_weights(fmt, synth.all_w13(w), synth.all_w2(w))
    x = synth.x_bits(w)
    wr = synth.router_bits(w)
    b = synth.router_bias(w)
    a13, a2 = synth.static_act_scales()
    threads = oracle.default_threads()
    n = 8
    rng = np.random.default_rng(0)

    def step():
        toks = rng.choice(w.T, size=n, replace=False).astype(np.int32)
        oracle.moe_forward(x, wr, b, w.k, W, act=1, a13_static=a13, a2_static=a2, tokens=toks, nthreads=threads)

    for _ in range(args.warmup):
        step()
    t0 = time.time()
    for _ in range(args.steps):
        step()
    dt = time.time() - t0
    v = n * args.steps / dt
    line = {"metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": workload_name(w), "sample_tokens_per_step": n},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": f"{n} random tokens per step of the {w.name} workload"},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_name(w) -> str:
    acts = {"fp8": "W8A8", "bf16": "bf16"}.get(w.fmt, "W4A4")
    s = (f"{w.name}: T={w.T} H={w.H} E={w.E} top-{w.k} I={w.I} {w.fmt.upper()} weights, "
         f"{acts} activations, {w.router} router")
    if w.shared_I:
        s += f", shared expert I={w.shared_I}"
    return s


# ------------------------------------------------------------- replicas ----
def max_over_ranks(value: float, device="cuda") -> float:
    """The slowest rank's time (no-op without an initialised process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _round_floats(v, digits: int = 4):
    if isinstance(v, float):
        return float(f"{v:.{digits}g}")
    if isinstance(v, dict):
        return {k: _round_floats(x, digits) for k, x in v.items()}
    if isinstance(v, list):
        return [_round_floats(x, digits) for x in v]
    return v


def job_throughput(tokens_per_rank: int, steps: int, world: int, slowest_s: float) -> float:
    """Whole-job tokens/s: every replica's tokens over the slowest replica's time."""
    return world * tokens_per_rank * steps / slowest_s


# ------------------------------------------------------------------ main ----
def main():
    args = parse()
    global PROFILE_RANGE
    PROFILE_RANGE = args.profile_range
    if args.impl == "reference":
        run_reference(args)
        return
    import torch
    import torch.distributed as dist
    from quantized_expert_ffn_top_b200 import ops, synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    ops.lib()
    pk, pk_kind = peaks()
    w = synth.workload(args.workload)
    act = ops.ACT_MATCH
    layer = build_layer(ops, synth, torch, w, static=True)
    l2 = torch.cuda.get_device_properties(local).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device="cuda")

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    clock = ClockSampler(local)
    barrier()
    clock.start()
    res = time_forward(ops, torch, layer, w, act, args.steps, args.warmup, flush)
    barrier()
    clocks = clock.stop()
    ms = float(np.mean(res["ms"]))
    total_s = max_over_ranks(float(np.sum(res["ms"])) / 1e3)
    ms = total_s * 1e3 / args.steps
    value = job_throughput(w.T, args.steps, world, total_s)

    # end to end: pinned host input -> device -> forward -> host output, in
    # token slices whose copies overlap the other slices' forwards; the
    # whole batch after one copy when that path fails its check
    barrier()
    method = f"moe_forward_host, {args.e2e_slices} token slices"
    try:
        res_e2e = time_forward_host(ops, torch, layer, w, act, args.steps, 2, flush, args.e2e_slices)
    except (RuntimeError, ops.MoeError) as exc:
        method = f"copy in, moe_forward, copy out (sliced path not used: {exc})"
        res_e2e = time_forward(ops, torch, layer, w, act, args.steps, 2, flush, stage=False, host_io=True)
    # whether any rank fell back (every rank runs this collective once)
    fell_back = max_over_ranks(0.0 if method.startswith("moe_forward_host") else 1.0) > 0
    e2e_s = max_over_ranks(float(np.sum(res_e2e["ms"])) / 1e3)
    e2e = {"value": job_throughput(w.T, args.steps, world, e2e_s), "unit": "tokens/s",
           "h2d_bytes_per_step": w.T * w.H * 2, "d2h_bytes_per_step": w.T * w.H * 2, "method": method}
    if not fell_back:
        e2e["tokens_off_by_routing_ties"] = res_e2e["bad_tokens"]

    alg = algorithmic(w, w.fmt, res["offsets"])
    stages = res["stages"]
    # dominant stage and its roofline
    dom = max(stages, key=stages.get) if stages else "ffn_up"
    peak_tensor = pk["bf16_tflops"] * (FP4_PER_BF16 if w.fmt != "fp8" else FP8_PER_BF16)
    if dom in ("ffn_up", "ffn_down"):
        flops = alg["flops_up"] if dom == "ffn_up" else alg["flops_down"]
        achieved = flops / (stages[dom] * 1e-3) / 1e12
        roof = {"kernel": dom, "bound": "tensor", "achieved": achieved, "peak": peak_tensor, "unit": "TFLOP/s",
                "frac": achieved / peak_tensor, "traffic": measured_traffic(dom, w.name),
                "peak_source": f"{pk_kind} bf16 x {FP4_PER_BF16 if w.fmt != 'fp8' else FP8_PER_BF16:g} nominal ratio"}
    else:
        roof = {"kernel": dom, "bound": "hbm", "achieved": None, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": None, "traffic": None, "peak_source": pk_kind}

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "nvfp4" if w.fmt == "nvfp4" else w.fmt, "data": "synthetic",
            "config": {"workload": workload_name(w), "global_batch": world * w.T, "parallelism": f"replicas x{world}",
                       "act_scales": "static", "l2": "flushed between steps (write of 2x L2 bytes)",
                       "routing": {"active_experts": alg["active_experts"], "max_over_mean": alg["max_over_mean"],
                                   "zero_experts": alg["zero_experts"]}},
            "stages_ms": stages, "roofline": roof, "e2e": e2e, "gpu_launches": int(res["launches"]),
            "clocks": clocks, "device_status": res["status"]}

    if not args.no_decode:
        wd = synth.workload("decode")
        dl = build_layer(ops, synth, torch, wd, static=True)
        rd = time_forward(ops, torch, dl, wd, act, max(args.steps, 20), args.warmup, flush)
        ffn_runs, d_off = time_grouped_ffn(ops, torch, dl, wd, act, max(args.steps, 20), args.warmup, flush)
        ad = algorithmic(wd, wd.fmt, d_off)
        ffn_ms = float(np.mean(ffn_runs))
        gbs = (ad["wbytes_up"] + ad["wbytes_down"]) / (ffn_ms * 1e-3) / 1e9 if ffn_ms else None
        line["decode"] = {"workload": workload_name(wd), "act_scales": "static", "ms_per_step": float(np.mean(rd["ms"])),
                          "tokens_per_s": wd.T / (float(np.mean(rd["ms"])) * 1e-3),
                          "expert_weight_bytes": ad["wbytes_up"] + ad["wbytes_down"],
                          "active_experts": ad["active_experts"], "ffn_ms": ffn_ms,
                          "ffn_timing": "moe_grouped_ffn alone, graph replay, L2 flushed", "weight_gbs": gbs,
                          # one fused kernel at this batch size; two launches otherwise
                          "traffic": measured_traffic("ffn", "decode") or (
                              lambda u, d: u + d if u is not None and d is not None else None)(
                              measured_traffic("ffn_up", "decode"), measured_traffic("ffn_down", "decode")),
                          "hbm_frac": gbs / pk["hbm_gbs"] if gbs else None, "stages_ms": rd["stages"]}
        # the metric's second half, where the driver's record keeps it
        line["roofline"]["decode"] = {"kernel": "moe_grouped_ffn (decode workload)", "bound": "hbm",
                                      "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                                      "frac": line["decode"]["hbm_frac"], "traffic": line["decode"]["traffic"],
                                      "bytes": ad["wbytes_up"] + ad["wbytes_down"], "ms": ffn_ms,
                                      "peak_source": pk_kind}
        del dl

    if not args.no_configs:
        line["configs"] = [config_report(ops, torch, synth, "prefill", act, 10, 3, flush, pk, static=False)] + [
            config_report(ops, torch, synth, n, act, 10, 3, flush, pk) for n in ("fp8_shared", "large", "bf16_prefill")]

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_oracle_sample(w, args.cpu_seconds, static=True)
    # the per-config and decode blocks at four significant digits, so the
    # line stays short
    for key in ("configs", "decode"):
        if key in line:
            line[key] = _round_floats(line[key])
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
