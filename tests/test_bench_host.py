"""Host-side arithmetic of the benchmark: the algorithmic FLOPs and bytes the
roofline divides by, the gate on stored ncu traffic figures, and the workload
label.  CPU only."""
import json

import numpy as np

import bench
from quantized_expert_ffn_top_b200 import synth


def _offsets(counts):
    return np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)


def test_algorithmic_work_of_the_prefill_layer():
    """2*S*H*2I and 2*S*I*H flops; per active expert 2I*H and H*I FP4 codes
    (half a byte each) plus one e4m3 scale per 16 values (NVFP4)."""
    w = synth.workload("prefill")
    S = w.T * w.k
    counts = np.zeros(w.E, dtype=np.int64)
    counts[:115] = S // 115
    counts[0] += S - counts.sum()
    a = bench.algorithmic(w, "nvfp4", _offsets(counts))
    assert a["flops_up"] == 2 * 32768 * 2048 * 1536 == 206158430208
    assert a["flops_down"] == 2 * 32768 * 768 * 2048
    assert a["active_experts"] == 115 and a["zero_experts"] == 13
    per13 = 1536 * 2048 // 2 + 1536 * 2048 // 16
    per2 = 2048 * 768 // 2 + 2048 * 768 // 16
    assert per13 + per2 == 2654208  # 2.654 MB of weights and scales per expert
    assert a["wbytes_up"] == 115 * per13 and a["wbytes_down"] == 115 * per2
    assert a["io_bytes"] == 4096 * 2048 * 2 * 2 + 128 * 2048 * 2


def test_algorithmic_weight_bytes_by_format():
    w = synth.workload("decode")
    counts = np.zeros(w.E, dtype=np.int64)
    counts[:27] = 1
    counts[0] += w.T * w.k - 27
    off = _offsets(counts)
    n13, n2 = 2 * w.I * w.H, w.H * w.I
    expect = {
        "nvfp4": (n13 // 2 + n13 // 16, n2 // 2 + n2 // 16),
        "mxfp4": (n13 // 2 + n13 // 32, n2 // 2 + n2 // 32),
        "fp8": (n13, n2),
        "bf16": (2 * n13, 2 * n2),
    }
    for fmt, (p13, p2) in expect.items():
        a = bench.algorithmic(w, fmt, off)
        assert a["wbytes_up"] == 27 * p13 and a["wbytes_down"] == 27 * p2, fmt
    # the decode layer's 27 active NVFP4 experts: 71.66 MB
    a = bench.algorithmic(w, "nvfp4", off)
    assert a["wbytes_up"] + a["wbytes_down"] == 71663616
    assert a["max_over_mean"] == counts.max() / counts.mean()


def test_stored_traffic_counts_only_for_unchanged_sources(monkeypatch, tmp_path):
    stored = json.load(open(bench.os.path.join(bench.ROOT, "profiles", "traffic.json")))
    for key, d in stored.items():
        assert d["dram_bytes_per_launch"] == d["read"] + d["write"], key
    wl, kern = "prefill", "ffn_up"
    got = bench.measured_traffic(kern, wl)
    if stored[f"{wl}/{kern}"]["sources_sha256"] == bench.gemm_sources_sha256():
        assert got == stored[f"{wl}/{kern}"]["dram_bytes_per_launch"]
    else:
        assert got is None
    monkeypatch.setattr(bench, "gemm_sources_sha256", lambda: "0" * 64)
    assert bench.measured_traffic(kern, wl) is None
    assert bench.measured_traffic("no_such_kernel", wl) is None


def test_workload_label_names_the_sizes():
    s = bench.workload_name(synth.workload("fp8_shared"))
    assert s.startswith("fp8_shared: T=512 H=2048 E=256 top-8 I=512 FP8 weights, W8A8 activations")
    assert s.endswith("shared expert I=512")
    assert "W4A4" in bench.workload_name(synth.workload("decode"))


def test_per_config_figures_are_rounded_but_keep_their_structure():
    d = {"ms": 0.123456789, "stages_ms": {"route": 0.0247123, "ffn_up": 0.0954}, "n": 7, "name": "x",
         "list": [1234567.89, 0.000123456]}
    r = bench._round_floats(d)
    assert r == {"ms": 0.1235, "stages_ms": {"route": 0.02471, "ffn_up": 0.0954}, "n": 7, "name": "x",
                 "list": [1235000.0, 0.0001235]}
    assert isinstance(r["n"], int)


def test_job_throughput_counts_every_rank():
    # value = tokens of all ranks / the slowest rank's time
    assert bench.job_throughput(4096, 20, 8, 0.02) == 4096 * 20 * 8 / 0.02
