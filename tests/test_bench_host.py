"""Host-side logic of bench.py that needs no GPU: the clock summary, the code-only
source hash that keys stored ncu counters, the workload config both arms report,
and the step roofline arithmetic."""
import sys
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parent.parent
sys.path.insert(0, str(ROOT))

import bench  # noqa: E402
from quantized_int8_gemm_q4_b200 import synth  # noqa: E402


def test_clock_summary_median_max_and_reasons():
    lines = [
        "0, 1965, 1965, 700.1, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1950, 1965, 990.5, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1965, 1965, 995.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "garbage line",
    ]
    c = bench.ClockSampler.summarize(lines)
    assert c["sm_mhz"] == 1965.0 and c["sm_max_mhz"] == 1965.0
    assert c["reasons"] == ["sw_power_cap"] and c["samples"] == 3
    assert bench.ClockSampler.summarize([]) is None


def test_source_hash_ignores_comments_only():
    a = ["int f(int x) {  // doubles x\n    return 2 * x;\n}\n"]
    b = ["// a new header comment\nint f(int x) {\n\n    return 2 * x;  // still doubles\n}\n"]
    c = ["int f(int x) {\n    return 3 * x;\n}\n"]
    assert bench.kernel_source_hash(a) == bench.kernel_source_hash(b)
    assert bench.kernel_source_hash(a) != bench.kernel_source_hash(c)


@pytest.mark.parametrize("name,layers,weight_bytes", [("llada-8b", 32, 4766023680), ("dream-7b", 28, 4607662080)])
def test_workload_config_is_the_workload(name, layers, weight_bytes):
    model = synth.MODELS[name]()
    cfg = bench.workload_config(model, 128, model.n_layers, 32, 1)
    assert cfg["layers"] == layers and cfg["canvas_tokens"] == 128
    assert cfg["weight_bytes_per_step"] == weight_bytes
    assert "graph" not in cfg  # implementation details are added by our arm only
    assert bench.workload_config(model, 128, model.n_layers, 32, 4)["parallelism"] == "replicas x4"


def test_step_roofline_matches_the_stated_target():
    model = synth.MODELS["llada-8b"]()
    gemms = bench.step_gemms(model, 128, model.n_layers)
    assert len(gemms) == 129
    t = bench.roofline_time(gemms, 6527.8, 4.5e15)
    assert abs(t * 1e3 - 0.8618) < 5e-4
    ops = sum(g.ops for g in gemms)
    assert abs(ops / 1e12 - 1.82) < 0.01  # 1.82 T int8 ops per step at canvas 128


def test_gather_last_step_shapes():
    """--gather-last: past attention the last layer runs on the requested rows only."""
    model = synth.MODELS["llada-8b"]()
    full = bench.step_gemms(model, 128, model.n_layers)
    g = bench.step_gemms(model, 128, model.n_layers, gather_last=True)
    assert [x.name for x in g] == [x.name for x in full]
    last = g[-5:-1]
    assert [x.M_out for x in last] == [128, 32, 32, 32]       # QKV still on the canvas
    assert all(a.M_out == b.M_out for a, b in zip(g[:-5], full[:-5]))
    h, f = model.hidden, model.ffn
    saved = 2 * (128 - 32) * (h * h + 2 * f * h + h * f)
    assert sum(x.ops for x in full) - sum(x.ops for x in g) == saved
    assert sum(x.weight_bytes for x in g) == sum(x.weight_bytes for x in full)
    cfg = bench.workload_config(model, 128, model.n_layers, 32, 1, gather_last=True)
    assert "requested rows only" in cfg["workload"]
    assert "requested rows only" not in bench.workload_config(model, 128, model.n_layers, 32, 1)["workload"]


def test_act_kernel_plan_matches_the_gemms():
    model = synth.MODELS["llada-8b"]()
    for gl in (False, True):
        plan = bench.act_kernel_plan(model, 128, model.n_layers, gl)
        gemms = bench.step_gemms(model, 128, model.n_layers, gl)
        assert len(plan) == len(gemms) == 129
        # each quantizer feeds the GEMM after it: same K and same activation rows
        for (kind, M, K), g in zip(plan, gemms):
            assert K == g.K
            assert M == g.M_act or (g.name == "output" and not gl)  # the output GEMM gathers rows
    kinds = [k for k, _, _ in bench.act_kernel_plan(model, 128, 2)]
    assert kinds == ["rmsnorm_quantize", "quantize_act", "rmsnorm_quantize", "swiglu_quantize"] * 2 + \
        ["rmsnorm_quantize"]


def test_act_rooflines():
    model = synth.MODELS["llada-8b"]()
    plan = bench.act_kernel_plan(model, 128, 1)
    # 2.78 MB of RMSNorm traffic in 5 us is 555.6 GB/s; swiglu 14.57 MB in 10 us
    d = [None, 0.004, 0.005, 0.010, 0.005]
    r = bench.act_rooflines(d, plan, 6527.8)
    rms = bench.act_bytes("rmsnorm_quantize", 128, 4096)
    assert abs(rms - 2777088) < 1   # 2 MiB of x + 16 KiB of gains + 0.64 MiB written
    assert r["rmsnorm_quantize"]["launches_timed"] == 2
    assert abs(r["rmsnorm_quantize"]["achieved_gbs"] - rms * 2 / 10e-6 / 1e9) < 0.1
    sw = bench.act_bytes("swiglu_quantize", 128, 12288)
    assert abs(r["swiglu_quantize"]["achieved_gbs"] - sw / 10e-6 / 1e9) < 0.1
    assert r["quantize_act"]["mean_us"] == 4.0
    assert abs(r["quantize_act"]["frac"] - r["quantize_act"]["achieved_gbs"] / 6527.8) < 1e-4


def test_split_durations_from_events():
    class Ev:
        def __init__(self, t):
            self.t = t

        def elapsed_time(self, other):
            return other.t - self.t

    # two steps of 3 (quantizer, GEMM) pairs: quantizers take 1, 2, 3 ms, GEMMs 10, 20, 30
    def step(t0):
        marks, t = [], t0
        for q, g in ((1, 10), (2, 20), (3, 30)):
            t += q
            marks.append(Ev(t))
            t += g
            marks.append(Ev(t))
        return marks
    gemm, quant, per = bench.split_durations([step(0.0), step(100.0)], 6)
    assert gemm == 60.0 and quant == 5.0   # the first quantizer of a step is not timed
    assert per == [None, 2.0, 3.0]


def test_parity_sample_covers_full_layers_and_sixty_fourths():
    model = synth.MODELS["llada-8b"]()
    smp = bench.parity_sample(model, model.n_layers, 6, 4)
    full = {l for (l, n), (a, b) in smp.items() if n == "down"}
    assert full == {0, 1, 2, 3, 4, 31}
    for l in range(model.n_layers):
        for p in model.layer:
            if l in full:
                assert smp[(l, p.name)] == (0, p.N)
            elif p.name == "down":
                assert (l, p.name) not in smp
            else:
                a, b = smp[(l, p.name)]
                assert b - a == p.N // 64 and 0 <= a and b <= p.N
    assert bench.parity_sample(model, model.n_layers, 6, 4) == smp  # seeded


def test_parity_ratio_is_the_tolerance():
    import numpy as np
    ref = np.array([[100.0, -2.0, 0.0]])
    T = np.array([[100.0, 1e6, 10.0]])
    got = ref + np.array([[1e-3, 0.5, 5e-6]])
    # 1e-3 / (1e-5*100) = 1, 0.5 / (1e-6*1e6) = 0.5, 5e-6 / (1e-6*10) = 0.5
    assert abs(bench.parity_ratio(got.astype(np.float32), ref, T) - 1.0) < 1e-3


def test_record_traffic_weights_the_step_launch_mix(tmp_path, monkeypatch):
    """--record-traffic: the five qgemm launches of a 1-layer step's ncu CSV (values with
    thousands separators, other kernels and ncu's own lines mixed in) become per-shape
    DRAM bytes and their mean over the full step's 129 launches, keyed to the current
    kernel source."""
    import csv
    import io
    import json
    import types
    hdr = ["ID", "Process ID", "Process Name", "Host Name", "Kernel Name", "Context", "Stream", "Block Size",
           "Grid Size", "Device", "CC", "Section Name", "Metric Name", "Metric Unit", "Metric Value"]
    shapes = [(1000, 0, 10000), (2000, 16, 20000), (3000, 32, 30000), (4000, 0, 40000), (50000, 64, 50000)]
    buf = io.StringIO()
    wr = csv.writer(buf, quoting=csv.QUOTE_ALL)
    wr.writerow(hdr)
    i = 0
    for rd, wt, ns in shapes:
        if i == 1:  # a quantizer launch between two GEMMs is ignored
            wr.writerow([str(i), "1", "python", "h", "void dllm::quantize_act_kernel(...)", "1", "7", "(256, 1, 1)",
                         "(16, 16, 1)", "0", "10.0", "", "dram__bytes_read.sum", "byte", "999"])
            i += 1
        for name, unit, val in (("dram__bytes_read.sum", "byte", rd), ("dram__bytes_write.sum", "byte", wt),
                                ("gpu__time_duration.sum", "nsecond", ns)):
            wr.writerow([str(i), "1", "python", "h", "void dllm::qgemm_kernel<12, false, false>(dllm::GemmArgs)",
                         "1", "7", "(512, 1, 1)", "(148, 1, 1)", "0", "10.0", "", name, unit, f"{val:,}"])
        i += 1
    path = tmp_path / "launches.csv"
    path.write_text("==PROF== Connected to process 1\n" + buf.getvalue())
    out_file = tmp_path / "traffic.json"
    monkeypatch.setattr(bench, "TRAFFIC_FILE", out_file)
    args = types.SimpleNamespace(record_traffic=str(path), model="llada-8b", canvas=128)
    bench.record_traffic(args)
    d = json.loads(out_file.read_text())
    assert d["kernel_source_sha"] == bench.kernel_source_hash()
    assert d["per_launch_shape"]["o"] == {"dram_read": 2000, "dram_write": 16, "us_cold": 20.0}
    expect = (32 * (1000 + 2016 + 3032 + 4000) + 50064) / 129
    assert d["per_launch_bytes"]["llada-8b_L128"] == round(expect)
    step = bench.step_gemms(synth.MODELS["llada-8b"](), 128, 32)
    assert len(step) == 129
    assert d["algorithmic_bytes_per_launch_llada-8b_L128"] == round(sum(g.bytes for g in step) / 129)
