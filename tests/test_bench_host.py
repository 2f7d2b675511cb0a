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
