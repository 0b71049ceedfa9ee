"""The benchmark's host-side arithmetic and its JSON line, without a GPU:
the clock regime that picks the peak, the roofline objects recomputed from
their own fields, the Hessian traffic tied to the profiled kernel source, and
the reference arm (the float64 checker on the host cores) printing one line
with the contract's keys."""
import hashlib
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from post_weight_quantization_accumulate_b200 import synth  # noqa: E402

PEAKS = {"hbm_gbs": 6450.3, "bf16_tflops": 1672.7, "bf16_tflops_sustained": 1414.8}


def test_regime_follows_the_clock_record():
    assert bench.regime({"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": []}) == "burst"
    assert bench.regime({"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"]}) == "sustained"
    assert bench.regime({"sm_mhz": 1500, "sm_max_mhz": 1965, "reasons": []}) == "sustained"
    assert bench.regime({}) == "sustained"


def test_hessian_roofline_recomputes_from_its_fields():
    spec = synth.WORKLOADS["q_proj_4096"]
    for clocks, reg in (({"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": []}, "burst"),
                        ({"sm_mhz": 1965, "sm_max_mhz": 1965, "reasons": ["sw_power_cap"]}, "sustained")):
        r = bench.hessian_roofline(spec, 3.2, clocks, PEAKS, "measured")
        flops = spec.n_tokens * spec.d_in * (spec.d_in + 1)
        assert r["flops_per_launch"] == flops
        assert r["achieved"] == pytest.approx(flops / 3.2e-3 / 1e12)
        peak = PEAKS["bf16_tflops"] if reg == "burst" else PEAKS["bf16_tflops_sustained"]
        assert r["peak"] == peak and r["frac"] == pytest.approx(r["achieved"] / peak)
        assert r["frac_burst"] == pytest.approx(r["achieved"] / PEAKS["bf16_tflops"])
        assert r["frac_sustained"] == pytest.approx(r["achieved"] / PEAKS["bf16_tflops_sustained"])
        assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
        if r["traffic"] is not None:
            assert r["traffic_over_alg_bytes"] == pytest.approx(r["traffic"] / r["alg_bytes"])


def test_profiled_traffic_is_tied_to_the_kernel_source(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("kernel v1\n")
    h = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    prof = tmp_path / "p.md"
    prof.write_text(f"traffic_bytes_per_launch: 4.5e9\nkernel_source_sha256_16: {h}\n")
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(prof))
    assert bench.profiled_traffic(str(src)) == 4.5e9
    src.write_text("kernel v2\n")            # the kernel changed since the capture
    assert bench.profiled_traffic(str(src)) is None


def test_lazy_batch_and_layer_lines():
    spec = synth.WORKLOADS["q_proj_4096"]
    stage = {"lazy_batch_ms": 0.5}
    line = bench.lazy_batch_line(spec, stage)
    fl = bench.lazy_flops(spec)
    assert line["flops_fp32"] == fl
    assert line["tf32_rate_tflops"] == pytest.approx(3 * fl / 0.5e-3 / 1e12)
    if line["peak"]:
        assert line["frac"] == pytest.approx(line["tf32_rate_tflops"] / line["peak"])
    # d_out (d_in^2 - sum of squared block widths): 32 blocks of 128 columns
    assert fl == spec.d_out * (spec.d_in ** 2 - 32 * 128 ** 2)
    lr = bench.layer_roofline(spec, 6.0, "burst", PEAKS)
    if lr is not None:
        assert lr["ideal_ms"] == pytest.approx(sum(lr["terms_ms"].values()))
        assert lr["frac"] == pytest.approx(lr["ideal_ms"] / 6.0)


@pytest.mark.timeout(600)
def test_reference_arm_prints_one_contract_line():
    env = dict(os.environ)
    env.setdefault("OMP_NUM_THREADS", str(min(8, os.cpu_count() or 1)))
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "0"], capture_output=True, text=True,
                         timeout=600, env=env, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "impl",
              "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0 and d["ms_per_step"] > 0
    assert d["config"]["workload"] == "q_proj_4096"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
