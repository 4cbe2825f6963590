"""The benchmark's reference arm (the CPU oracle as the reference) and its
JSON contract, on CPU: one line, the base keys, the oracle description."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "0", "--workload", "tiny_f32"],
                         capture_output=True, text=True, timeout=600, check=True).stdout
    lines = [ln for ln in out.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e", "impl"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["config"]["workload"].startswith("tiny_f32")


def test_ideal_bytes_follow_the_pages_model():
    sys.path.insert(0, ROOT)
    import bench
    from deformable_convolution_dcn4_b200.workloads import WORKLOADS
    wl = WORKLOADS["internimage_bf16"]
    ib = bench.ideal_bytes(wl, 56, 56)
    hwc = 64 * 56 * 56 * 128
    hwg = 64 * 56 * 56 * 8
    # (2HWC + 27HWG) * b forward; backward reads in, go, ow and writes gin, gow
    assert ib["dcn4_forward"] == (2 * hwc + 27 * hwg) * 2
    assert ib["dcn4_backward"] == (3 * hwc + 54 * hwg) * 2
    assert ib["msdcn_forward"] == (2 * hwc + 27 * hwg + hwg) * 2
