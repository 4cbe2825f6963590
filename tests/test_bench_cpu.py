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


def test_per_op_ideal_bytes_of_the_config_table():
    """op_ideal_bytes, which the per-config table divides by each op's time:
    the forward and backward as above, MSDCN with the raw scales, the fused
    forward with input and x read once, output written once and the
    sub-network's weights (the records stay on chip)."""
    sys.path.insert(0, ROOT)
    import bench
    from deformable_convolution_dcn4_b200.workloads import WORKLOADS
    wl = WORKLOADS["internimage_bf16"]
    hwc = 64 * 56 * 56 * 128
    hwg = 64 * 56 * 56 * 8
    J = 8 * 9 * 3
    assert bench.op_ideal_bytes(wl, 56, 56, "fwd") == (2 * hwc + 27 * hwg) * 2
    assert bench.op_ideal_bytes(wl, 56, 56, "bwd") == (3 * hwc + 54 * hwg) * 2
    assert bench.op_ideal_bytes(wl, 56, 56, "bwd_acc16") == (3 * hwc + 54 * hwg) * 2
    assert bench.op_ideal_bytes(wl, 56, 56, "msfwd") == (2 * hwc + 28 * hwg) * 2
    assert bench.op_ideal_bytes(wl, 56, 56, "msbwd") == (3 * hwc + 56 * hwg) * 2
    assert bench.op_ideal_bytes(wl, 56, 56, "fused") == (3 * hwc + 10 * 128 + J * 128 + J) * 2


def test_config_table_names_known_workloads_and_ops():
    """Every (config, workload, op) of the per-config table exists: the
    workloads are defined, each op has an ideal-byte model, and the fused
    forward appears where the sub-network's output grid is the input grid."""
    sys.path.insert(0, ROOT)
    import bench
    from deformable_convolution_dcn4_b200.workloads import WORKLOADS
    labels = set()
    for label, wname, ops in bench.CONFIG_TABLE:
        wl = WORKLOADS[wname]
        labels.add(label)
        for op in ops:
            assert bench.op_ideal_bytes(wl, wl.H, wl.W, op) > 0
            if op == "fused":
                assert wl.kind == "dcn4" and wl.stride == (1, 1) and wl.pad == (1, 1)
    assert {"c1", "c2", "c3a", "c3b", "c4", "c5"} <= labels
    assert any("fused" in ops for _, _, ops in bench.CONFIG_TABLE)
