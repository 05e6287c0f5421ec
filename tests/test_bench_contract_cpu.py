"""bench.py's reference arm (the oracle timed on host cores) runs without a
GPU: its JSON line carries the keys of the benchmark contract."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_contract_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--config", "small", "--steps", "1",
                        "--warmup", "0"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip().startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert "workload" in d["config"]


def test_roofline_traffic_is_keyed_to_kernel_and_workload():
    """roofline.traffic comes from the committed ncu summary only for the kernel
    source, model shape and segment length it was captured on."""
    import hashlib
    sys.path.insert(0, ROOT)
    import bench
    src = os.path.join(ROOT, "recurrent_memory_transformer_diag_b200", "csrc", "tc_gemm.cu")
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    rows = [ln.split() for ln in open(os.path.join(ROOT, "profiles", "traffic.txt")) if not ln.startswith("#")]
    rows = [r for r in rows if len(r) >= 5]
    assert rows, "traffic.txt holds no entry"
    for kernel, per_node, sha, config, seg_len in (r[:5] for r in rows):
        got = bench.read_traffic(kernel, config, int(seg_len))
        assert got == (float(per_node) if sha == h else None)
        assert bench.read_traffic(kernel, config, int(seg_len) + 1) is None
        assert bench.read_traffic(kernel, config + "x", int(seg_len)) is None


def test_weight_bytes_of_the_1b_shape():
    sys.path.insert(0, ROOT)
    import bench
    from recurrent_memory_transformer_diag_b200.inputs import CONFIGS
    # 16 layers x (3072 x 2048 QKV + 2048 x 2048 O + 3 x 8192 x 2048 MLP + (64 + 64 + 2048) x 2048 memory) x 2 bytes
    assert bench.weight_bytes(CONFIGS["1b"]) == 2 * 16 * (3072 * 2048 + 2048 * 2048 + 3 * 8192 * 2048
                                                        + (64 + 64 + 2048) * 2048)
