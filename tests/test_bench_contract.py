"""The parts of bench.py's output contract that run without a GPU.

The reference arm (the fp64 oracle timed on the host cores) prints the same
JSON line as the GPU arm, with "impl": "reference", a cpu_baseline describing
its own run and an e2e object with no host-device copies. The roofline's
`traffic` comes from the committed ncu record only while the kernel source is
the one the record was taken from.
"""

import io
import json
import os
import sys
from contextlib import redirect_stdout

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402

KEYS = {"metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
        "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"}


def test_reference_arm_line():
    args = type("A", (), {"steps": 1, "warmup": 0})()
    buf = io.StringIO()
    with redirect_stdout(buf):
        rc = bench.run_reference(args, 0, 1)
    assert rc == 0
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert KEYS <= set(line)
    assert line["impl"] == "reference" and line["n_gpus"] == 1 and line["steps"] == 1
    assert line["higher_is_better"] is True and line["scaling"] == "weak" and line["vs_baseline"] is None
    assert line["value"] > 0 and line["unit"] == "tokens/s"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] and cb["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0
    # the same workload description as the GPU arm
    gpu_cfg = bench.workload_config(4096, 1, 2048, 64, 8, 1024)
    assert line["config"]["workload"] == gpu_cfg["workload"]


def test_traffic_record_follows_the_kernel_source(tmp_path, monkeypatch):
    rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))["gate_up_T4096"]
    got = bench.committed_traffic("grouped_gemm.cu", "gate_up_T4096")
    assert got is None or got == rec["bytes_per_launch"]
    # a source that differs from the recorded one gives no traffic figure
    fake = tmp_path / "sparse_moe_transformer_route_b200" / "csrc"
    fake.mkdir(parents=True)
    (fake / "grouped_gemm.cu").write_text("// changed\n")
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"gate_up_T4096": rec}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.committed_traffic("grouped_gemm.cu", "gate_up_T4096") is None
    assert bench.committed_traffic("grouped_gemm.cu", "no_such_key") is None
