"""Host-side checks of bench.py's JSON line: the reference (oracle) arm prints
the same `config` object as the CUDA arm, so the two lines describe one
workload."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from sdpa_workloads import WORKLOADS  # noqa: E402


def test_arm_config_fields():
    w = WORKLOADS["lm_causal"]
    c = bench.arm_config(w, 1)
    assert c["workload"] == w.name and c["global_batch"] == 8
    assert c["parallelism"].startswith("dp1")
    assert c["l2"].startswith("inputs 403 MB")          # 3 x 8*16*4096*128 bf16
    c2 = bench.arm_config(w, 4)
    assert c2["global_batch"] == 32 and c2["parallelism"].startswith("dp4")
    f = bench.arm_config(WORKLOADS["fp8"], 1)             # e4m3 inputs: one byte each
    assert f["l2"].startswith("inputs 403 MB")           # 3 x 2*32*16384*128 bytes
    assert "fit in L2" in bench.arm_config(WORKLOADS["vit"], 1)["l2"]


def test_reference_line_uses_arm_config(monkeypatch, capsys):
    w = WORKLOADS["lm_causal"]
    monkeypatch.setattr(bench, "cpu_inputs", lambda w: (None, None, None, None))
    monkeypatch.setattr(bench, "oracle_rows_tflops", lambda *a: (0.5, 1e9))
    monkeypatch.delenv("RANK", raising=False)

    class A:
        steps, warmup, gpus, ref_budget_s = 2, 3, 2, 1.0
    bench.run_reference(A, w)
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["config"] == bench.arm_config(w, 2)
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
