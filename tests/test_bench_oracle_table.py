"""bench.py --oracle-table (the float64 oracle timed per workload, no GPU), on tiny stand-in
workloads so that it runs in a moment: one JSON line with derive + pack seconds per matrix,
the layer at every decode batch, and GEMM workloads scaled from a token sample."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from bit_gemv_rabit_b200 import inputs  # noqa: E402


def test_oracle_table_shape(monkeypatch, capsys):
    tiny = {
        "decode": dict(set=[("q", 64, 96), ("down", 32, 200)], batches=[1, 4], sigma=0.02,
                       w_outliers=0.0, x_outliers=0.0, cfg=7),
        "prefill": dict(set=[("gate", 48, 64)], batches=[512], sigma=0.02, w_outliers=0.0,
                        x_outliers=0.01, cfg=8),
    }
    monkeypatch.setattr(inputs, "WORKLOADS", tiny)
    assert bench.main(["--oracle-table", "--gemm-token-sample", "4"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["kind"] == "oracle" and line["cores"] >= 1
    dec = line["workloads"]["decode"]
    assert [r["matrix"] for r in dec] == ["q 64x96", "down 32x200"]
    assert all(r["derive_pack_s"] >= 0 and r["layer_b1_us"] > 0 and r["layer_b4_us"] > 0 for r in dec)
    pre = line["workloads"]["prefill"][0]
    assert pre["token_sample"] == 4 and pre["layer_m512_s"] > 0
