"""Host logic of bench.py on CPU: the reference arm's JSON line and the DRAM-traffic lookup.

The reference arm times the fp64 oracle on host cores, so it runs without a GPU; its line must
carry the same metric, workload and contract keys as the GPU arm.  The traffic lookup reads the
committed ncu summary and must answer only for the sources it was measured on.
"""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_reference_arm_prints_the_contract_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "3"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    d = json.loads(out.stdout.strip().splitlines()[-1])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "tokens/s"
    assert d["value"] > 0 and d["steps"] == 1 and d["warmup"] >= 3 and d["n_gpus"] == 1
    assert d["higher_is_better"] is True and d["vs_baseline"] is None
    assert d["config"]["workload"] == "train_fwdbwd_bf16_B8_H16_T2048_d128"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    e2e = d["e2e"]
    assert e2e["value"] == d["value"] and e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_traffic_record_matches_kernel_and_source_hash(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "dram_traffic.txt").write_text(
        "# | kernel | csrc_hash | parts | bytes_per_launch | read | write | algorithmic |\n"
        "| hgrn2_bwd_saved | aaaaaaaaaaaa | rev | 500 | 300 | 200 | 450 |\n"
        "| hgrn2_bwd_saved | bbbbbbbbbbbb | rev | 600 | 400 | 200 | 450 |\n"
        "| hgrn2_fwd_train | bbbbbbbbbbbb | fwd | not-a-number | 1 | 1 | 1 |\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "csrc_hash", lambda: "bbbbbbbbbbbb")
    assert bench.traffic_record("hgrn2_bwd_saved") == 600.0       # the row of the current sources
    assert bench.traffic_record("hgrn2_fwd_train") is None        # malformed figure
    assert bench.traffic_record("hgrn2_step") is None             # no row
    monkeypatch.setattr(bench, "csrc_hash", lambda: "cccccccccccc")
    assert bench.traffic_record("hgrn2_bwd_saved") is None        # sources changed since the capture


def test_committed_traffic_rows_name_kernels_the_bench_reports():
    # every row of the committed summary is well formed: a kernel the bench reports, a 12-digit
    # source hash and integer byte counts whose sum is the per-launch figure
    rows = []
    for line in open(os.path.join(ROOT, "profiles", "dram_traffic.txt")):
        if line.startswith("|"):
            rows.append([c.strip() for c in line.strip().strip("|").split("|")])
    assert rows
    for kernel, h, _, per_launch, rd, wr, alg in rows:
        assert kernel in ("hgrn2_fwd_train", "hgrn2_bwd_saved")
        assert len(h) == 12 and all(ch in "0123456789abcdef" for ch in h)
        assert int(per_launch) == int(rd) + int(wr) and int(alg) > 0
