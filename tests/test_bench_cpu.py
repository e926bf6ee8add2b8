"""The benchmark's host-side contract, without a GPU: the reference arm's JSON line
(the oracle timed on the host cores) and the CPU-baseline record."""
import json

import bench
import workloads as wl


def test_reference_arm_line(capsys):
    assert bench.main(["--impl", "reference", "--steps", "2", "--warmup", "1", "--workload", "tiny"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["steps"] == 2 and line["warmup"] == 3          # warm-up is raised to at least 3
    assert line["value"] > 0 and line["higher_is_better"] is True
    assert line["unit"] == bench.UNIT and line["metric"] == bench.METRIC
    assert line["config"]["workload"] == "tiny"
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_cpu_baseline_record():
    rec = bench.cpu_baseline(wl.get("tiny"))
    assert rec["kind"] == "oracle" and rec["unit"] == bench.UNIT and rec["value"] > 0
    assert "x one Muon step" in rec["sample"] and rec["cores"] >= 1


def test_elementwise_bytes_per_element():
    w = wl.get("square4096")
    mom, app = bench.elementwise_bytes(w)
    assert mom == 14 * w.elements          # G 2, B 4 + 4, X hi 2 + lo 2
