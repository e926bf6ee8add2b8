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
    """The method's counts: momentum G 2 (bf16) or 4 (fp32), B 4 + 4, X0 2 = 12 (14)
    B/elem; apply W 4 + 4, O 2 = 10 B/elem.  The bf16-pair iterate moves 2 B/elem more
    in each (X0's lo written, O's lo read)."""
    w = wl.get("square4096")
    mom, moved, app, app_moved = bench.elementwise_bytes(w)
    assert mom == 12 * w.elements and moved == 14 * w.elements
    assert app == 10 * w.elements and app_moved == 12 * w.elements
    t = wl.get("tiny")
    assert bench.elementwise_bytes(t)[0] == 14 * t.elements


def test_ns_figures_follow_their_stated_counts():
    """Every fraction in the bench line can be recomputed from the line's own fields."""
    w = wl.get("square4096")
    peaks = {"hbm_gbs": 6000.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    steps = 4
    phases = {"momentum_norm": (0.2, 4), "norm_finalize": (0.0, 0), "gram": (1.2, 20), "poly": (1.2, 20),
              "update": (2.0, 20), "apply": (0.16, 4)}
    f = bench.ns_figures(w, 1.25, 1.10, phases, steps, peaks)
    m = 4096.0
    sym = 5 * (3 * m ** 3 + m ** 3)
    assert f["ns5_symmetric"]["flops_per_step"] == sym
    assert abs(f["ns5_symmetric"]["ns_ms_per_step"] - (1.25 - 0.05)) < 1e-9
    assert abs(f["ns5_symmetric"]["tflops"] - round(sym / 1.2e-3 / 1e12, 2)) < 1e-6
    assert abs(f["ns5_symmetric"]["frac_sustained"] - round(sym / 1.2e-3 / 1e12 / 1400.0, 4)) < 1e-9
    assert abs(f["ns5_symmetric"]["tflops_burst"] - round(sym / 1.05e-3 / 1e12, 2)) < 1e-6
    assert abs(f["momentum_gbs"] - round(12 * w.elements / 0.05e-3 / 1e9, 1)) < 1e-6
    assert f["momentum_bytes_per_elem"] == 12 and f["momentum_moved_bytes_per_elem"] == 14
    assert f["apply"] == "apply_kernel" and abs(f["apply_ms"] - 0.04) < 1e-12
    assert abs(f["apply_gbs"] - round(10 * w.elements / 0.04e-3 / 1e9, 1)) < 1e-6
    assert abs(f["apply_frac_of_hbm"] - round(10 * w.elements / 0.04e-3 / 1e9 / 6000.0, 4)) < 1e-9
    assert abs(f["apply_gbs_moved"] - round(12 * w.elements / 0.04e-3 / 1e9, 1)) < 1e-6
    fused = dict(phases, apply=(0.0, 0))
    g = bench.ns_figures(w, 1.25, 1.10, fused, steps, peaks)
    assert g["apply_gbs"] is None and g["apply"].startswith("fused")
    nominal = 5 * (4 * m ** 3 + 2 * m ** 3)
    assert abs(f["ns5_tflops_nominal"] - round(nominal / 1.25e-3 / 1e12, 2)) < 1e-6
    assert abs(f["ns5_tflops_phase_sum"] - round(nominal / 1.1e-3 / 1e12, 2)) < 1e-6


def _ranks_worker(rank, world, port, out_dir):
    import os
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        v = bench.max_over_ranks(1.5 + rank, world)
        with open(os.path.join(out_dir, f"r{rank}.txt"), "w") as f:
            f.write(repr(v))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo(tmp_path):
    """The bench's timing reduction: every rank gets the slowest rank's time."""
    import socket
    import torch.multiprocessing as tmp
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    tmp.spawn(_ranks_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True)
    for r in range(2):
        assert float((tmp_path / f"r{r}.txt").read_text()) == 2.5
    assert bench.max_over_ranks(3.25, 1) == 3.25
