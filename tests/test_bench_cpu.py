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
