"""Host logic of bench.py's N > 1 path, on CPU: two gloo ranks set up through bench.py's own
dist_setup, meet at its barrier and agree on the max over ranks of their times (the
number rank 0 reports); the reference arm prints from rank 0 only."""
import json
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "WORLD_SIZE": str(world),
                       "RANK": str(rank), "LOCAL_RANK": str(rank)})
    sys.path.insert(0, ROOT)
    import bench

    class Args:
        impl = "reference"
    w, r, _ = bench.dist_setup(Args())
    try:
        bench.barrier(w)
        t = bench.max_over_ranks(10.0 + 5.0 * r, w)
        bench.barrier(w)
    finally:
        import torch.distributed as dist
        dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump({"world": w, "rank": r, "max": t}, f)


def test_two_gloo_ranks_agree_on_the_max_time(tmp_path):
    import torch.multiprocessing as mp
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    assert [x["rank"] for x in res] == [0, 1]
    assert all(x["world"] == world for x in res)
    assert all(x["max"] == 15.0 for x in res)      # max over ranks, the same on every rank


def test_reference_arm_prints_from_rank_zero_only(capsys, monkeypatch):
    sys.path.insert(0, ROOT)
    import bench

    class Args:
        gpus, steps, warmup = 2, 1, 3
    calls = []
    monkeypatch.setattr(bench, "threaded_sample", lambda *a, **k: calls.append("sample") or [[None]])
    monkeypatch.setattr(bench, "cpu_oracle_threads", lambda parts, target_s=8.0: (1.0, 0.1))
    monkeypatch.setattr(bench, "threaded_desc", lambda parts, sec: "stub sample")
    bench.reference_arm(Args(), 2, 1)
    assert capsys.readouterr().out == "" and calls == []
    bench.reference_arm(Args(), 2, 0)
    line = json.loads(capsys.readouterr().out)
    assert line["impl"] == "reference" and line["value"] == 1.0 and line["n_gpus"] == 2
    for key in ("metric", "unit", "steps", "warmup", "higher_is_better", "scaling", "dtype",
                "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == 1.0
    assert line["e2e"] == {"value": 1.0, "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
