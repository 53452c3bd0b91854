"""Host logic of the N > 1 bench path, run as world_size-2 gloo ranks on CPU.

With several GPUs every rank scans its own independent batch (weak scaling):
no collective touches the data path, only the barrier around the timed region
and the max over ranks of the step time.  These tests run that plumbing
(process group, barrier, max-reduction, per-rank seeding, whole-job value)
with the gloo backend, and check that the reference arm does no work on
ranks other than 0.
"""
import json
import os
import socket
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench as B
    from selective_state_space_28_b200 import inputs as I
    d = B.Dist()
    d.init("gloo")
    assert d.world == world and d.rank == rank and d.pg is not None
    d.barrier()
    # Each rank reports a different step time; all ranks must see the slowest.
    ms = 1.5 + rank * 0.75
    mx = d.max(ms, "cpu")
    # Each rank draws its own batch; a checksum of it goes through a gather
    # only here, in the test, to show that the ranks' batches differ.
    w = I.WORKLOADS["m1_toy_b1_l64_c32_n4_f32"]
    x = I.workload_inputs(w, device="cpu", seed=B.rank_seed(w.seed, rank))["x"]
    chk = torch.tensor([float(x.double().sum()), float(x.double().abs().sum())],
                       dtype=torch.float64)
    got = [torch.zeros(2, dtype=torch.float64) for _ in range(world)]
    d.pg.all_gather(got, chk)
    d.barrier()
    d.close()
    with open(os.path.join(out_dir, "rank%d.txt" % rank), "w") as f:
        json.dump({"max": mx, "sums": [g.tolist() for g in got]}, f)


def test_two_gloo_ranks_agree_on_max_and_draw_distinct_batches(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    res = []
    for r in range(world):
        d = json.loads((tmp_path / ("rank%d.txt" % r)).read_text())
        res.append((d["max"], d["sums"]))
    for mx, sums in res:
        assert mx == pytest.approx(1.5 + 0.75 * (world - 1))
        assert len(sums) == world
        assert sums[0] != sums[1]
    assert res[0][1] == res[1][1]


def test_rank_seeds_never_collide_with_buffer_set_seeds():
    # bench rotates up to n buffer sets per rank with seeds rank_seed + 1000*set.
    seeds = set()
    for rank in range(8):
        for sset in range(64):
            s = bench.rank_seed(12345, rank) + 1000 * sset
            assert s not in seeds
            seeds.add(s)


def test_job_value_is_all_ranks_units_over_slowest_time():
    # 4 ranks, 1e9 bytes each, slowest rank 2 ms -> 2e12 bytes/s.
    assert bench.job_value(1e9, 4, 2.0) == pytest.approx(2e12)
    assert bench.job_value(3.0, 1, 1000.0) == pytest.approx(3.0)


def test_reference_arm_does_nothing_on_other_ranks(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = bench.parse(["--impl", "reference", "--gpus", "2", "--steps", "3",
                        "--warmup", "3"])
    assert bench.run_reference(args) is None
    assert capsys.readouterr().out == ""
