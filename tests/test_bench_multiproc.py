"""The benchmark's multi-rank host logic on CPU: two gloo ranks.

Decode shards by sequence with no collective on the data path; the ranks only
agree on timings.  Checked here without a GPU: every rank gets its own seeded
sequences with the same layer shapes, the timings are reduced to the max over
ranks on every rank, the whole-job throughput counts all ranks' tokens over the
slowest rank's time, and the reference arm does its work on rank 0 only.
"""
import os
import socket

import pytest


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import json

    import torch
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    from checkpoint_input_replay_rssm_b200 import inputs as I

    wl = bench.rank_workload(rank, 8)
    tok = I.token(wl, 0, seqs=range(2))
    local = [10.0 + rank, 3.0 - rank, 7.5]
    got = bench.max_over_ranks(dist, local, torch.device("cpu"))
    value = bench.job_tokens_per_s(world, wl.batch, 16, got[0])
    json.dump({"seed": wl.seed, "shape": [wl.batch, wl.nheads, wl.headdim, wl.dstate],
               "x0": float(tok["x"][0, 0, 0]), "max": got, "value": value},
              open(os.path.join(out_dir, f"r{rank}.json"), "w"))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_shard_sequences_and_take_the_slowest_time(tmp_path):
    import json

    import torch.multiprocessing as mp

    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    r = [json.load(open(tmp_path / f"r{k}.json")) for k in range(world)]
    assert r[0]["shape"] == r[1]["shape"]
    assert r[0]["seed"] != r[1]["seed"] and r[0]["x0"] != r[1]["x0"]  # independent sequences
    for k in range(world):
        assert r[k]["max"] == [11.0, 3.0, 7.5]  # element-wise max over ranks, on every rank
        assert r[k]["value"] == pytest.approx(world * 8 * 16 / 11.0e-3)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    import argparse

    import bench

    bench.run_reference(argparse.Namespace(steps=2, warmup=3, gpus=2), rank=1)
    assert capsys.readouterr().out == ""


def test_single_process_reduction_is_identity():
    import bench

    assert bench.max_over_ranks(None, [1.5, 2], None) == [1.5, 2.0]


def test_reference_arm_prints_the_contract_line(capsys, oracle_built):
    """Rank 0 of the reference arm (the fp64 oracle on the host cores) prints one JSON
    line with the benchmark's keys, the same metric and unit as the main arm."""
    import argparse
    import json

    import bench

    bench.run_reference(argparse.Namespace(steps=2, warmup=3, gpus=1), rank=0)
    lines = [l for l in capsys.readouterr().out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "tokens/s"
    assert d["steps"] == 2 and d["warmup"] == 3 and d["value"] > 0 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == bench.WL.name
