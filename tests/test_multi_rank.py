"""Host-side logic of the data-parallel bench (one process per GPU, weak scaling) on two
gloo ranks on the CPU: each rank gets its own token stream of the same shape, the
slowest rank's time is what every rank reports, and the reference arm runs on rank 0
only. The GPU data path has no collective, so nothing else crosses ranks."""
import json
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime

    import bench
    from synth import configs, workloads
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ws, r, local = bench.dist_env()
        assert (ws, r, local) == (world, rank, rank)
        cfg = configs.PREFILL_D2048.with_(num_seqs=2, seq_len=512)
        tok, off = workloads.prefill_tokens(bench.rank_config(cfg, rank))
        # each rank times something different; all must report the slowest
        slowest = bench.max_over_ranks(10.0 + 5.0 * rank, world, torch.device("cpu"))
        dist.barrier()
        np.save(os.path.join(out_dir, f"tok{rank}.npy"), tok)
        np.save(os.path.join(out_dir, f"off{rank}.npy"), off)
        with open(os.path.join(out_dir, f"r{rank}.json"), "w") as f:
            json.dump({"slowest": slowest}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_split_batches_and_reduce_max(tmp_path):
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    t0, t1 = np.load(tmp_path / "tok0.npy"), np.load(tmp_path / "tok1.npy")
    o0, o1 = np.load(tmp_path / "off0.npy"), np.load(tmp_path / "off1.npy")
    assert t0.shape == t1.shape and np.array_equal(o0, o1)   # same shape of work per rank
    assert not np.array_equal(t0, t1)                        # but each rank its own tokens
    for r in range(world):
        assert json.load(open(tmp_path / f"r{r}.json"))["slowest"] == 15.0


def test_rank0_configured_workload_and_distinct_rank_seeds():
    sys.path.insert(0, ROOT)
    import bench
    from synth import configs
    cfg = configs.PREFILL_D2048
    assert bench.rank_config(cfg, 0) is cfg
    seeds = {bench.rank_config(cfg, r).seed for r in range(8)}
    assert len(seeds) == 8
    assert all(bench.rank_config(cfg, r).V_nk == cfg.V_nk for r in range(8))  # tables shared


def test_reference_arm_runs_on_rank0_only(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import argparse

    import bench
    from synth import configs
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = argparse.Namespace(gpus=2, steps=1, warmup=0, ref_step_seconds=0.1)
    assert bench.run_reference(args, configs.PREFILL_D2048) is None
    assert capsys.readouterr().out == ""  # no work, no line: rank 0 prints the only one
