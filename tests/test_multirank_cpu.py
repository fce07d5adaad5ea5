"""bench.py's multi-rank plumbing on the CPU with gloo, world size 2: the
step time is the max over ranks and the value counts every rank's tokens
(decode batches are independent replicas; no data-path collective)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    r, w, local = bench.dist_env()
    ms = 1.0 + 2.0 * rank  # rank 1 is the slow one
    t = bench.max_over_ranks(ms, w, device=torch.device("cpu"))
    tokens = 8
    value = tokens * w / (t / 1e3)
    q.put((r, w, local, t, value))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in res] == [0, 1]
    assert all(r[1] == 2 and r[0] == r[2] for r in res)
    assert all(r[3] == pytest.approx(3.0) for r in res)  # the max over ranks
    assert all(r[4] == pytest.approx(8 * 2 / 3e-3) for r in res)


def test_single_rank_env_defaults(monkeypatch):
    import bench
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.dist_env() == (0, 1, 0)
    assert bench.max_over_ranks(2.5, 1) == 2.5


def test_reference_arm_line_and_other_ranks(monkeypatch, capsys):
    # the oracle arm: rank 0 prints one line with the contract's keys; any
    # other rank exits 0 without work
    import json
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3", "--workloads", "2"]) == 0
    assert capsys.readouterr().out.strip() == ""
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    assert bench.main(["--impl", "reference", "--steps", "1", "--warmup", "3", "--workloads", "2"]) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["config"]["workload"] == "csa_decode_b1_ctx8k"
