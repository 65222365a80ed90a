"""The multi-rank logic of bench.py on CPU (not gpu): world size 2 over gloo.

Each rank contributes a different local time; max_over_ranks must return the
slowest on every rank, the barrier must release both, and the whole-job value
must count every rank's bytes over the slowest time (weak scaling)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        dev = torch.device("cpu")
        r, lr, w = bench.dist_env()
        local_ms = 100.0 + 50.0 * rank
        bench.barrier(dev)
        m = bench.max_over_ranks(local_ms, dev)
        v = bench.aggregate_value(10 ** 9, 4, w, m * 1e-3)
        q.put((r, lr, w, m, v))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_weak_scaling_value():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, (r, lr, w, m, v) in enumerate(res):
        assert (r, lr, w) == (rank, rank, 2)
        assert m == 150.0                      # the slowest rank's time on every rank
        assert v == pytest.approx(2 * 4 * 1e9 / 0.150 / 1e9)


def test_single_process_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, torch.device("cpu")) == 3.5
    assert bench.aggregate_value(2 * 10 ** 9, 10, 1, 2.0) == pytest.approx(10.0)


def test_algorithmic_bytes_match_the_closed_forms():
    """Byte model of the step against hand-counted sizes of the workload."""
    import bench
    n_used = 69760
    b = bench.algorithmic_bytes(n_used)
    assert b["swiglu_fwd"] == 805_568_512 and b["swiglu_bwd"] == 1_342_701_568
    assert b["router_weight_fwd"] == 469_827_584 and b["router_weight_bwd"] == 704_774_144
    assert b["unpermute"] == 606_076_928 and b["residual_add"] == 1_879_048_192
    assert b["act_sqrelu"] == 65536 * 1536 * 2 + n_used * 1536 * 2 + 4 * n_used + 4 * 65536
    assert b["act_swiglu"] == 65536 * 3072 * 2 + n_used * 1536 * 2 + 4 * n_used + 4 * 65536
    half = bench.algorithmic_bytes(n_used // 2, scale=0.5)
    assert half["residual_add"] == b["residual_add"] // 2


def test_reference_arm_runs_on_the_host(capsys):
    """The reference arm (the CPU oracle on a bounded sample) prints one JSON line."""
    import json
    import bench
    bench.main(["--impl", "reference", "--steps", "1", "--warmup", "0", "--cpu-sample", "0.01"])
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == "GB/s"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
