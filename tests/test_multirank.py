"""The N>1 host logic of bench.py on CPU: two gloo ranks.

Each rank owns a full, distinct batch (weak scaling, no collective on the
data path); the only collectives are the barrier and the max over ranks of
the device time.
"""
import os
import socket

import numpy as np
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import torch
    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        t = bench.max_over_ranks(1.0 + rank, world)
        cfg, d, flops = bench.prefill_inputs(rank)
        dcfg, dd, dbytes = bench.decode_inputs(rank, batch=4)
        digest = torch.tensor([float(d["q"][0, 0, 0, :8].astype(np.float64).sum()),
                               float(dd["kv_lens"].sum())], dtype=torch.float64)
        gathered = [torch.zeros(2, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(gathered, digest)
        out[rank] = (t, flops, dbytes > 0, [g.tolist() for g in gathered])
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_max_time_and_own_distinct_batches():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 2.0          # max over ranks
    assert res[0][1] == res[1][1] > 0             # same per-rank work (weak scaling)
    digests = res[0][3]
    assert digests[0] != digests[1]               # each rank generated its own batch


def _bench(*argv, env=None):
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    e = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    e.update(env or {})
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), *argv], capture_output=True, text=True,
                       env=e, timeout=300)
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    return r.returncode, (json.loads(lines[-1]) if lines else None), r.stdout + r.stderr


def test_bench_starts_its_own_ranks():
    """`bench.py --gpus 2` outside torchrun launches two ranks itself (gloo on a
    CPU-only host); rank 0 alone prints one line, which counts both ranks."""
    rc, line, log = _bench("--gpus", "2", "--only", "launcher", "--steps", "3", "--warmup", "3")
    assert rc == 0, log
    assert line is not None and line["n_gpus"] == 2, log
    assert log.count('"n_gpus"') == 1, log


def test_bench_refuses_a_rank_count_that_does_not_match():
    rc, line, log = _bench("--gpus", "2", "--only", "launcher", env={"WORLD_SIZE": "1", "RANK": "0"})
    assert rc != 0 and line is None, log
