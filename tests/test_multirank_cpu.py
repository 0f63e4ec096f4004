"""N > 1 host logic of the benchmark on CPU with gloo: every rank runs its own
replica on inputs drawn from its own seed (checked by gathering each rank's
first generated values); timings are reduced max-over-ranks and work
sum-over-ranks; the reference (oracle) arm runs on rank 0 only and the other
ranks exit at once."""
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world)})
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    dev = torch.device("cpu")
    mx = bench.reduce_over_ranks(1.5 + rank, "max", world, dev)
    sm = bench.reduce_over_ranks(10.0 * (rank + 1), "sum", world, dev)
    # each replica's inputs: the first values of its calibration q, made by the
    # benchmark's own generator from the rank's seed
    w = bench.synth.WORKLOADS[bench.WORKLOAD]
    mine = bench.randn_bf16((1, 64), bench.replica_seed(w, rank) + 1, dev).float()
    gathered = [torch.empty_like(mine) for _ in range(world)]
    dist.all_gather(gathered, mine)
    distinct = all(not torch.equal(gathered[i], gathered[j]) for i in range(world) for j in range(i + 1, world))
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, mx, sm, distinct))


@pytest.mark.parametrize("world", [2])
def test_timing_reductions_over_gloo_ranks(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, sm, distinct in res:
        assert mx == 1.5 + (world - 1)
        assert sm == 10.0 * world * (world + 1) / 2
        assert distinct            # replicas are independent: no two ranks draw the same inputs


def test_reference_arm_nonzero_rank_exits_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == ""
