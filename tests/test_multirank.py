"""Multi-rank host logic on CPU (gloo, world size 2).

The decode step shards across GPUs with no exchange: every (request, head)
update is independent (rcap.io post: a fixed-size state per request per
head).  Ranks that each step their own requests reproduce a single-process
step exactly, and bench.py's ranks meet only at the timing barrier and the
max-over-ranks reduction, exercised here with gloo.
"""

import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import oracle
import workload as W


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    import torch.distributed as dist
    d = bench.Dist(backend="gloo")
    cfg = W.CONFIGS["gdn"]
    p = W.make_plan(cfg)
    mine = list(range(rank, 4, world))               # requests of this rank
    plan = oracle.Plan(cfg.d, cfg.d, cfg.heads, cfg.gate_kind, cfg.unit_kind, 0, p.bits, p.w)
    pool = plan.new_pool(len(mine))
    slots = np.arange(len(mine), dtype=np.int32)
    plan.pack(pool, slots, W.initial_state(cfg, mine, heads=range(cfg.heads)))
    si = W.step_inputs(cfg, 0, p, mine)
    y, st = plan.decode_step(pool, slots, si.q, si.k, si.v, si.beta, si.gate)
    out = [None] * world
    dist.all_gather_object(out, {"reqs": mine, "y": y, "pool": pool, "st": st})
    d.barrier()
    m = d.max(float(rank + 1) * 1.5)
    if rank == 0:
        q.put((out, m))
    d.close()


@pytest.mark.timeout(300)
def test_two_ranks_shard_requests_without_exchange():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    out, m = q.get(timeout=240)
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    assert m == 3.0                                  # max over ranks of (rank+1)*1.5
    cfg = W.CONFIGS["gdn"]
    p = W.make_plan(cfg)
    plan = oracle.Plan(cfg.d, cfg.d, cfg.heads, cfg.gate_kind, cfg.unit_kind, 0, p.bits, p.w)
    pool = plan.new_pool(4)
    slots = np.arange(4, dtype=np.int32)
    plan.pack(pool, slots, W.initial_state(cfg, range(4)))
    si = W.step_inputs(cfg, 0, p, range(4))
    y, st = plan.decode_step(pool, slots, si.q, si.k, si.v, si.beta, si.gate)
    sb = plan.slot_bytes
    for part in out:
        assert part["st"] == 0
        for a, r in enumerate(part["reqs"]):
            assert np.array_equal(part["y"][a], y[r])
            assert np.array_equal(part["pool"][a * sb:(a + 1) * sb], pool[r * sb:(r + 1) * sb])


@pytest.mark.timeout(600)
def test_reference_arm_under_torchrun_prints_once():
    """bench.py --impl reference launched as the two-rank job: rank 0 alone
    times the oracle and prints one line; every rank exits 0."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
                        "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
                        "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3"],
                       cwd=root, capture_output=True, text=True, timeout=500)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"


def _rank_that_leaves(rank, world, port, q):
    """Rank 1 joins and leaves between steps (no collective in flight); rank 0
    then reaches the timing barrier and must get an error, not hang."""
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    import sys
    import time
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    d = bench.Dist(backend="gloo", timeout_s=20.0)
    d.barrier()                                      # both ranks are up
    if rank == 1:
        os._exit(0)                                  # gone without a word
    time.sleep(1.0)
    t0 = time.time()
    try:
        d.barrier()
        d.max(1.0)
        q.put(("no error", time.time() - t0))
    except Exception as e:                           # noqa: BLE001 -- any backend error will do
        q.put((type(e).__name__, time.time() - t0))
    q.close()
    q.join_thread()                                  # flushed before the hard exit below
    os._exit(0)


@pytest.mark.timeout(300)
def test_a_rank_that_leaves_ends_the_next_collective_with_an_error():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_that_leaves, args=(r, world, port, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    outcome, waited = q.get(timeout=120)
    for pr in procs:
        pr.join(timeout=60)
    assert outcome != "no error"
    assert waited < 60.0                             # bounded by the process-group timeout
