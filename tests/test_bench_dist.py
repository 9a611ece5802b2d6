"""The benchmark's multi-process plumbing on the CPU (gloo, world size 2): the
max-over-ranks timing reduction, the barrier, and the reference arm under the
distributed launcher (rank 0 prints one JSON line, rank 1 exits without work).
"""
import json
import os
import socket
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist

    w, r, _ = bench.dist_setup()
    try:
        assert (w, r) == (world, rank)
        bench.barrier(w)
        q.put((rank, bench.max_over_ranks(10.0 + 5.0 * rank, w)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert got == [(0, 15.0), (1, 15.0)]


def test_reference_arm_under_the_launcher():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "1", "--warmup", "1"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1  # rank 0 alone prints
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0


def _shard_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    from lossless_bf16_weight_huffman_b200 import shard, synth

    dist.init_process_group("gloo")
    try:
        loads = [s.numel for s in synth.llama8b_shaped()]
        mine = shard.partition(loads, world)[rank]
        got = [None] * world
        dist.all_gather_object(got, (rank, mine, sum(loads[i] for i in mine)))
        q.put(got)
    finally:
        dist.destroy_process_group()


def test_shard_partition_gloo_world2():
    """Each rank computes its share of the 8B-shaped set on its own; together
    the shares cover every tensor exactly once and the ranks' loads differ by
    at most one tensor's."""
    from lossless_bf16_weight_huffman_b200 import synth

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    views = [q.get(timeout=10) for _ in range(2)]
    assert views[0] == views[1]
    loads = [s.numel for s in synth.llama8b_shaped()]
    shares = [m for _, m, _ in views[0]]
    allidx = sorted(i for m in shares for i in m)
    assert allidx == list(range(len(loads)))
    tot = [t for _, _, t in views[0]]
    assert max(tot) - min(tot) <= max(loads)


def test_shard_partition_properties():
    import random

    from lossless_bf16_weight_huffman_b200 import shard

    rnd = random.Random(5)
    for trial in range(200):
        loads = [rnd.choice([1, 7, 4096, 10**6, 5 * 10**8]) for _ in range(rnd.randint(0, 60))]
        world = rnd.randint(1, 8)
        parts = shard.partition(loads, world)
        assert len(parts) == world
        assert sorted(i for p in parts for i in p) == list(range(len(loads)))
        tot = shard.rank_loads(loads, parts)
        if loads:
            assert max(tot) - min(tot) <= max(loads)
