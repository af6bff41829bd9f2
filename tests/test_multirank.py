"""Multi-rank host logic on CPU (gloo, world size 2).

The decode path shards by batch: every (batch, kv-head) pair is independent, so replicas need no
collective on the data path. These tests check (1) the benchmark's timing reduction (max over
ranks) and barrier, (2) that a batch split across ranks reproduces the unsplit result (with the
CPU oracle standing in for the per-rank compute), and (3) that the reference arm of bench.py runs
on rank 0 only under torchrun.
"""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import bench
    import oracle
    from block_sparse_attention_compressed_b200.workloads import WORKLOADS, generate
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # (1) timing reduction
        m = bench.max_over_ranks(1.5 + rank, world)
        bench.barrier(world)
        # (2) batch-sharded replicas: rank r takes sequences r, r + world, ...
        w = WORKLOADS["gqa4-bf16-32k-b1"].replace(name="mr", batch=4, seq_len=900, top_k=3,
                                                    needles=2)
        data = generate(w, device="cpu")
        mine = list(range(rank, w.batch, world))
        qr, _ = oracle.raw(data["q"][0][mine])
        kr, _ = oracle.raw(data["k"][0][mine])
        vr, _ = oracle.raw(data["v"][0][mine])
        P = oracle.make_problem(len(mine), w.num_q_heads, w.num_kv_heads, w.head_dim,
                                data["seq_cap"], oracle.BF16, w.n_init, w.n_local, w.top_k)
        res = oracle.decode(P, qr, kr, vr, [w.seq_len] * len(mine))
        out = torch.from_numpy(res["out"]).reshape(len(mine), -1)
        gathered = [torch.zeros_like(out) for _ in range(world)]
        dist.all_gather(gathered, out)
        q.put((rank, m, [g.numpy() for g in gathered] if rank == 0 else None))
    finally:
        dist.destroy_process_group()


def test_two_rank_sharding_and_timing():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    for _ in range(world):
        rank, m, g = q.get(timeout=300)
        results[rank] = (m, g)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert results[0][0] == results[1][0] == 2.5
    # unsplit reference
    sys.path.insert(0, ROOT)
    import oracle
    from block_sparse_attention_compressed_b200.workloads import WORKLOADS, generate
    w = WORKLOADS["gqa4-bf16-32k-b1"].replace(name="mr", batch=4, seq_len=900, top_k=3, needles=2)
    data = generate(w, device="cpu")
    qr, _ = oracle.raw(data["q"][0])
    kr, _ = oracle.raw(data["k"][0])
    vr, _ = oracle.raw(data["v"][0])
    P = oracle.make_problem(w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, data["seq_cap"],
                            oracle.BF16, w.n_init, w.n_local, w.top_k)
    full = oracle.decode(P, qr, kr, vr, [w.seq_len] * w.batch)["out"].reshape(w.batch, -1)
    g0, g1 = results[0][1]
    assert np.array_equal(np.concatenate([g0[0:1], g1[0:1], g0[1:2], g1[1:2]]), full)


def test_reference_arm_under_torchrun_rank0_only():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--gpus", "2", "--steps", "2", "--warmup", "1", "--impl", "reference",
           "--workload", "tiny-f32-2k", "--cpu-seconds", "1"]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    res = json.loads(lines[0])
    assert res["impl"] == "reference" and res["unit"] == "steps/s" and res["value"] > 0
    assert res["cpu_baseline"]["kind"] == "oracle"
    assert res["e2e"]["h2d_bytes_per_step"] == 0
