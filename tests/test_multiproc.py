"""Multi-process host logic of the benchmark on CPU (gloo, world size 2).

The forward shards by (batch, head) with no data-path exchange, so the only
collectives are the barrier around the timed region and the max over ranks of
the elapsed time. These tests run two real processes over gloo.
"""
import os
import subprocess
import sys
import json

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dist.barrier()
        local_ms = 10.0 + 5.0 * rank          # rank 1 is the slowest
        ms_max = bench.max_over_ranks(local_ms, world, torch.device("cpu"))
        value = bench.whole_job_tokens_per_s(world, 7, ms_max)
        q.put((rank, ms_max, value))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_max_over_ranks_and_whole_job_throughput():
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
    import bench
    for rank, ms_max, value in res:
        assert ms_max == 15.0                  # every rank sees the slowest rank's time
        assert value == pytest.approx(world * 7 * 2 * bench.B * bench.L / 0.015)


def test_single_rank_reduction_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
    assert bench.whole_job_tokens_per_s(1, 10, 1000.0) == pytest.approx(10 * 2 * bench.B * bench.L)


def test_reference_arm_under_torchrun_prints_once():
    """--impl reference under two ranks: rank 0 runs the oracle and prints one JSON
    line, the other rank exits 0 without work."""
    env = dict(os.environ, INFINI_REFERENCE_BUDGET_S="2", OMP_NUM_THREADS="2")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--steps", "1", "--warmup", "3"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["e2e"]["h2d_bytes_per_step"] == 0


def _shard_worker(rank, world, port, q):
    """Each rank holds one range of a Linear-mode sequence; the range's state sum is
    taken with the oracle (the GPU library's infini_attn_state_update on a GPU machine),
    exchanged with the package's gather_states over gloo, and composed as the
    sharded forward composes it."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import numpy as np
    import oracle
    from compressive_memory_transformer_b200.sharded import gather_states
    from synthetic_inputs import make_inputs
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, H, N, d = 1, 2, 32, 16
        seg_per_rank = [3, 2]                   # ranges of unequal length, in rank order
        L = N * sum(seg_per_rank)
        inp = make_inputs(B, H, L, d, torch.float32, seed=61, device="cpu", gen_device="cpu")
        f = {x: inp[x].double().numpy() for x in ("q", "k", "v", "beta")}
        lo = N * sum(seg_per_rank[:rank])
        hi = lo + N * seg_per_rank[rank]
        part = {x: f[x][:, :, lo:hi] for x in ("q", "k", "v")}
        _, dM, dz = oracle.forward(part["q"], part["k"], part["v"], f["beta"], N, oracle.LINEAR)
        dM_all, dz_all = gather_states(torch.from_numpy(dM), torch.from_numpy(dz))
        assert dM_all.shape == (world, B, H, d, d) and dz_all.shape == (world, B, H, d)
        M_pre = dM_all[:rank].sum(0).numpy()
        z_pre = dz_all[:rank].sum(0).numpy()
        out_r, _, _ = oracle.forward(part["q"], part["k"], part["v"], f["beta"], N, oracle.LINEAR,
                                     M_pre, z_pre)
        ref_out, ref_M, ref_z = oracle.forward(f["q"], f["k"], f["v"], f["beta"], N, oracle.LINEAR)
        err_out = float(np.max(np.abs(out_r - ref_out[:, :, lo:hi])))
        err_M = float(np.max(np.abs(dM_all.sum(0).numpy() - ref_M)) / np.max(np.abs(ref_M)))
        err_z = float(np.max(np.abs(dz_all.sum(0).numpy() - ref_z)) / np.max(np.abs(ref_z)))
        q.put((rank, err_out, err_M, err_z))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_linear_sequence_sharding_exchange():
    """Two ranks, one all-gather of the per-range Linear state sums: every rank's
    outputs and the final state equal the single-process forward's."""
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, err_out, err_M, err_z in res:
        assert err_out < 1e-12 and err_M < 1e-12 and err_z < 1e-12, (rank, err_out, err_M, err_z)
