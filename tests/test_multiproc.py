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


def _oracle_library(monkeypatch_target, beta):
    """Stand-ins for the three library calls of the sharded forward, computed by the
    oracle in float64 on the host (this CPU test has no CUDA library to run): the
    host logic around them (the exchange, the rank-order prefix, the validation of
    the ranges, the final state) is the shipped code."""
    import numpy as np
    import oracle

    def state_update(k, v, N, mode, stream=None):
        kk, vv = k.double().numpy(), v.double().numpy()
        _, M, z = oracle.forward(kk, kk, vv, np.zeros(k.shape[1]), N, mode)
        return torch.from_numpy(M).float(), torch.from_numpy(z).float()

    def state_sum(dM, dz, M_in=None, z_in=None, stream=None):
        M = dM.double().sum(0) + (0 if M_in is None else M_in.double())
        z = dz.double().sum(0) + (0 if z_in is None else z_in.double())
        return M.float(), z.float()

    def forward(q, k, v, beta_, N, mode, M_in=None, z_in=None, out=None, state_out=True,
                stream=None):
        f = lambda t: None if t is None else t.double().numpy()
        o, M, z = oracle.forward(f(q), f(k), f(v), f(beta_), N, mode, f(M_in), f(z_in))
        return torch.from_numpy(o), torch.from_numpy(M), torch.from_numpy(z)

    monkeypatch_target.infini_attn_state_update = state_update
    monkeypatch_target.infini_attn_state_sum = state_sum
    monkeypatch_target.infini_attn_forward = forward


def _shard_worker(rank, world, port, q, seg_per_rank, ragged):
    """Each rank holds one range of a Linear-mode sequence and runs the package's
    sequence_sharded_linear_forward on it (its library calls taken by the oracle)."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import numpy as np
    import oracle
    from compressive_memory_transformer_b200 import sharded
    from synthetic_inputs import make_inputs, normal_state
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, H, N, d = 1, 2, 32, 16
        lens = [N * n for n in seg_per_rank]
        lens[-1] -= ragged                      # the last range may end mid-segment
        L = sum(lens)
        inp = make_inputs(B, H, L, d, torch.float32, seed=61, device="cpu", gen_device="cpu")
        M0, z0 = normal_state(B, H, d, seed=62, scale_M=2.0, scale_z=10.0)
        _oracle_library(sharded, inp["beta"])
        lo = sum(lens[:rank])
        hi = lo + lens[rank]
        part = {x: inp[x][:, :, lo:hi] for x in ("q", "k", "v")}
        try:
            out_r, M_end, z_end = sharded.sequence_sharded_linear_forward(
                part["q"], part["k"], part["v"], inp["beta"], N, M0, z0)
        except ValueError as e:
            q.put((rank, "ValueError", str(e)))
            return
        f = {x: inp[x].double().numpy() for x in ("q", "k", "v", "beta")}
        ref_out, ref_M, ref_z = oracle.forward(f["q"], f["k"], f["v"], f["beta"], N,
                                               oracle.LINEAR, M0.double().numpy(),
                                               z0.double().numpy())
        err_out = float(np.max(np.abs(out_r.numpy() - ref_out[:, :, lo:hi])))
        err_M = float(np.max(np.abs(M_end.double().numpy() - ref_M)) / np.max(np.abs(ref_M)))
        err_z = float(np.max(np.abs(z_end.double().numpy() - ref_z)) / np.max(np.abs(ref_z)))
        q.put((rank, err_out, err_M, err_z))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _run_shards(seg_per_rank, ragged):
    world = len(seg_per_rank)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, q, seg_per_rank, ragged))
             for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return res


def test_linear_sequence_sharding_exchange():
    """Two ranks of unequal length (3 and 2 segments, the last one ragged), a non-zero
    incoming state, one all-gather of the per-range Linear state sums: every rank's
    outputs and the final state equal the single-process forward's (the state sums
    travel in float32, hence the 1e-6 bound)."""
    for rank, err_out, err_M, err_z in _run_shards([3, 2], ragged=5):
        assert err_out < 1e-5 and err_M < 1e-6 and err_z < 1e-6, (rank, err_out, err_M, err_z)


def test_linear_sequence_sharding_rejects_a_ragged_inner_range_on_every_rank():
    """A range that ends mid-segment on a rank other than the last raises ValueError on
    every rank together (each learns every range's length from the one all-gather), so
    no rank is left waiting in a collective."""
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_bad_range_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[1] for r in res] == ["ValueError", "ValueError"], res
    assert all("[0]" in r[2] for r in res), res


def _bad_range_worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    from compressive_memory_transformer_b200 import sharded
    from synthetic_inputs import make_inputs
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        N = 32
        L_r = N * 2 - 7 if rank == 0 else N * 2   # rank 0's range ends mid-segment
        inp = make_inputs(1, 2, L_r, 16, torch.float32, seed=63 + rank, device="cpu")
        _oracle_library(sharded, inp["beta"])
        try:
            sharded.sequence_sharded_linear_forward(inp["q"], inp["k"], inp["v"], inp["beta"], N)
            q.put((rank, "returned", ""))
        except ValueError as e:
            q.put((rank, "ValueError", str(e)))
    finally:
        dist.destroy_process_group()
