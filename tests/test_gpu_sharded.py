"""The sequence-sharded Linear forward as shipped (sharded.sequence_sharded_linear_forward),
run by two real processes over a gloo group, both on the one GPU of the test box: each
rank sums its range of the sequence with the CUDA library, the ranks exchange the sums
(staged through host memory, as gloo moves host tensors), and each rank runs its
forward from the incoming state plus the sums before it. The ranks never wait on one
another inside a kernel: the only exchange is the host-side all-gather.

Every rank's outputs and the final state are compared with one fp64 oracle forward over
the whole sequence at the bf16 tolerances of the parity tests."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from parity import check_bf16, run_oracle
from synthetic_inputs import make_inputs, normal_state

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
B, H, N = 1, 4, 256


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(lens):
    inp = make_inputs(B, H, sum(lens), 128, torch.bfloat16, seed=81, device="cpu",
                      gen_device="cpu")
    M0, z0 = normal_state(B, H, 128, seed=82, scale_M=3.0, scale_z=50.0)
    return inp, M0, z0


def _rank_main(rank, world, port, lens, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    torch.cuda.set_device(0)
    import compressive_memory_transformer_b200 as ia
    from compressive_memory_transformer_b200.sharded import sequence_sharded_linear_forward
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp, M0, z0 = _inputs(lens)
        lo = sum(lens[:rank])
        part = {x: inp[x][:, :, lo:lo + lens[rank]].contiguous().cuda() for x in ("q", "k", "v")}
        out, M, z = sequence_sharded_linear_forward(part["q"], part["k"], part["v"],
                                                    inp["beta"].cuda(), N, M0.cuda(), z0.cuda())
        torch.cuda.synchronize()
        status = ia.device_status()
        q.put((rank, status, out.float().cpu().numpy(), M.cpu().numpy(), z.cpu().numpy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("lens", [[3 * N, 2 * N - 100], [N, 4 * N]])
def test_two_ranks_match_one_forward(lens):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    world = len(lens)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, lens, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in range(world)), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    inp, M0, z0 = _inputs(lens)
    ref_out, ref_M, ref_z = run_oracle(inp, N, 0, M0, z0)
    bounds = np.cumsum([0] + lens)
    for rank, status, out, M, z in res:
        assert status == 0, f"rank {rank}: a bounded device wait ran out"
        lo, hi = bounds[rank], bounds[rank + 1]
        ref_r = (ref_out[:, :, lo:hi], ref_M, ref_z)
        check_bf16(torch.from_numpy(out), torch.from_numpy(M), torch.from_numpy(z), ref_r,
                   what=f"sharded Linear forward, rank {rank} of {lens}")
