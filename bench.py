#!/usr/bin/env python
"""Benchmark of the Infini-attention forward on B200.

Workload: the 1B-LM layer shape, B=4, H=8, d=128, segment N=2048, L=32768
(16 segments), bf16 q/k/v i.i.d. N(0,1), beta ~ N(0,1) per head, fp32 state
from zero. One step is one pass of the whole forward path in both memory-update
modes over the same batch: infini_attn_forward in Linear mode, then in
Linear+Delta mode (each = sigma(K) sums, z scan, per-segment state GEMMs, state
chain, fused attention + retrieval + gate). Tokens per step = 2 * B * L.

At N = 1 the line also carries, under "configs", the other full-size workloads
timed in the same run: the 1M-token stream of 512 graph-captured step calls, the
8B-model 500K forward and the segment-length sweep (--no-extra skips them).

Prints one JSON line (rank 0). Under torchrun (N > 1) every rank runs its own
batch (the path shards by (batch, head) with no exchange: weak scaling), the
ranks meet at barriers around the timed region, and the time is the max over
ranks.

--impl reference times the fp64 CPU oracle on the host cores instead (bounded
samples of the same workload) and prints the same line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "Infini-attn fwd tokens/s on 1 B200 (N=2048,d=128); % bf16 tensor peak"
UNIT = "tokens/s"
B, H, D, N, L = 4, 8, 128, 2048, 32768
WORKLOAD = (f"1B-LM layer shape: B={B}, H={H}, d={D}, N={N}, L={L} ({L // N} segments), "
            "bf16 q/k/v, fp32 state from zero; step = Linear forward + Linear+Delta forward")
# kernels per forward of the workload (several segments): Linear state, chain (which
# also scans z), attn; Linear+Delta zpart, zscan, state, chain, attn
LAUNCHES_PER_STEP = 3 + 5


def attn_flops_per_launch():
    """Algorithmic FLOPs of the fused attention + retrieval kernel for one forward:
    per token-head 2d(N+1) for the causal QK^T and PV pairs plus 2d^2 for sigma(Q)M."""
    return B * H * L * (2 * D * (N + 1) + 2 * D * D)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return j["bf16_tflops"], j.get("bf16_tflops_sustained", j["bf16_tflops"]), j["hbm_gbs"], "measured"
    return 1590.0, 1400.0, 6650.0, "fallback"


def measured_traffic(kernel_src, record):
    """dram read + write bytes per launch from the committed ncu capture, or None
    when the kernel source has changed since the counters were taken."""
    import hashlib
    p = os.path.join(ROOT, "profiles", record)
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    with open(os.path.join(ROOT, kernel_src), "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()
    if sha != rec.get("source_sha256"):
        return None
    return rec["dram_bytes_read"] + rec["dram_bytes_write"]


def usable_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i["num_threads"] for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


# ---------------------------------------------------------------------------
# multi-rank plumbing (no data-path collective: ranks work on their own batches)
# ---------------------------------------------------------------------------
def max_over_ranks(ms, world, device):
    """The slowest rank's time: every rank takes the same collective step."""
    t = torch.tensor([float(ms)], device=device, dtype=torch.float64)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_tokens_per_s(world, steps, ms_max, tokens_per_step_per_rank=2 * B * L):
    """Units processed by all ranks over the slowest rank's time (weak scaling)."""
    return world * steps * tokens_per_step_per_rank / (ms_max / 1e3)


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        self.proc = None
        self.path = None
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            self.sel = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            self.sel = str(device)

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.sel, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.3)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 8:
                    continue
                try:
                    rows.append((float(parts[0]), float(parts[1]), float(parts[2]), parts[3:]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        load = [r for r in rows if r[2] > 200.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in load for i, v in enumerate(r[3][1:5])
                          if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in load),
                "sm_max_mhz": max(r[1] for r in rows),
                "power_w_max": max(r[2] for r in rows),
                "samples": len(load), "reasons": reasons}


# ---------------------------------------------------------------------------
# CPU oracle timing (reported baseline; the oracle is timed as it stands)
# ---------------------------------------------------------------------------
def oracle_sample(q, k, v, beta, heads, modes):
    """Run the fp64 oracle on the given heads (full length) and modes; returns
    (seconds, token-heads processed)."""
    import oracle
    t0 = time.perf_counter()
    th = 0
    for (b, h) in heads:
        qh = q[b, h].to(torch.float64).numpy()
        kh = k[b, h].to(torch.float64).numpy()
        vh = v[b, h].to(torch.float64).numpy()
        g = oracle.gate_value(float(beta[h]))
        for mode in modes:
            oracle.head_forward(qh, kh, vh, g, N, mode)
            th += qh.shape[0]
    return time.perf_counter() - t0, th


def cpu_baseline(inp_cpu):
    heads = [(0, 0), (1, 3), (2, 5), (3, 7)]
    secs, th = oracle_sample(inp_cpu["q"], inp_cpu["k"], inp_cpu["v"], inp_cpu["beta"], heads,
                             (0, 1))
    return {"value": (th / H) / secs, "unit": UNIT, "cores": usable_cores(),
            "blas_threads": blas_threads(), "kind": "oracle",
            "sample": f"{len(heads)} of {B * H} heads (full L={L}) x Linear and Linear+Delta, "
                      f"fp64 numpy oracle, {secs:.1f} s; tokens = token-heads / H"}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def run_ours(args, rank, world, device):
    import compressive_memory_transformer_b200 as ia
    from synthetic_inputs import make_inputs

    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream()
    inp = make_inputs(B, H, L, D, torch.bfloat16, seed=rank, device=device, gen_device=device)
    q, k, v, beta = inp["q"], inp["k"], inp["v"], inp["beta"]
    outs = {m: (torch.empty_like(q), torch.empty((B, H, D, D), device=device),
                torch.empty((B, H, D), device=device)) for m in (ia.LINEAR, ia.DELTA)}
    ws = torch.empty(ia.workspace_size(B, H, L, N, D, ia.DELTA), dtype=torch.uint8, device=device)

    def forward(mode, evs=None):
        o, M, z = outs[mode]
        ia.infini_attn_forward_ex(q, k, v, beta, N, mode, out=o, M_out=M, z_out=z,
                                  workspace=ws, stage_events=evs)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for _ in range(args.warmup):
        forward(ia.LINEAR)
        forward(ia.DELTA)
    torch.cuda.synchronize()
    assert ia.device_status() == 0

    ev = [[[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(2)]
          for _ in range(args.steps)]
    # torch creates the CUDA event on its first record; the library then re-records
    # the same handles around its launches inside the timed region
    for e in (e for step in ev for mode in step for e in mode):
        e.record(stream)
    torch.cuda.synchronize()
    clocks = ClockSampler(device)
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        forward(ia.LINEAR, ev[i][0])
        forward(ia.DELTA, ev[i][1])
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    ms = t_start.elapsed_time(t_end)
    assert ia.device_status() == 0, "a bounded device wait ran out during the timed region"

    attn_ms = [ev[i][m][1].elapsed_time(ev[i][m][2]) for i in range(args.steps) for m in (0, 1)]
    state_ms = {m: statistics.mean(ev[i][m][0].elapsed_time(ev[i][m][1])
                                   for i in range(args.steps)) for m in (0, 1)}
    fwd_ms = {m: statistics.mean(ev[i][m][0].elapsed_time(ev[i][m][2])
                                 for i in range(args.steps)) for m in (0, 1)}

    ms_max = max_over_ranks(ms, world, device)

    # ---- end to end through the public call with host buffers ----
    # Every step copies its inputs from pinned host memory and reads its results back.
    # The copies and the kernels run on three streams with two sets of device buffers,
    # as a serving loop would: the host-to-device copy of step i + 1 and the
    # device-to-host copy of step i - 1 overlap the forwards of step i (PCIe moves both
    # directions at once). The timed region spans the first copy in to the last copy out.
    e2e = None
    if not args.no_e2e:
        qh, kh, vh = (x.cpu().pin_memory() for x in (q, k, v))
        oh = {m: torch.empty(q.shape, dtype=q.dtype).pin_memory() for m in (0, 1)}
        Mh = {m: torch.empty((B, H, D, D)).pin_memory() for m in (0, 1)}
        zh = {m: torch.empty((B, H, D)).pin_memory() for m in (0, 1)}
        ins = [(torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)) for _ in range(2)]
        res = [{m: (torch.empty_like(q), torch.empty((B, H, D, D), device=device),
                    torch.empty((B, H, D), device=device)) for m in (0, 1)} for _ in range(2)]
        s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
        mk = lambda: [torch.cuda.Event() for _ in range(2)]
        in_done, fwd_done, out_done = mk(), mk(), mk()
        for j in range(2):  # every slot starts free
            fwd_done[j].record(stream)
            out_done[j].record(stream)

        def e2e_step(i):
            j = i & 1
            qd, kd, vd = ins[j]
            s_in.wait_event(fwd_done[j])        # step i - 2's forwards are done with slot j
            with torch.cuda.stream(s_in):
                qd.copy_(qh, non_blocking=True)
                kd.copy_(kh, non_blocking=True)
                vd.copy_(vh, non_blocking=True)
                in_done[j].record(s_in)
            stream.wait_event(in_done[j])
            stream.wait_event(out_done[j])      # step i - 2's results have left slot j
            for m in (ia.LINEAR, ia.DELTA):
                o, M, z = res[j][m]
                ia.infini_attn_forward(qd, kd, vd, beta, N, m, out=o, M_out=M, z_out=z)
            fwd_done[j].record(stream)
            s_out.wait_event(fwd_done[j])
            with torch.cuda.stream(s_out):
                for m in (ia.LINEAR, ia.DELTA):
                    o, M, z = res[j][m]
                    oh[m].copy_(o, non_blocking=True)
                    Mh[m].copy_(M, non_blocking=True)
                    zh[m].copy_(z, non_blocking=True)
                out_done[j].record(s_out)

        e_steps = max(4, args.steps // 4)
        for i in range(max(3, args.warmup)):
            e2e_step(i)
        torch.cuda.synchronize()
        barrier()
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        s_in.wait_event(a)
        s_out.wait_event(a)
        for i in range(e_steps):
            e2e_step(i)
        stream.wait_event(out_done[(e_steps - 1) & 1])
        b_.record(stream)
        torch.cuda.synchronize()
        barrier()
        te_ms = max_over_ranks(a.elapsed_time(b_), world, device)
        h2d = 3 * q.numel() * q.element_size()
        d2h = 2 * (q.numel() * q.element_size() + B * H * (D * D + D) * 4)
        e2e = {"value": whole_job_tokens_per_s(world, e_steps, te_ms), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e_steps,
               "ms_per_step": te_ms / e_steps,
               "pipelined": "copies in of step i+1 and out of step i-1 overlap step i's "
                            "forwards (two device buffer sets, three streams)"}
        assert ia.device_status() == 0
        del ins, res

    if rank != 0:
        return None
    peak_burst, peak_sust, hbm, peak_src = load_peaks()
    avg_attn_s = statistics.mean(attn_ms) / 1e3
    achieved = attn_flops_per_launch() / avg_attn_s / 1e12
    line = {
        "metric": METRIC, "value": whole_job_tokens_per_s(world, args.steps, ms_max), "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) q/k/v, N(0,1) beta)",
        "config": {"workload": WORKLOAD, "B": B, "H": H, "d": D, "N": N, "L": L,
                   "modes": ["linear", "delta"], "per_rank_batch": B,
                   "l2": "inputs larger than L2 (q/k/v 768 MiB per forward), no flush"},
        # the timed region is tens of milliseconds at full clocks: the burst peak is
        # the denominator; the seconds-long power-capped figure is given beside it
        "roofline": {"kernel": "attn_kernel (fused local attention + retrieval + gate)",
                     "bound": "tensor", "achieved": achieved, "peak": peak_burst,
                     "unit": "TFLOP/s", "frac": achieved / peak_burst,
                     "traffic": measured_traffic(
                         "compressive_memory_transformer_b200/csrc/bf16_attn.cu",
                         "attn_kernel_c2_traffic.json"),
                     "peak_kind": f"bf16 dense, burst, {peak_src}",
                     "frac_of_sustained_peak": achieved / peak_sust,
                     "flops_per_launch": attn_flops_per_launch(),
                     "avg_launch_ms": avg_attn_s * 1e3},
        "modes": {
            "linear": {"tokens_per_s": B * L / (fwd_ms[0] / 1e3), "forward_ms": fwd_ms[0],
                       "state_kernels_ms": state_ms[0]},
            "delta": {"tokens_per_s": B * L / (fwd_ms[1] / 1e3), "forward_ms": fwd_ms[1],
                      "state_kernels_ms": state_ms[1]},
        },
        "gpu_launches": args.steps * LAUNCHES_PER_STEP,
        "clocks": clk,
    }
    if e2e is not None:
        line["e2e"] = e2e
    if world == 1 and not args.no_extra:
        # the other full-size workloads of the configuration list, each timed live in
        # this run (kernel fractions of the burst peak): they are reported beside the
        # headline, which stays the 1B-layer step above
        line["configs"] = {"c3_stream": extra_c3(args, device), "c4_8b_500k": extra_c4(args, device),
                           "c5_sweep": extra_c5(args, device)}
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline({"q": q.cpu(), "k": k.cpu(), "v": v.cpu(),
                                             "beta": beta.cpu()})
    return line


# ---------------------------------------------------------------------------
# reference arm: the oracle on the host cores
# ---------------------------------------------------------------------------
def run_reference(args):
    from synthetic_inputs import make_inputs
    import oracle
    inp = make_inputs(B, H, L, D, torch.bfloat16, seed=0, device="cpu")
    # one step = one head of the workload, full length, Linear and Linear+Delta; the
    # number of segments per step is cut so that the whole run stays within ~3 min
    q, k, v, beta = inp["q"], inp["k"], inp["v"], inp["beta"]
    t_cal, _ = oracle_sample(q[:, :, :N], k[:, :, :N], v[:, :, :N], beta, [(0, 0)], (0, 1))
    budget = float(os.environ.get("INFINI_REFERENCE_BUDGET_S", "150")) / max(1, args.steps + args.warmup)
    segs = int(max(1, min(L // N, budget // max(t_cal, 1e-3))))
    Ls = segs * N
    heads = [(b, h) for b in range(B) for h in range(H)]
    for i in range(args.warmup):
        b, h = heads[i % len(heads)]
        oracle_sample(q[:, :, :Ls], k[:, :, :Ls], v[:, :, :Ls], beta, [(b, h)], (0, 1))
    tot_s, tot_th = 0.0, 0
    for i in range(args.steps):
        b, h = heads[i % len(heads)]
        s_, th = oracle_sample(q[:, :, :Ls], k[:, :, :Ls], v[:, :, :Ls], beta, [(b, h)], (0, 1))
        tot_s += s_
        tot_th += th
    value = (tot_th / H) / tot_s
    sample = (f"per step one head of {B * H}, first {segs} of {L // N} segments, Linear and "
              f"Linear+Delta, fp64 numpy oracle; tokens = token-heads / H")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": tot_s / max(1, args.steps) * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": B, "H": H, "d": D, "N": N, "L": L,
                   "modes": ["linear", "delta"]},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": usable_cores(),
                         "blas_threads": blas_threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------------------
# the other workloads of the configuration list (extra lines, not the headline)
# ---------------------------------------------------------------------------
def _timed(fn, reps, stream):
    a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(reps):
        fn()
    b_.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b_) / reps


def _attn_tflops(Bc, Hc, Lc, Nc, ms):
    """Algorithmic TFLOP/s of the fused attention kernel over ms milliseconds."""
    return Bc * Hc * Lc * (2 * D * (Nc + 1) + 2 * D * D) / (ms / 1e3) / 1e12


def extra_c5(args, device):
    """Segment-length sweep: B=8, H=16, L=65536, N in {512, 1024, 2048, 4096}, both modes;
    per forward the state path and the attention kernel timed by the library's events."""
    import compressive_memory_transformer_b200 as ia
    from synthetic_inputs import make_inputs
    stream = torch.cuda.current_stream()
    peak_burst, peak_sust, _, src = load_peaks()
    Bc, Hc, Lc = 8, 16, 65536
    inp = make_inputs(Bc, Hc, Lc, D, torch.bfloat16, seed=0, device=device, gen_device=device)
    out = torch.empty_like(inp["q"])
    res = []
    for Nc in (512, 1024, 2048, 4096):
        for mode in (ia.LINEAR, ia.DELTA):
            ws = torch.empty(ia.workspace_size(Bc, Hc, Lc, Nc, D, mode), dtype=torch.uint8,
                             device=device)
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            for e in ev:
                e.record(stream)

            def f():
                ia.infini_attn_forward_ex(inp["q"], inp["k"], inp["v"], inp["beta"], Nc, mode,
                                          out=out, workspace=ws, stage_events=ev)
            for _ in range(3):
                f()
            torch.cuda.synchronize()
            tot = st = at = 0.0
            reps = max(3, args.steps // 3)
            for _ in range(reps):
                f()
                torch.cuda.synchronize()
                tot += ev[0].elapsed_time(ev[2])
                st += ev[0].elapsed_time(ev[1])
                at += ev[1].elapsed_time(ev[2])
            tot, st, at = tot / reps, st / reps, at / reps
            tf = _attn_tflops(Bc, Hc, Lc, Nc, at)
            res.append({"N": Nc, "mode": "delta" if mode else "linear",
                        "tokens_per_s": Bc * Lc / (tot / 1e3), "forward_ms": tot,
                        "state_ms": st, "attn_ms": at, "attn_tflops": tf,
                        "attn_frac": tf / peak_burst, "attn_frac_sustained": tf / peak_sust,
                        "attn_hbm_gbs": Bc * Hc * Lc * 1024 / (at / 1e3) / 1e9})
            del ws
    assert ia.device_status() == 0
    del inp, out
    torch.cuda.empty_cache()
    return {"config": "C5 segment-length sweep: B=8, H=16, d=128, L=65536, bf16",
            "peak": f"attn_frac of the {peak_burst} TFLOP/s burst bf16 peak ({src})",
            "results": res}


def extra_c4(args, device):
    """8B-model 500K stream: B=1, H=32, L=524288, N=2048, Linear+Delta, one forward."""
    import compressive_memory_transformer_b200 as ia
    from synthetic_inputs import make_inputs
    stream = torch.cuda.current_stream()
    peak_burst, peak_sust, _, src = load_peaks()
    Bc, Hc, Lc, Nc = 1, 32, 524288, 2048
    inp = make_inputs(Bc, Hc, Lc, D, torch.bfloat16, seed=0, device=device, gen_device=device)
    out = torch.empty_like(inp["q"])
    ws = torch.empty(ia.workspace_size(Bc, Hc, Lc, Nc, D, ia.DELTA), dtype=torch.uint8,
                     device=device)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(3)]
    for e in (e for row in evs for e in row):
        e.record(stream)
    it = [0]

    def f4():
        e = evs[it[0] % 3]
        it[0] += 1
        ia.infini_attn_forward_ex(inp["q"], inp["k"], inp["v"], inp["beta"], Nc, ia.DELTA,
                                  out=out, workspace=ws, stage_events=e)
    f4()
    f4()
    torch.cuda.synchronize()
    it[0] = 0
    ms = _timed(f4, 3, stream)
    at = sum(e[1].elapsed_time(e[2]) for e in evs) / 3
    st = sum(e[0].elapsed_time(e[1]) for e in evs) / 3
    tf = _attn_tflops(Bc, Hc, Lc, Nc, at)
    assert ia.device_status() == 0
    del inp, out, ws
    torch.cuda.empty_cache()
    return {"config": "C4 8B-model 500K stream: B=1, H=32, d=128, N=2048, L=524288, "
                      "Linear+Delta, one forward",
            "tokens_per_s": Bc * Lc / (ms / 1e3), "forward_ms": ms, "state_ms": st,
            "attn_ms": at, "attn_tflops": tf, "attn_frac": tf / peak_burst,
            "attn_frac_sustained": tf / peak_sust, "peak_source": src}


def extra_c3(args, device):
    """1M-token stream: 512 infini_attn_step calls (B=1, H=8, N=2048, Linear+Delta, the
    state carried in place), issued back to back and captured in one CUDA graph."""
    import compressive_memory_transformer_b200 as ia
    from synthetic_inputs import make_inputs
    stream = torch.cuda.current_stream()
    peak_burst, peak_sust, _, src = load_peaks()
    Bc, Hc, Nc, S = 1, 8, 2048, 512
    # the stream arrives segment by segment: [S][B, H, N, d], each segment contiguous
    seg = [make_inputs(Bc, Hc, Nc, D, torch.bfloat16, seed=1000 + i, device=device,
                       gen_device=device) for i in range(S)]
    beta = seg[0]["beta"]
    M = torch.zeros((Bc, Hc, D, D), device=device)
    z = torch.zeros((Bc, Hc, D), device=device)
    outs = [torch.empty_like(seg[0]["q"]) for _ in range(S)]

    def run_stream():
        for i in range(S):
            ia.infini_attn_step(seg[i]["q"], seg[i]["k"], seg[i]["v"], beta, ia.DELTA, M, z,
                                out=outs[i], M_out=M, z_out=z)
    run_stream()
    torch.cuda.synchronize()
    plain_ms = _timed(run_stream, 2, stream)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run_stream()
    g.replay()
    torch.cuda.synchronize()
    graph_ms = _timed(g.replay, 3, stream)
    del g
    assert ia.device_status() == 0
    step_ms = graph_ms / S
    # the attention kernel's algorithmic FLOPs per step over the whole step's time (the
    # state path runs beside it): a lower bound on the kernel's own fraction
    tf = _attn_tflops(Bc, Hc, Nc, Nc, step_ms)
    del seg, outs
    torch.cuda.empty_cache()
    return {"config": "C3 1M-token stream: B=1, H=8, d=128, N=2048, L=1048576 via 512 "
                      "infini_attn_step calls, Linear+Delta, state carried in place",
            "tokens_per_s_graph": Bc * S * Nc / (graph_ms / 1e3),
            "stream_ms_graph": graph_ms, "us_per_step_graph": step_ms * 1e3,
            "tokens_per_s_plain": Bc * S * Nc / (plain_ms / 1e3), "stream_ms_plain": plain_ms,
            "attn_tflops_over_step": tf, "attn_frac_over_step": tf / peak_burst,
            "peak_source": src}


def run_extra(args, device):
    """C3: 1M-token stream through 512 infini_attn_step calls (graph-captured),
    C4: 8B 500K single forward, C5: segment-length sweep, decode, backward, layer.
    One JSON line each."""
    import compressive_memory_transformer_b200 as ia
    from synthetic_inputs import make_inputs
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream()
    peak_burst, peak_sust, _, src = load_peaks()
    lines = []
    which = args.config
    if which in ("c5", "all"):
        lines.append(extra_c5(args, device))
    if which in ("c4", "all"):
        lines.append(extra_c4(args, device))
    if which in ("c3", "all"):
        lines.append(extra_c3(args, device))
    if which in ("decode", "all"):
        # token-level streaming decode on the 1B-layer heads: one segment of N tokens fed
        # one token per infini_attn_decode call (the segment-end call also folds the
        # segment into the state), and single calls in the middle of the segment
        Bc, Hc, Nc = 4, 8, 2048
        inp = make_inputs(Bc, Hc, Nc, D, torch.bfloat16, seed=7, device=device, gen_device=device)
        kc = torch.zeros((Bc, Hc, Nc, D), device=device, dtype=torch.bfloat16)
        vc = torch.zeros_like(kc)
        M = torch.zeros((Bc, Hc, D, D), device=device)
        z = torch.zeros((Bc, Hc, D), device=device)
        tok = [{x: inp[x][:, :, t:t + 1].contiguous() for x in ("q", "k", "v")}
               for t in range(Nc)]
        outs = [torch.empty_like(tok[0]["q"]) for _ in range(Nc)]
        beta = inp["beta"]

        def segment():
            for t in range(Nc):
                ia.infini_attn_decode(tok[t]["q"], tok[t]["k"], tok[t]["v"], beta, kc, vc, M, z,
                                      t, ia.DELTA, out=outs[t])
        segment()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            segment()
        g.replay()
        torch.cuda.synchronize()
        seg_ms = _timed(g.replay, 2, stream)
        del g

        def calls_at(pos, n, reps=64):
            q_ = inp["q"][:, :, pos:pos + n].contiguous()
            k_ = inp["k"][:, :, pos:pos + n].contiguous()
            v_ = inp["v"][:, :, pos:pos + n].contiguous()
            o_ = torch.empty_like(q_)

            def f():
                for _ in range(reps):
                    ia.infini_attn_decode(q_, k_, v_, beta, kc, vc, M, z, pos, ia.DELTA, out=o_)
            f()
            torch.cuda.synchronize()
            gg = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gg):
                f()
            gg.replay()
            torch.cuda.synchronize()
            ms = _timed(gg.replay, 3, stream) / reps
            del gg
            # bytes one call must move: the cache rows it attends to (K and V), the fp32
            # state, the new tokens' q/k/v in, their cache rows and outputs out
            byts = Bc * Hc * ((pos + n) * 2 * D * 2 + D * D * 4 + D * 4 + n * D * 2 * 6)
            return ms, byts
        ms1, by1 = calls_at(1024, 1)
        ms16, by16 = calls_at(1024, 16)
        assert ia.device_status() == 0
        hbm_peak = load_peaks()[2]
        lines.append({"config": "decode: B=4, H=8, d=128, N=2048, bf16, Linear+Delta, "
                                "infini_attn_decode",
                      "segment_one_token_per_call": {
                          "tokens_per_s": Bc * Nc / (seg_ms / 1e3),
                          "us_per_call": seg_ms * 1e3 / Nc, "graph_captured": True},
                      "one_token_at_pos1024": {
                          "us_per_call": ms1 * 1e3, "bytes": by1,
                          "hbm_gbs": by1 / (ms1 / 1e3) / 1e9,
                          "frac_hbm": by1 / (ms1 / 1e3) / 1e9 / hbm_peak},
                      "16_tokens_at_pos1024": {
                          "us_per_call": ms16 * 1e3, "tokens_per_s": Bc * 16 / (ms16 / 1e3),
                          "hbm_gbs": by16 / (ms16 / 1e3) / 1e9,
                          "frac_hbm": by16 / (ms16 / 1e3) / 1e9 / hbm_peak},
                      "hbm_peak_gbs": hbm_peak})
    if which in ("backward", "all"):
        # infini_attn_backward on the 1B-layer shape: gradients of q, k, v, beta and the
        # incoming state for a loss through the output (dout ~ N(0, 1), bf16)
        from synthetic_inputs import normal
        Bc, Hc, Lc, Nc = 4, 8, 32768, 2048
        inp = make_inputs(Bc, Hc, Lc, D, torch.bfloat16, seed=0, device=device, gen_device="cuda")
        dout = normal((Bc, Hc, Lc, D), torch.bfloat16, 0, 7, device="cuda").to(device)
        res = {}
        ws = torch.empty(ia.backward_workspace_size(Bc, Hc, Lc, Nc, D, ia.DELTA), dtype=torch.uint8,
                         device=device)
        for mode, name in ((ia.LINEAR, "linear"), (ia.DELTA, "delta")):
            evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(3)]
            for e in (e for row in evs for e in row):
                e.record(stream)  # torch creates the CUDA event on its first record
            it = [0]

            def f():
                e = evs[it[0] % 3]
                it[0] += 1
                e[0].record(stream)
                ia.infini_attn_backward(inp["q"], inp["k"], inp["v"], inp["beta"], Nc, mode, dout,
                                        workspace=ws, stage_events=e[1:])
            for _ in range(2):
                f()
            torch.cuda.synchronize()
            it[0] = 0
            ms = _timed(f, 3, stream)
            # per stage, averaged over the three timed calls: state rebuild, dq (with the
            # retrieval's backward), dk/dv (with the reverse state chain and the update's
            # backward)
            st_ms = [sum(e[k].elapsed_time(e[k + 1]) for e in evs) / 3 for k in range(3)]
            pairs = Bc * Hc * (Lc // Nc) * (Nc // 128) * (Nc // 128 + 1) // 2  # tile pairs
            att = pairs * 2 * 128 * 128 * D  # one 128 x 128 x 128 product over every pair
            # algorithmic products per token and head: the four gradient products of the
            # causal attention (dP = dout V^T, dV = P^T dout, dQ = dS K, dK = dS^T Q) over
            # (N + 1) / 2 keys on average, and the memory's d x d products (Linear: dnum M^T,
            # sigma(Q)^T dnum, V dM^T, sigma(K) dM; Delta adds U dM^T, dnumR M^T in place of
            # V dM^T and the chain's G_s dM_s, 2 d^3 per segment)
            mem = 8 * D * D if mode == ia.LINEAR else 10 * D * D + 2 * D ** 3 / Nc
            flops = Bc * Hc * Lc * (4 * D * (Nc + 1) + mem)
            tf = flops / (ms / 1e3) / 1e12
            res[name] = {"ms_per_call": ms, "tokens_per_s": Bc * Lc / (ms / 1e3),
                         "algorithmic_tflops": tf, "frac_of_sustained_bf16": tf / peak_sust,
                         "frac_of_burst_bf16": tf / peak_burst,
                         "stage_ms": {"state_rebuild": st_ms[0], "dq_kernel": st_ms[1],
                                      "chain_and_dkdv_kernel": st_ms[2]},
                         # executed tile products: dq 5 per tile pair (S, dP' twice, dQ),
                         # dk/dv 4 (S^T, dP'^T, dV, dK)
                         "dq_kernel_executed_tflops": 5 * att / (st_ms[1] / 1e3) / 1e12,
                         "dkdv_kernel_executed_tflops": 4 * att / (st_ms[2] / 1e3) / 1e12}
        assert ia.device_status() == 0
        del inp, dout, ws
        lines.append({"config": "backward: B=4, H=8, d=128, N=2048, L=32768, bf16, "
                                "infini_attn_backward (loss through out)",
                      **res, "peak_source": src,
                      "note": "one call: the state path rebuilt, then the dq kernel, the "
                              "reverse state chain, the dk/dv kernel (Delta: the z-gradient "
                              "scan and the dk fix-up) and the dbeta sum; executed tensor "
                              "work is about 2.3x the algorithmic count (S and dP' are "
                              "recomputed in both attention kernels)"})
    if which in ("layer", "all"):
        # one attention layer with its projections on the 1B-layer shape: x [B, L, 1024]
        # -> Q, K, V (8 heads of 128) -> forward -> W_O; and the projection GEMM alone
        from synthetic_inputs import normal
        Bc, Lc, Hc, Nc = 4, 32768, 8, 2048
        Dm = Hc * D
        x = normal((Bc, Lc, Dm), torch.bfloat16, 0, 0, device="cuda").to(device)
        Ws = [(normal((Dm, Dm), torch.float32, 0, 1 + i, device="cuda") / Dm ** 0.5).to(
            torch.bfloat16).to(device) for i in range(4)]
        beta = normal((Hc,), torch.float32, 0, 5, device="cuda").to(device)
        y = torch.empty_like(x)
        lws = torch.empty(ia.layer_workspace_size(Bc, Lc, Dm, Hc, Hc, Nc), dtype=torch.uint8,
                          device=device)
        res = {}
        for mode, name in ((ia.LINEAR, "linear"), (ia.DELTA, "delta")):
            def f(evs=None):
                ia.infini_attn_layer_forward(x, Ws[0], Ws[1], Ws[2], Ws[3], beta, Nc, mode, Hc,
                                             out=y, state_out=False, workspace=lws,
                                             stage_events=evs)
            for _ in range(2):
                f()
            torch.cuda.synchronize()
            ms = _timed(f, 5, stream)
            res[name] = {"ms_per_call": ms, "tokens_per_s": Bc * Lc / (ms / 1e3)}
            # the three stages of one call, from the events the layer records after the
            # grouped Q/K/V projection, after the forward and after W_O (mean of 5 calls)
            evs = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            for e in evs:
                e.record(stream)
            parts = [0.0, 0.0, 0.0]
            for _ in range(5):
                evs[0].record(stream)
                f(evs[1:])
                torch.cuda.synchronize()
                for i in range(3):
                    parts[i] += evs[i].elapsed_time(evs[i + 1]) / 5
            res[name]["stages_ms"] = {"qkv_projection": parts[0], "forward": parts[1],
                                      "output_projection": parts[2]}
        A2 = x.view(Bc * Lc, Dm)
        C2 = torch.empty((Bc * Lc, Dm), device=device, dtype=torch.bfloat16)
        g = lambda: ia.infini_attn_gemm_bf16(A2, Ws[0], out=C2)
        for _ in range(3):
            g()
        torch.cuda.synchronize()
        gms = _timed(g, 20, stream)
        gflop = 2.0 * Bc * Lc * Dm * Dm
        gtf = gflop / (gms / 1e3) / 1e12
        assert ia.device_status() == 0
        del x, Ws, y, A2, C2, lws
        lines.append({"config": "layer: B=4, L=32768, D_model=1024, H=H_kv=8, d=128, N=2048, "
                                "bf16, infini_attn_layer_forward (Q/K/V projections in one "
                                "grouped GEMM launch, forward, W_O)",
                      **res,
                      "projection_gemm": {"shape": "[131072 x 1024] @ [1024 x 1024]",
                                          "ms": gms, "tflops": gtf,
                                          "roofline": {"bound": "tensor", "achieved": gtf,
                                                       "peak": peak_burst, "unit": "TFLOP/s",
                                                       "frac": gtf / peak_burst,
                                                       "peak_kind": "burst (measured cuBLAS)"}},
                      "peak_source": src})
    return lines


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the C3 / C4 / C5 workloads reported beside the headline")
    ap.add_argument("--config", choices=["c2", "c3", "c4", "c5", "decode", "backward", "layer",
                                         "all"],
                    default="c2",
                    help="c2 (default) prints the headline line; the others print one extra "
                         "line per workload of the configuration list")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    device = torch.device("cuda", local)
    if args.config != "c2":
        for ln in run_extra(args, device):
            print(json.dumps(ln), flush=True)
        return
    try:
        line = run_ours(args, rank, world, device)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
