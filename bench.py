"""Benchmark of the block-sparse prefill attention path on B200.

One step = one pass of the whole path over one batch: pool (a1), block
scores + routing (a2-a4) and exact + 0th-order attention (a5-a7).  Default
workload: the DiT-video-shaped N = 32K case (B=1, H=12, d=128, top-k density
0.15).  Prints ONE JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--density X] [--impl psa|reference]

Timing: W untimed warm-up steps, then K timed steps.  Each step is bracketed
by CUDA events on the launching stream; a 512 MB buffer is rewritten between
steps (outside the events) so L2 (126 MB) starts cold every step.  Multi-GPU
(torchrun): every rank runs the same-size problem on its own seeded inputs
(weak scaling, no collective on the data path); the step time is the max
over ranks.  ``--impl reference`` times the fp64 CPU oracle on a bounded
sample of the same workload (the only other place this file runs it).
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from block_sparse_attention_psa_b200 import psa  # noqa: E402
from block_sparse_attention_psa_b200.inputs import WORKLOADS, make_qkv  # noqa: E402

METRIC = "block-sparse attn effective TFLOP/s & ms/call at N=32K; % of bf16 TC / HBM roofline"
DEFAULT_WORKLOAD = "dit_video_n32k"
L2_FLUSH_BYTES = 512 << 20


# ---------------------------------------------------------------- accounting
def dense_flops(B, H, N, d, causal):
    """Dense-equivalent FLOPs of attention: 4 B H N^2 d (half when causal)."""
    f = 4.0 * B * H * N * N * d
    return f / 2 if causal else f


def executed_flops(row_ptr, col_idx, B, H, M, d, causal):
    """Algorithmic FLOPs the sparse path executes (host, from the block lists):
    4 d b^2 per listed block pair (a causal diagonal block counts its b(b+1)/2
    visible pairs) + 4 d b per 0th-order term (unlisted candidate)."""
    b = 64
    rp = row_ptr.astype(np.int64)
    nsel = np.diff(rp)
    rows = np.arange(B * H * M)
    I = rows % M
    if causal:
        pcand = I                      # 0th-order candidates J < I
        n_diag = len(rows)             # routers always list the diagonal
        exact_pairs = b * b * (nsel.sum() - n_diag) + n_diag * b * (b + 1) // 2
        unlisted = pcand - (nsel - 1)
    else:
        exact_pairs = b * b * nsel.sum()
        unlisted = M - nsel
    return 4.0 * d * exact_pairs + 4.0 * d * b * unlisted.sum()


def issued_flops(row_ptr, B, H, M, d, causal, dense=False):
    """FLOPs the attention kernel's MMAs issue (host, from the block lists):
    per tile S^T = K Q^T (128 x 64 x d) and O^T += V^T P^T (d x 64 x 128: an
    M = d product).  A unit takes ceil(listed / 2) exact tiles
    and, when some candidate is unlisted, ceil(pooled candidates / 128) pooled
    tiles (at least one tile in all)."""
    rp = row_ptr.astype(np.int64)
    nsel = np.diff(rp)
    I = np.arange(B * H * M) % M
    cand = I + 1 if causal else np.full_like(I, M)
    pcand = I if causal else np.full_like(I, M)
    n_a2 = np.where((~np.bool_(dense)) & (pcand > 0) & (nsel < cand), (pcand + 127) // 128, 0)
    n_e = (nsel + 1) // 2
    tiles = np.maximum(n_a2 + n_e, 1)
    return float(tiles.sum()) * (2.0 * 128 * 64 * d + 2.0 * d * 64 * 128)


def pool_bytes(B, H, N, d):
    M = N // 64
    return 3 * B * H * N * d * 2 + 3 * B * H * M * d * 4


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of the SM clock and throttle reasons while running."""

    FIELDS = ("clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.rows = []
        self.proc = None
        try:
            self.target = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
        except Exception:
            self.target = None

    def start(self):
        cmd = ["nvidia-smi", "--query-gpu=" + ",".join(self.FIELDS), "--format=csv,noheader,nounits",
               "-lms", "50"]
        if self.target:
            cmd += ["--id=" + str(self.target)]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == len(self.FIELDS):
                self.rows.append(parts)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm = [float(r[0]) for r in self.rows if r[0].replace(".", "").isdigit()]
        smax = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({n for r in self.rows for n, val in zip(names, r[4:8]) if val.lower() == "active"})
        power = [float(r[2]) for r in self.rows if r[2].replace(".", "").isdigit()]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(self.rows),
                "power_w_max": max(power) if power else None}


# ---------------------------------------------------------------- GPU arm
class Step:
    """Device buffers and one step of the path for one workload."""

    def __init__(self, name, density, seed, device, dense=False, hyd=False):
        w = dict(WORKLOADS[name])
        self.name = name
        self.dense = dense  # psa_dense (every candidate exact) instead of pool -> route -> attn
        self.hyd = hyd      # first-order correction: + statistic, attention with the correction
        self.w = w
        self.B, self.H, self.N, self.d = w["B"], w["H"], w["N"], w["d"]
        self.M = self.N // 64
        self.causal = w["causal"]
        self.keep_first = w["keep_first"]
        self.mode, param = w["routing"]
        if isinstance(param, tuple):
            param = density if density is not None else param[0]
        elif density is not None:
            param = density
        self.param = float(param)
        q, k, v = make_qkv(self.B, self.H, self.N, self.d, w["gen"], seed)
        self.host = [x.pin_memory() for x in (q, k, v)]
        self.q, self.k, self.v = (x.to(device) for x in self.host)
        B, H, M, d = self.B, self.H, self.M, self.d
        f32 = dict(dtype=torch.float32, device=device)
        self.stats = tuple(torch.empty(B, H, M, d, **f32) for _ in range(3))
        cap = psa.psa_route_capacity(B, H, M, self.causal)
        i32 = dict(dtype=torch.int32, device=device)
        self.csr = (torch.empty(B * H * M + 1, **i32), torch.empty(cap, **i32), torch.empty(1, **i32),
                    torch.empty(B * H * M, dtype=torch.float32, device=device))
        self.ws = psa.workspace(B, H, self.N, d, device)
        self.hstat = torch.empty(B, H, d, d, dtype=torch.float32, device=device)
        self.out = torch.empty_like(self.q)
        self.out_host = torch.empty(self.out.shape, dtype=torch.bfloat16).pin_memory()
        self.stream = torch.cuda.current_stream()
        self.launches = launches_per_step(B, H, self.M, self.mode, dense, hyd)

    def run(self, ev=None, io=None, stream=None):
        """pool -> route -> [statistic ->] attention; ``ev`` = 5 events (or
        None entries) recorded before the pool, after it, after the routing,
        after the first-order statistic and after the attention call;
        ``io`` = (q, k, v, out) device tensors (default: the step's own) and
        ``stream`` the stream to issue on (default: the current one)."""
        q, k, v, out = io if io is not None else (self.q, self.k, self.v, self.out)
        s = stream if stream is not None else self.stream

        def mark(i):
            if ev is not None and ev[i] is not None:
                ev[i].record(s)

        if self.dense:
            # the dense baseline: one call (it pools the keys for its stabiliser itself)
            for i in range(4):
                mark(i)
            psa.psa_dense(q, k, v, self.causal, ws=self.ws, out=out, stream=s)
            mark(4)
            return
        mark(0)
        psa.psa_pool(q, k, v, out=self.stats, stream=s)
        mark(1)
        qbar, kbar, vsum = self.stats
        if self.mode == "topk":
            psa.psa_route_topk(qbar, kbar, self.param, self.causal, out=self.csr, ws=self.ws, stream=s)
        elif self.mode == "thresh_prob":
            psa.psa_route_thresh_prob(qbar, kbar, self.param, self.causal, self.keep_first, ws=self.ws,
                                      out=self.csr, stream=s)
        else:
            psa.psa_route_thresh(qbar, kbar, self.param, self.causal, self.keep_first, ws=self.ws,
                                 out=self.csr, stream=s)
        mark(2)
        if self.hyd:
            psa.psa_hyd_stat(k, v, kbar, vsum, ws=self.ws, out=self.hstat, stream=s)
        mark(3)
        if self.hyd:
            psa.psa_attn_hyd(q, k, v, kbar, vsum, self.hstat, self.csr[0], self.csr[1], self.causal, ws=self.ws,
                             out=out, row_max=self.csr[3], stream=s)
        else:
            psa.psa_attn(q, k, v, kbar, vsum, self.csr[0], self.csr[1], self.causal, ws=self.ws,
                         out=out, row_max=self.csr[3], stream=s)
        mark(4)

    def e2e_ms(self, nsteps):
        """Milliseconds per step with host buffers in and the host result out,
        through the same public calls, the way a caller would overlap them:
        step i's inputs go host -> device on one stream while step i-1
        computes on a second and step i-2's output goes device -> host on a
        third (two device buffer sets).  Timed on the device from the first
        input copy to the last output copy."""
        dev = self.q.device
        slots = [(self.q, self.k, self.v, self.out),
                 tuple(torch.empty_like(x) for x in (self.q, self.k, self.v, self.out))]
        host_out = [self.out_host, torch.empty(self.out.shape, dtype=self.out.dtype, pin_memory=True)]
        s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
        ev_in, ev_cmp, ev_out = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        start.record(s_in)
        for i in range(nsteps):
            b = i % 2
            q, k, v, out = slots[b]
            if i >= 2:
                s_in.wait_event(ev_cmp[b])   # step i-2 has finished reading these inputs
            with torch.cuda.stream(s_in):
                for dst, src in zip((q, k, v), self.host):
                    dst.copy_(src, non_blocking=True)
            ev_in[b].record(s_in)
            s_cmp.wait_event(ev_in[b])
            if i >= 2:
                s_cmp.wait_event(ev_out[b])  # step i-2's output has left this buffer
            self.run(io=(q, k, v, out), stream=s_cmp)
            ev_cmp[b].record(s_cmp)
            s_out.wait_event(ev_cmp[b])
            with torch.cuda.stream(s_out):
                host_out[b].copy_(out, non_blocking=True)
            ev_out[b].record(s_out)
        end.record(s_out)
        torch.cuda.synchronize()
        return start.elapsed_time(end) / nsteps

    def h2d_bytes(self):
        return sum(x.numel() * x.element_size() for x in self.host)

    def d2h_bytes(self):
        return self.out_host.numel() * self.out_host.element_size()


def launches_per_step(B: int, H: int, M: int, mode: str, dense: bool, hyd: bool = False) -> int:
    """Kernels of ours one step launches.  Every call that takes a workspace
    starts with one launch that zeroes its header.  psa_dense = 5 (header,
    key pooling, attention, rerun of flagged blocks, exact fixup); otherwise
    pool 1, route = header plus, per batch of heads, one score and one
    selection launch (the library batches as many heads as fit 256 MB of
    scores), plus scan and compaction for the threshold routers, and
    attention 5 (header, bf16 statistics, attention, rerun of flagged blocks,
    exact fixup); the first-order mode adds the statistic call (3: header,
    partial sums and their reduction) and the correction (1)."""
    if dense:
        return 5
    Mp = -(-M // 128) * 128
    per_batch = max(1, min(B * H, (256 << 20) // (M * Mp * 4)))
    nb = -(-(B * H) // per_batch)
    route = 1 + 2 * nb + (0 if mode == "topk" else 2)
    return 1 + route + 5 + (4 if hyd else 0)


def _flush(buf):
    buf.add_(1)


def _dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    return world, rank, local


def _barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The largest value over all ranks (device timing is the max over ranks)."""
    if world == 1:
        return x
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(flops_per_rank: float, world: int, ms_per_step: float) -> float:
    """Whole-job TFLOP/s: every rank processes its own problem of the same size."""
    return world * flops_per_rank / (ms_per_step * 1e-3) / 1e12


def gpu_arm(args):
    world, rank, local = _dist_setup()
    if args.gpus != world and world > 1:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE {world}")
    device = torch.device("cuda", local)
    st = Step(args.workload, args.density, seed=rank, device=device, dense=args.dense, hyd=args.hyd)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    for _ in range(args.warmup):
        st.run()
        _flush(flush)
    torch.cuda.synchronize()

    # routing of this batch, for the executed-FLOP count and density
    n_cand = st.B * st.H * (st.M * (st.M + 1) // 2 if st.causal else st.M * st.M)
    if st.dense:
        rows = st.B * st.H * st.M
        nsel = np.tile(np.arange(1, st.M + 1) if st.causal else np.full(st.M, st.M), st.B * st.H)
        rp = np.concatenate([[0], np.cumsum(nsel)])
        nnz = n_cand
        ex_flops = executed_flops(rp, None, st.B, st.H, st.M, st.d, st.causal)
        is_flops = issued_flops(rp, st.B, st.H, st.M, st.d, st.causal, dense=True)
        assert rp[-1] == nnz and len(rp) == rows + 1
    else:
        rp = st.csr[0].cpu().numpy()
        nnz = int(st.csr[2].item())
        ex_flops = executed_flops(rp, None, st.B, st.H, st.M, st.d, st.causal)
        is_flops = issued_flops(rp, st.B, st.H, st.M, st.d, st.causal)
    # first-order mode: the correction X = Q H (2 N d^2 per head) in the
    # attention call; the statistic (another 2 N d^2) is timed on its own
    hyd_apply_flops = 2.0 * st.B * st.H * st.N * st.d * st.d if st.hyd else 0.0
    ex_flops += hyd_apply_flops
    de_flops = dense_flops(st.B, st.H, st.N, st.d, st.causal)
    status = psa.psa_read_status(st.ws)
    fixup_rerun, fixup_exact = psa.psa_read_fixup_count(st.ws)

    clocks = ClockSampler(local)
    clocks.start()
    # the step: one event on each side, so nothing but the library's own
    # launches sits between its calls (each call's kernels are chained
    # launches that start while the previous kernel drains)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    _barrier(world)
    torch.cuda.synchronize()
    for i in range(args.steps):
        evs[i][0].record(st.stream)
        st.run()
        evs[i][1].record(st.stream)
        _flush(flush)
    torch.cuda.synchronize()
    # the per-call split: the same steps twice more, with events between
    # some calls (an event between two calls serialises them, so these times
    # feed the kernel split and the roofline, not the step time): once with
    # pool + routing as one chained pass, the statistic and the attention
    # call each between events; once with the pool alone between events
    def timed(marks):
        out = []
        for _ in range(args.steps):
            ev = [torch.cuda.Event(enable_timing=True) if m else None for m in marks]
            st.run(ev)
            _flush(flush)
            out.append(ev)
        torch.cuda.synchronize()
        return out
    split = timed((1, 0, 1, 1, 1))
    pool_only = timed((1, 1, 0, 0, 0))
    _barrier(world)
    clk = clocks.stop()
    step_ms = [a.elapsed_time(b) for a, b in evs]
    pool_ms = [e[0].elapsed_time(e[1]) for e in pool_only]
    pool_route_ms = [e[0].elapsed_time(e[2]) for e in split]
    stat_ms = [e[2].elapsed_time(e[3]) for e in split]
    attn_ms = [e[3].elapsed_time(e[4]) for e in split]
    total_ms = max_over_ranks(sum(step_ms), world)
    ms_per_step = total_ms / args.steps

    # end to end through the public API with host buffers
    e2e_steps = max(4, min(args.steps, 10))
    st.e2e_ms(2)
    torch.cuda.synchronize()
    _barrier(world)
    e2e_ms = max_over_ranks(st.e2e_ms(e2e_steps), world)

    peaks = _peaks()
    attn_avg = statistics.mean(attn_ms)
    stat_avg = statistics.mean(stat_ms)
    pool_avg = statistics.mean(pool_ms)
    pool_route_avg = statistics.mean(pool_route_ms)
    route_avg = pool_route_avg - pool_avg  # what the routing adds to the chained pass
    achieved = ex_flops / (attn_avg * 1e-3) / 1e12
    tc_peak = peaks["bf16_tflops"]
    line = {
        "metric": METRIC,
        "value": round(weak_scaling_value(de_flops, world, ms_per_step), 3),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded generator, seed = rank)",
        "config": {"workload": st.name, "B": st.B, "H": st.H, "N": st.N, "d": st.d, "block": 64,
                   "causal": st.causal, "routing": "dense (psa_dense)" if st.dense else f"{st.mode} {st.param}",
                   "variant": "first-order (psa_hyd_stat + psa_attn_hyd)" if st.hyd else "0th-order (psa_attn)",
                   "keep_first": st.keep_first,
                   "parallelism": f"replicas x{world} (independent problems)" if world > 1 else "1 GPU",
                   "l2": "flushed between steps (512 MB write outside the timed events)"},
        "roofline": {"bound": "tensor",
                     "kernel": "attn_kernel (psa_dense call)" if st.dense else
                     ("attn_kernel + hyd_apply_kernel (psa_attn_hyd call)" if st.hyd else "attn_kernel (psa_attn call)"),
                     "achieved": round(achieved, 2), "peak": tc_peak, "unit": "TFLOP/s",
                     "frac": round(achieved / tc_peak, 4),
                     # the capture is of psa_attn at the workload's own routing
                     "traffic": None if st.dense or st.hyd else recorded_traffic(st.name, args.density),
                     "peak_source": peaks["source"] + " bf16 burst"},
        "kernels": {"pool_ms": None if st.dense else round(pool_avg, 4),
                    "hyd_stat_ms": round(stat_avg, 4) if st.hyd else None,
                    "hyd_stat_gbs": round(2 * st.B * st.H * st.N * st.d * 2 / (stat_avg * 1e-3) / 1e9, 1)
                    if st.hyd else None,
                    "route_ms": None if st.dense else round(route_avg, 4), "attn_ms": round(attn_avg, 4),
                    "pool_gbs": None if st.dense else round(pool_bytes(st.B, st.H, st.N, st.d) / (pool_avg * 1e-3) / 1e9, 1),
                    "pool_hbm_frac": None if st.dense else round(pool_bytes(st.B, st.H, st.N, st.d) / (pool_avg * 1e-3)
                                                                 / 1e9 / peaks["hbm_gbs"], 4),
                    # pool and route as one chained pass (timed between two events)
                    # over the pooled inputs' HBM bytes (the routing itself reads
                    # only the pooled statistics)
                    "pool_route_ms": None if st.dense else round(pool_route_avg, 4),
                    "pool_route_hbm_frac": None if st.dense else round(
                        pool_bytes(st.B, st.H, st.N, st.d) / (pool_route_avg * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                    "attn_executed_tflops": round(achieved, 2),
                    "attn_effective_tflops": round(de_flops / (attn_avg * 1e-3) / 1e12, 2)},
        "flops": {"dense_equivalent": de_flops, "executed": ex_flops, "mma_issued": is_flops,
                  "mma_issued_tflops": round(is_flops / (attn_avg * 1e-3) / 1e12, 2)},
        "density": {"realised": round(nnz / n_cand, 5), "listed_blocks": nnz},
        "device_status": status,
        # query blocks of one step whose denominator left [2^-60, 2^60] under the
        # kernel's fixed per-block stabiliser: recomputed on the tensor cores with
        # per-query stabilisers (rerun), and those that still needed the exact
        # CUDA-core path; their cost is inside attn_ms
        "fixup": {"rerun_blocks": fixup_rerun, "exact_blocks": fixup_exact, "of": st.B * st.H * st.M,
                  "share": round(fixup_rerun / (st.B * st.H * st.M), 6)},
        "e2e": {"value": round(weak_scaling_value(de_flops, world, e2e_ms), 3), "unit": "TFLOP/s",
                "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": st.h2d_bytes(),
                "d2h_bytes_per_step": st.d2h_bytes(), "steps": e2e_steps,
                "overlap": "inputs in, compute, result out on three streams, two device buffer sets"},
        "gpu_launches": st.launches * (args.steps),
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # the oracle's sparse step at this workload's routing (also for --dense: the
        # oracle has no separate dense path; density 1.0 of the sweep is its dense case)
        line["cpu_baseline"] = cpu_baseline(st.name, st.param, budget_s=args.cpu_budget)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


def bwd_arm(args):
    """The backward of the 0th-order attention (psa_attn_bwd) on the
    workload's own block lists: pool, route and attention run once to give
    out and lse, dout is a seeded N(0, 1) tensor, and each timed step is one
    psa_attn_bwd call on inputs resident in HBM (L2 flushed between steps,
    outside the events).  FLOPs: 2.5x the forward's (five products per
    listed key pair and per pseudo-key instead of two: the scores and dP
    recomputed, dq, dk, dv / dkbar, dvsum)."""
    world, rank, local = _dist_setup()
    device = torch.device("cuda", local)
    st = Step(args.workload, args.density, seed=rank, device=device)
    if st.dense:
        raise SystemExit("--bwd times the routed path")
    st.run()
    qbar, kbar, vsum = st.stats
    out, lse = psa.psa_attn(st.q, st.k, st.v, kbar, vsum, st.csr[0], st.csr[1], st.causal, ws=st.ws,
                            want_lse=True, row_max=st.csr[3])
    gen = torch.Generator(device=device).manual_seed(1000 + rank)
    dout = torch.randn(st.q.shape, generator=gen, device=device).to(torch.bfloat16)
    grads = tuple(torch.empty_like(st.q) for _ in range(3))
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)

    def call():
        psa.psa_attn_bwd(st.q, st.k, st.v, kbar, vsum, st.csr[0], st.csr[1], out, lse, dout, st.causal,
                         ws=st.ws, grads=grads)

    for _ in range(args.warmup):
        call()
        _flush(flush)
    torch.cuda.synchronize()
    status = psa.psa_read_status(st.ws)
    rp = st.csr[0].cpu().numpy()
    fwd_ex = executed_flops(rp, None, st.B, st.H, st.M, st.d, st.causal)
    ex = 2.5 * fwd_ex
    de = 2.5 * dense_flops(st.B, st.H, st.N, st.d, st.causal)
    clocks = ClockSampler(local)
    clocks.start()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    _barrier(world)
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    for i in range(args.steps):
        evs[i][0].record(s)
        call()
        evs[i][1].record(s)
        _flush(flush)
    torch.cuda.synchronize()
    _barrier(world)
    clk = clocks.stop()
    ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in evs), world) / args.steps
    peaks = _peaks()
    achieved = ex / (ms * 1e-3) / 1e12
    line = {
        "metric": METRIC + " (backward of psa_attn)",
        "value": round(weak_scaling_value(de, world, ms), 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded generator, seed = rank)",
        "config": {"workload": st.name, "B": st.B, "H": st.H, "N": st.N, "d": st.d, "block": 64,
                   "causal": st.causal, "routing": f"{st.mode} {st.param}", "variant": "backward (psa_attn_bwd)",
                   "l2": "flushed between steps (512 MB write outside the timed events)"},
        "roofline": {"bound": "tensor", "kernel": "bwd_pseudo + bwd_dq + bwd_dkdv (psa_attn_bwd call)",
                     "achieved": round(achieved, 2), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": round(achieved / peaks["bf16_tflops"], 4), "traffic": None,
                     "peak_source": peaks["source"] + " bf16 burst"},
        "flops": {"dense_equivalent": de, "executed": ex},
        "device_status": status,
        # header, bf16 statistics, delta, bitmaps, pseudo + its reduction, dq, dk/dv
        "gpu_launches": 8 * args.steps,
        "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


def recorded_traffic(workload: str, density=None):
    """DRAM bytes per attention launch of this workload from the ncu record
    ``profiles/traffic.json`` (dram__bytes_read.sum + dram__bytes_write.sum of
    one captured launch), if the kernel source still hashes to the captured
    one and the capture used the same routing density override (else None:
    the counters no longer describe the kernel or the run)."""
    import hashlib

    rec = os.path.join(ROOT, "profiles", "traffic.json")
    src = os.path.join(ROOT, "block_sparse_attention_psa_b200", "csrc", "attn.cu")
    try:
        with open(rec) as f:
            entry = json.load(f)["attn_kernel"][workload]
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    except (OSError, KeyError, ValueError):
        return None
    if entry.get("attn_cu_sha256_prefix") != sha or entry.get("density") != density:
        return None
    return int(entry["dram_bytes_per_launch"])


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p["bf16_tflops_sustained"]), "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------- oracle arm
def _oracle_threads():
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads") for i in threadpool_info() if i.get("num_threads")]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def oracle_step_time(name, param, budget_s):
    """Time the fp64 oracle on a bounded sample of one step of the workload:
    pooling and block scores in full; routing of whole heads and attention on
    a seeded sample of query blocks of those heads until the budget is spent;
    both extrapolated (per head, per query block) to the whole step."""
    import oracle.psa_oracle as O

    w = WORKLOADS[name]
    B, H, N, d = w["B"], w["H"], w["N"], w["d"]
    M = N // 64
    causal = w["causal"]
    q, k, v = make_qkv(B, H, N, d, w["gen"], 0)
    f64 = lambda t: t.double().numpy()
    q, k, v = f64(q), f64(k), f64(v)
    t0 = time.perf_counter()
    qbar, kbar, vsum = O.pool(q, k, v)
    s = O.block_scores(qbar, kbar)
    t_full = time.perf_counter() - t0
    mode = w["routing"][0]
    rng = np.random.default_rng(0)
    t_route, heads = 0.0, 0
    t_attn, units = 0.0, 0
    for bh in range(B * H):
        b, h = divmod(bh, H)
        t1 = time.perf_counter()
        if mode == "topk":
            rp, ci = O.route_topk(s[b:b + 1, h:h + 1], param, causal)
        else:
            route = O.route_thresh_prob if mode == "thresh_prob" else O.route_thresh
            rp, ci = route(s[b:b + 1, h:h + 1], param, causal, w["keep_first"])
        t_route += time.perf_counter() - t1
        heads += 1
        for I in rng.permutation(M):
            t1 = time.perf_counter()
            O.attention(q[b:b + 1, h:h + 1], k[b:b + 1, h:h + 1], v[b:b + 1, h:h + 1],
                        kbar[b:b + 1, h:h + 1], vsum[b:b + 1, h:h + 1], rp, ci, causal, 64, [(0, 0, int(I))])
            t_attn += time.perf_counter() - t1
            units += 1
            if t_route + t_attn > budget_s:
                break
        if t_route + t_attn > budget_s:
            break
    per_step = t_full + t_route / heads * (B * H) + t_attn / units * (B * H * M)
    return per_step, units, B * H * M, t_full + t_route + t_attn


def cpu_baseline(name, param, budget_s=15.0):
    w = WORKLOADS[name]
    per_step, done, total, spent = oracle_step_time(name, param, budget_s)
    de = dense_flops(w["B"], w["H"], w["N"], w["d"], w["causal"])
    return {"value": round(de / per_step / 1e12, 6), "unit": "TFLOP/s", "cores": _oracle_threads(),
            "kind": "oracle",
            "sample": f"fp64 numpy oracle: pool + scores in full, routing + attention on {done} of {total} "
                      f"query blocks ({spent:.1f} s), extrapolated per query block; {per_step:.1f} s/step",
            "host_cpus": os.cpu_count()}


def reference_arm(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = WORKLOADS[args.workload]
    mode, param = w["routing"]
    if isinstance(param, tuple):
        param = param[0]
    if args.density is not None:
        param = args.density
    budget = max(2.0, min(args.cpu_budget, 120.0 / max(1, args.steps + args.warmup)))
    full_step_s, wall_s, sampled = [], [], []
    t_all = time.perf_counter()
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        per_step, done, total, spent = oracle_step_time(args.workload, param, budget)
        if i >= args.warmup:
            full_step_s.append(per_step)
            wall_s.append(time.perf_counter() - t0)
            sampled.append(done)
    wall_total = time.perf_counter() - t_all
    full_ms = statistics.mean(full_step_s) * 1e3
    de = dense_flops(w["B"], w["H"], w["N"], w["d"], w["causal"])
    value = de / (full_ms * 1e-3) / 1e12
    line = {
        "impl": "reference",
        # value: dense-equivalent FLOPs of one whole step over the oracle's time
        # for that step, EXTRAPOLATED from the sampled query blocks; ms_per_step
        # is the wall time each timed (sampled) step actually took
        "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(statistics.mean(wall_s) * 1e3, 1),
        "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded generator, seed 0)",
        "config": {"workload": args.workload, "B": w["B"], "H": w["H"], "N": w["N"], "d": w["d"],
                   "routing": f"{mode} {param}", "l2": "n/a (host)"},
        "extrapolated": True,
        "sampled_units": int(statistics.mean(sampled)), "total_units": total,
        "extrapolated_ms_per_full_step": round(full_ms, 1),
        "wall_s": round(wall_total, 1),
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": _oracle_threads(),
                         "kind": "oracle",
                         "sample": f"each step: pool + scores in full, routing + attention on "
                                   f"{int(statistics.mean(sampled))} of {total} query blocks (~{budget:.0f} s), "
                                   f"extrapolated per query block to {full_ms / 1e3:.1f} s per full step"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--density", type=float, default=None, help="override the routing parameter")
    ap.add_argument("--impl", default="psa", choices=["psa", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--dense", action="store_true", help="time psa_dense (density 1, every block exact) instead")
    ap.add_argument("--bwd", action="store_true",
                    help="time the backward (psa_attn_bwd) on the workload's block lists instead")
    ap.add_argument("--hyd", action="store_true",
                    help="time the first-order variant (psa_hyd_stat + psa_attn_hyd) instead of psa_attn")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        reference_arm(args)
    elif args.bwd:
        bwd_arm(args)
    else:
        gpu_arm(args)


if __name__ == "__main__":
    main()
