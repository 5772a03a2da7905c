"""Benchmark: Sol block-sparse attention forward (pool -> route -> attention) on B200.

One step = one full forward pass (sol_pool, sol_route, sol_attn_fwd) of one
synthetic sequence resident in HBM.  With --gpus N (one process per GPU,
launched by torch.distributed.run) every rank runs its own sequence of the
batch (weak scaling, no collective on the data path); the job value is the
total work over the slowest rank's time.

Metric: effective TFLOP/s = 4 * D * H * sum over query rows of the exact keys
they attend (centroid terms excluded) / time per step, with ms per call.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_video_sol_b200 import synth  # noqa: E402

WORKLOADS = {
    "h56_n32768": lambda: synth.h56_sweep(32768),
    "h56_n16384": lambda: synth.h56_sweep(16384),
    "h56_n8192": lambda: synth.h56_sweep(8192),
    "h56_n4096": synth.h56_n4096,
    "h56_joint": synth.h56_joint,
    "tiny": synth.tiny,
}
METRIC = "Sol-Attn ms/call & effective TFLOP/s at H=56,N=32768,d=128 bf16; % roofline"
L2_BYTES = 126 * 2 ** 20


def exact_work(row_ptr: np.ndarray, col_idx: np.ndarray, B: int, H: int, N: int) -> int:
    """sum over query rows of the exact keys they attend (rows x keys), from the CSR."""
    nb = -(-N // 64)
    nrows = np.minimum(np.arange(nb) * 64 + 64, N) - np.arange(nb) * 64
    keys = np.zeros(B * H * nb, np.int64)
    cnt = np.diff(row_ptr)
    rowid = np.repeat(np.arange(B * H * nb), cnt)
    np.add.at(keys, rowid, nrows[col_idx])
    return int((keys.reshape(B * H, nb) * nrows[None, :]).sum())


def route_stats(row_ptr, col_idx, B, H, N, prefix, q128, centroids):
    """Density over video query blocks, union waste of the attention's two-block tiles
    (MMA work over needed work on exact tiles), the exponentials per step, and the
    S tiles the attention kernel issues (each = QK^T and PV of 128 rows x 128 keys):
    ceil(union / 2) exact tiles per query tile, plus one per 128-block centroid chunk
    holding a block that a present half leaves unselected."""
    nb = -(-N // 64)
    rows = B * H * nb
    mask = np.zeros((rows, nb), bool)
    cnt = np.diff(row_ptr)
    mask[np.repeat(np.arange(rows), cnt), col_idx] = True
    mask = mask.reshape(B * H, nb, nb)
    n_dense = -(-prefix // (128 if q128 else 64))
    first_video = min(nb, n_dense * (2 if q128 else 1))
    video = mask[:, first_video:]
    dens_video = float(video.mean()) if video.size else 0.0
    a, b = mask[:, 0::2], mask[:, 1::2]
    present_b = np.arange(a.shape[1]) * 2 + 1 < nb
    b = np.concatenate([b, np.zeros_like(a[:, :a.shape[1] - b.shape[1]])], axis=1)
    uni = (a | b).sum(-1)                                 # [B*H, query tile]
    union = uni.sum()
    needed = a.sum() + b.sum()
    tiles = int(((uni + 1) // 2).sum())
    if centroids:
        unsel = ~a | (~b & present_b[None, :, None])      # a block some present half leaves out
        pad = (-nb) % 128
        unsel = np.concatenate([unsel, np.zeros(unsel.shape[:2] + (pad,), bool)], axis=-1)
        tiles += int(unsel.reshape(unsel.shape[0], unsel.shape[1], -1, 128).any(-1).sum())
    nrows = np.minimum(np.arange(nb) * 64 + 64, N) - np.arange(nb) * 64   # valid rows of each block
    exact_keys = (mask * nrows[None, None, :]).sum(-1)                    # [B*H, query block]
    exps = int((exact_keys * nrows[None, :]).sum())
    if centroids:   # one term per unselected key block
        exps += int(((~mask).sum(-1) * nrows[None, :]).sum())
    return dens_video, float(2 * union / max(needed, 1)), exps, tiles


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return dict(hbm=pk["hbm_gbs"], bf16=pk["bf16_tflops"], bf16_sus=pk.get("bf16_tflops_sustained"),
                    source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, source="fallback")


def source_hash(names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "block_sparse_video_sol_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str):
    """DRAM bytes per launch from a committed ncu summary, if the kernel's source is unchanged."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None, None
    with open(path) as f:
        t = json.load(f).get(kernel)
    if not t or source_hash(t["sources"]) != t["source_sha"]:
        return None, None
    return t["bytes_per_launch"], t.get("note")


class ClockSampler:
    """nvidia-smi samples of SM clock / throttle reasons during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index, self.rows, self.proc = index, [], None
        self.t0, self.t1 = 0.0, float("inf")

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 8:
                self.rows.append((time.perf_counter(), parts))

    def mark(self, start: bool):
        """Host time at the start / end of the timed region: only samples read in
        between (plus one sampling interval for the output's delay) are summarised."""
        if start:
            self.t0 = time.perf_counter()
        else:
            self.t1 = time.perf_counter()

    def __exit__(self, *exc):
        if self.proc:
            time.sleep(0.25)
            self.proc.terminate()
            self.proc.wait(timeout=5)

    def summary(self):
        rows = [r for t, r in self.rows if self.t0 <= t <= self.t1 + 0.05] or [r for _, r in self.rows]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = max(float(r[2]) for r in rows if r[2].replace(".", "").isdigit())
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i].lower() == "active"})
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_min_mhz": min(sm) if sm else None,
                "sm_max_mhz": mx, "reasons": reasons, "samples": len(rows),
                "window": "samples read during the timed region"}


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    return ws, int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0"))


def shard_b_offset(rank: int, w: synth.Workload) -> int:
    """Batch index of this rank's first sequence: rank r runs sequences r*B .. r*B+B-1 of the job."""
    return rank * w.B


def shard_heads(rank: int, world: int, H: int) -> list:
    """Heads of one call that rank r runs when the call is split by head: a contiguous run,
    sizes differing by at most one.  Every stage is per head, so no collective is needed
    when the heads arrive sharded (as after a head-parallel QKV projection)."""
    return list(range(rank * H // world, (rank + 1) * H // world))


def job_reduce(values, device, world: int):
    """Max-over-ranks of the timing entries and sum of the work entry.

    ``values`` = (timed ms, e2e ms, work); returns the same triple for the whole
    job: the slowest rank's times and the total work.  Collective only when
    world > 1 (plumbing, not the data path).
    """
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if world > 1:
        mx, sm = t.clone(), t.clone()
        dist.all_reduce(mx, op=dist.ReduceOp.MAX)
        dist.all_reduce(sm, op=dist.ReduceOp.SUM)
        return mx[0].item(), mx[1].item(), sm[2].item()
    return t[0].item(), t[1].item(), t[2].item()


def oracle_sample(w: synth.Workload, heads, b_offset=0):
    """Time the fp64 oracle on a head subset of the workload; returns (seconds, rows x keys)."""
    from oracle import sol_ref
    q, k, v = (synth.bf16_bits_to_f64(x) for x in synth.generate(w, heads=heads, b_offset=b_offset))
    t0 = time.perf_counter()
    if w.topk_ratio is not None:
        out = sol_ref.sol_forward(q, k, v, prefix=w.prefix, bq=64 if w.compressed else 128,
                                  topk_ratio=w.topk_ratio, compressed=w.compressed,
                                  log_mass_bias_on=int(w.log_mass_bias) == 1, reweight_on=int(w.log_mass_bias) == 2,
                                  reblock=w.reblock, qk_int8=w.qk_int8)
    else:
        out = sol_ref.sol_forward(q, k, v, tau=w.tau, prefix=w.prefix, log_mass_bias_on=int(w.log_mass_bias) == 1,
                                  reweight_on=int(w.log_mass_bias) == 2, reblock=w.reblock, qk_int8=w.qk_int8)
    dt = time.perf_counter() - t0
    nk = sol_ref.block_rows(w.N, 64)
    nq = sol_ref.block_rows(w.N, 128 if (w.topk_ratio is not None and not w.compressed) else 64)
    work = int(sum(((nk[None, :] * out["sel"][b, h]).sum(1) * nq).sum()
                   for b in range(w.B) for h in range(len(heads))))
    return dt, work


def routing_config(w: synth.Workload) -> dict:
    rb = ({"reblock": True} if w.reblock else {}) | ({"qk": "int8 residual keys"} if w.qk_int8 else {})
    if w.topk_ratio is None:
        return {"routing": "threshold", **rb}
    if w.compressed:
        return {"routing": "topk+compressed", "topk_ratio": w.topk_ratio, "q_block": 64, **rb}
    return {"routing": "topk", "topk_ratio": w.topk_ratio, "q_block": 128, **rb}


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [os.cpu_count() or 1])
    except Exception:
        return os.cpu_count() or 1


def run_reference(args, w):
    ws, rank, _ = dist_env()
    if rank != 0:
        return
    heads = list(range(min(args.ref_heads or 1, w.H)))
    for _ in range(args.warmup):
        oracle_sample(w, heads[:1])
    times, works = [], []
    for _ in range(args.steps):
        dt, work = oracle_sample(w, heads)
        times.append(dt)
        works.append(work)
    sec = float(np.mean(times))
    # The whole call (all heads) would take minutes per step on the host, so each step runs
    # a head sample; ms_per_step is that sample's time scaled to all heads (an extrapolation,
    # labelled in the line), while value is a plain rate measured on the sample itself.
    ms_call = sec * 1e3 * w.H / len(heads)
    val = 4 * w.D * float(np.mean(works)) / sec / 1e12
    sample = f"{len(heads)} of {w.H} heads of {w.name} per step (full pool/route/attention of those heads)"
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_call,
            "ms_per_step_basis": (f"extrapolated: {sec * 1e3:.0f} ms measured per step on {len(heads)} of "
                                  f"{w.H} heads, x {w.H / len(heads):g}"),
            "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "D": w.D, "tau": w.tau,
                       "prefix": w.prefix, "log_mass_bias": w.log_mass_bias, **routing_config(w)},
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


def run_ours(args, w):
    import torch
    import torch.distributed as dist
    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", device_id=dev, timeout=__import__("datetime").timedelta(seconds=300))
    from block_sparse_video_sol_b200 import sol

    # this rank's work (pinned host copies for e2e): batch element `rank` of a world-size batch,
    # or with --shard heads its run of heads of the one call
    by_heads = args.shard == "heads"
    heads = shard_heads(rank, world, w.H) if by_heads else None
    Hr = len(heads) if by_heads else w.H
    shape = (w.B, w.N, Hr, w.D)
    host = [torch.empty(shape, dtype=torch.bfloat16).pin_memory() for _ in range(3)]
    synth.generate(w, heads=heads, out=tuple(h.view(torch.int16).numpy().view(np.uint16) for h in host),
                   b_offset=0 if by_heads else shard_b_offset(rank, w))
    q, k, v = (h.to(dev) for h in host)
    p = sol.make_params(w.B, w.N, Hr, w.D, tau=w.tau, prefix_len=w.prefix, log_mass_bias=w.log_mass_bias,
                        topk_ratio=w.topk_ratio, compressed=w.compressed, qk_int8=w.qk_int8)
    stream = torch.cuda.current_stream()
    # pool (+ anchor, K/V; + residual key codes), route + scan + compact, plan + attention
    launches_per_step = (3 if w.log_mass_bias else 1) + (1 if w.qk_int8 else 0) + 3 + 2
    if w.reblock:
        # the adaptive partition, then the Sol passes on head-major copies in its order
        rb = sol.alloc_reblock(p, dev)
        o_out = torch.empty_like(q)
        rp_, rq, rk, rv, buf = rb.hm, rb.qp, rb.kp, rb.vp, rb.buf
        launches_per_step += 4 + sol.reblock_levels(w.N - 64 * (-(-w.prefix // 64))) + 4   # partition, 3 gathers + scatter
    else:
        buf = sol.alloc_buffers(p, dev)
        rp_, rq, rk, rv = p, q, k, v
    n_ev = 7 if w.reblock else 4

    def step(ev=None):
        def mark(i):
            if ev:
                ev[i].record()
        mark(0)
        j = 0
        if w.reblock:
            sol.sol_reblock(p, q, k, rb.ws, rb.perm)
            mark(1)
            for x, xp in ((q, rb.qp), (k, rb.kp), (v, rb.vp)):
                sol.sol_gather_rows(p, rb.perm, x, xp)
            mark(2)
            j = 2
        sol.sol_pool(rp_, rq, rk, rv, buf.ws)
        mark(j + 1)
        sol.sol_route(rp_, buf.ws, buf.row_ptr, buf.col_idx)
        mark(j + 2)
        sol.sol_attn_fwd(rp_, rq, rk, rv, buf.ws, buf.row_ptr, buf.col_idx, buf.o)
        mark(j + 3)
        if w.reblock:
            sol.sol_scatter_rows(p, rb.perm, buf.o, o_out)
            mark(6)

    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if args.flush_l2 else None

    for _ in range(args.warmup):
        step()
    sol.sol_last_device_status()
    rp = buf.row_ptr.cpu().numpy().astype(np.int64)
    ci = buf.col_idx[:int(rp[-1])].cpu().numpy().astype(np.int64)
    work = exact_work(rp, ci, w.B, Hr, w.N)
    nb = -(-w.N // 64)
    density = rp[-1] / (w.B * Hr * nb * nb)
    sla = w.topk_ratio is not None and not w.compressed
    dens_video, union_waste, exps, tiles = route_stats(rp, ci, w.B, Hr, w.N, w.prefix, sla, not sla)
    issued_flop = 4.0 * 128 * 128 * w.D * tiles   # what the tensor cores execute (QK^T + PV per S tile)
    flop = 4.0 * w.D * work   # work is summed over every (b, h)
    cent_flop = 4.0 * w.D * w.B * Hr * w.N * nb

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        clocks.mark(True)
        t0.record()
        for s in range(args.steps):
            if flush is not None:
                flush.zero_()   # 256 MB through L2 before each step (outside the per-kernel events)
            step(evs[s])
        t1.record()
        torch.cuda.synchronize()
        clocks.mark(False)
    if world > 1:
        dist.barrier()
    sol.sol_last_device_status()
    total_ms = t0.elapsed_time(t1)
    per = np.array([[e[i].elapsed_time(e[i + 1]) for i in range(n_ev - 1)] for e in evs]).mean(axis=0)
    if w.reblock:
        reblock_ms, gather_ms, pool_ms, route_ms, attn_ms, scatter_ms = per
    else:
        pool_ms, route_ms, attn_ms = per

    # e2e through the C ABI's host-buffer entry point: every step copies q, k, v from pinned host
    # memory, runs the forward pass and copies o back (pipelined over head chunks inside the call)
    o_host = torch.empty(shape, dtype=torch.bfloat16).pin_memory()
    staging = None if w.reblock else torch.empty(sol.sol_host_staging_bytes(p), dtype=torch.uint8, device=dev)
    h2d = 3 * q.numel() * q.element_size()
    d2h = o_host.numel() * o_host.element_size()
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    def e2e_step():
        if w.reblock:   # pinned host -> device copies, the reblocked pass, the output back
            for hsrc, dsts in zip(host, (q, k, v)):
                dsts.copy_(hsrc, non_blocking=True)
            sol.forward_reblocked(p, q, k, v, o_out, rb)
            o_host.copy_(o_out, non_blocking=True)
        else:
            sol.sol_forward_host(p, host[0], host[1], host[2], o_host, staging)
    e2e_step()   # warm-up (creates the copy streams)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(e2e_steps):
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    del staging

    total_ms, e2e_ms, flop_all = job_reduce((total_ms, e2e_ms, flop), dev, world)
    if rank == 0:
        peaks = read_peaks()
        ms_step = total_ms / args.steps
        value = flop_all / (ms_step * 1e-3) / 1e12
        attn_tf = flop / (attn_ms * 1e-3) / 1e12
        issued_tf = issued_flop / (attn_ms * 1e-3) / 1e12
        traffic, tnote = profiled_traffic("sol_attn_fwd")
        in_bytes = 3 * w.B * w.N * Hr * w.D * 2
        # route: fp32 centroids in, bitmap + counts + CSR out (not its bound: it is ALU work)
        route_bytes = 2 * w.B * Hr * nb * w.D * 4 + w.B * Hr * nb * (4 * (-(-nb // 32)) + 8) + 4 * int(rp[-1])
        pool_bytes = (2 if sla else 3) * w.B * w.N * Hr * w.D * 2   # the SLA variant pools no V
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "strong" if by_heads else "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "D": w.D, "tau": w.tau,
                       "prefix": w.prefix, "log_mass_bias": w.log_mass_bias, **routing_config(w),
                       "global_batch": w.B if by_heads else w.B * world,
                       "parallelism": (f"heads split {world} ways ({Hr} of {w.H} heads on rank 0), no collective"
                                       if by_heads else f"dp{world} (one sequence per GPU)"),
                       "l2": (f"inputs larger than L2 ({in_bytes / 1e9:.2f} GB per step vs 126 MB)"
                              + (", 256 MB written before each step" if args.flush_l2 else ", no flush"))},
            # The attention kernel runs for milliseconds back to back under the 1 kW cap
            # (sw_power_cap active, SM clock ~1.4 GHz in its phase trace), the regime of the
            # sustained bf16 figure; the burst fraction is kept beside it.
            "roofline": {"kernel": "sol_attn_fwd", "bound": "tensor", "achieved": attn_tf,
                         "peak": peaks["bf16_sus"], "unit": "TFLOP/s", "frac": attn_tf / peaks["bf16_sus"],
                         "peak_source": f"{peaks['source']} bf16 sustained (a kernel timed inside a long run "
                                        "under the power cap)",
                         "frac_of_burst": attn_tf / peaks["bf16"],
                         "issued_mma_tflops": issued_tf, "issued_frac": issued_tf / peaks["bf16_sus"],
                         "issued_note": "tensor-core work executed: 4*128*128*D per S tile (exact tiles = "
                                        "ceil(union/2) per query tile, plus centroid tiles); achieved counts "
                                        "only the exact keys the rows need",
                         "traffic": traffic, "traffic_note": tnote},
            "kernels": {
                "sol_pool": {"ms": pool_ms, "GB/s": pool_bytes / (pool_ms * 1e-3) / 1e9,
                             "frac_hbm": pool_bytes / (pool_ms * 1e-3) / 1e9 / peaks["hbm"]},
                "sol_route": {"ms": route_ms,
                              "TFLOP/s_fp32": 2.0 * w.B * Hr * nb * nb * w.D / (route_ms * 1e-3) / 1e12,
                              "GB/s": route_bytes / (route_ms * 1e-3) / 1e9},
                "sol_attn_fwd": {"ms": attn_ms, "TFLOP/s_effective": attn_tf,
                                 "TFLOP/s_incl_centroids": (flop + cent_flop) / (attn_ms * 1e-3) / 1e12},
                **({"sol_reblock": {"ms": reblock_ms},
                    "sol_gather_rows": {"ms": gather_ms, "GB/s": 2 * in_bytes / (gather_ms * 1e-3) / 1e9},
                    "sol_scatter_rows": {"ms": scatter_ms,
                                         "GB/s": 2 * in_bytes / 3 / (scatter_ms * 1e-3) / 1e9}} if w.reblock else {}),
            },
            "density": float(density), "density_video_blocks": dens_video,
            "union_waste": union_waste, "exponentials_per_step": exps,
            "exact_flop_per_step": flop, "clocks": clocks.summary(),
            "e2e": {"value": flop_all / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                    "api": ("pinned host copies + sol_reblock, gathers, pool/route/attention, scatter"
                            if w.reblock else "sol_forward_host, pinned host buffers, 4-head chunks")},
            "gpu_launches": launches_per_step * args.steps,
        }
        if world == 1 and not args.no_cpu_baseline:
            heads = list(range(min(args.ref_heads or 6, w.H)))
            dt, swork = oracle_sample(w, heads)
            line["cpu_baseline"] = {"value": 4 * w.D * swork / dt / 1e12, "unit": "TFLOP/s", "cores": cpu_threads(),
                                    "kind": "oracle",
                                    "sample": f"{len(heads)} of {w.H} heads of {w.name} ({dt:.1f} s)"}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="h56_n32768", choices=sorted(WORKLOADS))
    ap.add_argument("--tau", type=float, default=None)
    ap.add_argument("--log-mass-bias", action="store_true", help="centroid terms with the log-mass bias")
    ap.add_argument("--reweight", action="store_true",
                    help="anchor-weighted key/value summaries with the log-mass bias")
    ap.add_argument("--topk-ratio", type=float, default=None,
                    help="Top-K routing (the SLA variant: 128-row query blocks, no centroid terms)")
    ap.add_argument("--compressed", action="store_true",
                    help="with --topk-ratio: keep the compressed branch (64-row blocks, sink, centroid terms)")
    ap.add_argument("--qk-int8", action="store_true",
                    help="exact logits from INT8 query codes and INT8 per-block residual key codes")
    ap.add_argument("--reblock", action="store_true",
                    help="order the rows by the adaptive partition first (sol_reblock, gathers, scatter)")
    ap.add_argument("--shard", default="batch", choices=["batch", "heads"],
                    help="with --gpus N: one sequence per GPU (batch, weak scaling) or the heads of one "
                         "call split over the GPUs (heads, strong scaling)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-heads", type=int, default=None,
                    help="heads per oracle sample (default: 1 for --impl reference steps, 6 for cpu_baseline)")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--flush-l2", action="store_true",
                    help="write 256 MB before each timed step (ms_per_step then includes it; the per-kernel times do not)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = WORKLOADS[args.workload]()
    if args.log_mass_bias and args.reweight:
        ap.error("--log-mass-bias and --reweight are exclusive")
    mode = 2 if args.reweight else int(args.log_mass_bias)
    if args.topk_ratio is not None and (args.tau is not None or (mode and not args.compressed)):
        ap.error("--topk-ratio takes no tau, and centroid options only with --compressed")
    if args.compressed and args.topk_ratio is None:
        ap.error("--compressed needs --topk-ratio")
    if args.tau is not None or mode or args.topk_ratio is not None or args.reblock or args.qk_int8:
        import dataclasses
        w = dataclasses.replace(w, tau=w.tau if args.tau is None else args.tau, log_mass_bias=mode,
                                topk_ratio=args.topk_ratio, compressed=args.compressed, reblock=args.reblock,
                                qk_int8=args.qk_int8,
                                name=w.name + (f"_tau{args.tau:g}" if args.tau is not None else "")
                                     + synth.mode_suffix(mode)
                                     + (f"_topk{args.topk_ratio:g}" if args.topk_ratio is not None else "")
                                     + ("_compressed" if args.compressed else "")
                                     + ("_reblock" if args.reblock else "")
                                     + ("_int8" if args.qk_int8 else ""))
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
