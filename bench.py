"""Benchmark of the Sol-Attn forward (pool + fused forward) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload wan_75k] [--beta B | --density D]

One step = one pass of the whole hot path over one batch of synthetic input:
solattn_pool (block means, key mean and covariance) followed by
solattn_forward (on-the-fly routing, exact kept blocks, zeroth-order correction)
at the Wan2.1-14B-like 720p shape: 75,600 tokens (21x45x80 latent grid), 40
heads, d = 128, beta calibrated for a 15 % mean kept-block density.

Prints one JSON line. value = kept-block TFLOP/s of the whole step (kept-block
FLOPs = 4 d n_i n_j summed over kept (i, j) pairs), whole job over all ranks.
Multi-GPU (torchrun): every rank runs its own copy of the workload on its own
GPU (heads are independent; no collective on the data path; weak scaling), or
with --shard heads its contiguous share of the (batch, head) pairs (strong
scaling, the survey's head partition); timing is the max over ranks and value
counts every rank's work.

e2e = the same step through solattn_forward_host: q, k, v in pinned host
memory, out, lse and density back to pinned host memory, the copies inside the
timed region (overlapped with the computation of other head chunks).

--impl reference runs the CPU oracle (the only other implementation of this
method available here) on the host cores, on a bounded sample of the same
workload per step.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_attention_cov_b200.inputs import WORKLOADS, make_qkv  # noqa: E402

METRIC = "Sol-Attn fwd ms & kept-block TFLOP/s (% BF16 peak) at 75.6K tokens, 1×B200"
UNIT = "TFLOP/s (kept-block)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return dict(FALLBACK_PEAKS)


def load_beta(workload, target=None):
    p = os.path.join(ROOT, "tests", "golden", "calibrated_beta.json")
    d = json.load(open(p))[workload]
    if target is None:
        return d["beta"], d
    return d["targets"][f"{target:.2f}"]["beta"], d


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock/throttle sampling in the background during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []      # (arrival time, csv line)
        self.window = None   # (start, end) of the timed region, monotonic seconds

    def mark(self, start, end):
        self.window = (start, end)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        lines = [ln for t, ln in self.lines if self.window is None or self.window[0] <= t <= self.window[1]]
        for ln in lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm), "samples_total": len(self.lines),
                "window": "samples taken between the first and the last timed step"}


# --------------------------------------------------------------------------- traffic record
TRAFFIC_RECORD = os.path.join(ROOT, "profiles", "solattn_fwd_pp_kernel.traffic.txt")
FWD_SOURCES = [os.path.join(ROOT, "block_sparse_attention_cov_b200", "csrc", f)
               for f in ("forward_pp.cu", "fwd_common.cuh", "ptx.cuh")]


def fwd_source_digest():
    """sha256 over the two-group kernel's sources (the kernel and the headers
    it compiles in), in a fixed order."""
    h = hashlib.sha256()
    for f in FWD_SOURCES:
        h.update(open(f, "rb").read())
    return h.hexdigest()


def fwd_traffic(heads):
    """DRAM bytes (read + write) of one forward launch at `heads` heads, from the
    committed ncu record of a small capture scaled by the units processed; None
    when the record is missing or was taken on another version of the kernel
    source (its sha256 over forward_pp.cu, fwd_common.cuh and ptx.cuh no
    longer matches)."""
    try:
        rec = dict(ln.split(":", 1) for ln in open(TRAFFIC_RECORD).read().splitlines() if ":" in ln)
        rec = {k.strip(): v.strip() for k, v in rec.items()}
        digest = fwd_source_digest()
        if rec.get("source_sha256") != digest:
            return None
        per_head = (float(rec["dram_bytes_read"]) + float(rec["dram_bytes_write"])) / float(rec["heads"])
        return per_head * heads
    except (OSError, KeyError, ValueError):
        return None


# --------------------------------------------------------------------------- helpers
def kept_flops(stats, dens, beta, N, d, rule="threshold", n_forced=0):
    """Algorithmic kept-block FLOPs: 4 d n_i sum_{j in S_i} n_j over every (b, h, i).
    Only the last key block can be partial; with the threshold rule whether row
    i keeps it is recomputed from the pooled statistics (bookkeeping only); with
    the top-k / top-p rules it is counted as a full block (an overcount below
    1e-4 of the work at 75.6K tokens)."""
    nb = math.ceil(N / 64)
    n_last = N - 64 * (nb - 1)
    n_i = torch.full((nb,), 64.0, device=dens.device, dtype=torch.float64)
    n_i[-1] = n_last
    cols = 64.0 * dens.double()
    if n_last < 64 and rule == "threshold" and n_forced < nb:
        qbar, kbar = stats.view("qbar").double(), stats.view("kbar").double()
        s = 1.0 / math.sqrt(d)
        sh = s * (qbar @ kbar[..., -1, :].unsqueeze(-1)).squeeze(-1)
        mu = s * (qbar @ stats.view("kmean").double().unsqueeze(-1)).squeeze(-1)
        sigma = s * ((qbar @ stats.view("kcov").double()) * qbar).sum(-1).clamp_min(0.0).sqrt()
        tau = torch.where(sigma == 0, torch.full_like(mu, math.inf), mu + beta * sigma)
        cols = cols - (64 - n_last) * (sh > tau).double()
    return float((4.0 * d * n_i * cols).sum().item())


def dense_flops(B, H, N, d):
    return 4.0 * d * N * N * B * H


def union_flops(stats, beta, N, d, n_forced=0):
    """Tensor-core work of the threshold rule's 128-row units (bookkeeping on
    the pooled statistics): a unit multiplies every key block kept by either of
    its two query blocks for all 128 rows, 4 d 128 64 FLOPs per block (QK^T and
    PV). Its ratio to the kept-block FLOPs is what the tensor pipe does per
    useful FLOP."""
    qbar, kbar = stats.view("qbar").double(), stats.view("kbar").double()
    B, H, nb, _ = qbar.shape
    s = 1.0 / math.sqrt(d)
    mu = s * (qbar @ stats.view("kmean").double().unsqueeze(-1)).squeeze(-1)
    sigma = s * ((qbar @ stats.view("kcov").double()) * qbar).sum(-1).clamp_min(0.0).sqrt()
    tau = torch.where(sigma == 0, torch.full_like(mu, math.inf), mu + beta * sigma)
    blocks = 0.0
    for b in range(B):
        for h in range(H):
            mask = (s * (qbar[b, h] @ kbar[b, h].T)) > tau[b, h].unsqueeze(-1)
            if n_forced:
                mask[:, :n_forced] = True
            if nb % 2:
                mask = torch.cat([mask, torch.zeros_like(mask[:1])])
            blocks += float((mask[0::2] | mask[1::2]).sum().item())
    return 4.0 * d * 128 * 64 * blocks


def density_stats(dens, nb):
    """Distribution of the per-row kept fraction |S_i| / N_b over every (b, h, i)."""
    x = dens.double().flatten().cpu().numpy() / nb
    return {"mean": float(x.mean()), "std": float(x.std()), "min": float(x.min()), "max": float(x.max()),
            "p5": float(np.percentile(x, 5)), "p50": float(np.percentile(x, 50)), "p95": float(np.percentile(x, 95))}


def pool_bytes(B, H, N, d):
    nb = math.ceil(N / 64)
    return 3 * B * H * N * d * 2 + (3 * nb * d + d + d * d) * B * H * 4 + 2 * nb * d * B * H * 2


def cpu_threads():
    """BLAS threads numpy uses (the oracle's matrix products)."""
    try:
        from threadpoolctl import threadpool_info

        n = [x.get("num_threads", 1) for x in threadpool_info() if x.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:  # noqa: BLE001
        return 1


def cpu_info():
    """Cores this process may run on, the CPU model and the BLAS threads."""
    model = "unknown"
    try:
        for ln in open("/proc/cpuinfo"):
            if ln.startswith("model name"):
                model = ln.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return {"cores": len(os.sched_getaffinity(0)), "cpu_model": model, "blas_threads": cpu_threads()}


SAMPLE_BLOCKS = 32  # per head: the first and last query block and 30 seeded random ones


def sample_rows(nb, head, seed=0):
    """The stratified sample of query blocks of one head."""
    rng = np.random.default_rng(seed * 100003 + head)
    inner = np.arange(1, nb - 1)  # the random ones are drawn between the first and the last
    extra = rng.choice(inner, min(len(inner), SAMPLE_BLOCKS - 2), replace=False).tolist() if len(inner) else []
    return sorted({0, nb - 1, *extra})


def row_kept_flops(mask, N, d):
    """Kept-block FLOPs of every query block i: 4 d n_i sum_{j in S_i} n_j."""
    from oracle import solattn_oracle as orc

    n = orc.block_counts(N).astype(np.float64)
    return 4.0 * d * n * (mask.astype(np.float64) @ n)


def oracle_head_sample(q, k, v, beta, head_pos, head_id, seed=0, out_gpu=None, lse_gpu=None):
    """The oracle (fp32 working precision, multithreaded BLAS) on the stratified
    sample of one head. Returns (seconds, kept FLOPs of the sample, error sums):
    with the GPU's out / lse of this head ([N, d], [N] numpy), the squared
    error and squared norm of out over the sampled rows, its max abs error and
    the max lse error (outside the timed call)."""
    from oracle import solattn_oracle as orc

    N, d = q.shape[2], q.shape[3]
    nb = math.ceil(N / 64)
    rows = sample_rows(nb, head_id, seed)
    qq, kk, vv = (x[0, head_pos].float().numpy() for x in (q, k, v))
    t0 = time.perf_counter()
    o, l, _ = orc.attend(qq, kk, vv, beta, rows=rows, dtype=np.float32)
    secs = time.perf_counter() - t0
    r = orc.route(qq, kk, beta, dtype=np.float32)
    errs = None
    if out_gpu is not None:
        tok = np.concatenate([np.arange(64 * i, min(64 * i + 64, N)) for i in rows])
        e = out_gpu[tok].astype(np.float64) - o[tok].astype(np.float64)
        errs = (float((e * e).sum()), float((o[tok].astype(np.float64) ** 2).sum()), float(np.abs(e).max()),
                float(np.abs(lse_gpu[tok].astype(np.float64) - l[tok]).max()))
    return secs, float(row_kept_flops(r["mask"], N, d)[rows].sum()), errs


def routing_oracle(q, k, beta, dens_gpu):
    """The routing oracle (fp64) over every query block of every head: time,
    near ties (|s_hat - tau| <= 1e-4), query blocks whose GPU kept count
    differs from the oracle's by more than their near ties, and the kept FLOPs
    of every row (for the extrapolation of the CPU time)."""
    from oracle import solattn_oracle as orc

    B, H, N, d = q.shape
    secs, ties, bad, flops = 0.0, 0, 0, []
    for h in range(H):
        qq, kk = q[0, h].double().numpy(), k[0, h].double().numpy()
        t0 = time.perf_counter()
        r = orc.route(qq, kk, beta)
        secs += time.perf_counter() - t0
        near = (np.abs(r["shat"] - r["tau"][:, None]) <= 1e-4).sum(1)
        ties += int(near.sum())
        bad += int((np.abs(dens_gpu[0, h].astype(np.int64) - r["density"]) > near).sum())
        flops.append(row_kept_flops(r["mask"], N, d))
    return secs, ties, bad, np.stack(flops)


def cpu_baseline_leg(q, k, v, beta, dens_gpu, seed=0, out_gpu=None, lse_gpu=None):
    """CPU baseline as the oracle stands: fp32 multithreaded BLAS on the
    stratified sample of every head (first, last, 30 random query blocks),
    with the full forward's CPU time extrapolated from it by kept FLOPs; the
    routing oracle over every block (also the near-tie and kept-count parity
    of the GPU run); the tiny and mid workloads timed in full."""
    from oracle import solattn_oracle as orc

    B, H, N, d = q.shape
    nb = math.ceil(N / 64)
    r_secs, ties, bad, row_flops = routing_oracle(q, k, beta, dens_gpu)
    s_secs, s_flops = 0.0, 0.0
    err2 = ref2 = emax = lmax = 0.0
    for h in range(H):
        t, f, errs = oracle_head_sample(q, k, v, beta, h, h, seed,
                                        None if out_gpu is None else out_gpu[0, h],
                                        None if lse_gpu is None else lse_gpu[0, h])
        s_secs += t
        s_flops += f
        if errs is not None:
            err2, ref2 = err2 + errs[0], ref2 + errs[1]
            emax, lmax = max(emax, errs[2]), max(lmax, errs[3])
    total_flops = float(row_flops.sum())
    full = {}
    for name, wl_beta in (("tiny", 1.0), ("mid", 1.0)):
        wl = WORKLOADS[name]
        qt, kt, vt = make_qkv(wl, seed=0)
        t0 = time.perf_counter()
        for h in range(wl.H):
            orc.attend(*(x[0, h].float().numpy() for x in (qt, kt, vt)), wl_beta, dtype=np.float32)
        full[name] = {"seconds": round(time.perf_counter() - t0, 3), "beta": wl_beta, "heads": wl.H, "N": wl.N}
    info = cpu_info()
    return {
        "value": s_flops / s_secs / 1e12, "unit": UNIT, "cores": info["cores"], "kind": "oracle",
        "sample": f"oracle fp32, {H} heads x {SAMPLE_BLOCKS} query blocks (first, last, 30 seeded random); "
                  f"{s_secs:.1f} s of CPU time",
        "cpu_model": info["cpu_model"], "blas_threads": info["blas_threads"],
        "sample_seconds": s_secs, "sample_kept_tflop": s_flops / 1e12,
        "full_forward_seconds_extrapolated": s_secs * total_flops / s_flops,
        "routing_oracle_seconds_all_blocks": r_secs,
        "full_runs": full,
    }, {"near_ties": ties, "density_mismatch_rows": bad, "rows": int(H * nb),
        "output_error": None if out_gpu is None else {
            "rel_l2": math.sqrt(err2 / ref2), "max_abs": emax, "max_lse": lmax,
            "against": f"oracle fp32 on the stratified sample ({H} heads x {SAMPLE_BLOCKS} query blocks)"}}


def max_over_ranks(values, world, device):
    """Element-wise max of per-rank timings (ms) over all ranks; identity for
    one rank. Every rank must call it with the same number of values."""
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_value(flops_per_rank, ms, world):
    """Whole-job throughput in TFLOP/s: every rank processes its own copy of the
    workload (weak scaling), the job takes the slowest rank's time."""
    return world * flops_per_rank / (ms * 1e-3) / 1e12


def sum_over_ranks(value, world, device):
    """Sum of one per-rank number over all ranks; identity for one rank."""
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


def head_slice(B, H, rank, world):
    """(b, h) pairs of this rank when the B*H independent pairs are split over
    the ranks: contiguous, balanced (sizes differ by at most one), every pair
    on exactly one rank."""
    pairs = [(b, h) for b in range(B) for h in range(H)]
    lo, hi = len(pairs) * rank // world, len(pairs) * (rank + 1) // world
    return pairs[lo:hi]


# --------------------------------------------------------------------------- reference arm
def run_reference(args, rank, world):
    """The oracle as it stands (fp32 working precision, multithreaded BLAS) on
    the host cores. Step s times the stratified sample of head s % H (first,
    last and 30 seeded random query blocks): the same per-head samples the
    cpu_baseline leg of the GPU arm times for every head."""
    if rank != 0:
        return
    wl = WORKLOADS[args.workload]
    beta = args.beta if args.beta is not None else load_beta(args.workload, args.density)[0]
    heads = sorted({s_ % wl.H for s_ in range(args.warmup + args.steps)})
    q, k, v = make_qkv(wl, 0, heads=[(0, h) for h in heads])
    pos = {h: i for i, h in enumerate(heads)}
    times, flops = [], 0.0
    for step in range(args.warmup + args.steps):
        h = step % wl.H
        t, f, _ = oracle_head_sample(q, k, v, beta, pos[h], h)
        if step >= args.warmup:
            times.append(t)
            flops += f
    secs = sum(times)
    val = flops / secs / 1e12
    info = cpu_info()
    desc = (f"oracle fp32 per step: {SAMPLE_BLOCKS} query blocks (first, last, 30 seeded random) of head "
            f"step % {wl.H}; {secs:.1f} s of CPU time over {args.steps} steps")
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": args.workload, "B": wl.B, "H": wl.H, "N": wl.N, "d": wl.d, "beta": beta,
                   "sample": desc},
        "cpu_baseline": {"value": val, "unit": UNIT, "cores": info["cores"], "kind": "oracle", "sample": desc,
                         "cpu_model": info["cpu_model"], "blas_threads": info["blas_threads"]},
        "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank):
    import block_sparse_attention_cov_b200 as sa
    from block_sparse_attention_cov_b200 import _lib

    _lib.lib()  # fail loudly if the extension is missing
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = WORKLOADS[args.workload]
    if args.heads:
        wl = dataclasses.replace(wl, H=args.heads)
    beta = args.beta if args.beta is not None else load_beta(args.workload, args.density)[0]
    B, H, N, d = wl.B, wl.H, wl.N, wl.d
    peaks = load_peaks()

    sharded = args.shard == "heads" and world > 1
    if sharded:
        # strong scaling: this rank's contiguous share of the (b, h) pairs,
        # attended as one batch of heads (the pairs are independent)
        mine = head_slice(B, H, rank, world)
        if not mine:
            raise SystemExit(f"--shard heads needs at least {world} (batch, head) pairs")
        q_h, k_h, v_h = make_qkv(wl, seed=0, heads=mine)
        B, H = 1, len(mine)
    else:
        q_h, k_h, v_h = make_qkv(wl, seed=0)
    q, k, v = (x.to(dev) for x in (q_h, k_h, v_h))
    stream = torch.cuda.current_stream()
    ws = sa.workspace(dev)
    stats = sa.pool(q, k, v)
    out = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    nb = math.ceil(N / 64)
    dens = torch.empty((B, H, nb), dtype=torch.int32, device=dev)

    rule_kw = {"rule": args.rule, "topk": args.topk, "topp": args.topp, "n_forced": args.n_forced,
               "correction": args.correction}

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        sa.pool(q, k, v, stats)
        if ev is not None:
            ev[1].record(stream)
        sa.forward(q, k, v, stats, beta, out=out, lse=lse, density=dens, ws=ws, **rule_kw)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if sa.status(ws) != 0:
        raise RuntimeError(f"device status {sa.status(ws)} after warm-up")
    kflops = kept_flops(stats, dens, beta, N, d, args.rule, args.n_forced)
    mean_density = float(dens.double().mean().item()) / nb
    # work of the whole job: every rank's own share (sharded) or copy (replicas)
    job_kflops = sum_over_ranks(kflops, world, dev) if sharded else world * kflops
    # the union of each unit's two kept sets: what the tensor pipe multiplies
    uflops = union_flops(stats, beta, N, d, args.n_forced) if args.rule == "threshold" else None
    job_uflops = None if uflops is None else (sum_over_ranks(uflops, world, dev) if sharded else world * uflops)

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    cvd = os.environ.get("CUDA_VISIBLE_DEVICES")
    clocks = ClockSampler(cvd.split(",")[local_rank] if cvd else str(local_rank))
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    w0 = time.monotonic()
    t_start.record(stream)
    for s in range(args.steps):
        step(evs[s])
    t_end.record(stream)
    torch.cuda.synchronize()
    clocks.mark(w0, time.monotonic())
    clk = clocks.stop()
    if world > 1:
        torch.distributed.barrier()
    st = sa.status(ws)
    if st != 0:
        raise RuntimeError(f"device status {st} in the timed region")
    ms_total = t_start.elapsed_time(t_end)
    pool_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    fwd_ms = float(np.mean([e[1].elapsed_time(e[2]) for e in evs]))
    ms_total, pool_ms, fwd_ms = max_over_ranks([ms_total, pool_ms, fwd_ms], world, dev)
    ms_step = ms_total / args.steps

    # dense comparison path on the same inputs
    dense_ms = None
    if not args.skip_dense:
        sa.dense(q, k, v, out=out, lse=lse, ws=ws)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        reps = 2
        for _ in range(reps):
            sa.dense(q, k, v, out=out, lse=lse, ws=ws)
        e1.record(stream)
        torch.cuda.synchronize()
        dense_ms = e0.elapsed_time(e1) / reps
        step()  # restore the Sol-Attn outputs
        torch.cuda.synchronize()

    # end to end through the C ABI's host-buffer entry point (solattn_forward_host):
    # pinned host inputs in, pinned host outputs back, copies overlapped with
    # the pool + forward of other head chunks
    e2e = None
    if not args.skip_e2e and args.rule == "threshold" and args.n_forced == 0 and args.correction == "block":
        qp, kp, vp = (x.pin_memory() for x in (q_h, k_h, v_h))
        out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        lse_h = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
        dens_h = torch.empty(dens.shape, dtype=dens.dtype).pin_memory()
        scratch = sa.host_scratch(B, H, N, d, device=dev)

        def e2e_step():
            sa.forward_host(qp, kp, vp, beta, out_h, lse_h, dens_h, scratch=scratch)

        e2e_step()
        torch.cuda.synchronize()
        if sa.status(scratch) != 0:
            raise RuntimeError(f"device status {sa.status(scratch)} in the end-to-end path")
        reps = max(1, min(args.steps, 5))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(reps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        if sa.status(scratch) != 0:
            raise RuntimeError(f"device status {sa.status(scratch)} in the end-to-end path")
        if not torch.equal(dens_h, dens.cpu()):
            raise RuntimeError("end-to-end density differs from the device path")
        (e2e_ms,) = max_over_ranks([e0.elapsed_time(e1) / reps], world, dev)
        h2d = sum(x.numel() * x.element_size() for x in (qp, kp, vp))
        d2h = sum(x.numel() * x.element_size() for x in (out_h, lse_h, dens_h))
        e2e = {"value": job_kflops / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
               "path": "solattn_forward_host: pinned host buffers, head chunks copied in / attended / "
                       "copied back on three streams"}
        del scratch

    if rank != 0:
        return

    fwd_tflops = job_kflops / world / (fwd_ms * 1e-3) / 1e12  # per GPU
    # The timed loop runs the kernel back to back; once it lasts a second or
    # more the GPU sits at its power cap, so the sustained GEMM figure (taken
    # the same way) is the like-for-like denominator, else the burst one.
    if ms_total >= 1000.0 and peaks.get("bf16_tflops_sustained"):
        peak_tc, peak_kind = peaks["bf16_tflops_sustained"], " (bf16 sustained: %.1f s timed loop)" % (ms_total / 1e3)
    else:
        peak_tc, peak_kind = peaks["bf16_tflops"], " (bf16 burst)"
    pbytes = pool_bytes(B, H, N, d)
    pool_gbs = pbytes / (pool_ms * 1e-3) / 1e9
    # the threshold rule with the block-level correction runs on the two-group
    # kernel (whose ncu traffic record bench reports); the other variants on
    # the one-unit kernel
    two_group = args.rule == "threshold" and args.correction == "block"
    cpu, parity = None, None
    if not args.skip_cpu and world == 1 and args.rule == "threshold" and not args.n_forced:
        cpu, parity = cpu_baseline_leg(q_h, k_h, v_h, beta, dens.cpu().numpy(), out_gpu=out.float().cpu().numpy(),
                                       lse_gpu=lse.cpu().numpy())
    line = {
        "metric": METRIC,
        "value": job_kflops / (ms_step * 1e-3) / 1e12,
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "strong" if sharded else "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded random-Fourier-feature Q/K, Gaussian V; bf16)",
        "config": {
            "workload": args.workload, "B": wl.B, "H": wl.H, "N": N, "d": d, "grid": list(wl.grid), "beta": beta,
            "rule": args.rule, **({"topk": args.topk} if args.rule == "topk" else {}),
            **({"topp": args.topp} if args.rule == "topp" else {}),
            **({"n_forced": args.n_forced} if args.n_forced else {}),
            **({"correction": args.correction} if args.correction != "block" else {}),
            "mean_density": mean_density, "global_batch": 1 if sharded else B * world, "seq_len": N,
            "parallelism": (f"(batch, head) pairs sharded over {world} ranks, {H} on this rank" if sharded
                            else f"heads-independent replicas x{world}"),
            "l2": "inputs (3 x %.0f MB) larger than the 126 MB L2; no explicit flush" % (B * H * N * d * 2 / 1e6),
        },
        "fwd_ms": fwd_ms,
        "pool_ms": pool_ms,
        "fwd_kept_tflops": fwd_tflops,
        "fwd_frac_bf16_peak": fwd_tflops / peaks["bf16_tflops"],
        "fwd_frac_bf16_sustained": fwd_tflops / peaks["bf16_tflops_sustained"],
        "pool_gbs": pool_gbs,
        "pool_frac_hbm": pool_gbs / peaks["hbm_gbs"],
        "dense_ms": dense_ms,
        "speedup_vs_dense": (dense_ms / fwd_ms) if dense_ms else None,
        "kept_tflop_per_step": job_kflops / 1e12,
        "union_tflop_per_step": None if uflops is None else job_uflops / 1e12,
        "pair_efficiency": None if uflops is None else job_kflops / job_uflops,
        "density": density_stats(dens, nb),
        "near_ties": None if parity is None else parity["near_ties"],
        "density_mismatch_rows": None if parity is None else parity["density_mismatch_rows"],
        "output_error": None if parity is None else parity["output_error"],
        "roofline": {
            "bound": "tensor",
            "achieved": fwd_tflops,
            "peak": peak_tc,
            "unit": "TFLOP/s",
            "frac": fwd_tflops / peak_tc,
            "traffic": fwd_traffic(B * H) if two_group else None,
            "kernel": "solattn_fwd_pp_kernel (fused forward)" if two_group
                      else "solattn_fwd_kernel (fused forward, one-unit kernel)",
            "peak_source": peaks["source"] + peak_kind,
        },
        "pool_roofline": {
            "bound": "hbm", "achieved": pool_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": pool_gbs / peaks["hbm_gbs"], "algorithmic_bytes": pbytes,
        },
        "cpu_baseline": cpu,
        "e2e": e2e,
        "clocks": clk,
        # per step: pool_means, key_stats and the fused forward (the forward's
        # workspace reset is a cudaMemsetAsync, not a kernel)
        "gpu_launches": 3 * args.steps,
    }
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- suite
def run_suite(args):
    """One JSON line per configuration of the length sweep (16K-128K tokens x
    5/10/15/30 % density, 24 heads), the HunyuanVideo-like attention (10 / 15
    %) and the kept-set rules at the Wan-like 15 % (threshold, top-k, top-p):
    forward ms, kept-block TFLOP/s and its fraction of the bf16 burst peak, the
    dense path's ms and the speed-up, the per-row density distribution and the
    clocks of each timed loop, and for the threshold rule the near ties and the
    rows whose kept count differs from the fp64 routing oracle. Inputs resident
    on the GPU; warm-up calls, then a timed loop of at least 5 calls and about
    0.8 s (so that the clock sampler sees it several times)."""
    import block_sparse_attention_cov_b200 as sa
    from block_sparse_attention_cov_b200 import _lib

    _lib.lib()
    dev = torch.device("cuda", 0)
    peaks = load_peaks()
    stream = torch.cuda.current_stream()
    cvd = os.environ.get("CUDA_VISIBLE_DEVICES")

    def timed(fn, reps, warm=2, window_ms=800.0):
        for _ in range(warm):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        torch.cuda.synchronize()
        reps = max(reps, math.ceil(window_ms / max(e0.elapsed_time(e1), 1e-3)))
        clocks = ClockSampler(cvd.split(",")[0] if cvd else "0")
        clocks.start()
        time.sleep(0.2)
        w0 = time.monotonic()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        clocks.mark(w0, time.monotonic())
        return e0.elapsed_time(e1) / reps, clocks.stop()

    plan = [(name, None) for name in ("sweep_16k", "sweep_32k", "sweep_64k", "sweep_128k", "hunyuan_119k")]
    plan.append(("wan_75k", "rules"))
    for name, mode in plan:
        wl = WORKLOADS[name]
        q_h, k_h, v_h = make_qkv(wl, seed=0)
        q, k, v = (x.to(dev) for x in (q_h, k_h, v_h))
        B, H, N, d = q.shape
        nb = math.ceil(N / 64)
        ws = sa.workspace(dev)
        stats = sa.pool(q, k, v)
        out = torch.empty_like(q)
        lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
        dens = torch.empty((B, H, nb), dtype=torch.int32, device=dev)
        dense_ms, _ = timed(lambda: sa.dense(q, k, v, out=out, lse=lse, ws=ws), 2, 1)
        beta15 = load_beta(name, 0.15)[0]
        if mode == "rules":
            runs = [("threshold", {"rule": "threshold"}, beta15),
                    ("topk", {"rule": "topk", "topk": args.topk}, 0.0),
                    ("topp", {"rule": "topp", "topp": args.topp}, 0.0)]
        else:
            targets = json.load(open(os.path.join(ROOT, "tests", "golden", "calibrated_beta.json")))[name]["targets"]
            runs = [(f"{float(t):.0%}", {"rule": "threshold"}, targets[t]["beta"]) for t in sorted(targets)]
        for label, kw, beta in runs:
            fwd = lambda: sa.forward(q, k, v, stats, beta, out=out, lse=lse, density=dens, ws=ws, **kw)
            ms, clk = timed(fwd, 5, 3)
            if sa.status(ws) != 0:
                raise RuntimeError(f"device status {sa.status(ws)} in {name} {label}")
            kfl = kept_flops(stats, dens, beta, N, d, kw["rule"])
            tf = kfl / (ms * 1e-3) / 1e12
            line = {"suite": name, "config": label, "rule": kw["rule"], "beta": beta,
                    **({"topk": kw["topk"]} if "topk" in kw else {}), **({"topp": kw["topp"]} if "topp" in kw else {}),
                    "B": B, "H": H, "N": N, "d": d, "fwd_ms": ms, "kept_tflop": kfl / 1e12, "kept_tflops": tf,
                    "frac_bf16_burst": tf / peaks["bf16_tflops"], "dense_ms": dense_ms,
                    "speedup_vs_dense": dense_ms / ms, "density": density_stats(dens, nb), "clocks": clk}
            if kw["rule"] == "threshold":
                uf = union_flops(stats, beta, N, d)
                line["pair_efficiency"] = kfl / uf
                _, ties, bad, _ = routing_oracle(q_h, k_h, beta, dens.cpu().numpy())
                line["near_ties"], line["density_mismatch_rows"] = ties, bad
            print(json.dumps(line), flush=True)
        del q, k, v, q_h, k_h, v_h, stats, out, lse, dens
        torch.cuda.empty_cache()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="wan_75k", choices=sorted(WORKLOADS))
    ap.add_argument("--beta", type=float, default=None)
    ap.add_argument("--density", type=float, default=None,
                    help="use the calibrated beta of this mean kept-block density (e.g. 0.05 on the sweeps)")
    ap.add_argument("--heads", type=int, default=None, help="override the head count (small profiling cases)")
    ap.add_argument("--rule", choices=["threshold", "topk", "topp"], default="threshold",
                    help="kept-set rule (the method is 'threshold'; top-k / top-p are the ablation rules)")
    ap.add_argument("--topk", type=int, default=177, help="top-k rule: blocks per query block (15 %% of 1182)")
    ap.add_argument("--topp", type=float, default=0.1612,
                    help="top-p rule: mass fraction (0.1612 gives a 15 %% mean density on the Wan-like inputs)")
    ap.add_argument("--n-forced", type=int, default=0, help="leading key blocks always kept")
    ap.add_argument("--correction", choices=["block", "token"], default="block",
                    help="skipped-block correction: block-level proxy score (the method) or per token")
    ap.add_argument("--shard", choices=["replicas", "heads"], default="replicas",
                    help="multi-GPU layout: every rank runs the whole workload (weak scaling), or the (batch, "
                         "head) pairs are split over the ranks (strong scaling); no collective on the data path "
                         "either way")
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--skip-dense", action="store_true")
    ap.add_argument("--suite", action="store_true",
                    help="one JSON line per configuration of the sweep, the Hunyuan-like workload and the rules")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        backend = "nccl" if args.impl == "ours" else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    try:
        if args.suite:
            run_suite(args)
        elif args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
