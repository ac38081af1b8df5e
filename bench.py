"""Benchmark of the Token Sparse Attention prefill path on B200.

One step = one pass of the whole hot path (proxy scores, coverage budget,
per-head top-k, gather, compressed causal attention, scatter) over one
synthetic 128K-token prefill (32 query / 8 KV heads, d = 128, w = 128,
tau = 0.05), through the C ABI.  Metric: effective TFLOP/s = dense causal
attention FLOPs of the workload / TSA time (the speedup over our dense causal
kernel on the same tensors is reported beside it).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--tau T] [--impl reference]

With --gpus N > 1 (under torchrun) the ranks split the query heads of the
one sequence (--shard heads, the default: every step runs on each rank's
heads, and the budget, which is global over a sequence's heads, is combined
by one all-reduce of B integers per step; strong scaling), or every rank
runs its own sequence (--shard replicas: no collective; weak scaling).  The
step time is the max over ranks.  --impl reference times the CPU oracle on a
bounded sample of the same workload on the host cores (rank 0 only).
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "Token-sparse prefill attention ms and effective TFLOP/s at 128K vs dense; % BF16/HBM roofline"
UNIT = "TFLOP/s (effective: dense causal attention FLOPs / TSA time)"
DEFAULT_WORKLOAD = "c4_L128K_gqa"
KERNELS_PER_FORWARD = 9  # score x3, budget, budget finalize, select, gather, attention, scatter
# DRAM bytes per kept (head, row) of the forward's attention kernel, from ncu
# dram__bytes_read.sum + dram__bytes_write.sum of one launch; DRAM traffic
# grows with kept rows, not with FLOPs (algorithmic: 3 x 256 B read + 256 B
# written per kept row).
ATTN_DRAM_BYTES_PER_KEPT_ROW = 805.7e6 / (32 * 25147)
ATTN_TRAFFIC_NOTE = ("ncu dram__bytes_read.sum + dram__bytes_write.sum of one launch of the same kernel on the 32K "
                     "workload (805.7 MB for 32 x 25147 kept rows), scaled by kept rows")
SMS = 148
EX2_PER_CLK_SM = 16   # ex2.approx on B200, measured: one warp instruction per 8 clocks per SMSP


def stage_algorithmic_bytes(wl, kept_np, idx) -> dict:
    """Algorithmic HBM bytes of the HBM-bound stages for one forward.

    gather:  Q rows of every kept (head, row), the UNIQUE K and V rows each
             KV group reads (the union of its query heads' selections), and
             the three compressed rows written per kept (head, row);
    scatter: every output row written plus the kept compressed rows read;
    score:   one read of K, the window rows of Q, and the fp32 scores.
    idx: the device index tensor [B, Hq, L] of the forward just timed."""
    import torch
    B, Hq, Hkv, L, d = wl.B, wl.Hq, wl.Hkv, wl.L, wl.d
    G = Hq // Hkv
    per_head = kept_np if kept_np.ndim == 2 else np.repeat(np.asarray(kept_np)[:, None], Hq, axis=1)
    kept = int(per_head.sum())
    row = d * 2
    uniq = 0
    for b in range(B):
        for g in range(Hkv):
            mask = torch.zeros(L, dtype=torch.bool, device=idx.device)
            for h in range(g * G, (g + 1) * G):
                mask[idx[b, h, :int(per_head[b, h])].long()] = True
            uniq += int(mask.sum().item())
    return {"gather": kept * row + 2 * uniq * row + 3 * kept * row,
            "scatter": B * Hq * L * row + kept * row,
            "score": B * Hkv * L * row + B * Hq * wl.w * row + B * Hq * L * 4}


def dense_flops(wl) -> float:
    return float(wl.B) * wl.Hq * 2.0 * wl.d * wl.L * (wl.L + 1)


def compressed_flops(wl, kept) -> float:
    """FLOPs of causal attention over the kept rows: kept is one count per
    sequence (every head keeps it) or one per (sequence, head)."""
    kept = np.asarray(kept, dtype=np.float64)
    per = 2.0 * wl.d * kept * (kept + 1)
    return float(per.sum() * (wl.Hq if kept.ndim == 1 else 1))


def peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            m = json.load(f)
        return {"hbm_gbs": m["hbm_gbs"], "bf16": m["bf16_tflops"], "bf16_sustained": m["bf16_tflops_sustained"],
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16": 1590.0, "bf16_sustained": 1400.0, "source": "fallback"}


# ---------------------------------------------------------------- ranks
def rank_workload(wl, rank: int):
    """Each rank processes its own sequence(s): same shape, own seed."""
    return wl.with_(seed=wl.seed + 1000 * rank)


def max_over_ranks(x: float, dist, device) -> float:
    """Step time of the whole job: the slowest rank (identity without dist)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(wl, world: int, ms: float, sharded: bool = False) -> float:
    """Whole-job effective TFLOP/s: the dense-equivalent FLOPs of all ranks
    over the max-over-ranks step time (replicas: every rank its own
    sequence; heads: the ranks share one sequence's heads)."""
    return (1 if sharded else world) * dense_flops(wl) / (ms * 1e-3) / 1e12


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during timing."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        rows = []
        if self.path and os.path.exists(self.path):
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) >= 9:
                        rows.append(parts)
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        load = [s for s in sm if mx and s > 0.5 * max(mx)] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------- oracle leg
def oracle_sample(wl, tau: float, rows: int = 1536, heads: int = 2, keep_recent: int = 0) -> dict:
    """Time the CPU oracle on a bounded sample of the workload and scale it to
    the whole step: steps 1-4 and 6 at full length for the first `heads`
    query heads of sequence 0 (their own KV heads), and step 5 for the `rows`
    most expensive compressed rows of each.  The step estimate is the mean
    per-head cost times the head count, with step 5 scaled by causal pairs."""
    import oracle as O
    try:
        from threadpoolctl import threadpool_info
        cores = max([t.get("num_threads", 1) for t in threadpool_info()] or [1])
    except Exception:  # pragma: no cover
        cores = 1
    heads = min(heads, wl.Hq)
    sub = wl.with_(B=1, Hq=heads, Hkv=max(1, heads // wl.G) if heads >= wl.G else 1)
    q, k, v = W.generate(sub)
    G = sub.Hq // sub.Hkv
    L, d = wl.L, wl.d
    scale = O.default_scale(d)
    fixed = attn = 0.0
    pairs_sample = pairs_full = 0.0
    ks = []
    t_start = time.perf_counter()
    for h in range(heads):
        t0 = time.perf_counter()
        s32 = O.proxy_scores_head(q[0, h, L - wl.w:], k[0, h // G], L, scale)
        kh = max(L - O.pruned_count_head(s32, tau), keep_recent)
        sel = O.select_head(s32, kh, keep_recent)
        qc, kc, vc = q[0, h][sel], k[0, h // G][sel], v[0, h // G][sel]
        t1 = time.perf_counter()
        r = np.arange(max(kh - rows, 0), kh)
        oc = O.attention_rows(qc, kc, vc, r, scale)
        t2 = time.perf_counter()
        full = np.zeros((L, d))
        full[sel[r]] = oc
        t3 = time.perf_counter()
        fixed += (t1 - t0) + (t3 - t2)
        attn += t2 - t1
        pairs_sample += float(np.sum(r + 1))
        pairs_full += kh * (kh + 1) / 2.0
        ks.append(int(kh))
    sample_seconds = time.perf_counter() - t_start
    per_head = (fixed + attn * pairs_full / pairs_sample) / heads
    t_full = wl.B * wl.Hq * per_head
    return {"seconds_full_step_est": t_full, "cores": cores, "host_cores": len(os.sched_getaffinity(0)),
            "sample_seconds": sample_seconds, "k_head": ks,
            "sample": (f"steps 1-4,6 at L={L} for query heads 0..{heads - 1} of sequence 0, step 5 for the last "
                       f"{rows} compressed rows of each (k={ks}); the mean per-head time scaled by head count, "
                       f"step 5 by causal pair count, to the full step ({sample_seconds:.1f} s measured)")}


L2_BYTES = 126 << 20   # B200 L2


def l2_note(wl) -> str:
    """Whether the step's inputs exceed L2 (the timing rule between timed
    iterations: flush L2 or use inputs larger than it), with their sizes."""
    q = wl.B * wl.Hq * wl.L * wl.d * 2
    kv = wl.B * wl.Hkv * wl.L * wl.d * 2
    mib = lambda n: f"{n / 2**30:.3g} GiB" if n >= 2**30 else f"{n / 2**20:.3g} MiB"
    sizes = f"Q {mib(q)}, K/V {mib(kv)} each"
    if q + 2 * kv > L2_BYTES:
        return f"inputs larger than L2 ({sizes})"
    return f"inputs fit in L2 ({sizes}): a small case, not a headline timing"


def config_of(args, wl, world: int) -> dict:
    """The workload description both arms print."""
    shard = getattr(args, "shard", "heads")
    return {"workload": wl.name, "B": wl.B, "Hq": wl.Hq, "Hkv": wl.Hkv, "L": wl.L, "d": wl.d, "w": wl.w,
            "tau": args.tau, "budget_mode": args.budget_mode, "keep_recent": args.keep_recent,
            "layout": args.layout, "parallelism": f"{shard}{world}" if world > 1 else "single",
            "l2": l2_note(wl)}


def run_reference(args, wl, rank: int) -> int:
    if rank != 0:
        return 0
    # each step a smaller sample (one head, 768 attention rows) so that the
    # default --steps/--warmup run ends in a few minutes
    one = lambda: oracle_sample(wl, args.tau, rows=768, heads=1, keep_recent=args.keep_recent)
    for _ in range(args.warmup):
        one()
    runs = [one() for _ in range(args.steps)]
    t = statistics.median(r["seconds_full_step_est"] for r in runs)
    value = dense_flops(wl) / t / 1e12
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "impl": "reference", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(args, wl, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": runs[0]["cores"], "host_cores": runs[0]["host_cores"],
                         "kind": "oracle", "sample": runs[0]["sample"]},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- varlen leg
def run_varlen(args, wl) -> int:
    """One packed varlen batch (sequence b: the first L_b tokens of sequence b
    of the workload), timed like the headline step on one GPU.  Effective
    TFLOP/s counts the dense causal FLOPs of every sequence."""
    import torch
    import token_sparse_attention_tsa_b200 as T
    lengths = [int(x) for x in args.varlen.split(",")]
    Lmax = max(lengths)
    wl = wl.with_(B=len(lengths), L=Lmax)
    qh, kh, vh = W.generate(wl)
    pack = lambda x: np.ascontiguousarray(np.concatenate(
        [x[b, :, :n].transpose(1, 0, 2) for b, n in enumerate(lengths)], axis=0))
    q, k, v = (torch.from_numpy(pack(x)).view(torch.bfloat16).cuda() for x in (qh, kh, vh))
    del qh, kh, vh
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lengths)]), dtype=torch.int32, device="cuda")
    p = T.params(wl.B, wl.Hq, wl.Hkv, Lmax, wl.d, wl.w, args.tau, budget_mode=args.budget_mode,
                 keep_recent=args.keep_recent, cu_seqlens=cu, total_tokens=q.shape[0])
    ws = T.new_workspace(p, full=True)
    o = torch.empty_like(q)
    scores = torch.empty((wl.B, wl.Hq, Lmax), device="cuda")
    idx = torch.empty((wl.B, wl.Hq, Lmax), dtype=torch.int32, device="cuda")
    kept = torch.empty((wl.B, wl.Hq) if args.budget_mode == "per_head" else (wl.B,), dtype=torch.int32,
                       device="cuda")
    fwd = lambda: T.tsa_forward(p, q, k, v, o, ws, scores, idx, kept)
    for _ in range(args.warmup):
        fwd()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    with ClockSampler(0) as clk:
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            fwd()
        b.record(stream)
        torch.cuda.synchronize()
    ms = a.elapsed_time(b) / args.steps
    status, flags = T.get_device_status(ws)
    if status != 0:
        print(json.dumps({"error": f"device status {status} flags {flags}"}), file=sys.stderr)
        return 3
    kept_np = kept.cpu().numpy()
    per_head = kept_np if kept_np.ndim == 2 else np.repeat(kept_np[:, None], wl.Hq, axis=1)
    dense = sum(wl.Hq * 2.0 * wl.d * n * (n + 1) for n in lengths)
    comp = float((2.0 * wl.d * per_head.astype(np.float64) * (per_head + 1)).sum())
    od = torch.empty_like(q)
    for _ in range(2):
        T.tsa_attend_dense(p, q, k, v, od, None, ws)
    torch.cuda.synchronize()
    a.record(stream)
    T.tsa_attend_dense(p, q, k, v, od, None, ws)
    b.record(stream)
    torch.cuda.synchronize()
    dense_ms = a.elapsed_time(b)
    line = {"metric": METRIC + " (packed varlen batch)", "value": dense / (ms * 1e-3) / 1e12, "unit": UNIT,
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": wl.name, "varlen_lengths": lengths, "Hq": wl.Hq, "Hkv": wl.Hkv, "d": wl.d,
                       "w": wl.w, "tau": args.tau, "budget_mode": args.budget_mode, "layout": "packed token-major"},
            "kept_rows_fraction": float(per_head.sum()) / (wl.Hq * sum(lengths)),
            "achieved_tflops": comp / (ms * 1e-3) / 1e12, "dense_ms": dense_ms,
            "speedup_vs_dense": dense_ms / ms, "gpu_launches": KERNELS_PER_FORWARD * args.steps,
            "clocks": clk.summary()}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------- sweep leg
def run_sweep(args, wl) -> int:
    """The forward over a grid of coverage thresholds and context lengths
    (the workload's shape otherwise), one JSON line per point, on one GPU:
    the forward's time, keep fraction, effective and achieved TFLOP/s, the
    stage breakdown, and the dense baselines (our kernel and torch SDPA) on
    the same tensors.  These are supporting lines, not the headline."""
    import torch
    import token_sparse_attention_tsa_b200 as T
    T.load()
    stream = torch.cuda.current_stream()
    taus = [float(x) for x in args.sweep_tau.split(",")] if args.sweep_tau else [args.tau]
    lengths = [int(x) for x in args.sweep_L.split(",")] if args.sweep_L else [wl.L]
    pk = peaks()

    def timed(fn, n):
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n

    for L in lengths:
        wl_l = wl.with_(L=L, w=min(wl.w, L))
        qh, kh, vh = W.generate(wl_l)
        q, k, v = (torch.from_numpy(x).view(torch.bfloat16).cuda() for x in (qh, kh, vh))
        del qh, kh, vh
        o = torch.empty_like(q)
        shape3 = (wl.B, wl.Hq, L)
        scores = torch.empty(shape3, device="cuda")
        idx = torch.empty(shape3, dtype=torch.int32, device="cuda")
        k_seq = torch.empty((wl.B,), dtype=torch.int32, device="cuda")
        k_head = torch.empty((wl.B, wl.Hq), dtype=torch.int32, device="cuda")
        qc, kc, vc = (torch.empty((wl.B, wl.Hq, L, wl.d), dtype=torch.bfloat16, device="cuda") for _ in range(3))
        p0 = T.params(wl.B, wl.Hq, wl.Hkv, L, wl.d, wl_l.w, taus[0])
        ws = T.new_workspace(p0)
        od = torch.empty_like(q)
        T.tsa_attend_dense(p0, q, k, v, od, None, ws)
        dense_ms = timed(lambda: T.tsa_attend_dense(p0, q, k, v, od, None, ws), 2)
        sdpa_ms = None
        try:
            from torch.nn.attention import SDPBackend, sdpa_kernel
            sdpa = torch.nn.functional.scaled_dot_product_attention
            with sdpa_kernel([SDPBackend.CUDNN_ATTENTION, SDPBackend.FLASH_ATTENTION]):
                sdpa(q, k, v, is_causal=True, enable_gqa=True)
                sdpa_ms = timed(lambda: sdpa(q, k, v, is_causal=True, enable_gqa=True), 2)
        except Exception:
            sdpa_ms = None
        for tau in taus:
            p = T.params(wl.B, wl.Hq, wl.Hkv, L, wl.d, wl_l.w, tau)
            fwd = lambda: T.tsa_forward(p, q, k, v, o, ws, scores, idx, k_seq)
            for _ in range(args.warmup):
                fwd()
            with ClockSampler(0) as clk:
                ms = timed(fwd, args.steps)
            evs = [torch.cuda.Event(enable_timing=True) for _ in range(7)]
            names = ["score", "budget", "select", "gather", "attend", "scatter"]
            acc = {n: 0.0 for n in names}
            reps = 2
            for _ in range(reps):
                evs[0].record(stream)
                T.tsa_score(p, q, k, scores, ws); evs[1].record(stream)
                T.tsa_budget(p, scores, k_head, k_seq, ws); evs[2].record(stream)
                T.tsa_select(p, scores, k_seq, idx, ws); evs[3].record(stream)
                T.tsa_gather_qkv(p, q, k, v, idx, k_seq, qc, kc, vc, ws); evs[4].record(stream)
                T.tsa_attend(p, qc, kc, vc, k_seq, qc, None, ws); evs[5].record(stream)
                T.tsa_scatter(p, qc, idx, k_seq, o, ws); evs[6].record(stream)
                torch.cuda.synchronize()
                for i, n in enumerate(names):
                    acc[n] += evs[i].elapsed_time(evs[i + 1]) / reps
            st = T.get_device_status(ws)
            kept = k_seq.cpu().numpy()
            cfl = compressed_flops(wl_l, kept)
            line = {"metric": METRIC + " (sweep point)", "sweep": True, "n_gpus": 1, "steps": args.steps,
                    "warmup": args.warmup, "dtype": "bf16", "data": "synthetic",
                    "config": {"workload": wl.name, "L": L, "B": wl.B, "Hq": wl.Hq, "Hkv": wl.Hkv, "d": wl.d,
                               "w": wl_l.w, "tau": tau},
                    "ms_per_step": ms, "k_seq": kept.tolist(), "keep_fraction": (kept / L).tolist(),
                    "effective_tflops": dense_flops(wl_l) / (ms * 1e-3) / 1e12,
                    "achieved_tflops": cfl / (ms * 1e-3) / 1e12,
                    "attend_tflops": cfl / (acc["attend"] * 1e-3) / 1e12,
                    "attend_frac_sustained": cfl / (acc["attend"] * 1e-3) / 1e12 / pk["bf16_sustained"],
                    "dense_ms": dense_ms, "speedup_vs_dense": dense_ms / ms, "sdpa_dense_ms": sdpa_ms,
                    "speedup_vs_sdpa": (sdpa_ms / ms) if sdpa_ms else None,
                    "stage_ms": acc, "overhead_frac": (acc["score"] + acc["budget"] + acc["select"]) / acc["attend"],
                    "status": st, "clocks": clk.summary()}
            print(json.dumps(line), flush=True)
        del q, k, v, o, qc, kc, vc, od, ws
        torch.cuda.empty_cache()
    return 0


# ---------------------------------------------------------------- GPU leg
def run_gpu(args, wl, rank: int, world: int, local_rank: int) -> int:
    import torch
    import token_sparse_attention_tsa_b200 as T

    dist = None
    # one rank per GPU; with fewer GPUs than ranks (a test of the sharded
    # path's plumbing only) ranks share devices round-robin
    dev = torch.device("cuda", local_rank % torch.cuda.device_count())
    torch.cuda.set_device(dev)
    if world > 1:   # the device is set first, so NCCL binds each rank to its own GPU
        import datetime
        import torch.distributed as dist_mod
        dist = dist_mod
        backend = os.environ.get("TSA_BENCH_BACKEND", "nccl")   # gloo: host-side exchange, for plumbing tests
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300),
                                device_id=dev if backend == "nccl" else None)
    T.load()
    stream = torch.cuda.current_stream()

    def barrier():
        if dist is not None:
            dist.barrier()

    def rank_max(x: float) -> float:
        return max_over_ranks(x, dist, dev)

    # inputs: this rank's own sequence (replicas), or this rank's heads of
    # the one sequence (heads: the same sequence on every rank, split by
    # query head with the key/value heads they read)
    sharded = world > 1 and args.shard == "heads"
    if sharded:
        h0, h1, kv0, kv1 = T.shard_heads(wl.Hq, wl.Hkv, world, rank)
        qh, kh, vh = W.generate(wl)
        qh, kh, vh = (np.ascontiguousarray(x[:, a:b]) for x, (a, b) in
                      zip((qh, kh, vh), ((h0, h1), (kv0, kv1), (kv0, kv1))))
        wl_all, wl = wl, wl.with_(Hq=h1 - h0, Hkv=kv1 - kv0)    # wl: this rank's part from here on
    else:
        wl_all = wl
        qh, kh, vh = W.generate(rank_workload(wl, rank))
    if args.layout == "blhd":   # the caller's tensors token-major [B, L, H, d]
        qh, kh, vh = (np.ascontiguousarray(x.transpose(0, 2, 1, 3)) for x in (qh, kh, vh))
    pin = [torch.from_numpy(x).view(torch.bfloat16).pin_memory() for x in (qh, kh, vh)]
    q, k, v = [x.to(dev, non_blocking=True) for x in pin]
    o = torch.empty_like(q)
    p = T.params(wl.B, wl.Hq, wl.Hkv, wl.L, wl.d, wl.w, args.tau, budget_mode=args.budget_mode,
                 keep_recent=args.keep_recent, layout=args.layout)
    ws = T.new_workspace(p, full=True, device=dev)
    scores = torch.empty((wl.B, wl.Hq, wl.L), dtype=torch.float32, device=dev)
    idx = torch.empty((wl.B, wl.Hq, wl.L), dtype=torch.int32, device=dev)
    k_seq = torch.empty((wl.B,), dtype=torch.int32, device=dev)
    k_head = torch.empty((wl.B, wl.Hq), dtype=torch.int32, device=dev)
    # rows kept per head as the later calls read them: the sequence budget,
    # or in the per-head mode each head's own count
    kept = k_head if args.budget_mode == "per_head" else k_seq
    shape = (wl.B, wl.Hq, wl.L, wl.d)
    qc, kc, vc = (torch.empty(shape, dtype=torch.bfloat16, device=dev) for _ in range(3))
    torch.cuda.synchronize()

    k_part = torch.empty((wl.B,), dtype=torch.int32, device=dev)

    def forward():
        if sharded:   # steps 1-2 here, the budget exchanged over the ranks, steps 3-6 here
            T.forward_sharded(p, wl_all.Hq, q, k, v, o, ws, scores_out=scores, idx_out=idx, k_seq_out=kept,
                              k_part=k_part)
        else:
            T.tsa_forward(p, q, k, v, o, ws, scores, idx, kept)

    # the kernels tsa_forward runs, one ABI call each (with head sharding, the
    # budget's all-reduce over the ranks between the budget and the selection)
    exchange_op = T.budget_reduce_op(args.budget_mode) if sharded else None
    stage_names = ["score", "budget"] + (["exchange"] if exchange_op is not None else []) + \
        ["select", "gather", "attend", "scatter"]

    def staged(evs):
        n = iter(range(len(evs)))
        evs[next(n)].record(stream)
        T.tsa_score(p, q, k, scores, ws)
        evs[next(n)].record(stream)
        T.tsa_budget(p, scores, k_head, k_seq, ws)
        evs[next(n)].record(stream)
        if exchange_op == "max":
            dist.all_reduce(k_seq, op=dist.ReduceOp.MAX)
            evs[next(n)].record(stream)
        elif exchange_op == "sum":    # mean budget: the heads' counts summed over the ranks, as tsa_forward_end
            tot = k_head.sum(dim=1, dtype=torch.int64)
            dist.all_reduce(tot, op=dist.ReduceOp.SUM)
            k_seq.copy_(torch.div(tot + wl_all.Hq - 1, wl_all.Hq, rounding_mode="floor").to(torch.int32))
            evs[next(n)].record(stream)
        T.tsa_select(p, scores, kept, idx, ws)
        evs[next(n)].record(stream)
        T.tsa_gather_qkv(p, q, k, v, idx, kept, qc, kc, vc, ws)
        evs[next(n)].record(stream)
        T.tsa_attend(p, qc, kc, vc, kept, qc, None, ws)      # output over qc in place, as tsa_forward
        evs[next(n)].record(stream)
        T.tsa_scatter(p, qc, idx, kept, o, ws)
        evs[next(n)].record(stream)

    # the stage calls tsa_forward does not use, timed for comparison next to
    # the pair it does use (attention into a compressed output, then the
    # scatter), in the same iterations so that all see the same clocks: the
    # attention with the scatter folded into its epilogue (plus the zero fill
    # of the unselected rows), and the variant that also gathers by index
    unfused_names = ["attend_then_scatter", "attend_scatter_fused", "attend_gathered"]
    oc = torch.empty_like(qc)

    def unfused(evs):
        evs[0].record(stream)
        T.tsa_attend(p, qc, kc, vc, kept, oc, None, ws)
        T.tsa_scatter(p, oc, idx, kept, o, ws)
        evs[1].record(stream)
        T.tsa_attend_scatter(p, qc, kc, vc, idx, kept, o, None, ws)
        evs[2].record(stream)
        T.tsa_attend_gathered(p, q, k, v, idx, kept, o, None, ws)
        evs[3].record(stream)

    def timed(fn, n):
        barrier()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        barrier()
        return rank_max(a.elapsed_time(b) / n)

    for _ in range(args.warmup):
        forward()
    torch.cuda.synchronize()

    # ---- headline: tsa_forward, inputs resident in HBM (all > L2)
    with ClockSampler(dev.index) as clk:
        ms = timed(forward, args.steps)
    clocks = clk.summary()
    kept_np = kept.cpu().numpy()
    ks = kept_np.max(axis=1).tolist() if kept_np.ndim == 2 else kept_np.tolist()
    kept_rows = int(kept_np.sum()) * (wl.Hq if kept_np.ndim == 1 else 1)

    # ---- per-stage breakdown (same kernels, one ABI call per stage)
    def breakdown(fn, names):
        acc = {n: [] for n in names}
        for it in range(args.warmup + args.steps):
            evs = [torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
            barrier()
            fn(evs)
            torch.cuda.synchronize()
            if it >= args.warmup:
                for i, n in enumerate(names):
                    acc[n].append(evs[i].elapsed_time(evs[i + 1]))
        return {n: rank_max(statistics.mean(v)) for n, v in acc.items()}

    stage_ms = breakdown(staged, stage_names)
    unfused_ms = breakdown(unfused, unfused_names)

    # ---- dense baselines on the same tensors
    od = torch.empty_like(q)
    dense_ms = timed(lambda: T.tsa_attend_dense(p, q, k, v, od, None, ws), max(2, args.steps // 2))
    sdpa_ms = None
    try:  # library baseline (context only); fused backends only, never the O(L^2)-memory one
        from torch.nn.attention import SDPBackend, sdpa_kernel
        sdpa = torch.nn.functional.scaled_dot_product_attention
        hm = (lambda x: x.transpose(1, 2)) if args.layout == "blhd" else (lambda x: x)
        sq, sk, sv = hm(q), hm(k), hm(v)
        with sdpa_kernel([SDPBackend.CUDNN_ATTENTION, SDPBackend.FLASH_ATTENTION]):
            sdpa(sq, sk, sv, is_causal=True, enable_gqa=True)
            sdpa_ms = timed(lambda: sdpa(sq, sk, sv, is_causal=True, enable_gqa=True), 2)
    except Exception:
        sdpa_ms = None

    # ---- optional: block-sparse composition on the compressed sequence
    blocks = None
    if args.blocks:
        nbw = int(args.blocks.split(":")[1])
        nb = (wl.L + 127) // 128
        ii = torch.arange(nb, device=dev)[:, None]
        jj = torch.arange(nb, device=dev)[None, :]
        band = (((ii - jj) <= nbw) | (jj == 0)) & (jj <= ii)
        bmask = band.to(torch.uint8).expand(wl.B, wl.Hq, nb, nb).contiguous()

        def blocks_fwd():
            T.tsa_score(p, q, k, scores, ws)
            T.tsa_budget(p, scores, k_head, k_seq, ws)
            T.tsa_select(p, scores, kept, idx, ws)
            T.tsa_gather_qkv(p, q, k, v, idx, kept, qc, kc, vc, ws)
            T.tsa_attend_blocks(p, qc, kc, vc, idx, kept, bmask, o, None, ws)

        for _ in range(2):
            blocks_fwd()
        bms = timed(blocks_fwd, max(2, args.steps // 2))
        kb_rows = ks[0]
        nbk = (kb_rows + 127) // 128
        frac = float(band[:nbk, :nbk].sum().item()) / (nbk * (nbk + 1) / 2)
        blocks = {"mask": f"sink block + local band of {nbw} blocks (128 compressed tokens each)",
                  "ms_per_step": bms, "effective_tflops": dense_flops(wl) / (bms * 1e-3) / 1e12,
                  "causal_tile_fraction_kept": frac, "speedup_vs_tsa": ms / bms}

    # ---- end to end: pinned host inputs -> device -> tsa_forward -> host
    # output, every step.  Steps are pipelined the way a serving loop runs
    # them: step i+1's inputs go up on a copy stream and step i-1's output
    # comes back on another while step i computes (two device buffer sets;
    # events order each set's reuse).
    o_hosts = [torch.empty(tuple(o.shape), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    sets = [(q, k, v, o), tuple(torch.empty_like(x) for x in (q, k, v, o))]
    h2d_s, d2h_s = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

    def e2e_run(n):
        ev = lambda: torch.cuda.Event(enable_timing=True)
        start, end = ev(), ev()
        comp_done, d2h_done = [None] * n, [None] * n
        start.record(stream)
        h2d_s.wait_event(start)
        for i in range(n):
            sq, sk, sv, so = sets[i % 2]
            if i >= 2:
                h2d_s.wait_event(comp_done[i - 2])         # step i-2 has finished reading this set
            with torch.cuda.stream(h2d_s):
                for dst, src in zip((sq, sk, sv), pin):
                    dst.copy_(src, non_blocking=True)
            up = torch.cuda.Event()
            up.record(h2d_s)
            stream.wait_event(up)
            if i >= 2:
                stream.wait_event(d2h_done[i - 2])         # this set's previous output is back on the host
            if sharded:
                T.forward_sharded(p, wl_all.Hq, sq, sk, sv, so, ws, scores_out=scores, idx_out=idx, k_seq_out=kept,
                                  k_part=k_part)
            else:
                T.tsa_forward(p, sq, sk, sv, so, ws, scores, idx, kept, stream=stream)
            comp_done[i] = torch.cuda.Event()
            comp_done[i].record(stream)
            d2h_s.wait_event(comp_done[i])
            with torch.cuda.stream(d2h_s):
                o_hosts[i % 2].copy_(so, non_blocking=True)
            d2h_done[i] = torch.cuda.Event()
            d2h_done[i].record(d2h_s)
        stream.wait_event(d2h_done[n - 1])
        end.record(stream)
        torch.cuda.synchronize()
        return start.elapsed_time(end) / n

    e2e_run(2)
    barrier()
    e2e_steps = max(8, args.steps)
    e2e_ms = rank_max(e2e_run(e2e_steps))
    h2d = sum(x.numel() * x.element_size() for x in pin)
    d2h = o_hosts[0].numel() * o_hosts[0].element_size()

    status, flags = T.get_device_status(ws)
    if status != 0:
        print(json.dumps({"error": f"device status {status} flags {flags}"}), file=sys.stderr)
        return 3

    # ---- roofline of the dominant kernel (attention: a dense contraction)
    pk = peaks()
    cflops = compressed_flops(wl, kept_np)
    attn_ms = stage_ms["attend"]
    achieved = cflops / (attn_ms * 1e-3) / 1e12
    roof = {"bound": "tensor", "kernel": "attend2_kernel<128,false,false,false> (attention, compressed output)",
            "achieved": achieved,
            "peak": pk["bf16_sustained"], "unit": "TFLOP/s", "frac": achieved / pk["bf16_sustained"],
            "traffic": (ATTN_DRAM_BYTES_PER_KEPT_ROW * kept_rows) if ATTN_DRAM_BYTES_PER_KEPT_ROW else None,
            "traffic_note": ATTN_TRAFFIC_NOTE,
            "peak_note": f"bf16_tflops_sustained of {pk['source']} peaks (kernel timed inside a long step)"}
    hbm = pk["hbm_gbs"]
    stage_bytes = stage_algorithmic_bytes(wl, kept_np, idx)
    times = {n: stage_ms[n] for n in stage_bytes}
    stage_roof = {n: {"bytes": b, "GB/s": b / (times[n] * 1e-3) / 1e9, "frac_hbm": b / (times[n] * 1e-3) / 1e9 / hbm}
                  for n, b in stage_bytes.items()}
    # the proxy score is bound by its exponentials: 2 B Hq w L of them (two passes)
    exps = 2.0 * wl.B * wl.Hq * wl.w * wl.L
    ex2_peak = EX2_PER_CLK_SM * SMS * (clocks.get("sm_mhz") or 1965.0) * 1e6
    stage_roof["score"]["exp_per_s"] = exps / (stage_ms["score"] * 1e-3)
    stage_roof["score"]["exp_frac"] = stage_roof["score"]["exp_per_s"] / ex2_peak
    stage_roof["score"]["exp_peak_note"] = (f"{EX2_PER_CLK_SM} ex2/clk/SM x {SMS} SMs x the median sampled SM clock "
                                            "(ex2.approx: one warp instruction per 8 clocks per SMSP, measured)")

    job_flops = dense_flops(wl_all) * (1 if sharded else world)   # the work of all ranks together
    value = job_value(wl_all, world, ms, sharded)
    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        s = oracle_sample(wl_all, args.tau, keep_recent=args.keep_recent)
        cpu = {"value": dense_flops(wl_all) / s["seconds_full_step_est"] / 1e12, "unit": UNIT,
               "cores": s["cores"], "host_cores": s["host_cores"], "kind": "oracle", "sample": s["sample"],
               "sample_seconds": s["sample_seconds"]}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "strong" if sharded else "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": config_of(args, wl_all, world),
        "k_seq": ks, "keep_fraction": [x / wl.L for x in ks],
        "kept_fraction_all_heads": kept_rows / float(wl.B * wl.Hq * wl.L),
        "dense_ms": dense_ms, "speedup_vs_dense": dense_ms / ms, "sdpa_dense_ms": sdpa_ms,
        "effective_tflops": value,
        "achieved_tflops": cflops / (ms * 1e-3) / 1e12 * (world if sharded else 1),
        "stage_ms": stage_ms, "unfused_stage_ms": unfused_ms, "stage_hbm": stage_roof,
        "overhead_frac": (sum(stage_ms.values()) - attn_ms) / attn_ms,
        "roofline": roof, "cpu_baseline": cpu,
        "e2e": {"value": job_flops / (e2e_ms * 1e-3) / 1e12, "unit": UNIT, "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "note": "every step copies its inputs up and its output back; copies of neighbouring steps "
                        "overlap this step's compute on separate streams (pipeline fill and drain included)"},
        "gpu_launches": KERNELS_PER_FORWARD * args.steps, "clocks": clocks,
    }
    if blocks is not None:
        line["block_sparse"] = blocks
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main() -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--tau", type=float, default=None)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(W.WORKLOADS))
    ap.add_argument("--impl", default="tsa", choices=["tsa", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--budget-mode", default="max", choices=["max", "mean", "per_head"])
    ap.add_argument("--keep-recent", type=int, default=0)
    ap.add_argument("--layout", default="bhld", choices=["bhld", "blhd"])
    ap.add_argument("--shard", default="heads", choices=["heads", "replicas"],
                    help="with --gpus N > 1: split the query heads of the one sequence over the ranks (one "
                         "all-reduce of the budget per step; strong scaling), or give every rank its own "
                         "sequence (no collective; weak scaling)")
    ap.add_argument("--blocks", default=None,
                    help="band:N -- also time the path with a block-sparse mask on the compressed sequence "
                         "(sink block + local band of N blocks)")
    ap.add_argument("--varlen", default=None,
                    help="comma-separated sequence lengths: time a packed varlen batch of the workload's "
                         "first L_b tokens per sequence instead of the headline step")
    ap.add_argument("--sweep-tau", default=None, help="comma-separated tau values: print one sweep line each")
    ap.add_argument("--sweep-L", default=None, help="comma-separated context lengths for the sweep")
    args = ap.parse_args()
    wl = W.WORKLOADS[args.workload]
    if args.tau is None:
        args.tau = wl.tau
    wl = wl.with_(tau=args.tau)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, wl, rank)
    if args.varlen:
        return run_varlen(args, wl)
    if args.sweep_tau or args.sweep_L:
        return run_sweep(args, wl)
    return run_gpu(args, wl, rank, world, local_rank)


if __name__ == "__main__":
    sys.exit(main())
