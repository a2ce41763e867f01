#!/usr/bin/env python
"""Benchmark of the LightningIndexer hot path (scheduler -> score -> Top-k).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step is one full indexer call (all three kernels) over one batch of the
named synthetic workload, with inputs resident in HBM.  The ``sfa_*``
workloads instead time one call of the sparse attention consumer
(li_sparse_attention) over its own synthetic inputs.  The default workload
is the TileLang test shape (B=2, S1=512, S2=4096, G=32, D=64, k=1024, fp16,
no mask).  L2 is flushed before every timed step (a 256 MiB device write,
then a 256 MiB read of a second buffer so no dirty lines are left behind),
outside the timed interval; each step is timed with CUDA events on the
launching stream and the per-step times are summed.  Under torchrun every
rank runs its own copy of the workload (independent problems, weak scaling,
no data-path collective); the job time is the max over ranks.

The JSON line reports queries/s (value), the effective TFLOP/s, the roofline
of the dominant kernel measured live with per-stage CUDA events, an
end-to-end figure through the C ABI with host buffers (copies inside the
timed region), and the fp64 oracle timed on the host cores on a bounded
sample (cpu_baseline).  `--impl reference` times that oracle alone as the
reference arm.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "indexer queries/s and effective TFLOP/s at 1 B200; % of tensor/HBM roofline"
UNIT = "queries/s"
DEFAULT_WORKLOAD = "cfg2"
FLUSH_BYTES = 256 << 20
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

WORKLOAD_DESC = {
    "tiny": "tiny: B=1 S1=32 S2=256 N1=8 D=128 k=64 mode0 bf16",
    "cfg2": "B=2 S1=512 S2=4096 G=32 D=64 k=1024 mode0 fp16 q/k, fp32 w (TileLang test shape)",
    "dsa_prefill": "DSA prefill: B=1 S1=S2=8192 N1=64 D=128 k=2048 mode3 bf16, values on",
    "paged_decode": "paged decode: B=64 S1=1 N1=64 D=128 PA block 128, lengths U[4096,65536], k=2048 mode3 bf16",
    "quant_varlen": "quant varlen TND {2k,4k,8k,16k} N1=64 D=128 fp8 e4m3 + fp32 scales, k=2048 mode3",
    "quant_varlen_int8": "quant varlen TND {2k,4k,8k,16k} N1=64 D=128 int8 + fp16 scales/weights, k=2048 mode3",
    "quant_int8_pa": "quant int8 PA (VllmQuant README A3 example): B=24 S1=4 S2=512 N1=64 D=128 block 128, fp16 scales/weights, k=512 mode0",
    "dsa_prefill_window": "DSA prefill with sink/local window: B=1 S1=S2=8192 N1=64 D=128 k=2048 mode3 bf16, init_num=16 local_num=512, values on",
    "sfa_prefill": "sparse attention consumer of DSA prefill: 8192 rows x 64 heads, K=2048 selected keys (causal), D=Dv=128 bf16",
    "sfa_decode": "sparse attention consumer of paged decode: 64 rows x 64 heads over a PA pool (block 128, lengths U[4096,65536]), K=2048, D=Dv=128 bf16",
}
SFA_METRIC = "sparse attention query rows/s at 1 B200 (the indexer's consumer); % of tensor roofline"
SFA_UNIT = "rows/s"
RETURN_VALUE = {"tiny": 1, "cfg2": 1, "dsa_prefill": 1, "paged_decode": 0, "quant_varlen": 0,
                "quant_varlen_int8": 0, "quant_int8_pa": 0, "dsa_prefill_window": 1}


SEEDS = {"tiny": 0, "cfg2": 1, "dsa_prefill": 2, "paged_decode": 3, "quant_varlen": 4,
         "quant_int8_pa": 5, "quant_varlen_int8": 6, "dsa_prefill_window": 7}


def make_workload(name, rank=0):
    """The named workload; rank r > 0 draws an independent problem of the same
    shape (seed offset by r), as weak scaling over independent problems."""
    import synth
    fn = synth.WORKLOADS[name]
    if name in ("tiny",):
        return fn(seed=SEEDS[name] + rank)
    return fn(seed=SEEDS[name] + rank, return_value=RETURN_VALUE[name])


def job_value(rows_per_rank, steps, world, max_total_ms):
    """Whole-job queries/s: every rank's rows over the slowest rank's time."""
    return world * rows_per_rank * steps / (max_total_ms * 1e-3)


def work_counts(p, inp):
    """Host-side algorithmic work: visible pairs, FLOPs and compulsory bytes."""
    import torch
    B = p.B
    aq, ak = inp.get("act_q"), inp.get("act_k")
    if p.layout_q == "TND":
        cq = [0] + aq.tolist()
        Sq = [cq[b + 1] - cq[b] for b in range(B)]
    else:
        Sq = aq.tolist() if aq is not None else [p.S1] * B
    if p.layout_k == "TND":
        ck = [0] + ak.tolist()
        Sk = [ck[b + 1] - ck[b] for b in range(B)]
    elif p.layout_k == "BSND":
        Sk = ak.tolist() if ak is not None else [p.S2] * B
    else:
        Sk = ak.tolist()
    pairs = 0
    rows_nvis = 0
    for b in range(B):
        if p.sparse_mode == 0:
            pairs += Sq[b] * Sk[b]
        else:
            for i in range(Sq[b]):
                pairs += max(0, min(Sk[b], i + 1 + Sk[b] - Sq[b]))
    rows_nvis = pairs
    es = 1 if p.dtype_qk in ("e4m3", "int8") else 2
    esw = 4 if p.dtype_w == "fp32" else 2
    nbytes = lambda t: 0 if t is None else t.numel() * t.element_size()
    keys_visible = sum(Sk)
    kv_bytes = keys_visible * p.D * es
    compulsory = (nbytes(inp["query"]) + kv_bytes + nbytes(inp["weights"])
                  + nbytes(inp.get("q_scale"))
                  + keys_visible * (4 if p.dtype_scale == "fp32" else 2) * int(p.quant)
                  + nbytes(inp.get("block_table")) + nbytes(aq) + nbytes(ak)
                  + p.rows * p.sparse_count * (4 + 4 * p.return_value))
    topk_bytes = rows_nvis * 4 + p.rows * p.sparse_count * (4 + 4 * p.return_value)
    return dict(pairs=pairs, flops=2.0 * p.N1 * p.D * pairs, compulsory_bytes=compulsory,
                topk_bytes=topk_bytes, score_bytes=compulsory - p.rows * p.sparse_count *
                (4 + 4 * p.return_value) + pairs * 4, es=es, esw=esw)


def load_peaks():
    if os.path.exists(PEAKS_FILE):
        with open(PEAKS_FILE) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def traffic_record(workload, kernel):
    """Per-launch DRAM bytes from the committed ncu summary, if the kernel
    source is unchanged since the capture; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(workload, {}).get(kernel)
    if not rec:
        return None
    src = os.path.join(ROOT, "sparse_attention_top_n1_b200", "csrc", rec["source"])
    if not os.path.exists(src):
        return None
    sha = hashlib.sha1(open(src, "rb").read()).hexdigest()
    return rec["bytes_per_launch"] if sha == rec["sha1"] else None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.Q,
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.out,
                stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[j] for r in rows for j in range(4) if r[5 + j] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    return ws, rank, local


def allreduce_max(x, device="cuda"):
    """Max of a host float over all ranks (timing only; no data-path use)."""
    import torch
    import torch.distributed as dist
    if not dist.is_initialized():
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_initialized():
        dist.barrier()


def cpu_model():
    """The host CPU's model name (for the CPU baseline record)."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def cpu_oracle_sample(p, inp, budget_s=12.0, max_rows=None, seed=0):
    """Time the fp64 oracle on a bounded sample of query rows (host cores)."""
    import numpy as np

    import oracle
    oracle.build()
    nthreads = os.cpu_count() or 1
    R = p.rows
    rng = np.random.default_rng(seed)
    probe = sorted(rng.choice(R, size=min(R, max(nthreads, 8)), replace=False).tolist())
    t0 = time.perf_counter()
    oracle.run(p, inp, rows=probe, nthreads=nthreads)
    t_probe = time.perf_counter() - t0
    per_row = t_probe / len(probe)
    n = int(min(R if max_rows is None else max_rows, max(len(probe), budget_s / max(per_row, 1e-9))))
    rows = sorted(rng.choice(R, size=n, replace=False).tolist())
    t0 = time.perf_counter()
    oracle.run(p, inp, rows=rows, nthreads=nthreads)
    dt = time.perf_counter() - t0
    return {"value": len(rows) / dt, "unit": UNIT, "cores": nthreads, "kind": "oracle",
            "cpu_model": cpu_model(), "nproc": os.cpu_count(),
            "sample": "%d of %d query rows (seeded uniform sample), fp64 C oracle, %.2f s"
                      % (len(rows), R, dt)}, rows, dt


def run_reference(args, ws, rank):
    """The reference arm: the fp64 oracle on the host cores, bounded samples."""
    if rank != 0:
        return 0
    import numpy as np

    import oracle
    p, inp = make_workload(args.workload)
    oracle.build()
    nthreads = os.cpu_count() or 1
    R = p.rows
    rng = np.random.default_rng(1)
    probe = sorted(rng.choice(R, size=min(R, max(nthreads, 8)), replace=False).tolist())
    t0 = time.perf_counter()
    oracle.run(p, inp, rows=probe, nthreads=nthreads)
    per_row = (time.perf_counter() - t0) / len(probe)
    total_steps = args.steps + args.warmup
    step_budget = max(0.5, min(6.0, 150.0 / max(total_steps, 1)))
    n = int(min(R, max(len(probe), step_budget / max(per_row, 1e-9))))
    times = []
    for s in range(total_steps):
        rows = sorted(rng.choice(R, size=n, replace=False).tolist())
        t0 = time.perf_counter()
        oracle.run(p, inp, rows=rows, nthreads=nthreads)
        dt = time.perf_counter() - t0
        if s >= args.warmup:
            times.append(dt)
    tot = sum(times)
    value = n * len(times) / tot
    line = {"metric": METRIC, "value": value, "unit": UNIT, "impl": "reference", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": WORKLOAD_DESC[args.workload], "rows_per_step": n},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": nthreads, "kind": "oracle",
                             "cpu_model": cpu_model(), "nproc": os.cpu_count(),
                             "sample": "%d of %d query rows per step, fp64 C oracle" % (n, R)},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def blas_threads():
    """Threads the numpy oracle's matrix products may use (its BLAS pool)."""
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def sfa_workload(name, rank=0):
    """The named sparse attention workload; rank r > 0 draws an independent
    problem of the same shape (seed offset by r)."""
    from synth import sfa as ssfa
    if name == "sfa_prefill":
        return ssfa.make_sfa_prefill(seed=9 + rank)
    return ssfa.make_sfa_decode(seed=10 + rank)


def sfa_counts(p, inp):
    """Valid (row, selected key) pairs, FLOPs and gathered bytes of one call."""
    idx = inp["sparse_indices"].reshape(p.rows, p.sparse_count)
    pairs = int((idx >= 0).sum())
    flops = 2.0 * p.N1 * (p.D + p.Dv) * pairs
    gathered = pairs * (p.D + p.Dv) * 2
    io = p.rows * p.N1 * (p.D + p.Dv) * 2 + idx.numel() * 4 + p.rows * p.N1 * 4
    return pairs, flops, gathered, io


def sfa_reference(args, rank):
    """Reference arm for the sparse attention workloads: the fp64 oracle on
    bounded row samples on the host cores."""
    if rank != 0:
        return 0
    import numpy as np

    import oracle.sfa as osfa
    p, inp = sfa_workload(args.workload)
    rng = np.random.default_rng(1)
    probe = sorted(rng.choice(p.rows, size=min(p.rows, 8), replace=False).tolist())
    t0 = time.perf_counter()
    osfa.run(p, inp, rows=probe)
    per_row = (time.perf_counter() - t0) / len(probe)
    total_steps = args.steps + args.warmup
    step_budget = max(0.5, min(6.0, 150.0 / max(total_steps, 1)))
    n = int(min(p.rows, max(2, step_budget / max(per_row, 1e-9))))
    times = []
    for st in range(total_steps):
        rows = sorted(rng.choice(p.rows, size=n, replace=False).tolist())
        t0 = time.perf_counter()
        osfa.run(p, inp, rows=rows)
        if st >= args.warmup:
            times.append(time.perf_counter() - t0)
    tot = sum(times)
    value = n * len(times) / tot
    line = {"metric": SFA_METRIC, "value": value, "unit": SFA_UNIT, "impl": "reference", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": WORKLOAD_DESC[args.workload], "rows_per_step": n},
            "cpu_baseline": {"value": value, "unit": SFA_UNIT, "cores": blas_threads(), "kind": "oracle",
                             "cpu_model": cpu_model(), "nproc": os.cpu_count(),
                             "sample": "%d of %d rows per step, fp64 numpy oracle" % (n, p.rows)},
            "e2e": {"value": value, "unit": SFA_UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def sfa_main(args, ws, rank, local):
    """One step = one li_sparse_attention call over the whole workload."""
    import torch

    import sparse_attention_top_n1_b200 as li
    from sparse_attention_top_n1_b200 import build as libbuild
    if not os.path.exists(li.LIB_PATH):
        libbuild.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    p, inp = sfa_workload(args.workload, rank)
    pairs, flops, gathered, io = sfa_counts(p, inp)
    d = {k: v.to(dev) for k, v in inp.items()}
    pr = li.make_sfa_params(p)
    out = torch.empty((p.rows, p.N1, p.Dv), dtype=d["query"].dtype, device=dev)
    lse = torch.empty((p.rows, p.N1), dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    clean = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def flush_l2():
        flush.zero_()
        clean.sum()

    def call():
        li.li_sparse_attention(pr, d["query"], d["key"], d["value"], d["sparse_indices"], d.get("act_q"),
                               d.get("act_k"), d.get("block_table"), out, lse, status)

    clocks = ClockSampler(local)
    if not args.plain:
        clocks.start()
    t_warm = time.perf_counter()
    nw = 0
    while nw < args.warmup or (not args.plain and time.perf_counter() - t_warm < 0.8):
        flush_l2()
        call()
        nw += 1
    torch.cuda.synchronize()
    mk = lambda: torch.cuda.Event(enable_timing=True)
    K = args.steps
    st_ev = [mk() for _ in range(K)]
    en_ev = [mk() for _ in range(K)]
    barrier()
    torch.cuda.synchronize()
    launches = 0
    torch.cuda.nvtx.range_push("timed steps")
    for s_ in range(K):
        flush_l2()
        st_ev[s_].record()
        call()
        en_ev[s_].record()
        launches += li.li_last_launch_count()
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    barrier()
    own = sum(st_ev[s_].elapsed_time(en_ev[s_]) for s_ in range(K))
    total_ms = allreduce_max(own)
    clk = clocks.stop()
    if int(status.item()):
        raise SystemExit("device status 0x%x" % int(status.item()))
    peaks, peak_src = load_peaks()
    ms = total_ms / K
    tflops = flops / (ms * 1e-3) / 1e12
    roof = {"bound": "tensor", "achieved": tflops, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
            "frac": tflops / peaks["bf16_tflops"], "traffic": traffic_record(args.workload, "sfa"), "kernel": "sfa",
            "peak_source": "bf16 burst peak (tcgen05 cuBLAS), %s; this kernel issues m16n8k16 mma.sync" % peak_src}
    e2e = None
    if not (args.no_e2e or args.plain):
        host = {k: v.pin_memory() for k, v in inp.items()}
        hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        h2d = sum(v.numel() * v.element_size() for v in host.values())
        d2h = hout.numel() * hout.element_size()
        e_st = [mk() for _ in range(K + args.warmup)]
        e_en = [mk() for _ in range(K + args.warmup)]
        for s_ in range(K + args.warmup):
            flush_l2()
            e_st[s_].record()
            for k2, v in host.items():
                d[k2].copy_(v, non_blocking=True)
            call()
            hout.copy_(out, non_blocking=True)
            e_en[s_].record()
        torch.cuda.synchronize()
        e_ms = allreduce_max(sum(e_st[s_].elapsed_time(e_en[s_]) for s_ in range(args.warmup, K + args.warmup)))
        e2e = {"value": ws * p.rows * K / (e_ms * 1e-3), "unit": SFA_UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h}
    cpu = None
    if rank == 0 and ws == 1 and not (args.no_cpu_baseline or args.plain):
        import numpy as np

        import oracle.sfa as osfa
        rng = np.random.default_rng(0)
        probe = sorted(rng.choice(p.rows, size=min(p.rows, 8), replace=False).tolist())
        t0 = time.perf_counter()
        osfa.run(p, inp, rows=probe)
        per = (time.perf_counter() - t0) / len(probe)
        n = int(min(p.rows, max(1, 12.0 / max(per, 1e-9))))
        rows = sorted(rng.choice(p.rows, size=n, replace=False).tolist())
        t0 = time.perf_counter()
        osfa.run(p, inp, rows=rows)
        dt = time.perf_counter() - t0
        cpu = {"value": n / dt, "unit": SFA_UNIT, "cores": blas_threads(), "kind": "oracle",
               "cpu_model": cpu_model(), "nproc": os.cpu_count(),
               "sample": "%d of %d rows (seeded uniform sample), fp64 numpy oracle, %.2f s" % (n, p.rows, dt)}
    line = {
        "metric": SFA_METRIC, "value": ws * p.rows * K / (total_ms * 1e-3), "unit": SFA_UNIT, "n_gpus": ws,
        "steps": K, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD_DESC[args.workload], "rows": p.rows, "selected_pairs": pairs,
                   "l2": "flushed before every timed step (256 MiB write, then a 256 MiB read of a second buffer)",
                   "parallelism": "independent replica per GPU" if ws > 1 else "1 GPU"},
        "effective_tflops": tflops,
        "gathered_gbs": gathered / (ms * 1e-3) / 1e9,
        "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches, "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOAD_DESC))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-stage-events", action="store_true",
                    help="do not record per-kernel CUDA events inside the timed steps")
    ap.add_argument("--plain", action="store_true",
                    help="exactly W warm-up and K timed calls, no clock sampling, e2e or "
                         "CPU baseline (a fixed launch sequence for ncu)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    ws, rank, local = dist_setup()
    if args.workload.startswith("sfa_"):
        rc = sfa_reference(args, rank) if args.impl == "reference" else sfa_main(args, ws, rank, local)
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return rc
    if args.impl == "reference":
        rc = run_reference(args, ws, rank)
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return rc

    import torch

    import sparse_attention_top_n1_b200 as li
    from sparse_attention_top_n1_b200 import build as libbuild
    if not os.path.exists(li.LIB_PATH):
        libbuild.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    p, inp = make_workload(args.workload, rank)
    counts = work_counts(p, inp)
    d = {k: v.to(dev) for k, v in inp.items()}
    pr = li.make_params(p)
    wsb = li.alloc_workspace(pr, dev)
    shape = li.li_output_shape(pr)
    idx = torch.empty(shape, dtype=torch.int32, device=dev)
    val = torch.empty(shape, dtype=torch.float32, device=dev) if p.return_value else None
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    clean = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)   # fp32: summed without a cast

    def flush_l2():
        """Evict L2: write a buffer larger than L2, then read a second one, so
        that the written lines are back in HBM before the next step starts and
        the timed step does not inherit their write-back."""
        flush.zero_()
        clean.sum()
    quant = bool(p.quant)

    def call(q, k, w, qs, ks, aq, ak, bt, oi, ov):
        if quant:
            li.li_quant_indexer(pr, q, k, w, qs, ks, aq, ak, bt, oi, ov, wsb)
        else:
            li.li_indexer(pr, q, k, w, aq, ak, bt, oi, ov, wsb)

    args_dev = (d["query"], d["key"], d["weights"], d.get("q_scale"), d.get("k_scale"),
                d.get("act_q"), d.get("act_k"), d.get("block_table"), idx, val)
    clocks = ClockSampler(local)
    if not args.plain:
        clocks.start()
    # W warm-up steps, then more of the same until the clock sampler has seen
    # the GPU under this load for a while (its period is 200 ms)
    t_warm = time.perf_counter()
    nwarm = 0
    while nwarm < args.warmup or (not args.plain and time.perf_counter() - t_warm < 0.8):
        flush_l2()
        call(*args_dev)
        nwarm += 1
        if nwarm % 16 == 0:
            torch.cuda.synchronize()
    torch.cuda.synchronize()
    flags = li.li_read_device_status(wsb)
    if flags:
        raise SystemExit("device status 0x%x during warm-up" % flags)

    K = args.steps
    mk = lambda: torch.cuda.Event(enable_timing=True)

    def timed_steps(stage_events):
        """K steps, L2 flushed before each outside the timed interval.  With
        stage_events, the library records per-kernel events inside each step
        (which keeps the kernels from overlapping their launch with the
        previous kernel's tail, so the step itself gets a little slower)."""
        starts = [mk() for _ in range(K)]
        ends = [mk() for _ in range(K)]
        prof = [[mk() for _ in range(4)] for _ in range(K)]
        for e in [x for row in prof for x in row]:      # torch creates events lazily
            e.record()
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        nlaunch = 0
        torch.cuda.nvtx.range_push("timed steps%s" % (" (stage events)" if stage_events else ""))
        for s in range(K):
            flush_l2()
            if stage_events:
                li.li_set_profile_events(prof[s])
            torch.cuda.nvtx.range_push("step %d" % s)
            starts[s].record()
            call(*args_dev)
            ends[s].record()
            torch.cuda.nvtx.range_pop()
            nlaunch += li.li_last_launch_count()
        torch.cuda.nvtx.range_pop()
        li.li_set_profile_events(None)
        torch.cuda.synchronize()
        barrier()
        step_ms = [starts[s].elapsed_time(ends[s]) for s in range(K)]
        stage = {"scheduler": [], "score": [], "topk": []}
        if stage_events:
            for s in range(K):
                e = prof[s]
                stage["scheduler"].append(e[0].elapsed_time(e[1]))
                stage["score"].append(e[1].elapsed_time(e[2]))
                stage["topk"].append(e[2].elapsed_time(e[3]))
        return sum(step_ms), stage, nlaunch

    # timed region 1: the job value, nothing between the kernels
    own_ms, _, launches = timed_steps(False)
    total_ms = allreduce_max(own_ms)
    # timed region 2: the same steps with per-kernel events, for the roofline
    staged_ms = 0.0
    stage = {"scheduler": [], "score": [], "topk": []}
    if not args.no_stage_events:
        own_staged, stage, _ = timed_steps(True)
        staged_ms = allreduce_max(own_staged)
    clk = clocks.stop()
    avg = {k: (sum(v) / len(v) if v else float("nan")) for k, v in stage.items()}

    peaks, peak_src = load_peaks()
    score_tflops = counts["flops"] / (avg["score"] * 1e-3) / 1e12
    topk_gbs = counts["topk_bytes"] / (avg["topk"] * 1e-3) / 1e9
    tensor_peak = peaks["bf16_tflops"] * (2.0 if counts["es"] == 1 else 1.0)
    tensor_note = ("bf16 burst peak x2 (nominal 8-bit/bf16 ratio, fp8 and int8 alike), %s" % peak_src
                   if counts["es"] == 1 else "bf16 burst peak (fp16 has the same rate), %s" % peak_src)
    kern = {
        "score": {"bound": "tensor", "achieved": score_tflops, "peak": tensor_peak,
                  "unit": "TFLOP/s", "frac": score_tflops / tensor_peak, "ms": avg["score"],
                  "peak_source": tensor_note,
                  "traffic": traffic_record(args.workload, "score")},
        "topk": {"bound": "hbm", "achieved": topk_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                 "frac": topk_gbs / peaks["hbm_gbs"], "ms": avg["topk"],
                 "peak_source": "hbm copy peak, %s" % peak_src,
                 "traffic": traffic_record(args.workload, "topk")},
    }
    dom = max(("score", "topk"), key=lambda k: kern[k]["ms"])
    roof = {k: kern[dom][k] for k in ("bound", "achieved", "peak", "unit", "frac", "traffic")}
    roof["kernel"] = dom

    n = ws
    value = job_value(p.rows, K, n, total_ms)
    eff_tflops = n * counts["flops"] * K / (total_ms * 1e-3) / 1e12
    whole_frac = max(counts["flops"] / (tensor_peak * 1e12),
                     counts["compulsory_bytes"] / (peaks["hbm_gbs"] * 1e9)) / (total_ms * 1e-3 / K)

    # end to end through the C ABI with host buffers: H2D of the inputs from
    # pinned memory, the call, D2H of the outputs, all inside the timed region
    e2e = None
    if not (args.no_e2e or args.plain):
        host = {k: v.pin_memory() for k, v in inp.items()}
        hidx = torch.empty(shape, dtype=torch.int32).pin_memory()
        hval = torch.empty(shape, dtype=torch.float32).pin_memory() if p.return_value else None
        h2d = sum(v.numel() * v.element_size() for v in host.values())
        d2h = hidx.numel() * 4 + (hval.numel() * 4 if hval is not None else 0)
        e_st = [mk() for _ in range(K + args.warmup)]
        e_en = [mk() for _ in range(K + args.warmup)]
        for s in range(K + args.warmup):
            flush_l2()
            e_st[s].record()
            for k2, v in host.items():
                d[k2].copy_(v, non_blocking=True)
            call(*args_dev)
            hidx.copy_(idx, non_blocking=True)
            if hval is not None:
                hval.copy_(val, non_blocking=True)
            e_en[s].record()
        torch.cuda.synchronize()
        e_ms = allreduce_max(sum(e_st[s].elapsed_time(e_en[s]) for s in range(args.warmup, K + args.warmup)))
        e2e = {"value": n * p.rows * K / (e_ms * 1e-3), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    flags = li.li_read_device_status(wsb)
    if flags:
        raise SystemExit("device status 0x%x after timing" % flags)

    cpu = None
    if rank == 0 and n == 1 and not (args.no_cpu_baseline or args.plain):
        cpu, _, _ = cpu_oracle_sample(p, inp)

    dtype = {"bf16": "bf16", "fp16": "fp16", "e4m3": "fp8_e4m3", "int8": "int8"}[p.dtype_qk]
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": n, "steps": K,
        "warmup": args.warmup, "ms_per_step": total_ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": dtype, "data": "synthetic",
        "config": {"workload": WORKLOAD_DESC[args.workload], "rows": p.rows,
                   "visible_pairs": counts["pairs"], "sparse_count": p.sparse_count,
                   "return_value": p.return_value,
                   "l2": "flushed before every timed step (256 MiB write, then a 256 MiB read of a second buffer)",
                   "parallelism": "independent replica per GPU" if n > 1 else "1 GPU"},
        "ms_per_step_with_stage_events": (staged_ms / K) if staged_ms else None,
        "effective_tflops": eff_tflops,
        "whole_call_roofline_frac": whole_frac,
        "roofline": roof,
        "kernels": kern,
        "stage_ms": avg,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if ws > 1:
        import torch.distributed as dist
        barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
