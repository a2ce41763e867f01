#!/usr/bin/env python
"""Benchmark of the LightningIndexer hot path (scheduler -> score -> Top-k).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step is one full indexer call (all three kernels) over one batch of the
named synthetic workload, with inputs resident in HBM.  The default workload
is the largest of the five configurations: the quantised varlen prefill (TND,
sequences of 2048/4096/8192/16384 tokens, 64 heads, D = 128, fp8 e4m3 q/k
with fp32 dequant scales, k = 2048, right-down causal).  With one GPU the
same run also times the other four configurations (tiny, the TileLang test
shape, DSA prefill and paged decode) and reports each under ``per_config``,
with its stage times, roofline, clocks and oracle baseline.

L2 is flushed before every timed step (a 256 MiB device write, then a
256 MiB read of a second buffer so no dirty lines are left behind), outside
the timed interval; each step is timed with CUDA events on the launching
stream and the per-step times are summed.

Under torchrun (N > 1) the problem is split by query rows: each rank takes a
contiguous row range balanced by visible pairs, keeps its own copy of the
keys and runs its rows through the ordinary entry points (one to three calls
per step).  Nothing crosses ranks on the data path; the job time is the max
over ranks and the value is the problem's rows over that time (strong
scaling).

The JSON line reports queries/s (value), the effective TFLOP/s, per-kernel
rooflines measured live with per-stage CUDA events (each kernel's bound is
the slower of its FLOPs at the tensor peak of its operand type and its bytes
at the HBM peak), an end-to-end figure through the C ABI with host buffers
(copies inside the timed region), and the fp64 oracle timed on the host cores
on a bounded sample (cpu_baseline).  The fp8 and int8 dense tensor peaks are
measured in the same run (cuBLAS through torch, 8192^3, best of 10), since
the driver's peak file holds only bf16.  `--impl reference` times the oracle
alone as the reference arm.
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
DEFAULT_WORKLOAD = "quant_varlen"
# the five configurations of the benchmark, timed together when N = 1
CONFIGS = ("tiny", "cfg2", "dsa_prefill", "paged_decode", "quant_varlen")
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
SFA_METRIC = "sparse attention query rows/s at 1 B200 (the indexer's consumer); % of tensor/HBM roofline"
SFA_UNIT = "rows/s"
RETURN_VALUE = {"tiny": 1, "cfg2": 1, "dsa_prefill": 1, "paged_decode": 0, "quant_varlen": 0,
                "quant_varlen_int8": 0, "quant_int8_pa": 0, "dsa_prefill_window": 1}
SEEDS = {"tiny": 0, "cfg2": 1, "dsa_prefill": 2, "paged_decode": 3, "quant_varlen": 4,
         "quant_int8_pa": 5, "quant_varlen_int8": 6, "dsa_prefill_window": 7}
DTYPE_NAME = {"bf16": "bf16", "fp16": "fp16", "e4m3": "fp8_e4m3", "int8": "int8"}


def make_workload(name, seed_offset=0):
    """The named workload (seed offset only for tests of independent draws)."""
    import synth
    fn = synth.WORKLOADS[name]
    if name in ("tiny",):
        return fn(seed=SEEDS[name] + seed_offset)
    return fn(seed=SEEDS[name] + seed_offset, return_value=RETURN_VALUE[name])


def job_value(rows, steps, max_total_ms):
    """Whole-job queries/s: the problem's rows per step over the slowest rank's time."""
    return rows * steps / (max_total_ms * 1e-3)


def seq_lengths(p, inp):
    """Per-batch query and key lengths (host lists)."""
    aq, ak = inp.get("act_q"), inp.get("act_k")
    B = p.B
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
    return Sq, Sk


def work_counts(p, inp):
    """Host-side algorithmic work of one call: visible pairs, FLOPs, and the
    bytes each kernel must move at least.

    * score kernel: its inputs (query, each key once, weights, scales, block
      table, lengths) plus one fp32 score per visible pair written;
    * Top-k kernel: one fp32 score per visible pair read plus the outputs;
    * whole call: the inputs plus the outputs (the score rows are an
      intermediate and do not count).
    """
    Sq, Sk = seq_lengths(p, inp)
    pairs = 0
    for b in range(p.B):
        if p.sparse_mode == 0:
            pairs += Sq[b] * Sk[b]
        else:
            for i in range(Sq[b]):
                pairs += max(0, min(Sk[b], i + 1 + Sk[b] - Sq[b]))
    es = 1 if p.dtype_qk in ("e4m3", "int8") else 2
    nbytes = lambda t: 0 if t is None else t.numel() * t.element_size()
    keys = sum(Sk)
    inputs = (nbytes(inp["query"]) + keys * p.D * es + nbytes(inp["weights"])
              + nbytes(inp.get("q_scale"))
              + keys * (4 if p.dtype_scale == "fp32" else 2) * int(p.quant)
              + nbytes(inp.get("block_table")) + nbytes(inp.get("act_q")) + nbytes(inp.get("act_k")))
    outputs = p.rows * p.sparse_count * (4 + 4 * p.return_value)
    return dict(pairs=pairs, flops=2.0 * p.N1 * p.D * pairs, compulsory_bytes=inputs + outputs,
                score_bytes=inputs + pairs * 4, topk_bytes=pairs * 4 + outputs, es=es)


def load_peaks():
    if os.path.exists(PEAKS_FILE):
        with open(PEAKS_FILE) as f:
            d = json.load(f)
        return d, "measured (MEASURED_PEAKS.json)"
    print("bench: MEASURED_PEAKS.json is absent; rooflines use the fallback peaks "
          "(6650 GB/s, 1590 TFLOP/s bf16) and say so", file=sys.stderr)
    return FALLBACK_PEAKS, "fallback (MEASURED_PEAKS.json absent)"


def measure_8bit_peaks(dev, n=8192, reps=10):
    """Dense fp8 e4m3 and int8 tensor throughput of this GPU through cuBLAS
    (torch._scaled_mm / torch._int_mm), n^3 GEMMs, best of `reps` after 3
    warm-up calls, CUDA events.  A figure below the bf16 peak is not trusted
    (that library path is not on the 8-bit tensor cores) and left None."""
    import torch
    out = {"how": "torch._scaled_mm e4m3 (bf16 out) and torch._int_mm int8, %d^3, best of %d, CUDA events"
           % (n, reps)}
    g = torch.Generator(device=dev)
    g.manual_seed(0)

    def best(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return 2.0 * n ** 3 / (min(ts) * 1e-3) / 1e12

    try:
        a = torch.randn(n, n, device=dev, generator=g).to(torch.float8_e4m3fn)
        b = torch.randn(n, n, device=dev, generator=g).to(torch.float8_e4m3fn).t()
        one = torch.ones((), device=dev, dtype=torch.float32)
        out["fp8_tflops"] = best(lambda: torch._scaled_mm(a, b, scale_a=one, scale_b=one,
                                                          out_dtype=torch.bfloat16))
        del a, b
    except Exception as e:  # pragma: no cover - depends on the torch build
        out["fp8_tflops"] = None
        out["fp8_error"] = str(e)[:120]
    try:
        a = torch.randint(-64, 64, (n, n), device=dev, dtype=torch.int8, generator=g)
        b = torch.randint(-64, 64, (n, n), device=dev, dtype=torch.int8, generator=g)
        out["int8_tops"] = best(lambda: torch._int_mm(a, b))
        del a, b
    except Exception as e:  # pragma: no cover
        out["int8_tops"] = None
        out["int8_error"] = str(e)[:120]
    torch.cuda.empty_cache()
    return out


def tensor_peak(dtype_qk, peaks, peak_src, p8):
    """(peak TFLOP/s, description) of the score MMA's operand type."""
    bf16 = peaks["bf16_tflops"]
    if dtype_qk in ("bf16", "fp16"):
        return bf16, "bf16 dense burst peak (fp16 has the same rate), %s" % peak_src
    key = "fp8_tflops" if dtype_qk == "e4m3" else "int8_tops"
    v = (p8 or {}).get(key)
    if v and v >= bf16:
        return v, "%s dense peak measured in this run (%s)" % ("fp8" if dtype_qk == "e4m3" else "int8", p8["how"])
    return 2.0 * bf16, "assumed: 2x the bf16 peak (nominal 8-bit/16-bit ratio; the in-run measurement failed)"


def roofline(ms, flops, nbytes, t_peak, t_src, hbm, hbm_src, traffic=None):
    """Bound = the slower of flops at the tensor peak and bytes at HBM bandwidth."""
    t_t = flops / (t_peak * 1e12) if flops else 0.0
    t_b = nbytes / (hbm * 1e9)
    sec = ms * 1e-3
    if t_t >= t_b:
        r = {"bound": "tensor", "achieved": flops / sec / 1e12, "peak": t_peak, "unit": "TFLOP/s",
             "peak_source": t_src}
    else:
        r = {"bound": "hbm", "achieved": nbytes / sec / 1e9, "peak": hbm, "unit": "GB/s",
             "peak_source": "HBM copy peak, %s" % hbm_src}
    r["frac"] = max(t_t, t_b) / sec
    r["ms"] = ms
    r["algorithmic_bytes"] = nbytes
    r["flops"] = flops
    r["traffic"] = traffic
    return r


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
    """Rank, world size and this rank's GPU.  The process group carries only
    the barriers and the max of the timings: NCCL by default; LI_BENCH_BACKEND
    =gloo runs it on the host, which lets several ranks share a GPU (their
    kernels never wait on one another) to exercise the sharded path."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime

        import torch
        import torch.distributed as dist
        local = local % max(1, torch.cuda.device_count())
        torch.cuda.set_device(local)
        dist.init_process_group(os.environ.get("LI_BENCH_BACKEND", "nccl"),
                                timeout=datetime.timedelta(seconds=120))
    return ws, rank, local


def allreduce_max(x, device=None):
    """Max of a host float over all ranks (timing only; no data-path use)."""
    import torch
    import torch.distributed as dist
    if not dist.is_initialized():
        return x
    if device is None:
        device = "cpu" if dist.get_backend() == "gloo" else "cuda"
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


def cpu_oracle_sample(p, inp, budget_s=12.0, seed=0):
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
    per_row = (time.perf_counter() - t0) / len(probe)
    n = int(min(R, max(len(probe), budget_s / max(per_row, 1e-9))))
    rows = sorted(rng.choice(R, size=n, replace=False).tolist())
    t0 = time.perf_counter()
    oracle.run(p, inp, rows=rows, nthreads=nthreads)
    dt = time.perf_counter() - t0
    return {"value": len(rows) / dt, "unit": UNIT, "cores": nthreads, "kind": "oracle",
            "cpu_model": cpu_model(), "nproc": os.cpu_count(),
            "sample": "%d of %d query rows (seeded uniform sample), fp64 C oracle, %.2f s"
                      % (len(rows), R, dt)}


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
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "f64",
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


# ------------------------------------------------------------------ indexer

def make_flush(dev):
    import torch
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    clean = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)   # fp32: summed without a cast

    def flush_l2():
        """Evict L2: write a buffer larger than L2, then read a second one, so
        that the written lines are back in HBM before the next step starts and
        the timed step does not inherit their write-back."""
        flush.zero_()
        clean.sum()
    return flush_l2


class Calls:
    """This rank's calls of one step: the whole problem at N = 1, else the
    pieces of its row range (sparse_attention_top_n1_b200.shard)."""

    def __init__(self, li, p, inp, dev, ws, rank):
        import dataclasses

        import torch

        from sparse_attention_top_n1_b200 import shard
        self.li = li
        self.p = p
        self.quant = bool(p.quant)
        shape = (p.rows, p.sparse_count)
        self.idx = torch.empty(shape, dtype=torch.int32, device=dev)
        self.val = torch.empty(shape, dtype=torch.float32, device=dev) if p.return_value else None
        self.d = {k: v.to(dev) for k, v in inp.items()}
        self.host_inputs = inp
        if ws == 1:
            self.pieces = [(p, self.d, 0, p.rows, inp)]
        else:
            plan = shard.shard(p, ws, inp.get("act_q"), inp.get("act_k"), inp.get("cmp_residual_k"))[rank]
            to_dev = lambda a: torch.from_numpy(a).to(dev)
            self.pieces = [(dataclasses.replace(p, **pc.fields), shard.piece_inputs(pc, p, self.d, to_dev),
                            pc.r0, pc.r1, shard.piece_inputs(pc, p, inp)) for pc in plan]
        self.calls = []
        for sp, sd, r0, r1, _ in self.pieces:
            pr = li.make_params(sp)
            if sd.get("cmp_residual_k") is not None:
                pr.cmp_residual_k = sd["cmp_residual_k"].data_ptr()
            wsb = li.alloc_workspace(pr, dev)
            oi = self.idx[r0:r1]
            ov = self.val[r0:r1] if self.val is not None else None
            self.calls.append((pr, sd, wsb, oi, ov))
        self.rows_here = sum(r1 - r0 for _, _, r0, r1, _ in self.pieces)

    def __call__(self, prof=None):
        li = self.li
        n = 0
        for j, (pr, sd, wsb, oi, ov) in enumerate(self.calls):
            if prof is not None:
                li.li_set_profile_events(prof[j])
            if self.quant:
                li.li_quant_indexer(pr, sd["query"], sd["key"], sd["weights"], sd.get("q_scale"),
                                    sd.get("k_scale"), sd.get("act_q"), sd.get("act_k"),
                                    sd.get("block_table"), oi, ov, wsb)
            else:
                li.li_indexer(pr, sd["query"], sd["key"], sd["weights"], sd.get("act_q"),
                              sd.get("act_k"), sd.get("block_table"), oi, ov, wsb)
            n += li.li_last_launch_count()
        if prof is not None:
            li.li_set_profile_events(None)
        return n

    def device_flags(self):
        f = 0
        for _, _, wsb, _, _ in self.calls:
            f |= self.li.li_read_device_status(wsb)
        return f


def e2e_pieces(p):
    """Row pieces for the end-to-end leg: one per 4096 query rows, up to 8."""
    return max(1, min(8, p.rows // 4096))


def time_e2e_pipelined(li, p, inp, calls, dev, npieces, steps, warmup, flush_l2):
    """End to end with host buffers, the transfers overlapped with the work:
    the query rows are split into `npieces` contiguous, pair-balanced pieces
    (the same row split as the multi-GPU path), each its own li_indexer /
    li_quant_indexer call.  One stream copies the key-side inputs and then
    each piece's query-side inputs host -> device, one runs the calls in
    order as their inputs land, one copies each piece's output rows back as
    it completes; the timed region runs from the first copy to the last.
    Every byte a call reads is copied every step.  The pieces' outputs are
    checked bit for bit against the whole-problem call's."""
    import dataclasses

    import torch

    from sparse_attention_top_n1_b200 import shard
    aq, ak, cr = inp.get("act_q"), inp.get("act_k"), inp.get("cmp_residual_k")
    cost = shard.row_costs(p, aq, ak, cr)
    plan = [pc for r0, r1 in shard.split_rows(cost, npieces) for pc in shard.pieces_for_range(p, r0, r1, aq, ak, cr)]
    d = calls.d
    pin = lambda t: t.contiguous().pin_memory()
    # key-side tensors, whole, once per step (pieces share them)
    key_side = [k for k in ("key", "k_scale", "block_table") if d.get(k) is not None]
    shared = [(pin(inp[k]), d[k]) for k in key_side]
    pieces = []
    for pc in plan:
        sp = dataclasses.replace(p, **pc.fields)
        dev_in = shard.piece_inputs(pc, p, d, lambda a: torch.from_numpy(a).to(dev))
        host_in = shard.piece_inputs(pc, p, inp)
        copies = [(pin(host_in[k]), dev_in[k]) for k in dev_in if k not in key_side]
        pr = li.make_params(sp)
        if dev_in.get("cmp_residual_k") is not None:
            pr.cmp_residual_k = dev_in["cmp_residual_k"].data_ptr()
        wsb = li.alloc_workspace(pr, dev)
        oi = calls.idx[pc.r0:pc.r1]
        ov = calls.val[pc.r0:pc.r1] if calls.val is not None else None
        hi = torch.empty(oi.shape, dtype=oi.dtype).pin_memory()
        hv = torch.empty(ov.shape, dtype=ov.dtype).pin_memory() if ov is not None else None
        pieces.append((pr, dev_in, copies, wsb, oi, ov, hi, hv))
    # the whole-problem call's result (the last timed call left it here): the
    # pieces must reproduce it bit for bit
    ref_i = calls.idx.clone()
    ref_v = calls.val.clone() if calls.val is not None else None
    h2d = sum(h.numel() * h.element_size() for h, _ in shared)
    h2d += sum(h.numel() * h.element_size() for pc in pieces for h, _ in pc[2])
    d2h = p.rows * p.sparse_count * (4 + 4 * p.return_value)
    s_in, s_run, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    main = torch.cuda.current_stream(dev)
    mk = lambda: torch.cuda.Event(enable_timing=True)
    st, en = [mk() for _ in range(steps + warmup)], [mk() for _ in range(steps + warmup)]
    for s_ in range(steps + warmup):
        flush_l2()
        st[s_].record(main)
        for x in (s_in, s_run, s_out):
            x.wait_stream(main)
        with torch.cuda.stream(s_in):
            for h, dv in shared:
                dv.copy_(h, non_blocking=True)
        for pr, dev_in, copies, wsb, oi, ov, hi, hv in pieces:
            with torch.cuda.stream(s_in):
                for h, dv in copies:
                    dv.copy_(h, non_blocking=True)
            landed = s_in.record_event()
            s_run.wait_event(landed)
            with torch.cuda.stream(s_run):
                if p.quant:
                    li.li_quant_indexer(pr, dev_in["query"], dev_in["key"], dev_in["weights"], dev_in.get("q_scale"),
                                        dev_in.get("k_scale"), dev_in.get("act_q"), dev_in.get("act_k"),
                                        dev_in.get("block_table"), oi, ov, wsb)
                else:
                    li.li_indexer(pr, dev_in["query"], dev_in["key"], dev_in["weights"], dev_in.get("act_q"),
                                  dev_in.get("act_k"), dev_in.get("block_table"), oi, ov, wsb)
            done = s_run.record_event()
            s_out.wait_event(done)
            with torch.cuda.stream(s_out):
                hi.copy_(oi, non_blocking=True)
                if hv is not None:
                    hv.copy_(ov, non_blocking=True)
        main.wait_stream(s_out)
        main.wait_stream(s_run)
        en[s_].record(main)
    torch.cuda.synchronize()
    for pr, dev_in, copies, wsb, oi, ov, hi, hv in pieces:
        f = li.li_read_device_status(wsb)
        if f:
            raise SystemExit("end-to-end piece: device status 0x%x" % f)
    if not torch.equal(calls.idx, ref_i) or (ref_v is not None and not torch.equal(
            calls.val.view(torch.int32), ref_v.view(torch.int32))):
        raise SystemExit("end-to-end pieces differ from the whole-problem call")
    e_ms = sum(st[s_].elapsed_time(en[s_]) for s_ in range(warmup, steps + warmup))
    return {"value": p.rows * steps / (e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "pieces": len(pieces),
            "overlap": "host->device copies, the calls and device->host copies on three streams, by row piece"}


def time_indexer(name, args, ctx, steps, warmup, cpu_budget, with_e2e=True):
    """Time `steps` calls of workload `name` on this rank; returns the record."""
    import torch
    li, dev, ws, rank = ctx["li"], ctx["dev"], ctx["ws"], ctx["rank"]
    p, inp = make_workload(name)
    counts = work_counts(p, inp)
    calls = Calls(li, p, inp, dev, ws, rank)
    flush_l2 = ctx["flush"]
    clocks = ClockSampler(ctx["local"])
    if not args.plain:
        clocks.start()
    # W warm-up steps, then more of the same until the clock sampler has seen
    # the GPU under this load for a while (its period is 200 ms)
    t_warm = time.perf_counter()
    nwarm = 0
    while nwarm < warmup or (not args.plain and time.perf_counter() - t_warm < 0.8):
        flush_l2()
        calls()
        nwarm += 1
        if nwarm % 16 == 0:
            torch.cuda.synchronize()
    torch.cuda.synchronize()
    flags = calls.device_flags()
    if flags:
        raise SystemExit("%s: device status 0x%x during warm-up" % (name, flags))

    K = steps
    mk = lambda: torch.cuda.Event(enable_timing=True)
    ncalls = len(calls.calls)

    def timed_steps(stage_events):
        """K steps, L2 flushed before each outside the timed interval.  With
        stage_events, the library records per-kernel events inside each call
        (which keeps the kernels from overlapping their launch with the
        previous kernel's tail, so the step itself gets a little slower)."""
        starts = [mk() for _ in range(K)]
        ends = [mk() for _ in range(K)]
        prof = [[[mk() for _ in range(4)] for _ in range(ncalls)] for _ in range(K)]
        for e in [x for st in prof for c in st for x in c]:      # torch creates events lazily
            e.record()
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        nlaunch = 0
        torch.cuda.nvtx.range_push("timed steps%s" % (" (stage events)" if stage_events else ""))
        for s in range(K):
            flush_l2()
            torch.cuda.nvtx.range_push("step %d" % s)
            starts[s].record()
            nlaunch += calls(prof[s] if stage_events else None)
            ends[s].record()
            torch.cuda.nvtx.range_pop()
        torch.cuda.nvtx.range_pop()
        torch.cuda.synchronize()
        barrier()
        step_ms = [starts[s].elapsed_time(ends[s]) for s in range(K)]
        stage = {"scheduler": [], "score": [], "topk": []}
        if stage_events:
            for s in range(K):
                sch = sc = tk = 0.0
                for e in prof[s]:
                    sch += e[0].elapsed_time(e[1])
                    sc += e[1].elapsed_time(e[2])
                    tk += e[2].elapsed_time(e[3])
                stage["scheduler"].append(sch)
                stage["score"].append(sc)
                stage["topk"].append(tk)
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
    # the slowest rank's stage times (the roofline of the job)
    avg = {k: allreduce_max(v) for k, v in avg.items()}

    peaks, peak_src, p8 = ctx["peaks"], ctx["peak_src"], ctx["p8"]
    tpk, tsrc = tensor_peak(p.dtype_qk, peaks, peak_src, p8)
    hbm = peaks["hbm_gbs"]
    share = 1.0 / ws            # each rank does about 1/N of the pairs and rows
    kern = {}
    if avg["score"] == avg["score"]:          # not NaN
        kern["score"] = roofline(avg["score"], counts["flops"] * share,
                                 counts["score_bytes"] * share, tpk, tsrc, hbm, peak_src,
                                 traffic_record(name, "score") if ws == 1 else None)
        kern["topk"] = roofline(avg["topk"], 0.0, counts["topk_bytes"] * share, tpk, tsrc, hbm,
                                peak_src, traffic_record(name, "topk") if ws == 1 else None)
    ms_step = total_ms / K
    whole = roofline(ms_step, counts["flops"], counts["compulsory_bytes"], tpk * ws, tsrc,
                     hbm * ws, peak_src)
    dom = max(kern, key=lambda k: kern[k]["ms"]) if kern else None
    roof = None
    if dom:
        roof = {k: kern[dom][k] for k in ("bound", "achieved", "peak", "unit", "frac", "traffic",
                                          "peak_source")}
        roof["kernel"] = dom + "_kernel"

    # end to end through the C ABI with host buffers: H2D of this rank's inputs
    # from pinned memory, the call, D2H of its output rows, all timed
    e2e = None
    npieces = e2e_pieces(p) if ws == 1 else 1
    if with_e2e and not (args.no_e2e or args.plain) and npieces > 1:
        e2e = time_e2e_pipelined(li, p, inp, calls, dev, npieces, K, warmup, flush_l2)
    elif with_e2e and not (args.no_e2e or args.plain):
        # every device tensor a call reads is refreshed once per step (pieces
        # that share one, such as a paged pool, copy it once)
        hosts = []
        h2d = 0
        seen = set()
        for (sp, sd, r0, r1, hin), (pr, dd, wsb, oi, ov) in zip(calls.pieces, calls.calls):
            hp = {}
            for k, v in hin.items():
                if k not in dd or (dd[k].data_ptr(), dd[k].numel()) in seen:
                    continue
                seen.add((dd[k].data_ptr(), dd[k].numel()))
                hp[k] = v.contiguous().pin_memory()
            h2d += sum(v.numel() * v.element_size() for v in hp.values())
            hosts.append((hp, dd))
        hidx = torch.empty(calls.idx.shape, dtype=torch.int32).pin_memory()
        hval = torch.empty(calls.idx.shape, dtype=torch.float32).pin_memory() if p.return_value else None
        d2h = calls.rows_here * p.sparse_count * (4 + 4 * p.return_value)
        e_st = [mk() for _ in range(K + warmup)]
        e_en = [mk() for _ in range(K + warmup)]
        for s in range(K + warmup):
            flush_l2()
            e_st[s].record()
            for hp, dd in hosts:
                for k2, v in hp.items():
                    dd[k2].copy_(v, non_blocking=True)
            calls()
            for _, _, r0, r1, _ in calls.pieces:
                hidx[r0:r1].copy_(calls.idx[r0:r1], non_blocking=True)
                if hval is not None:
                    hval[r0:r1].copy_(calls.val[r0:r1], non_blocking=True)
            e_en[s].record()
        torch.cuda.synchronize()
        e_ms = allreduce_max(sum(e_st[s].elapsed_time(e_en[s]) for s in range(warmup, K + warmup)))
        e2e = {"value": p.rows * K / (e_ms * 1e-3), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    flags = calls.device_flags()
    if flags:
        raise SystemExit("%s: device status 0x%x after timing" % (name, flags))

    cpu = None
    if rank == 0 and ws == 1 and cpu_budget > 0 and not (args.no_cpu_baseline or args.plain):
        cpu = cpu_oracle_sample(p, inp, budget_s=cpu_budget)

    rec = {
        "workload": name, "config": WORKLOAD_DESC[name], "dtype": DTYPE_NAME[p.dtype_qk],
        "rows": p.rows, "visible_pairs": counts["pairs"], "sparse_count": p.sparse_count,
        "return_value": p.return_value, "steps": K, "warmup": warmup,
        "ms_per_step": ms_step, "value": job_value(p.rows, K, total_ms), "unit": UNIT,
        "ms_per_step_with_stage_events": (staged_ms / K) if staged_ms else None,
        "effective_tflops": counts["flops"] * K / (total_ms * 1e-3) / 1e12,
        "whole_call_roofline": {k: whole[k] for k in ("bound", "achieved", "peak", "unit", "frac")},
        "roofline": roof, "kernels": kern, "stage_ms": avg,
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches, "clocks": clk,
        "calls_per_step_this_rank": len(calls.calls),
    }
    del calls
    torch.cuda.empty_cache()
    return rec


# ------------------------------------------------------------------ sparse attention

def sfa_workload(name, seed_offset=0):
    from synth import sfa as ssfa
    if name == "sfa_prefill":
        return ssfa.make_sfa_prefill(seed=9 + seed_offset)
    return ssfa.make_sfa_decode(seed=10 + seed_offset)


def sfa_counts(p, inp):
    """Valid (row, selected key) pairs, FLOPs, gathered bytes and the bytes one
    call must move at least (query, output, lse, index rows, and each distinct
    selected key/value row once)."""
    import numpy as np
    idx = inp["sparse_indices"].reshape(p.rows, p.sparse_count).numpy()
    valid = idx >= 0
    pairs = int(valid.sum())
    flops = 2.0 * p.N1 * (p.D + p.Dv) * pairs
    gathered = pairs * (p.D + p.Dv) * 2
    # distinct selected keys per batch
    if p.layout_q == "BSND":
        bounds = [(b * p.S1, (b + 1) * p.S1) for b in range(p.B)]
    else:
        c = [0] + inp["act_q"].tolist()
        bounds = [(c[b], c[b + 1]) for b in range(p.B)]
    distinct = 0
    for lo, hi in bounds:
        sel = idx[lo:hi][valid[lo:hi]]
        distinct += int(np.unique(sel).size)
    io = p.rows * p.N1 * (p.D + p.Dv) * 2 + idx.size * 4 + p.rows * p.N1 * 4
    return pairs, flops, gathered, io + distinct * (p.D + p.Dv) * 2


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


def sfa_e2e_pipelined(li, p, inp, d, pr_whole, out, lse, status, npieces, steps, warmup, flush_l2):
    """End to end with host buffers for a one-batch BSND problem, transfers
    overlapped with the work: the query rows are split into `npieces`
    contiguous pieces (one li_sparse_attention call each); one stream copies
    the keys and values and then each piece's query and index rows in, one
    runs the calls as their inputs land, one copies each piece's output rows
    out.  The pieces' outputs are checked bit for bit against the whole call."""
    import dataclasses

    import torch
    dev = out.device
    ref_o, ref_l = out.clone(), lse.clone()
    shared = [(inp[k].contiguous().pin_memory(), d[k]) for k in ("key", "value")]
    bounds = [p.rows * j // npieces for j in range(npieces + 1)]
    pieces = []
    for r0, r1 in zip(bounds, bounds[1:]):
        pr = li.make_sfa_params(dataclasses.replace(p, S1=r1 - r0))
        q_d, i_d = d["query"][:, r0:r1], d["sparse_indices"][r0:r1]
        copies = [(inp["query"][:, r0:r1].contiguous().pin_memory(), q_d),
                  (inp["sparse_indices"][r0:r1].contiguous().pin_memory(), i_d)]
        ho = torch.empty(out[r0:r1].shape, dtype=out.dtype).pin_memory()
        pieces.append((pr, q_d, i_d, copies, out[r0:r1], lse[r0:r1], ho))
    h2d = sum(h.numel() * h.element_size() for h, _ in shared)
    h2d += sum(h.numel() * h.element_size() for pc in pieces for h, _ in pc[3])
    d2h = out.numel() * out.element_size()
    s_in, s_run, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    main = torch.cuda.current_stream(dev)
    mk = lambda: torch.cuda.Event(enable_timing=True)
    st, en = [mk() for _ in range(steps + warmup)], [mk() for _ in range(steps + warmup)]
    for s_ in range(steps + warmup):
        flush_l2()
        st[s_].record(main)
        for x in (s_in, s_run, s_out):
            x.wait_stream(main)
        with torch.cuda.stream(s_in):
            for h, dv in shared:
                dv.copy_(h, non_blocking=True)
        for pr, q_d, i_d, copies, o_d, l_d, ho in pieces:
            with torch.cuda.stream(s_in):
                for h, dv in copies:
                    dv.copy_(h, non_blocking=True)
            landed = s_in.record_event()
            s_run.wait_event(landed)
            with torch.cuda.stream(s_run):
                li.li_sparse_attention(pr, q_d, d["key"], d["value"], i_d, None, None, None, o_d, l_d, status)
            done = s_run.record_event()
            s_out.wait_event(done)
            with torch.cuda.stream(s_out):
                ho.copy_(o_d, non_blocking=True)
        main.wait_stream(s_out)
        main.wait_stream(s_run)
        en[s_].record(main)
    torch.cuda.synchronize()
    if not (torch.equal(out.view(torch.int16), ref_o.view(torch.int16))
            and torch.equal(lse.view(torch.int32), ref_l.view(torch.int32))):
        raise SystemExit("sparse attention end-to-end pieces differ from the whole call")
    e_ms = allreduce_max(sum(st[s_].elapsed_time(en[s_]) for s_ in range(warmup, steps + warmup)))
    return {"value": p.rows * steps / (e_ms * 1e-3), "unit": SFA_UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "pieces": len(pieces),
            "overlap": "host->device copies, the calls and device->host copies on three streams, by row piece"}


def sfa_main(args, ws, rank, local):
    """One step = one li_sparse_attention call over the whole workload; under
    torchrun every rank runs its own problem of the same shape (weak scaling)."""
    import torch

    import sparse_attention_top_n1_b200 as li
    from sparse_attention_top_n1_b200 import build as libbuild
    if not os.path.exists(li.LIB_PATH):
        libbuild.build()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    p, inp = sfa_workload(args.workload, rank)
    pairs, flops, gathered, compulsory = sfa_counts(p, inp)
    d = {k: v.to(dev) for k, v in inp.items()}
    pr = li.make_sfa_params(p)
    out = torch.empty((p.rows, p.N1, p.Dv), dtype=d["query"].dtype, device=dev)
    lse = torch.empty((p.rows, p.N1), dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    flush_l2 = make_flush(dev)

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
    kern = roofline(ms, flops, compulsory, peaks["bf16_tflops"],
                    "bf16 dense burst peak, %s" % peak_src, peaks["hbm_gbs"], peak_src,
                    traffic_record(args.workload, "sfa"))
    roof = {k: kern[k] for k in ("bound", "achieved", "peak", "unit", "frac", "traffic", "peak_source")}
    roof["kernel"] = "sfa_kernel"
    e2e = None
    sfa_pieces = (min(8, p.rows // 2048) if (p.layout_q == "BSND" and p.B == 1 and "act_q" not in inp)
                  else 1)
    if not (args.no_e2e or args.plain) and sfa_pieces > 1:
        e2e = sfa_e2e_pipelined(li, p, inp, d, pr, out, lse, status, sfa_pieces, K, args.warmup, flush_l2)
        e2e["value"] *= ws
    elif not (args.no_e2e or args.plain):
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
        "effective_tflops": flops / (ms * 1e-3) / 1e12,
        "gathered_gbs": gathered / (ms * 1e-3) / 1e9,
        "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches, "clocks": clk,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def summary(rec):
    """The per-config entry of the JSON line."""
    keep = ("config", "dtype", "rows", "visible_pairs", "steps", "ms_per_step", "value", "unit",
            "effective_tflops", "stage_ms", "roofline", "kernels", "whole_call_roofline",
            "cpu_baseline", "e2e", "gpu_launches", "clocks")
    return {k: rec[k] for k in keep}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOAD_DESC))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="time only --workload (no per_config records of the other configurations)")
    ap.add_argument("--no-stage-events", action="store_true",
                    help="do not record per-kernel CUDA events inside the timed steps")
    ap.add_argument("--plain", action="store_true",
                    help="exactly W warm-up and K timed calls of --workload, no clock sampling, "
                         "e2e, CPU baseline or per-config records (a fixed launch sequence for ncu)")
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
    peaks, peak_src = load_peaks()
    p8 = None if args.plain else measure_8bit_peaks(dev)
    ctx = {"li": li, "dev": dev, "ws": ws, "rank": rank, "local": local, "peaks": peaks,
           "peak_src": peak_src, "p8": p8, "flush": make_flush(dev)}

    head = time_indexer(args.workload, args, ctx, args.steps, args.warmup, cpu_budget=12.0)
    per_config = None
    if ws == 1 and not (args.plain or args.no_per_config):
        per_config = {}
        pc_steps = max(3, min(args.steps, 10))
        for name in CONFIGS:
            if name == args.workload:
                per_config[name] = summary(head)
                continue
            per_config[name] = summary(time_indexer(name, args, ctx, pc_steps, 3, cpu_budget=4.0))

    line = {
        "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": head["dtype"],
        "data": "synthetic",
        "config": {"workload": head["config"], "rows": head["rows"],
                   "visible_pairs": head["visible_pairs"], "sparse_count": head["sparse_count"],
                   "return_value": head["return_value"],
                   "l2": "flushed before every timed step (256 MiB write, then a 256 MiB read of a second buffer)",
                   "parallelism": ("query rows split over %d GPUs, balanced by visible pairs, keys replicated, "
                                   "no data-path collective" % ws) if ws > 1 else "1 GPU"},
        "ms_per_step_with_stage_events": head["ms_per_step_with_stage_events"],
        "effective_tflops": head["effective_tflops"],
        "whole_call_roofline": head["whole_call_roofline"],
        "roofline": head["roofline"],
        "kernels": head["kernels"],
        "stage_ms": head["stage_ms"],
        "cpu_baseline": head["cpu_baseline"],
        "e2e": head["e2e"],
        "gpu_launches": head["gpu_launches"],
        "clocks": head["clocks"],
        "tensor_peaks_8bit": p8,
        "per_config": per_config,
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
