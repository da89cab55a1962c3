"""Benchmark of the FP8 paged decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload gqa|ragged|wide|long] [--no-bf16] [--no-cpu-baseline]
                    [--sweep]

A step is one pass of the whole hot path over one decode batch:
kvq_append (the new token of every sequence) -> kvq_validate (page tags ->
abort mask) -> kvq_decode (split-KV attention + log-sum-exp combine).  The
default workload is the GQA decode batch: 32 sequences x 8,192 tokens, page
16, 64 query / 8 KV heads, head_dim 128, E4M3 cache with per-head scales.
The cache (537 MB of codes) is larger than L2, so no flush is needed.

`value` is KV GB/s: cache bytes one decode step reads / device time per step
(CUDA events, steps replayed from a CUDA graph, max over ranks).  N > 1 runs
N independent replicas (one per GPU, no collective on the data path) and
reports the aggregate.  `--impl reference` times the CPU oracle on a bounded
sample of the same workload.

The JSON line also carries: `roofline` (the decode call against the measured
HBM copy bandwidth, or for the wide shape the measured bf16 tensor peak),
`e2e` (the step through the Python API with its inputs copied from pinned
host memory and its results read back every step, host traffic overlapped
with the neighbouring steps; serial and eager forms beside it),
`cpu_baseline` (the oracle on host cores), the BF16 cache on the same shape,
the bulk prompt quantize, clocks sampled during the timed region and the
number of kernel launches timed.  `--workload long` runs the 1,000-step loop
with the tag check's cost; `--sweep` the FP8 / BF16 capacity and
concurrency sweep.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "FP8 paged decode attention: KV GB/s (% of HBM peak) and decode tokens/s"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="gqa")
    ap.add_argument("--num-ctas", type=int, default=0)
    ap.add_argument("--no-bf16", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--loop-steps", type=int, default=1000,
                    help="decode steps of the long workload's loop")
    ap.add_argument("--sweep", action="store_true",
                    help="capacity and concurrency sweep (FP8 vs BF16 at B = 1..64) instead of the bench line")
    ap.add_argument("--seqs", type=int, default=0,
                    help="keep only the first N sequences (smaller case for profiling)")
    return ap.parse_args()


def measured_traffic(workload, seqs):
    """DRAM bytes per decode launch from the committed ncu record, or None when
    the kernel source changed since the capture or the workload differs."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if seqs or not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    for r in rec.values():
        src = os.path.join(ROOT, r["source"])
        if not os.path.exists(src) or r.get("workload") != workload:
            continue
        h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        if h == r["source_sha256_prefix"]:
            return r["dram_bytes_per_launch"]
    return None


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def tensor_peak():
    """Dense bf16 TFLOP/s of this GPU (burst: the decode launch is timed on its own)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    return FALLBACK_BF16_TFLOPS, "fallback"


def is_wide(spec) -> bool:
    """The 128-query-head, one-KV-head shape served by the tensor-core kernel."""
    return spec.num_q_heads // spec.num_kv_heads >= 64


def decode_roofline(spec, wl, alg_bytes, ms_dec, traffic):
    """Roofline of one kvq_decode launch.  The 8-head kernel moves bytes
    (bound: HBM).  The wide kernel is a pair of dense contractions per token,
    QK^T (a bf16 query against keys that are exact in f16) and PV (f16), so it
    is bound by the tensor cores at the f16/bf16 rate: 2 * Hq * (Dk + Dv) FLOPs
    per decoded token."""
    if is_wide(spec):
        tokens = int(np.minimum(wl.seq_lens, wl.max_pages * spec.page_size).sum())
        flops = 2.0 * spec.num_q_heads * (spec.head_dim_k + spec.head_dim_v) * tokens
        peak, kind = tensor_peak()
        achieved = flops / (ms_dec * 1e-3) / 1e12
        return {"bound": "tensor",
                "kernel": "kvq_decode (wide_prep_kernel + wide_decode_kernel + lse_combine_kernel)",
                "achieved": achieved, "peak": peak, "peak_kind": kind + " (bf16 burst)",
                "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                "algorithmic_flops_per_launch": flops, "algorithmic_bytes_per_launch": alg_bytes,
                "ms_per_launch": ms_dec}
    hbm, kind = peaks()
    achieved = alg_bytes / (ms_dec * 1e-3) / 1e9
    return {"bound": "hbm", "kernel": "kvq_decode (gqa_decode_kernel + lse_combine_kernel)",
            "achieved": achieved, "peak": hbm, "peak_kind": kind, "unit": "GB/s",
            "frac": achieved / hbm, "traffic": traffic,
            "algorithmic_bytes_per_launch": alg_bytes, "ms_per_launch": ms_dec}


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML reads only)
# ---------------------------------------------------------------------------
class ClockSampler:
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting", 0x1: "gpu_idle", 0x10: "sync_boost"}

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.ok = False
        self.samples = []
        self.period = period_s
        try:
            import pynvml
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            try:
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report nothing rather than guess
            self.err = str(e)

    def _run(self):
        nv = self.nv
        while not self.stop:
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((sm, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.stop = False
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self.stop = True
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": "NVML unavailable" if not self.ok else "no samples"}
        mhz = [s for s, _ in self.samples]
        bits = 0
        for _, r in self.samples:
            bits |= r
        reasons = sorted(n for b, n in self.REASONS.items() if bits & b and n != "gpu_idle")
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(mhz)}


# ---------------------------------------------------------------------------
# timing helpers
# ---------------------------------------------------------------------------
def time_graph(graph, K, stream):
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(K):
        graph.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / K


def capture(fn, stream):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    return g


def dist_setup(args):
    """One process per GPU under torchrun (NCCL); without CUDA (the multi-rank
    tests on the host) the same plumbing runs over gloo."""
    if args.gpus <= 1 and "WORLD_SIZE" not in os.environ:
        return 0, 1, 0
    import torch.distributed as dist
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if torch.cuda.is_available():
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    return rank, world, local


def max_over_ranks(x: float, world: int) -> float:
    """The largest of the ranks' values (timings are taken as the slowest rank's)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(world: int, bytes_per_rank: float, ms_max: float) -> float:
    """Whole-job throughput: every rank's bytes over the slowest rank's time."""
    return world * bytes_per_rank / (ms_max * 1e-3) / 1e9


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


# ---------------------------------------------------------------------------
# CPU oracle baseline (bounded sample of the same workload)
# ---------------------------------------------------------------------------
def oracle_sample(spec_name, n_groups, seed=0):
    """Oracle cache for the first (sequence, KV head) groups of the workload.

    Returns (step, kv_bytes, description): step() runs the oracle's
    append (new tokens) + validate + decode (the groups' query heads)."""
    import oracle
    from fp8_kv_paged_kvq_b200 import workloads as W
    full = W.spec_by_name(spec_name, seed)
    H, G = full.num_kv_heads, full.group
    nseq = min(full.B, -(-n_groups // H))
    n_groups = min(n_groups, nseq * H)
    spec = W.Spec(full.name + "_sample", list(full.seq_lens)[:nseq], full.page_size,
                  full.num_q_heads, H, full.head_dim_k, full.head_dim_v, v_alias=full.v_alias,
                  kv_dtype=full.kv_dtype, scale_mode=full.scale_mode, outlier_p=full.outlier_p,
                  n_stale=0, sm_scale=full.sm_scale)
    wl = W.make_workload(spec, seed=seed, device="cpu")
    s = spec
    P, ps = wl.num_pages, s.page_size
    fp8 = s.kv_dtype == W.FP8
    el = np.uint8 if fp8 else np.uint16
    kp = np.zeros((P, H, ps, s.head_dim_k), el)
    vp = None if s.v_alias else np.zeros((P, H, ps, s.head_dim_v), el)
    mode = {W.SCALE_TENSOR: 0, W.SCALE_HEAD: 1, W.SCALE_TOKEN: 2}[s.scale_mode]
    if mode == 2:
        ks = np.ones((P, H, ps), np.float32)
        vs = None if s.v_alias else np.ones((P, H, ps), np.float32)
    else:
        n = 1 if mode == 0 else H
        ks, vs = np.ones(n, np.float32), (None if s.v_alias else np.ones(n, np.float32))
    oc = oracle.Cache(oracle.FP8 if fp8 else oracle.BF16, mode, P, ps, H, s.head_dim_k,
                      s.head_dim_v, kp, vp, ks, vs, wl.page_tags.copy())

    def bits(t):
        return t.contiguous().view(torch.int16).numpy().view(np.uint16)

    hist = [(bits(k), None if v is None else bits(v), sl) for k, v, sl in wl.hist_chunks()]
    if fp8 and mode != 2:
        oc.k_scale[:] = oracle.scales(np.concatenate([h[0] for h in hist]), mode == 1)
        if vs is not None:
            oc.v_scale[:] = oracle.scales(np.concatenate([h[1] for h in hist]), mode == 1)
    for k, v, sl in hist:
        oracle.append(oc, k, v, sl)
    del hist
    kn, vn, slots = wl.new_tokens()
    knb, vnb = bits(kn), (None if vn is None else bits(vn))
    qb = bits(wl.q())
    rows = np.array([(g // H) * s.num_q_heads + (g % H) * G + i
                     for g in range(n_groups) for i in range(G)], np.int32)
    row_bytes = wl.kv_row_bytes + (4 if (fp8 and mode == 2) else 0)
    kv = sum(int(wl.seq_lens[g // H]) for g in range(n_groups)) * row_bytes

    def step():
        oracle.append(oc, knb, vnb, slots)
        m = oracle.validate(oc.page_tags, wl.block_table, wl.expected_tags, wl.seq_lens, ps)
        oracle.decode(oc, qb, wl.block_table, wl.seq_lens, m, wl.sm_scale, rows=rows)

    desc = (f"{n_groups} (sequence, KV head) groups = {rows.size} query rows of the {full.name} "
            f"workload ({kv / 1e6:.1f} MB of cache), step = append + validate + decode")
    return step, kv, desc


def cpu_baseline(spec_name, budget_s, seed=0):
    """The oracle as it stands, timed on the host cores on a sample of the
    workload sized to about budget_s seconds (one step)."""
    from fp8_kv_paged_kvq_b200 import workloads as W
    full = W.spec_by_name(spec_name, seed)
    step1, _, _ = oracle_sample(spec_name, 1, seed)
    t0 = time.perf_counter()
    step1()
    t1 = time.perf_counter() - t0
    n = max(1, min(full.B * full.num_kv_heads, int(budget_s / max(t1, 1e-6))))
    step, kv, desc = oracle_sample(spec_name, n, seed)
    t0 = time.perf_counter()
    step()
    dt = time.perf_counter() - t0
    return {"value": kv / dt / 1e9, "unit": "GB/s", "cores": len(os.sched_getaffinity(0)),
            "kind": "oracle", "sample": desc, "seconds": dt}


# ---------------------------------------------------------------------------
# the reference arm: the oracle as it stands
# ---------------------------------------------------------------------------
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    oracle.build()
    # per-step budget so that warm-up + steps end in a few minutes
    per_step = max(0.02, 150.0 / max(1, args.steps + args.warmup))
    step1, _, _ = oracle_sample(args.workload, 1)
    t0 = time.perf_counter()
    step1()
    t1 = time.perf_counter() - t0
    n = max(1, int(per_step / max(t1, 1e-6)))
    step, kv, desc = oracle_sample(args.workload, n)
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / max(1, args.steps)
    cores = len(os.sched_getaffinity(0))
    value = kv / dt / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_desc(args.workload), "sample": desc},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_desc(name, seqs=0):
    from fp8_kv_paged_kvq_b200 import workloads as W
    s = W.spec_by_name(name)
    if seqs:
        s.seq_lens = list(s.seq_lens)[:seqs]
    lens = sorted(set(s.seq_lens))
    ltxt = f"{s.B} seq x {lens[0]} tok" if len(lens) == 1 else f"{s.B} seq, {min(lens)}..{max(lens)} tok"
    return (f"{name}: {ltxt}, page {s.page_size}, {s.num_q_heads}q/{s.num_kv_heads}kv heads, "
            f"d{s.head_dim_k}/{s.head_dim_v}, {s.kv_dtype} {s.scale_mode} scales")


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def run_ours(args):
    rank, world, local = dist_setup(args)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    import fp8_kv_paged_kvq_b200 as kvq
    from fp8_kv_paged_kvq_b200 import build as kvq_build
    from fp8_kv_paged_kvq_b200 import workloads as W
    from fp8_kv_paged_kvq_b200.pipeline import DecodeBatch
    if rank == 0:
        kvq_build.build()
    barrier(world) if world > 1 else None
    kvq.lib()

    spec = W.spec_by_name(args.workload)
    if args.seqs:
        spec.seq_lens = list(spec.seq_lens)[: args.seqs]
    wl = W.make_workload(spec, seed=0, device=dev)
    db = DecodeBatch(wl, device=dev, num_ctas=args.num_ctas)
    db.prefill()
    torch.cuda.synchronize()
    kv_bytes = wl.kv_bytes_read()
    s = spec
    alg_bytes = (kv_bytes + s.B * s.num_q_heads * s.head_dim_k * 2          # q
                 + int(np.ceil(wl.seq_lens / s.page_size).sum()) * 4        # block table
                 + s.B * s.num_q_heads * (s.head_dim_v + 1) * 4)            # out + lse
    stream = torch.cuda.Stream(device=dev)
    hbm, hbm_kind = peaks()

    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            db.step(check_tags=True, stream=stream)
        torch.cuda.synchronize()
        g_step = capture(lambda: db.step(check_tags=True, stream=stream), stream)
        g_nochk = capture(lambda: db.step(check_tags=False, stream=stream), stream)
        g_dec = capture(lambda: db.decode(use_abort=True, stream=stream), stream)
        for g in (g_step, g_nochk, g_dec):
            for _ in range(3):
                g.replay()
        torch.cuda.synchronize()

        # ---- the timed region: K steps ----
        barrier(world)
        sampler = ClockSampler(local)
        with sampler:
            ms_step = time_graph(g_step, args.steps, stream)
        barrier(world)
        ms_step = max_over_ranks(ms_step, world)
        # dominant kernel (kvq_decode: split-KV kernel + combine), same data
        ms_dec = max_over_ranks(time_graph(g_dec, args.steps, stream), world)
        ms_nochk = max_over_ranks(time_graph(g_nochk, args.steps, stream), world)
    assert kvq.device_error() == 0, "device-side wait timed out"

    # ---- e2e through the public API with host buffers ----
    e2e = run_e2e(db, args, stream, kv_bytes, world)

    # ---- BF16 cache, same shapes ----
    bf16 = None
    if not args.no_bf16 and s.kv_dtype == W.FP8 and not s.v_alias:
        del g_step, g_nochk, g_dec
        bf16 = run_bf16(wl, args, stream, world, dev)

    value = whole_job_gbs(world, kv_bytes, ms_step)
    # kernels per step: append, validate, then decode (wide: query pre-pass +
    # decode + combine; otherwise decode + combine)
    launches = 2 + (3 if is_wide(s) else 2)
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16 mma / f32 accumulate (e4m3 cache)",
        "data": "synthetic",
        "config": {"workload": workload_desc(args.workload, args.seqs),
                   "step": "kvq_append + kvq_validate + kvq_decode (split-KV + LSE combine)",
                   "l2": f"inputs exceed L2: {kv_bytes / 1e6:.0f} MB of cache read per step",
                   "timing": "CUDA graph replay, CUDA events, max over ranks",
                   "parallelism": "replicas" if world > 1 else "single GPU"},
        "decode_tokens_per_s": world * s.B / (ms_step * 1e-3),
        "hbm_frac_of_step": value / world / hbm,
        "validate_overhead_pct": 100.0 * (ms_step - ms_nochk) / ms_nochk,
        "ms_per_step_without_validation": ms_nochk,
        "roofline": decode_roofline(s, wl, alg_bytes, ms_dec,
                                    measured_traffic(args.workload, args.seqs)),
        "gpu_launches": launches * args.steps,
        "clocks": sampler.summary(),
        "e2e": e2e,
    }
    if bf16:
        line["bf16_same_shape"] = bf16
        line["fp8_vs_bf16_step_time"] = ms_step / bf16["ms_per_step"]
    if not is_wide(s) and s.kv_dtype == W.FP8 and not args.seqs:
        line["bulk_append"] = run_bulk_append(s, dev, stream)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.workload, budget_s=10.0)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_long(args):
    """The long workload as its decode loop: every step appends one token per
    sequence with page reallocation and tag bumps; even steps validate with
    0.01% of expected tags made stale (those requests abort for that step), odd
    steps skip the check.  Step time = device time of append + validate +
    decode replayed from a CUDA graph; bytes count decoded (non-aborted) rows."""
    rank, world, local = dist_setup(args)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    import fp8_kv_paged_kvq_b200 as kvq
    from fp8_kv_paged_kvq_b200 import build as kvq_build
    from fp8_kv_paged_kvq_b200 import workloads as W
    from fp8_kv_paged_kvq_b200.pipeline import DecodeLoop
    if rank == 0:
        kvq_build.build()
    barrier(world)
    spec = W.spec_by_name("long")
    wl = W.make_workload(spec, seed=0, device=dev)
    steps = args.loop_steps
    loop = DecodeLoop(wl, steps, device=dev, num_ctas=args.num_ctas)
    loop.batch.prefill()
    torch.cuda.synchronize()
    row = spec.num_kv_heads * (spec.head_dim_k + spec.head_dim_v)
    stream = torch.cuda.Stream(device=dev)
    recs = []
    with torch.cuda.stream(stream):
        loop.capture(stream)
        torch.cuda.synchronize()
        barrier(world)
        sampler = ClockSampler(local)
        with sampler:
            for ls in W.loop_steps(wl, steps):
                # kind 0: check + stale tags, 1: clean check, 2: no check; the
                # second half of each six-step cycle replays the graphs with
                # events between the kernels, for the per-kernel breakdown
                kind = ls.step % 3
                detailed = (ls.step // 3) % 2 == 1
                chk = kind != 2
                idx = loop.prepare(ls, chk, inject_stale=(kind == 0))
                ev = loop.run(chk, stream, detailed)
                loop.restore(idx)
                torch.cuda.synchronize()
                ms_step = ev[0].elapsed_time(ev[-1])
                parts = tuple(ev[i].elapsed_time(ev[i + 1]) for i in range(3)) if detailed else (0, 0, 0)
                aborted = {b for b, _ in ls.stale} if kind == 0 else set()
                kv = sum(int(ls.seq_lens[b]) for b in range(spec.B) if b not in aborted) * row
                recs.append((kind, detailed, ms_step) + parts + (kv, len(aborted)))
    assert kvq.device_error() == 0, "device-side wait timed out"
    kind = np.array([r[0] for r in recs])
    det = np.array([r[1] for r in recs])
    ms = np.array([r[2] for r in recs])
    t_app = np.array([r[3] for r in recs])
    t_val = np.array([r[4] for r in recs])
    t_dec = np.array([r[5] for r in recs])
    kv = np.array([r[6] for r in recs], dtype=np.float64)
    # the tracker's view must match what the device did
    host_tags = loop.tracker.tags
    dev_tags = loop.batch.cache.page_tags.cpu().numpy().view(np.uint32)
    tags_ok = bool(np.array_equal(host_tags, dev_tags))
    def mean(x):
        return float(max_over_ranks(float(np.mean(x)), world))
    plain = ~det                                  # steps timed only at their boundaries
    step_clean, step_nochk = mean(ms[plain & (kind == 1)]), mean(ms[plain & (kind == 2)])
    # in the detailed graphs the no-check step records the same events around an
    # empty slot: its gap is the event overhead, subtracted from the validate slot
    val = mean(t_val[det & (kind == 1)]) - mean(t_val[det & (kind == 2)])
    gbs = whole_job_gbs(world, kv[plain].sum(), max_over_ranks(float(ms[plain].sum()), world))
    hbm, hbm_kind = peaks()
    line = {
        "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": world, "steps": steps,
        "warmup": 1, "ms_per_step": float(ms[plain].mean()), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "f16 mma / f32 accumulate (e4m3 cache)", "data": "synthetic",
        "config": {"workload": workload_desc("long"),
                   "loop": f"{steps} steps: append 1 token/seq with page reallocation + tag "
                           "bump; steps cycle validate+stale tags / validate / no validation",
                   "l2": "inputs exceed L2: >3 GB of cache read per step",
                   "timing": "CUDA graph per step between CUDA events; step time and value "
                             "from the half of the steps with events only around the step"},
        "decode_tokens_per_s": world * spec.B / (ms[plain].mean() * 1e-3),
        "hbm_frac_of_step": gbs / world / hbm,
        "ms_per_step_with_validation": step_clean,
        "ms_per_step_without_validation": step_nochk,
        "ms_per_step_with_validation_and_stale_tags": mean(ms[plain & (kind == 0)]),
        "p95_ms_with_validation": float(np.percentile(ms[plain & (kind == 1)], 95)),
        "p95_ms_without_validation": float(np.percentile(ms[plain & (kind == 2)], 95)),
        "ms_validate_kernel": val,
        "ms_decode_with_validation": mean(t_dec[det & (kind == 1)]),
        "ms_decode_without_validation": mean(t_dec[det & (kind == 2)]),
        "ms_decode_with_stale_aborts": mean(t_dec[det & (kind == 0)]),
        "ms_append": mean(t_app[det]),
        "validate_overhead_pct": 100.0 * (step_clean - step_nochk) / step_nochk,
        "validate_overhead_note": "steps cycle: validate with 0.01% stale tags / validate with "
                                  "clean tags / no validation; overhead compares the last two, "
                                  "each timed only at the step's boundaries",
        "aborted_requests_per_stale_step": float(np.mean([r[7] for r in recs if r[0] == 0])),
        "pages_reallocated": int(sum(len(l.new_pages) for l in W.loop_steps(wl, steps))),
        "host_tracker_matches_device_tags": tags_ok,
        "clocks": sampler.summary(), "gpu_launches": int(4 * np.sum(kind != 2) + 3 * np.sum(kind == 2)),
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_e2e(db, args, stream, kv_bytes, world):
    """Same step through the public API, its inputs copied from pinned host
    memory and its results (out, lse, abort mask) read back, every step:
    - value: two CUDA graphs (DecodeBatch.capture_io_pipelined) replayed in
      turn; each replay runs one step while copying in the next step's inputs
      and copying out the previous step's results on side streams;
    - serial: one graph per step holding its copies, append, validate, decode
      and read-back in order (DecodeBatch.capture_io_step);
    - eager: the same calls issued one by one from Python each step."""
    K = args.e2e_steps
    names = [n for n in db.IO_IN if getattr(db, n) is not None]
    pin = lambda t: torch.empty(t.shape, dtype=t.dtype).pin_memory()
    host_in = [{n: getattr(db, n).detach().cpu().pin_memory() for n in names} for _ in range(2)]
    host_out = [{n: pin(getattr(db, n)) for n in db.IO_OUT} for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host_in[0].values())
    d2h = sum(t.numel() * t.element_size() for t in host_out[0].values())

    def one():
        for n, h in host_in[0].items():
            getattr(db, n).copy_(h, non_blocking=True)
        db.step(check_tags=True, stream=stream)
        for n, h in host_out[0].items():
            h.copy_(getattr(db, n), non_blocking=True)

    def timed(fns):
        for i in range(6):
            fns[i % len(fns)]()
        barrier(world)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(K):
            fns[i % len(fns)]()
        e1.record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(e0.elapsed_time(e1) / K, world)

    with torch.cuda.stream(stream):
        ms_eager = timed([one])
        g = db.capture_io_step(host_in[0], host_out[0], stream)
        ms_serial = timed([g.replay])
        del g
        ga, gb = db.capture_io_pipelined(host_in, host_out, stream)
        ms = timed([ga.replay, gb.replay])
        del ga, gb
    gbs = lambda m: whole_job_gbs(world, kv_bytes, m)
    return {"value": gbs(ms), "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms,
            "steps": K, "path": "python binding -> C ABI; two CUDA graphs in turn, each a step "
                                "(append, validate, decode) with the next step's host->device "
                                "copies and the previous step's device->host copies beside it",
            "serial": {"value": gbs(ms_serial), "ms_per_step": ms_serial,
                       "path": "one CUDA graph per step: copies in, step, copies out, in order"},
            "eager": {"value": gbs(ms_eager), "ms_per_step": ms_eager,
                      "path": "the same calls launched one by one from Python"}}


def run_bf16(wl_fp8, args, stream, world, dev):
    from fp8_kv_paged_kvq_b200 import workloads as W
    from fp8_kv_paged_kvq_b200.pipeline import DecodeBatch
    db = DecodeBatch(wl_fp8, device=dev, num_ctas=args.num_ctas, kv_dtype=W.BF16)
    db.prefill()
    with torch.cuda.stream(stream):
        for _ in range(max(3, args.warmup)):
            db.step(check_tags=True, stream=stream)
        g = capture(lambda: db.step(check_tags=True, stream=stream), stream)
        gd = capture(lambda: db.decode(use_abort=True, stream=stream), stream)
        for _ in range(3):
            g.replay()
            gd.replay()
        barrier(world)
        ms = max_over_ranks(time_graph(g, args.steps, stream), world)
        msd = max_over_ranks(time_graph(gd, args.steps, stream), world)
    kv = 2 * wl_fp8.kv_bytes_read()
    hbm, _ = peaks()
    res = {"ms_per_step": ms, "kv_gbs": whole_job_gbs(world, kv, ms),
           "decode_ms_per_launch": msd, "decode_kv_gbs": kv / (msd * 1e-3) / 1e9,
           "decode_frac_of_hbm": kv / (msd * 1e-3) / 1e9 / hbm,
           "decode_tokens_per_s": world * wl_fp8.B / (ms * 1e-3)}
    del g, gd, db
    torch.cuda.empty_cache()
    return res


def run_bulk_append(spec, dev, stream, tokens=65536, iters=20):
    """Bulk quantize: a prompt's worth of BF16 K/V (tokens x Hkv x D) through
    kvq_append into FP8 pages scattered by a random page permutation, as at
    the prefill -> decode hand-over.  Algorithmic bytes: the BF16 reads, the
    code writes and the slot mapping."""
    import fp8_kv_paged_kvq_b200 as kvq
    s = spec
    ps, H, Dk, Dv = s.page_size, s.num_kv_heads, s.head_dim_k, s.head_dim_v
    pages = -(-tokens // ps)
    g = torch.Generator(device=dev).manual_seed(11)
    cache = kvq.PagedCache(kvq.FP8_E4M3, kvq.SCALE_HEAD, pages, ps, H, Dk, Dv, device=dev)
    k = torch.randn(tokens, H, Dk, device=dev, generator=g).to(torch.bfloat16)
    v = torch.randn(tokens, H, Dv, device=dev, generator=g).to(torch.bfloat16)
    # per-head scales from the data (amax / 448), as at the hand-over; not
    # powers of two, so every value takes the checked product quotient
    kvq.scale_from_amax(kvq.amax(k, True), out=cache.k_scale)
    kvq.scale_from_amax(kvq.amax(v, True), out=cache.v_scale)
    pow2 = bool(((cache.k_scale.view(torch.int32) & 0x7FFFFF) == 0).any() or
                ((cache.v_scale.view(torch.int32) & 0x7FFFFF) == 0).any())
    perm = torch.randperm(pages, device=dev, generator=g).to(torch.int32)
    t = torch.arange(tokens, device=dev, dtype=torch.int32)
    slots = (perm[t // ps] * ps + t % ps).contiguous()
    with torch.cuda.stream(stream):
        for _ in range(3):
            kvq.append(cache, k, v, slots, stream=stream)
        gr = capture(lambda: kvq.append(cache, k, v, slots, stream=stream), stream)
        ms = time_graph(gr, iters, stream)
    nbytes = tokens * H * (Dk + Dv) * 3 + tokens * 4
    hbm, kind = peaks()
    del gr
    return {"tokens": tokens, "ms": ms, "gbs": nbytes / (ms * 1e-3) / 1e9,
            "frac_of_hbm": nbytes / (ms * 1e-3) / 1e9 / hbm, "peak_kind": kind,
            "bytes": nbytes, "note": "bf16 K/V read + e4m3 codes written + slot mapping",
            "scales": "per head, amax / 448 of the data" + (" (some powers of two)" if pow2 else "")}


def run_sweep(args):
    """Capacity and concurrency sweep on the gqa shape (64 query / 8 KV heads,
    d 128, page 16, 8,192 tokens per sequence): FP8 and BF16 decode time at
    B = 1, 8, 16, 32, 64, and the tokens a fixed memory budget holds in each
    format (cache bytes per token read from the allocated pages)."""
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    import fp8_kv_paged_kvq_b200 as kvq
    from fp8_kv_paged_kvq_b200 import build as kvq_build
    from fp8_kv_paged_kvq_b200 import workloads as W
    from fp8_kv_paged_kvq_b200.pipeline import DecodeBatch
    kvq_build.build()
    stream = torch.cuda.Stream(device=dev)
    hbm, _ = peaks()
    rows = []
    budget = 80 * 2**30                       # bytes of cache in the capacity comparison
    per_token = {}
    for B in (1, 8, 16, 32, 64):
        row = {"B": B}
        for dt in (W.FP8, W.BF16):
            spec = W.spec_by_name("gqa")
            spec.seq_lens = [8192] * B
            spec.kv_dtype = dt
            wl = W.make_workload(spec, seed=0, device=dev)
            db = DecodeBatch(wl, device=dev)
            db.prefill()
            c = db.cache
            nbytes = sum(x.numel() * x.element_size() for x in
                         (c.k_pages, c.v_pages, c.k_scale, c.v_scale) if x is not None)
            per_token[dt] = nbytes / (wl.num_pages * spec.page_size)
            with torch.cuda.stream(stream):
                for _ in range(3):
                    db.decode(use_abort=False, stream=stream)
                gd = capture(lambda: db.decode(use_abort=False, stream=stream), stream)
                ms = time_graph(gd, args.steps, stream)
            kv = wl.kv_bytes_read()               # bytes of this cache format
            row[dt] = {"ms": ms, "kv_gbs": kv / (ms * 1e-3) / 1e9,
                       "frac_of_hbm": kv / (ms * 1e-3) / 1e9 / hbm,
                       "decode_tokens_per_s": B / (ms * 1e-3)}
            del gd, db
            torch.cuda.empty_cache()
        row["fp8_over_bf16_time"] = row[W.FP8]["ms"] / row[W.BF16]["ms"]
        rows.append(row)
    line = {"sweep": "gqa shape, 8,192 tokens per sequence, decode call only",
            "rows": rows,
            "capacity": {"budget_bytes": budget,
                         "fp8_bytes_per_token": per_token[W.FP8],
                         "bf16_bytes_per_token": per_token[W.BF16],
                         "fp8_tokens": int(budget // per_token[W.FP8]),
                         "bf16_tokens": int(budget // per_token[W.BF16])},
            "steps": args.steps}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    elif args.sweep:
        run_sweep(args)
    elif args.workload == "long":
        run_long(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
