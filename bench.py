"""Benchmark of the FP8 paged decode path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload long|gqa|ragged|wide] [--no-extra] [--no-bf16]
                    [--no-cpu-baseline] [--sweep]

A decode step is one pass of the whole hot path over one batch:
kvq_append (the new token of every sequence, with tag bumps for reallocated
pages) -> kvq_validate (page tags -> abort mask) -> kvq_decode (split-KV
attention + log-sum-exp combine).

Default workload (the long-context one): 4 sequences of 262,144 tokens and 60
of 8,192, page 16, 64 query / 8 KV heads, head_dim 128, E4M3 cache with
per-head scales, decoded for 1,000 steps that each append a token per
sequence (pages that fill up are replaced by reallocated pages whose tags the
append bumps).  Steps cycle through three kinds: the tag check with 0.01% of
the expected tags made stale (those requests abort), the tag check with
every tag right ("clean"), and no check.  For this workload --steps and
--warmup count passes over the 1,000-step loop; every pass repeats the same
tag history.

`value` is KV GB/s on the clean steps (cache bytes a step reads / its device
time, CUDA events around each step), `ms_per_step` their mean, and the tag
check's cost compares the clean steps with the unchecked ones (mean and
p95).  `roofline` is the decode call (decode kernel + combine, timed between
events inside the steps) against the measured HBM copy bandwidth.  `e2e` is
the loop through the Python API with every step's inputs copied from pinned
host memory and its results read back.  `cpu_baseline` is the CPU oracle on
a sample of the same workload, on all host cores and on one.  The line also
carries the other decode batches (`configs`): the GQA batch (32 x 8,192), the
ragged batch (64 sequences of 1k-32k tokens, FP8 and BF16 caches) and the
wide-group batch (128 query heads on one KV head, 576/512 dims, tensor
cores), each with its own step statistics and roofline.

N > 1 runs N independent replicas (one per GPU, no collective on the data
path) and reports the aggregate.  `--impl reference` times the CPU oracle on
a bounded sample of the workload.  `--sweep` runs the FP8 / BF16 capacity
and concurrency sweep instead.
"""
from __future__ import annotations

import argparse
import datetime
import json
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
DTYPE = "f16 mma / f32 accumulate (e4m3 cache)"


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="long")
    ap.add_argument("--num-ctas", type=int, default=0)
    ap.add_argument("--no-bf16", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="only the headline workload, not the other decode batches")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--loop-steps", type=int, default=1000,
                    help="decode steps of the long workload's loop")
    ap.add_argument("--min-seconds", type=float, default=0.5,
                    help="least device time of each timed single-batch measurement")
    ap.add_argument("--idle-seconds", type=float, default=3.0,
                    help="idle time before each single-batch measurement")
    ap.add_argument("--sweep", action="store_true",
                    help="capacity and concurrency sweep (FP8 vs BF16 at B = 1..64) instead of the bench line")
    ap.add_argument("--seqs", type=int, default=0,
                    help="keep only the first N sequences (smaller case for profiling)")
    return ap.parse_args(argv)


def measured_traffic(kernel, units):
    """DRAM bytes of one decode launch from the committed ncu record (bytes per
    unit x the launch's units), or None when the kernel source changed since
    the capture.  Records without a per-unit figure give their per-launch
    bytes for the workload they were taken on."""
    import hashlib
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    for name, r in rec.items():
        if not name.startswith(kernel):
            continue
        src = os.path.join(ROOT, r["source"])
        if not os.path.exists(src):
            continue
        h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        if h != r["source_sha256_prefix"]:
            return None
        if "dram_bytes_per_unit" in r:
            return r["dram_bytes_per_unit"] * units
        return None
    return None


def gqa_units(spec, seq_lens):
    """Work units of the 8-head decode kernel: 16-token tiles per (sequence, KV head)."""
    lens = np.asarray(seq_lens, np.int64)
    return int(((lens + 15) // 16).sum()) * spec.num_kv_heads


def wide_units(seq_lens):
    """Work units of the tensor-core kernel: 64-token blocks per sequence."""
    lens = np.asarray(seq_lens, np.int64)
    return int(((lens + 63) // 64).sum())


def decode_traffic(spec, seq_lens):
    """Recorded DRAM bytes of the launch that decodes these rows, or None."""
    if is_wide(spec):
        return measured_traffic("wide_decode_kernel", wide_units(seq_lens))
    return measured_traffic("gqa_decode_kernel", gqa_units(spec, seq_lens))


def _peaks_file():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return json.load(f)
    return None


def peaks():
    d = _peaks_file()
    if d:
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def tensor_peak():
    """Dense bf16 TFLOP/s of this GPU (burst: the decode launch is timed on its own)."""
    d = _peaks_file()
    if d:
        return float(d["bf16_tflops"]), "measured"
    return FALLBACK_BF16_TFLOPS, "fallback"


def is_wide(spec) -> bool:
    """The 128-query-head, one-KV-head shape served by the tensor-core kernel."""
    return spec.num_q_heads // spec.num_kv_heads >= 64


def decode_alg_bytes(spec, seq_lens):
    """Algorithmic bytes of one kvq_decode call: the cache bytes the rows read
    (codes, + per-token scales in TOKEN mode), the query, the block-table
    entries, out and lse."""
    s = spec
    lens = np.minimum(np.asarray(seq_lens, np.int64), 1 << 40)
    el = 1 if s.kv_dtype == "fp8" else 2
    row = el * (s.head_dim_k + (0 if s.v_alias else s.head_dim_v))
    if s.scale_mode == "token" and s.kv_dtype == "fp8":
        row += 4
    kv = int(lens.sum()) * s.num_kv_heads * row
    return (kv + s.B * s.num_q_heads * s.head_dim_k * 2
            + int(np.ceil(lens / s.page_size).sum()) * 4
            + s.B * s.num_q_heads * (s.head_dim_v + 1) * 4)


def decode_roofline(spec, seq_lens, ms_dec, traffic, alg_bytes=None):
    """Roofline of one kvq_decode launch.  The 8-head kernel moves bytes
    (bound: HBM).  The wide kernel is a pair of dense contractions per token,
    QK^T (a bf16 query against keys that are exact in f16) and PV (f16), so it
    is bound by the tensor cores at the f16/bf16 rate: 2 * Hq * (Dk + Dv) FLOPs
    per decoded token."""
    alg = decode_alg_bytes(spec, seq_lens) if alg_bytes is None else alg_bytes
    if is_wide(spec):
        tokens = int(np.asarray(seq_lens, np.int64).sum())
        flops = 2.0 * spec.num_q_heads * (spec.head_dim_k + spec.head_dim_v) * tokens
        peak, kind = tensor_peak()
        achieved = flops / (ms_dec * 1e-3) / 1e12
        return {"bound": "tensor",
                "kernel": "kvq_decode (wide_prep_kernel + wide_decode_kernel + lse_combine_kernel)",
                "achieved": achieved, "peak": peak, "peak_kind": kind + " (bf16 burst)",
                "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                "algorithmic_flops_per_launch": flops, "algorithmic_bytes_per_launch": alg,
                "hbm_frac": alg / (ms_dec * 1e-3) / 1e9 / peaks()[0],
                "ms_per_launch": ms_dec}
    hbm, kind = peaks()
    achieved = alg / (ms_dec * 1e-3) / 1e9
    return {"bound": "hbm", "kernel": "kvq_decode (gqa_decode_kernel + lse_combine_kernel)",
            "achieved": achieved, "peak": hbm, "peak_kind": kind, "unit": "GB/s",
            "frac": achieved / hbm, "traffic": traffic,
            "algorithmic_bytes_per_launch": alg, "ms_per_launch": ms_dec}


def stats(ms):
    ms = np.asarray(ms, np.float64)
    return {"mean": float(ms.mean()), "min": float(ms.min()), "median": float(np.median(ms)),
            "p95": float(np.percentile(ms, 95)), "n": int(ms.size)}


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
def time_replays(replay, stream, min_s, min_n=20, chunk=64):
    """Per-call device times (ms) of `replay`, with CUDA events on `stream`
    around every call, repeated until at least min_n calls and min_s seconds."""
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(chunk + 1)]
    times = []
    torch.cuda.synchronize()
    while len(times) < min_n or sum(times) < min_s * 1e3:
        ev[0].record(stream)
        for j in range(chunk):
            replay()
            ev[j + 1].record(stream)
        torch.cuda.synchronize()
        times += [ev[j].elapsed_time(ev[j + 1]) for j in range(chunk)]
    return np.array(times)


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


def _oracle_rate(spec_name, budget_s, threads, seed=0):
    import oracle
    from fp8_kv_paged_kvq_b200 import workloads as W
    full = W.spec_by_name(spec_name, seed)
    used = oracle.set_threads(threads)
    step1, kv1, _ = oracle_sample(spec_name, 1, seed)
    t0 = time.perf_counter()
    step1()
    t1 = time.perf_counter() - t0
    n = max(1, min(full.B * full.num_kv_heads, int(budget_s / max(t1, 1e-6))))
    step, kv, desc = oracle_sample(spec_name, n, seed)
    t0 = time.perf_counter()
    step()
    dt = time.perf_counter() - t0
    return {"value": kv / dt / 1e9, "unit": "GB/s", "cores": used, "kind": "oracle",
            "sample": desc, "seconds": dt}


def cpu_baseline(spec_name, budget_s, seed=0):
    """The oracle as it stands, timed on the host's cores (all, then one) on a
    sample of the workload sized to about budget_s seconds (one step)."""
    import oracle
    oracle.build()
    allc = len(os.sched_getaffinity(0))
    res = _oracle_rate(spec_name, budget_s, allc, seed)
    one = _oracle_rate(spec_name, budget_s / 2, 1, seed)
    oracle.set_threads(allc)
    res["one_core"] = one
    return res


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
# one decode batch (gqa, ragged, wide): the step, the decode call, e2e
# ---------------------------------------------------------------------------
REPS = 8   # calls per CUDA graph in the single-batch measurements


def measure_batch(name, args, dev, stream, world, e2e=True, bf16=True, cpu=True):
    """Step and decode-call statistics of one decode batch.  The step
    (append -> validate -> decode) and the decode call are each captured
    REPS times back to back in one CUDA graph, replayed with events around
    every replay until args.min_seconds of device time; a call's time is a
    replay's time / REPS, so the graph's launch and the events are not charged
    to every call.  The inputs exceed L2, so no flush is needed."""
    from fp8_kv_paged_kvq_b200 import workloads as W
    from fp8_kv_paged_kvq_b200.pipeline import DecodeBatch
    spec = W.spec_by_name(name)
    if args.seqs:
        spec.seq_lens = list(spec.seq_lens)[: args.seqs]
    wl = W.make_workload(spec, seed=0, device=dev)
    db = DecodeBatch(wl, device=dev, num_ctas=args.num_ctas)
    db.prefill()
    torch.cuda.synchronize()
    kv_bytes = wl.kv_bytes_read()
    s = spec
    # start from an idle GPU: a batch measured right after the long loop's
    # seconds under the power cap would inherit that power state
    torch.cuda.synchronize()
    time.sleep(args.idle_seconds)
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    with torch.cuda.stream(stream), sampler:
        for _ in range(3):
            db.step(check_tags=True, stream=stream)
        torch.cuda.synchronize()
        reps = lambda f: (lambda: [f() for _ in range(REPS)])
        g_step = capture(reps(lambda: db.step(check_tags=True, stream=stream)), stream)
        g_nochk = capture(reps(lambda: db.step(check_tags=False, stream=stream)), stream)
        g_dec = capture(reps(lambda: db.decode(use_abort=True, stream=stream)), stream)
        for g in (g_step, g_nochk, g_dec):
            for _ in range(3):
                g.replay()
        barrier(world)
        t_step = time_replays(g_step.replay, stream, args.min_seconds) / REPS
        t_nochk = time_replays(g_nochk.replay, stream, args.min_seconds) / REPS
        t_dec = time_replays(g_dec.replay, stream, args.min_seconds) / REPS
    st, sn, sd = stats(t_step), stats(t_nochk), stats(t_dec)
    ms_step = max_over_ranks(st["mean"], world)
    hbm, _ = peaks()
    lens = np.minimum(wl.seq_lens, wl.max_pages * s.page_size)
    res = {"workload": workload_desc(name, args.seqs),
           "kv_bytes_per_step": kv_bytes,
           "kv_gbs": whole_job_gbs(world, kv_bytes, ms_step),
           "hbm_frac_of_step": kv_bytes / (ms_step * 1e-3) / 1e9 / hbm,
           "decode_tokens_per_s": world * s.B / (ms_step * 1e-3),
           "ms_per_step": st, "ms_per_step_without_validation": sn, "ms_decode_call": sd,
           "validate_overhead_pct": 100.0 * (st["mean"] - sn["mean"]) / sn["mean"],
           "roofline": decode_roofline(s, lens, max_over_ranks(sd["mean"], world),
                                       decode_traffic(s, lens)),
           "timing": f"CUDA graphs of {REPS} back-to-back calls, events around every "
                     f"replay, >= {args.min_seconds} s each, per call = replay / {REPS}; "
                     "min/median/p95 are over replays; inputs exceed L2; "
                     f"after {args.idle_seconds} s idle",
           "clocks": sampler.summary()}
    assert_no_device_error()
    if e2e:
        res["e2e"] = run_e2e(db, args, stream, kv_bytes, world)
    del g_step, g_nochk, g_dec
    if bf16 and not args.no_bf16 and s.kv_dtype == W.FP8 and not s.v_alias:
        res["bf16_same_shape"] = run_bf16(wl, args, stream, world, dev)
        res["fp8_vs_bf16_step_time"] = st["mean"] / res["bf16_same_shape"]["ms_per_step"]["mean"]
    del db
    torch.cuda.empty_cache()
    if cpu and not args.no_cpu_baseline and world == 1:
        res["cpu_baseline"] = cpu_baseline(name, budget_s=4.0)
    return res


def assert_no_device_error():
    import fp8_kv_paged_kvq_b200 as kvq
    assert kvq.device_error() == 0, "device-side wait timed out"


def run_e2e(db, args, stream, kv_bytes, world):
    """Same step through the public API, its inputs copied from pinned host
    memory and its results (out, lse, abort mask) read back, every step:
    two CUDA graphs (DecodeBatch.capture_io_pipelined) replayed in turn; each
    replay runs one step while copying in the next step's inputs and copying
    out the previous step's results on side streams."""
    names = [n for n in db.IO_IN if getattr(db, n) is not None]
    pin = lambda t: torch.empty(t.shape, dtype=t.dtype).pin_memory()
    host_in = [{n: getattr(db, n).detach().cpu().pin_memory() for n in names} for _ in range(2)]
    host_out = [{n: pin(getattr(db, n)) for n in db.IO_OUT} for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host_in[0].values())
    d2h = sum(t.numel() * t.element_size() for t in host_out[0].values())
    with torch.cuda.stream(stream):
        ga, gb = db.capture_io_pipelined(host_in, host_out, stream)
        flip = [0]

        def one():
            (ga if flip[0] == 0 else gb).replay()
            flip[0] ^= 1
        for _ in range(6):
            one()
        barrier(world)
        t = time_replays(one, stream, args.min_seconds / 2)
        del ga, gb
    ms = max_over_ranks(float(t.mean()), world)
    return {"value": whole_job_gbs(world, kv_bytes, ms), "unit": "GB/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms,
            "steps": int(t.size),
            "path": "python binding -> C ABI; two CUDA graphs in turn, each a step (append, "
                    "validate, decode) with the next step's host->device copies and the "
                    "previous step's device->host copies beside it"}


def run_bf16(wl_fp8, args, stream, world, dev):
    from fp8_kv_paged_kvq_b200 import workloads as W
    from fp8_kv_paged_kvq_b200.pipeline import DecodeBatch
    db = DecodeBatch(wl_fp8, device=dev, num_ctas=args.num_ctas, kv_dtype=W.BF16)
    db.prefill()
    with torch.cuda.stream(stream):
        for _ in range(3):
            db.step(check_tags=True, stream=stream)
        g = capture(lambda: [db.step(check_tags=True, stream=stream) for _ in range(REPS)], stream)
        gd = capture(lambda: [db.decode(use_abort=True, stream=stream) for _ in range(REPS)], stream)
        for _ in range(3):
            g.replay()
            gd.replay()
        barrier(world)
        t = stats(time_replays(g.replay, stream, args.min_seconds) / REPS)
        td = stats(time_replays(gd.replay, stream, args.min_seconds) / REPS)
    ms = max_over_ranks(t["mean"], world)
    msd = max_over_ranks(td["mean"], world)
    kv = 2 * wl_fp8.kv_bytes_read()
    hbm, _ = peaks()
    spec16 = W.Spec(**{**wl_fp8.spec.__dict__, "kv_dtype": W.BF16})
    lens = np.minimum(wl_fp8.seq_lens, wl_fp8.max_pages * spec16.page_size)
    res = {"ms_per_step": t, "kv_gbs": whole_job_gbs(world, kv, ms),
           "ms_decode_call": td, "decode_kv_gbs": kv / (msd * 1e-3) / 1e9,
           "decode_frac_of_hbm": kv / (msd * 1e-3) / 1e9 / hbm,
           "roofline": decode_roofline(spec16, lens, msd, None),
           "decode_tokens_per_s": world * wl_fp8.B / (ms * 1e-3)}
    del g, gd, db
    torch.cuda.empty_cache()
    return res


def run_bulk_append(spec, dev, stream, tokens=65536):
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
    perm = torch.randperm(pages, device=dev, generator=g).to(torch.int32)
    t = torch.arange(tokens, device=dev, dtype=torch.int32)
    slots = (perm[t // ps] * ps + t % ps).contiguous()
    with torch.cuda.stream(stream):
        for _ in range(3):
            kvq.append(cache, k, v, slots, stream=stream)
        gr = capture(lambda: kvq.append(cache, k, v, slots, stream=stream), stream)
        t = stats(time_replays(gr.replay, stream, 0.2))
    nbytes = tokens * H * (Dk + Dv) * 3 + tokens * 4
    hbm, kind = peaks()
    del gr
    return {"tokens": tokens, "ms": t, "gbs": nbytes / (t["mean"] * 1e-3) / 1e9,
            "frac_of_hbm": nbytes / (t["mean"] * 1e-3) / 1e9 / hbm, "peak_kind": kind,
            "bytes": nbytes, "note": "bf16 K/V read + e4m3 codes written + slot mapping",
            "scales": "per head, amax / 448 of the data"}


# ---------------------------------------------------------------------------
# the long workload: the 1,000-step loop
# ---------------------------------------------------------------------------
def run_long(args, rank, world, local, dev):
    from fp8_kv_paged_kvq_b200 import workloads as W
    from fp8_kv_paged_kvq_b200.pipeline import CLEAN, NOCHECK, STALE, DecodeLoop
    spec = W.spec_by_name("long")
    wl = W.make_workload(spec, seed=0, device=dev)
    n = args.loop_steps
    loop = DecodeLoop(wl, n, device=dev, num_ctas=args.num_ctas)
    loop.batch.prefill()
    torch.cuda.synchronize()
    loop.snapshot_tags()
    stream = torch.cuda.Stream(device=dev)
    # kinds cycle in twelve steps: stale / clean / no check, then stale / no
    # check / clean, so that clean and unchecked steps follow the same mix of
    # neighbours; every other cycle of three steps runs each call as its own
    # graph with events between them (the decode call's time), the others as
    # one graph per step with events only at the step's boundaries (the step
    # times)
    order = (STALE, CLEAN, NOCHECK, STALE, CLEAN, NOCHECK,
             STALE, NOCHECK, CLEAN, STALE, NOCHECK, CLEAN)
    kinds = [order[i % 12] for i in range(n)]
    detailed = [(i // 3) % 2 == 1 for i in range(n)]
    loop.capture(stream, kinds, detailed)
    row = spec.num_kv_heads * (spec.head_dim_k + spec.head_dim_v)
    lens = np.stack([ls.seq_lens for ls in loop.plan]).astype(np.int64)
    aborted = [{b for b, _ in ls.stale} if kinds[ls.step] == STALE else set() for ls in loop.plan]
    kv = np.array([sum(int(lens[i, b]) for b in range(spec.B) if b not in aborted[i]) * row
                   for i in range(n)], np.float64)
    alg_dec = np.array([decode_alg_bytes(spec, [lens[i, b] for b in range(spec.B)
                                                if b not in aborted[i]]) for i in range(n)])

    def new_events():
        return [[torch.cuda.Event(enable_timing=True) for _ in range(4 if d else 2)]
                for d in detailed]

    evsets = [new_events(), new_events()]
    rec = []

    def harvest(evs):
        for i, ev in enumerate(evs):
            t = [ev[j].elapsed_time(ev[j + 1]) for j in range(len(ev) - 1)]
            rec.append((i, sum(t)) + tuple(t if len(t) == 3 else (0.0, 0.0, 0.0)))

    for _ in range(max(3, args.warmup)):
        loop.replay_pass(stream)
    torch.cuda.synchronize()
    loop.batch.cache.page_tags.copy_(loop.tags0)
    barrier(world)
    sampler = ClockSampler(local)
    t_wall = time.perf_counter()
    with sampler:
        # passes alternate between two event sets: pass p + 1 is queued before
        # pass p's events are read, so the device never waits for the host
        for p in range(args.steps):
            loop.replay_pass(stream, evsets[p % 2])
            if p > 0:
                evsets[(p - 1) % 2][-1][-1].synchronize()
                harvest(evsets[(p - 1) % 2])
        torch.cuda.synchronize()
        harvest(evsets[(args.steps - 1) % 2])
    barrier(world)
    wall = time.perf_counter() - t_wall
    assert_no_device_error()
    tags_ok = bool(np.array_equal(loop.batch.cache.page_tags.cpu().numpy().view(np.uint32),
                                  loop.final_tags()))
    idx = np.array([r[0] for r in rec])
    ms = np.array([r[1] for r in rec])
    t_app, t_val, t_dec = (np.array([r[k] for r in rec]) for k in (2, 3, 4))
    kind = np.array([kinds[i] for i in idx])
    det = np.array([detailed[i] for i in idx])
    plain = ~det
    clean, nochk, stale = plain & (kind == CLEAN), plain & (kind == NOCHECK), plain & (kind == STALE)
    dclean = det & (kind == CLEAN)
    m = lambda x: max_over_ranks(float(x), world)
    ms_clean = m(ms[clean].mean())
    value = whole_job_gbs(world, kv[idx[clean]].sum(), m(ms[clean].sum()))
    sc, sn, ss = stats(ms[clean]), stats(ms[nochk]), stats(ms[stale])
    # decode call (decode kernel + combine) timed between events in the clean
    # detailed steps: algorithmic bytes / time, summed over those steps
    dec_ms = m(t_dec[dclean].sum()) / dclean.sum()
    dec_bytes = alg_dec[idx[dclean]].mean()
    dec_units = np.mean([gqa_units(spec, [lens[i, b] for b in range(spec.B)
                                          if b not in aborted[i]]) for i in idx[dclean]])
    roof = decode_roofline(spec, lens[n // 2], dec_ms,
                           measured_traffic("gqa_decode_kernel", dec_units), alg_bytes=dec_bytes)
    roof["note"] = ("decode call between events inside the clean steps of the timed passes; "
                    "algorithmic bytes and time averaged over those steps; traffic = DRAM "
                    "bytes per 16-token tile from an ncu capture of the 8-head kernel on 8 "
                    "of the gqa batch's sequences, times the tiles of the average step")
    hbm, _ = peaks()
    launches = sum(3 if k == NOCHECK else 4 for k in kinds) * args.steps
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(3, args.warmup),
        "ms_per_step": ms_clean, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": DTYPE, "data": "synthetic",
        "config": {"workload": workload_desc("long"),
                   "loop": f"{n} decode steps per pass: append 1 token/seq with page "
                           "reallocation + tag bump, then the tag check, then decode; steps "
                           "cycle check with 0.01% stale tags / clean check / no check (and "
                           "stale / no check / clean)",
                   "steps_and_warmup": f"passes over the {n}-step loop (each pass resets the "
                                       "live tags and repeats the same tag history)",
                   "ms_per_step": "one decode step (append + validate + decode), mean over "
                                  "the clean steps",
                   "value": "KV bytes of the clean steps / their device time",
                   "l2": "inputs exceed L2: >3 GB of cache read per step",
                   "timing": "one CUDA graph per step, CUDA events at step boundaries, "
                             "max over ranks",
                   "parallelism": "replicas" if world > 1 else "single GPU"},
        "decode_tokens_per_s": world * spec.B / (ms_clean * 1e-3),
        "hbm_frac_of_step": value / world / hbm,
        "ms_per_step_stats": sc,
        "ms_per_step_without_validation": sn,
        "ms_per_step_with_stale_tags": ss,
        "validate_overhead_pct": 100.0 * (sc["mean"] - sn["mean"]) / sn["mean"],
        "validate_overhead_p95_pct": 100.0 * (sc["p95"] - sn["p95"]) / sn["p95"],
        "validate_overhead_median_pct": 100.0 * (sc["median"] - sn["median"]) / sn["median"],
        "validate_overhead_note": "clean steps (check on, every tag right) against steps "
                                  "without the check, each timed at its boundaries only",
        "ms_decode_call": stats(t_dec[dclean]),
        "ms_validate_call": stats(t_val[dclean]),
        "ms_append_call": stats(t_app[dclean]),
        "aborted_requests_per_stale_step": float(np.mean([len(a) for a in aborted if a]
                                                         or [0])),
        "pages_reallocated_per_pass": int(sum(len(ls.new_pages) for ls in loop.plan)),
        "host_tracker_matches_device_tags": tags_ok,
        "roofline": roof,
        "gpu_launches": launches,
        "timed_region_s": wall,
        "clocks": sampler.summary(),
    }
    if not args.no_e2e:
        line["e2e"] = run_long_e2e(loop, stream, world, row, spec)
    del loop
    torch.cuda.empty_cache()
    return line


def run_long_e2e(loop, stream, world, row, spec):
    """The loop through the public API with host buffers: every step's inputs
    (query, new K/V, slots, lengths, reallocated pages, new block-table and
    expected-tag entries) copied from pinned host memory and its results
    (out, lse, abort mask, abort count) read back, host traffic overlapped
    with the neighbouring steps.  Every step runs the clean check."""
    io = loop.io_setup(stream)
    loop.io_pass(stream, steps=50)                    # warm-up
    barrier(world)
    e0, e1, counts = loop.io_pass(stream)
    ms_total = max_over_ranks(e0.elapsed_time(e1), world)
    lens = np.stack([ls.seq_lens for ls in loop.plan]).astype(np.int64)
    kv = float(lens.sum()) * row
    n = len(counts)
    assert all(c == 0 for c in counts), "clean steps must abort nothing"
    return {"value": whole_job_gbs(world, kv, ms_total), "unit": "GB/s",
            "h2d_bytes_per_step": io["h2d_bytes_per_step"],
            "d2h_bytes_per_step": io["d2h_bytes_per_step"],
            "ms_per_step": ms_total / n, "steps": n,
            "path": "python binding -> C ABI; two CUDA graphs in turn, each a step (block-table "
                    "entries, append, validate, decode) with the next step's host->device "
                    "copies and the previous step's device->host copies beside it; every "
                    "step's abort count read back and checked"}


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
    if rank == 0:
        kvq_build.build()
    barrier(world)
    kvq.lib()
    stream = torch.cuda.Stream(device=dev)
    if args.workload == "long":
        line = run_long(args, rank, world, local, dev)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline("long", budget_s=8.0)
        extra = [] if args.no_extra else ["gqa", "ragged", "wide"]
    else:
        # a single decode batch as the headline: K timed steps after W warm-up steps
        res = measure_batch(args.workload, args, dev, stream, world, e2e=not args.no_e2e,
                            cpu=False)
        st = res["ms_per_step"]
        line = {"metric": METRIC, "value": res["kv_gbs"], "unit": "GB/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": st["mean"],
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": DTYPE, "data": "synthetic",
                "config": {"workload": res["workload"],
                           "step": "kvq_append + kvq_validate + kvq_decode",
                           "timing": res["timing"],
                           "parallelism": "replicas" if world > 1 else "single GPU"}}
        line.update({k: v for k, v in res.items() if k not in ("workload", "kv_gbs")})
        line["gpu_launches"] = ((2 + (3 if is_wide(W.spec_by_name(args.workload)) else 2))
                                * st["n"] * REPS)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(args.workload, budget_s=8.0)
        extra = []
    if extra:
        line["configs"] = {}
        for name in extra:
            line["configs"][name] = measure_batch(name, args, dev, stream, world,
                                                  e2e=(name == "gqa"), bf16=(name != "wide"))
        s = W.spec_by_name("gqa")
        line["bulk_append"] = run_bulk_append(s, dev, stream)
        if world == 1:
            line["concurrency"] = run_concurrency(args, dev, stream)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def decode_call_at(B, dt, args, dev, stream, hbm):
    """Decode-call time on the gqa shape (64 query / 8 KV heads, d 128, page
    16) with B sequences of 8,192 tokens in cache format dt: CUDA graphs of
    REPS back-to-back calls, events around every replay.  Returns the timing
    record and the cache bytes per token of the allocated pages."""
    from fp8_kv_paged_kvq_b200 import workloads as W
    from fp8_kv_paged_kvq_b200.pipeline import DecodeBatch
    spec = W.spec_by_name("gqa")
    spec.seq_lens = [8192] * B
    spec.kv_dtype = dt
    wl = W.make_workload(spec, seed=0, device=dev)
    db = DecodeBatch(wl, device=dev)
    db.prefill()
    c = db.cache
    nbytes = sum(x.numel() * x.element_size() for x in
                 (c.k_pages, c.v_pages, c.k_scale, c.v_scale) if x is not None)
    per_token = nbytes / (wl.num_pages * spec.page_size)
    with torch.cuda.stream(stream):
        for _ in range(3):
            db.decode(use_abort=False, stream=stream)
        gd = capture(lambda: [db.decode(use_abort=False, stream=stream)
                              for _ in range(REPS)], stream)
        for _ in range(3):
            gd.replay()
        t = stats(time_replays(gd.replay, stream, args.min_seconds) / REPS)
    kv = wl.kv_bytes_read()               # bytes of this cache format
    rec = {"ms": t, "kv_gbs": kv / (t["mean"] * 1e-3) / 1e9,
           "frac_of_hbm": kv / (t["mean"] * 1e-3) / 1e9 / hbm,
           "decode_tokens_per_s": B / (t["mean"] * 1e-3)}
    del gd, db
    torch.cuda.empty_cache()
    return rec, per_token


def run_concurrency(args, dev, stream):
    """FP8 decode call at low concurrency (B = 1, 8, 16 sequences of 8,192
    tokens, gqa shape), each after the same idle time as the carried batches."""
    from fp8_kv_paged_kvq_b200 import workloads as W
    hbm, _ = peaks()
    out = {"workload": "gqa shape, B x 8,192 tokens, FP8 head scales, decode call only",
           "timing": f"CUDA graphs of {REPS} back-to-back calls, >= {args.min_seconds} s each, "
                     f"after {args.idle_seconds} s idle"}
    for B in (1, 8, 16):
        time.sleep(args.idle_seconds)
        out[f"B{B}"], _ = decode_call_at(B, W.FP8, args, dev, stream, hbm)
    return out


def run_sweep(args):
    """Capacity and concurrency sweep on the gqa shape (64 query / 8 KV heads,
    d 128, page 16, 8,192 tokens per sequence): FP8 and BF16 decode time at
    B = 1, 8, 16, 32, 64, and the tokens a fixed memory budget holds in each
    format (cache bytes per token read from the allocated pages)."""
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    from fp8_kv_paged_kvq_b200 import build as kvq_build
    from fp8_kv_paged_kvq_b200 import workloads as W
    kvq_build.build()
    stream = torch.cuda.Stream(device=dev)
    hbm, _ = peaks()
    rows = []
    budget = 80 * 2**30                       # bytes of cache in the capacity comparison
    per_token = {}
    for B in (1, 8, 16, 32, 64):
        row = {"B": B}
        for dt in (W.FP8, W.BF16):
            row[dt], per_token[dt] = decode_call_at(B, dt, args, dev, stream, hbm)
        row["fp8_over_bf16_time"] = row[W.FP8]["ms"]["mean"] / row[W.BF16]["ms"]["mean"]
        rows.append(row)
    line = {"sweep": "gqa shape, 8,192 tokens per sequence, decode call only",
            "rows": rows,
            "capacity": {"budget_bytes": budget,
                         "fp8_bytes_per_token": per_token[W.FP8],
                         "bf16_bytes_per_token": per_token[W.BF16],
                         "fp8_tokens": int(budget // per_token[W.FP8]),
                         "bf16_tokens": int(budget // per_token[W.BF16])}}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    elif args.sweep:
        run_sweep(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
