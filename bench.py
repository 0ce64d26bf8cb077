"""Benchmark of the quantized attention forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl sage|reference]

One step = the whole hot path over one batch: the Q/K and V pre-passes
(sage_quant_qkv) and the fused attention kernel (sage_attn_fwd_quantized),
inputs resident in HBM.  L2 is flushed (a 256 MiB device write) between
timed steps; each step is bracketed by CUDA events on the launching stream.
Metric: effective TOPS = 4*B*H*N^2*d / t (summed over ranks; weak scaling,
each rank processes its own batch of heads with no collective on the data
path).  Prints one JSON line on rank 0.

The default workload is n16k (B=2 H=32 N=16384 d=128, non-causal, bf16,
INT8 Q/K with FP8 P~ and V); the same shape in FP4 mode (the fp4 workload)
is timed after it, kernel-only, and reported under "also"
(--also none skips it).

--impl reference times the CPU oracle (NumPy FP64, the method restated) on
the host cores, on a bounded sample of the same workload per step.
"""

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from quantized_attention_quant_b200.workloads import WORKLOADS, make_qkv  # noqa: E402

L2_FLUSH_BYTES = 256 << 20
DEFAULT_WORKLOAD = "n16k"
DEFAULT_ALSO = {"n16k": "fp4"}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    p.add_argument("--impl", default="sage", choices=["sage", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--ubench", action="store_true",
                   help="run the microbenchmarks of include/sage_ubench.h instead (one JSON line)")
    p.add_argument("--also", default=None,
                   help="comma-separated workloads timed after the main one (kernel-only "
                        "lines under 'also'); 'none' for none")
    a = p.parse_args()
    if a.also is None:
        a.also = DEFAULT_ALSO.get(a.workload, "none")
    a.also = [x for x in a.also.split(",") if x and x != "none"]
    for x in a.also:
        if x not in WORKLOADS:
            p.error(f"unknown workload in --also: {x}")
    if a.warmup < 3:
        a.warmup = 3
    return a


def visible_pairs(w):
    """(query, key) pairs the masked softmax keeps, per head."""
    return w.N * (w.N + 1) // 2 if w.causal else w.N * w.N


def work_ops(w, heads):
    """Algorithmic tensor-core operations: 4 d per visible pair (2d for
    Q K^T, 2d for P~V)."""
    return 4.0 * w.d * visible_pairs(w) * heads


def prepass_bytes(w, heads):
    """Algorithmic HBM bytes of the pre-pass: read Q, K, V once (2 B per
    element each), write the three code tensors (1 B per element in the
    8-bit modes, 0.5 B + one UE4M3 scale per 16 elements in FP4 mode)."""
    elem = heads * w.N * w.d
    write = 1.0 if w.mode != "fp4" else 0.5 + 1.0 / 16
    return elem * 3 * (2.0 + write)


def percentile(xs, p):
    xs = sorted(xs)
    if not xs:
        return None
    i = (len(xs) - 1) * p / 100.0
    lo = int(math.floor(i))
    hi = min(lo + 1, len(xs) - 1)
    return xs[lo] + (xs[hi] - xs[lo]) * (i - lo)


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, \
            "fallback"


# ---------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid=None):
        cmd = ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
               "-lms", "200"]
        if uuid:
            cmd += ["-i", uuid]
        try:
            self.p = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                      text=True)
        except OSError:
            self.p = None
        self.t0 = time.time()

    def stop(self):
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.p.terminate()
        out, _ = self.p.communicate(timeout=10)
        rows = [r.split(",") for r in out.strip().splitlines() if r.count(",") >= 8]
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------- sage arm

def rank_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_workload(w, rank):
    """Weak scaling: rank r draws its own batch (seed offset by rank)."""
    return w.with_(seed=w.seed + 1000 * rank)


def config_of(w, world):
    """The JSON `config` of a run: the workload one rank processes, and the
    job-wide head count (weak scaling: every rank its own batch of heads)."""
    return {"workload": f"{w.name}: B={w.B} H={w.H} N={w.N} d={w.d} "
                        f"{'causal' if w.causal else 'non-causal'} {w.dtype} {w.mode}",
            "global_batch_heads": w.B * w.H * world, "seq_len": w.N, "head_dim": w.d,
            "causal": w.causal, "input_dtype": w.dtype, "mode": w.mode,
            "l2": "flushed between timed steps (256 MiB device write)",
            "parallelism": f"dp{world} (heads sharded by batch, no collective)"}


def max_over_ranks(values, world, device):
    """Element-wise max of a list of floats over all ranks (identity at
    world 1).  Every rank must call it, in the same order."""
    if world == 1:
        return list(values)
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_throughput(ops_per_rank, world, t_ms):
    """Whole-job TOPS: the work of all ranks over the slowest rank's time."""
    return ops_per_rank * world / (t_ms * 1e-3) / 1e12


class Runner:
    """The timed step of one workload on one rank: device inputs, the code
    buffers, and the two library calls of a step."""

    def __init__(self, w, dev):
        import torch

        import quantized_attention_quant_b200 as sage
        self.torch, self.sage = torch, sage
        self.lib = sage.library()
        self.w, self.dev = w, dev
        self.mode = sage.MODES[w.mode]
        self.dt = sage.DTYPES[w.dtype]
        qh, kh, vh = make_qkv(w)
        self.host = [t.pin_memory() for t in (qh, kh, vh)]
        self.q, self.k, self.v = (t.to(dev) for t in self.host)
        self.o = torch.empty_like(self.q)
        names = ["q_codes", "q_scales", "q_sf", "k_codes", "k_scales", "k_sf", "k_mean",
                 "v_codes", "v_scales", "v_sf"]
        self.bufs = {}
        for n in names:
            nb = sage.buffer_bytes(w.mode, n, w.B, w.H, w.N, w.d)
            self.bufs[n] = torch.empty(nb, dtype=torch.uint8, device=dev) if nb else None
        self.P = {n: (b.data_ptr() if b is not None else None) for n, b in self.bufs.items()}
        self.stream = torch.cuda.current_stream(dev)

    def check(self, s):
        if s != 0:
            raise RuntimeError(self.lib.sage_status_string(s).decode())

    def step(self, ev_mid=None):
        """Both pre-passes (the V pass overlapped with the Q/K pass), then the
        attention kernel on the codes; ev_mid is recorded between them."""
        import ctypes
        w, P, sptr = self.w, self.P, self.stream.cuda_stream
        self.check(self.lib.sage_quant_qkv(
            self.q.data_ptr(), self.k.data_ptr(), self.v.data_ptr(), self.dt, w.B, w.H, w.N, w.d,
            self.mode, P["q_codes"], P["q_scales"], P["q_sf"], P["k_codes"], P["k_scales"],
            P["k_sf"], P["k_mean"], P["v_codes"], P["v_scales"], P["v_sf"], sptr))
        if ev_mid is not None:
            ev_mid.record(self.stream)
        self.check(self.lib.sage_attn_fwd_quantized(
            self.mode, P["q_codes"], P["q_scales"], P["q_sf"], P["k_codes"], P["k_scales"],
            P["k_sf"], P["v_codes"], P["v_scales"], P["v_sf"], self.o.data_ptr(), self.dt,
            w.B, w.H, w.N, w.d, int(w.causal), ctypes.c_float(w.sm_scale), sptr))

    def launches_per_step(self):
        """sage_quant_qkv: one cluster-fused launch in the 8-bit modes up to 8
        tiles (1024 tokens) per head and 16 heads, else 2 (Q/K) + 2 (V in the
        8-bit modes) or 1 (V in FP4); attention: 1."""
        w = self.w
        if w.mode != "fp4" and -(-w.N // 128) <= 8 and w.B * w.H <= 16:
            return 1 + 1
        return 2 + (1 if w.mode == "fp4" else 2) + 1

    def time(self, steps, warmup, flush):
        """Per timed step: (step ms, pre-pass ms, attention ms), CUDA events
        on the launching stream, L2 flushed before every step."""
        torch = self.torch
        for _ in range(warmup):
            flush.zero_()
            self.step()
        torch.cuda.synchronize()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        for e0, e1, e2 in ev:
            flush.zero_()                  # outside the events
            e0.record(self.stream)
            self.step(e1)
            e2.record(self.stream)
        torch.cuda.synchronize()
        return [(a.elapsed_time(c), a.elapsed_time(b), b.elapsed_time(c)) for a, b, c in ev]

    def time_e2e(self, steps, flush):
        """The public C-ABI call on host buffers, sage_attn_fwd_host: pinned
        Q, K, V in host memory, O written back to host memory, every copy
        (chunked and overlapped with the compute by the library) inside the
        events."""
        import ctypes
        torch, sage, w = self.torch, self.sage, self.w
        qh, kh, vh = self.host
        oh = torch.empty_like(qh).pin_memory()
        lib = sage.library()
        dt = 1 if qh.dtype == torch.bfloat16 else 0
        mode = sage.MODES[w.mode]

        def call():
            st = lib.sage_attn_fwd_host(qh.data_ptr(), kh.data_ptr(), vh.data_ptr(), oh.data_ptr(),
                                        dt, w.B, w.H, w.N, w.d, int(bool(w.causal)),
                                        ctypes.c_float(0.0), mode, self.stream.cuda_stream)
            if st != 0:
                raise RuntimeError(lib.sage_status_string(st).decode())

        for _ in range(2):
            call()
        torch.cuda.synchronize()
        ms = []
        for _ in range(steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(self.stream)
            call()
            e1.record(self.stream)
            torch.cuda.synchronize()
            ms.append(e0.elapsed_time(e1))
        elem = w.B * w.H * w.N * w.d
        return ms, 3 * elem * 2, elem * 2

    def free(self):
        del self.q, self.k, self.v, self.o, self.bufs, self.host
        self.torch.cuda.empty_cache()


def summarize(w, world, times, sms, dev_name=None):
    """Throughput, percentiles and the attention roofline of a list of
    (step, pre-pass, attention) times (already the max over ranks)."""
    steps = [t[0] for t in times]
    pre = [t[1] for t in times]
    attn = [t[2] for t in times]
    t_step, t_pre, t_attn = (sum(x) / len(x) for x in (steps, pre, attn))
    heads = w.B * w.H
    peaks, src = measured_peaks()
    ratio = 4.0 if w.mode == "fp4" else 2.0             # vs bf16, nominal dense ratios
    peak = peaks["bf16_tflops"] * ratio
    achieved = work_ops(w, heads) / (t_attn * 1e-3) / 1e12
    pre_gbs = prepass_bytes(w, heads) / (t_pre * 1e-3) / 1e9
    return {
        "value": round(job_throughput(w.ops, world, t_step), 2),
        "value_done": round(job_throughput(work_ops(w, heads), world, t_step), 2),
        "ms_per_step": round(t_step, 4),
        "step_ms_p50": round(percentile(steps, 50), 4),
        "step_ms_p95": round(percentile(steps, 95), 4),
        "attn_kernel_ms": round(t_attn, 4),
        "attn_kernel_ms_p50": round(percentile(attn, 50), 4),
        "attn_kernel_ms_p95": round(percentile(attn, 95), 4),
        "prepass_ms": round(t_pre, 4),
        "prepass_gbs": round(pre_gbs, 1),
        "prepass_hbm_frac": round(pre_gbs / peaks["hbm_gbs"], 4),
        "roofline": {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(peak, 1),
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "traffic": read_traffic(w.name),
                     "kernel": attention_kernel(w, sms),
                     "peak_source": f"{src} bf16 burst x{ratio:g} (nominal dense ratio)",
                     "work": "4 d ops per visible (q,k) pair"},
        # the secondary bound: one exponential per visible (q,k) pair against the
        # SFU's 16 per clock per SM (at the maximum SM clock)
        "exp_rate": exp_rate(w, heads, t_attn, sms),
    }


def exp_rate(w, heads, t_attn_ms, sms, sm_mhz=None):
    mhz = float(sm_mhz or measured_peaks()[0].get("sm_max_mhz") or 1965.0)
    per_clk = visible_pairs(w) * heads / (t_attn_ms * 1e-3) / (sms * mhz * 1e6)
    return {"exps_per_clk_per_sm": round(per_clk, 2), "sfu_frac": round(per_clk / 16.0, 4),
            "sm_mhz": mhz}


def run_sage(args):
    import torch
    import torch.distributed as dist

    import quantized_attention_quant_b200 as sage

    rank, world, local = rank_env()
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    sage.library()
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    w0 = WORKLOADS[args.workload]
    w = rank_workload(w0, rank)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    run = Runner(w, dev)

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    clocks = ClockSampler(uuid)

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    times = run.time(args.steps, args.warmup, flush)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    status = sage.device_status()
    if status != 0:
        raise RuntimeError(f"device status {status}")
    e2e_ms, h2d, d2h = run.time_e2e(max(3, args.steps // 4), flush)
    clk = clocks.stop()

    # max over ranks, step by step
    flat = [x for t in times for x in t] + [sum(e2e_ms) / len(e2e_ms)]
    flat = max_over_ranks(flat, world, dev)
    times = [tuple(flat[3 * i:3 * i + 3]) for i in range(len(times))]
    t_e2e = flat[-1]
    summ = summarize(w0, world, times, sms)
    out = {
        "metric": "attention fwd effective TOPS (4*B*H*N^2*d/t)",
        "value": summ.pop("value"),
        "unit": "TOPS",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": summ.pop("ms_per_step"),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": {"fp4": "fp4e2m1", "fp8": "fp8e4m3"}.get(w.mode, "int8+fp8e4m3"),
        "data": "synthetic",
        "config": config_of(w0, world),
    }
    out.update(summ)
    out["value_done_note"] = ("value counts 4*B*H*N^2*d as the metric is written; value_done "
                              "counts 4*d per visible (q,k) pair (half of it, plus the "
                              "diagonal, in causal runs)")
    out["e2e"] = {"value": round(job_throughput(w0.ops, world, t_e2e), 2), "unit": "TOPS",
                  "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                  "ms_per_step": round(t_e2e, 4),
                  "call": "sage_attn_fwd_host (pinned host Q, K, V in; O back to host; copies "
                          "chunked by heads and overlapped with the compute)"}
    out["gpu_launches"] = run.launches_per_step() * args.steps
    out["clocks"] = clk
    run.free()

    # further workloads, kernel-only (the same timed step)
    also = []
    for name in args.also:
        wa = rank_workload(WORKLOADS[name], rank)
        ra = Runner(wa, dev)
        if world > 1:
            dist.barrier()
        ta = ra.time(args.steps, args.warmup, flush)
        flat = max_over_ranks([x for t in ta for x in t], world, dev)
        ta = [tuple(flat[3 * i:3 * i + 3]) for i in range(len(ta))]
        sa = summarize(WORKLOADS[name], world, ta, sms)
        sa["config"] = config_of(WORKLOADS[name], world)
        sa["gpu_launches"] = ra.launches_per_step() * args.steps
        also.append(sa)
        ra.free()
    status = sage.device_status()
    if status != 0:
        raise RuntimeError(f"device status {status}")
    if also:
        out["also"] = also
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(w0, budget_s=12.0)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


def attention_kernel(w, sms):
    """The attention kernel the library runs for this workload: FP4, or
    INT8/FP8 one CTA per (query tile, head), or INT8/FP8 persistent when the
    items are short (the rule of use_persistent_attention in the library)."""
    if w.mode == "fp4":
        return "attn_fp4_kernel"
    ntiles = -(-w.N // 128)
    mean = (ntiles + 1) // 2 if w.causal else ntiles
    return ("attn_i8f8_persist_kernel" if mean <= 64 and ntiles * w.B * w.H > sms
            else "attn_i8f8_kernel")


def read_traffic(workload):
    """DRAM bytes per attention launch from the committed ncu summary, if it
    was taken on the current kernel (else null)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            entry = json.load(f).get(workload)
        if not entry:
            return None
        with open(os.path.join(ROOT, entry["kernel_source"]), "rb") as f:
            current = hashlib.sha256(f.read()).hexdigest()
        return entry["bytes"] if current == entry["kernel_source_sha256"] else None
    except (OSError, ValueError, KeyError):
        return None


# --------------------------------------------------------- oracle timing

def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(w, heads, rows=None, exact=False):
    """Run the oracle on the given heads -- the emulated quantized path, or
    with exact=True the FP64 exact attention; returns seconds."""
    from oracle import attention as att
    from quantized_attention_quant_b200.workloads import to_numpy32
    q, k, v = (to_numpy32(t) for t in make_qkv(w, heads))
    t0 = time.perf_counter()
    if exact:
        att.exact_attention(q, k, v, w.causal, w.sm_scale, rows=rows)
    else:
        att.emulated_sage_attention(q, k, v, w.causal, w.sm_scale, mode=w.mode, rows=rows)
    return time.perf_counter() - t0


def sample_rows(w):
    """Query rows of one head that fill about a second of oracle time, and the
    effective (metric) pair count they stand for: N keys per query row, as
    in 4*B*H*N^2*d."""
    target_pairs = 6e6 if w.mode == "fp4" else 2.5e7
    if w.N * w.N <= target_pairs:
        return None, w.N * w.N
    n = max(128, int(target_pairs / w.N))
    rows = __import__("numpy").linspace(0, w.N - 1, n).astype(int)
    return rows, len(rows) * w.N


def _oracle_rate(w, rows, pairs, budget_s, exact=False):
    """Heads run within the budget and the oracle's rate on them (TOPS of
    the metric's 4 d ops per pair)."""
    t = 0.0
    h = 0
    while t < budget_s and h < w.B * w.H:
        t += oracle_sample(w, [(h // w.H, h % w.H)], rows, exact=exact)
        h += 1
    return h, 4.0 * w.d * pairs * h / t / 1e12, t


def cpu_baseline(w, budget_s=12.0):
    """The oracle on the host cores: the emulated quantized path (the
    baseline), the exact FP64 attention beside it, and the emulated path
    again on one BLAS thread."""
    rows, pairs = sample_rows(w)
    h, value, t = _oracle_rate(w, rows, pairs, budget_s)
    _, exact, _ = _oracle_rate(w, rows, pairs, budget_s / 4, exact=True)
    single = None
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1, user_api="blas"):
            _, single, _ = _oracle_rate(w, rows, pairs, budget_s / 4)
    except ImportError:
        pass
    desc = (f"{h} head(s), {'all' if rows is None else len(rows)} query rows each, "
            f"emulated quantized path (pre-pass of the sampled heads included)")
    return {"value": round(value, 6), "unit": "TOPS", "cores": blas_threads(),
            "kind": "oracle", "sample": desc, "seconds": round(t, 2),
            "exact_fp64_value": round(exact, 6),
            "emulated_1_thread_value": None if single is None else round(single, 6)}


def run_reference(args):
    rank, world, _ = rank_env()
    if rank != 0:
        return
    w = WORKLOADS[args.workload]
    rows, pairs = sample_rows(w)
    times = []
    for i in range(args.warmup + args.steps):
        h = i % (w.B * w.H)
        t = oracle_sample(w, [(h // w.H, h % w.H)], rows)
        if i >= args.warmup:
            times.append(t)
    t_step = sum(times) / len(times)
    value = 4.0 * w.d * pairs / t_step / 1e12
    desc = (f"per step one head, {'all' if rows is None else len(rows)} query rows, "
            f"emulated quantized path (NumPy FP64 oracle)")
    out = {
        "impl": "reference",
        "metric": "attention fwd effective TOPS (4*B*H*N^2*d/t)",
        "value": round(value, 6), "unit": "TOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(t_step * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, world),
        "cpu_baseline": {"value": round(value, 6), "unit": "TOPS", "cores": blas_threads(),
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": round(value, 6), "unit": "TOPS", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def run_ubench():
    """The microbenchmarks behind the kernels' design (libsage_ubench.so):
    tcgen05 MMA throughput per kind, accumulator and tile width, the SFU
    exponential rate, FP32 against packed FP16x2, and the FP64 FMA rate."""
    import ctypes

    import torch

    from quantized_attention_quant_b200 import build as qb
    qb.build()
    torch.cuda.init()
    lib = ctypes.CDLL(qb.UBENCH_LIB)
    lib.sage_ubench_mma.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                    ctypes.POINTER(ctypes.c_double)]
    lib.sage_ubench_exp.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                    ctypes.POINTER(ctypes.c_double)]
    lib.sage_ubench_dfma.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_double)]
    out = {"ubench": "tcgen05 MMA, SFU exponential and FP64 FMA rates", "mma_tops": {},
           "exp_per_clk_per_sm": {}, "dfma_per_clk_per_sm": {}}
    kinds = {"f8f6f4_e4m3_f32acc": (0, 32), "f8f6f4_e4m3_f16acc": (1, 32), "i8_s32acc": (2, 32),
             "mxf4nvf4_e2m1_ue4m3x16_f32acc": (3, 64)}
    for name, (kind, kdim) in kinds.items():
        for n in (128, 256):
            v = ctypes.c_double(0.0)
            st = lib.sage_ubench_mma(kind, n, 8192, 5, ctypes.byref(v))
            out["mma_tops"][f"{name}_M128_N{n}_K{kdim}"] = round(v.value, 1) if st == 0 \
                else f"status {st}"
    for name, mode in (("ex2_f32", 0), ("ex2_f16x2", 1)):
        for threads in (128, 256, 512):
            v = ctypes.c_double(0.0)
            st = lib.sage_ubench_exp(mode, threads, 4096, ctypes.byref(v))
            out["exp_per_clk_per_sm"][f"{name}_{threads}thr"] = round(v.value, 2) if st == 0 \
                else f"status {st}"
    for threads in (256, 512, 1024):
        v = ctypes.c_double(0.0)
        st = lib.sage_ubench_dfma(threads, 4096, ctypes.byref(v))
        out["dfma_per_clk_per_sm"][f"{threads}thr"] = round(v.value, 2) if st == 0 \
            else f"status {st}"
    out["device"] = torch.cuda.get_device_name(0)
    print(json.dumps(out), flush=True)


def main():
    args = parse()
    if args.ubench:
        run_ubench()
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_sage(args)


if __name__ == "__main__":
    main()
