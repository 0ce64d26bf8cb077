"""Benchmark of the quantized attention forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl sage|reference]

One step = the whole hot path over one batch: the Q/K pre-pass
(sage_quant_qk), the V pre-pass (sage_quant_v) and the fused attention
kernel (sage_attn_fwd_quantized), inputs resident in HBM.  L2 is flushed (a 256 MiB device write) between
timed steps; each step is bracketed by CUDA events on the launching stream.
Metric: effective TOPS = 4*B*H*N^2*d / t (summed over ranks; weak scaling,
each rank processes its own batch of heads with no collective on the data
path).  Prints one JSON line on rank 0.

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
DEFAULT_WORKLOAD = "llm"


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    p.add_argument("--impl", default="sage", choices=["sage", "reference"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    a = p.parse_args()
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


def run_sage(args):
    import ctypes

    import torch
    import torch.distributed as dist

    import quantized_attention_quant_b200 as sage

    rank, world, local = rank_env()
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    lib = sage.library()
    w0 = WORKLOADS[args.workload]
    w = rank_workload(w0, rank)
    B, H, N, d = w.B, w.H, w.N, w.d
    mode = sage.MODES[w.mode]
    dt = sage.DTYPES[w.dtype]

    qh, kh, vh = make_qkv(w)
    qh, kh, vh = qh.pin_memory(), kh.pin_memory(), vh.pin_memory()
    q, k, v = qh.to(dev), kh.to(dev), vh.to(dev)
    o = torch.empty_like(q)

    def buf(name):
        n = sage.buffer_bytes(w.mode, name, B, H, N, d)
        return torch.empty(n, dtype=torch.uint8, device=dev) if n else None

    names = ["q_codes", "q_scales", "q_sf", "k_codes", "k_scales", "k_sf", "k_mean",
             "v_codes", "v_scales", "v_sf"]
    bufs = {n: buf(n) for n in names}
    P = {n: (bufs[n].data_ptr() if bufs[n] is not None else None) for n in names}
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    sptr = stream.cuda_stream
    sm_scale = w.sm_scale

    def check(s):
        if s != 0:
            raise RuntimeError(lib.sage_status_string(s).decode())

    def step(ev_attn=None):
        # both pre-passes (the V pass overlapped with the Q/K pass), then
        # the attention kernel on the codes
        check(lib.sage_quant_qkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), dt, B, H, N, d, mode,
                                 P["q_codes"], P["q_scales"], P["q_sf"], P["k_codes"],
                                 P["k_scales"], P["k_sf"], P["k_mean"], P["v_codes"],
                                 P["v_scales"], P["v_sf"], sptr))
        if ev_attn:
            ev_attn[0].record(stream)
        check(lib.sage_attn_fwd_quantized(mode, P["q_codes"], P["q_scales"], P["q_sf"],
                                          P["k_codes"], P["k_scales"], P["k_sf"], P["v_codes"],
                                          P["v_scales"], P["v_sf"], o.data_ptr(), dt, B, H, N, d,
                                          int(w.causal), ctypes.c_float(sm_scale), sptr))
        if ev_attn:
            ev_attn[1].record(stream)

    # sage_quant_qkv: one cluster-fused launch in the 8-bit modes up to 8
    # tiles (1024 tokens) per head and 16 heads, else 2 (Q/K) + 2 (V in FP8)
    # or 1 (V in FP4); attention: 1
    if w.mode != "fp4" and -(-N // 128) <= 8 and B * H <= 16:
        launches_per_step = 1 + 1
    else:
        launches_per_step = 2 + (1 if w.mode == "fp4" else 2) + 1

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    clocks = ClockSampler(uuid)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    ea = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    for i in range(args.steps):
        flush.zero_()                      # L2 flush between timed steps (outside the events)
        ev[i][0].record(stream)
        step(ea[i])
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    attn_ms = [a.elapsed_time(b) for a, b in ea]
    status = sage.device_status()
    if status != 0:
        raise RuntimeError(f"device status {status}")

    # end to end through the public API: pinned host inputs in, O back to host
    oh = torch.empty_like(qh).pin_memory()
    for _ in range(2):
        oh.copy_(sage.sage_attn_fwd(qh.to(dev, non_blocking=True), kh.to(dev, non_blocking=True),
                                    vh.to(dev, non_blocking=True), w.causal, None, w.mode).to(
                                        "cpu", non_blocking=True))
    torch.cuda.synchronize()
    e2e_ms = []
    for _ in range(max(3, args.steps // 4)):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        qd = qh.to(dev, non_blocking=True)
        kd = kh.to(dev, non_blocking=True)
        vd = vh.to(dev, non_blocking=True)
        od = sage.sage_attn_fwd(qd, kd, vd, w.causal, None, w.mode)
        oh.copy_(od, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms.append(e0.elapsed_time(e1))
    clk = clocks.stop()

    # max over ranks
    t_step = sum(step_ms) / len(step_ms)
    t_attn = sum(attn_ms) / len(attn_ms)
    t_e2e = sum(e2e_ms) / len(e2e_ms)
    t_step, t_attn, t_e2e = max_over_ranks([t_step, t_attn, t_e2e], world, dev)

    heads = B * H
    value = job_throughput(w.ops, world, t_step)        # 4 B H N^2 d, all ranks
    e2e_val = job_throughput(w.ops, world, t_e2e)
    peaks, src = measured_peaks()
    ratio = 4.0 if w.mode == "fp4" else 2.0             # vs bf16, nominal dense ratios
    peak = peaks["bf16_tflops"] * ratio
    achieved = work_ops(w, heads) / (t_attn * 1e-3) / 1e12
    traffic = read_traffic(args.workload)
    elem = B * H * N * d
    out = {
        "metric": "attention fwd effective TOPS (4*B*H*N^2*d/t)",
        "value": round(value, 2),
        "unit": "TOPS",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(t_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": {"fp4": "fp4e2m1", "fp8": "fp8e4m3"}.get(w.mode, "int8+fp8e4m3"),
        "data": "synthetic",
        "config": config_of(w0, world),
        "attn_kernel_ms": round(t_attn, 4),
        "prepass_ms": round(t_step - t_attn, 4),
        "roofline": {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(peak, 1),
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "traffic": traffic,
                     "kernel": attention_kernel(w, torch.cuda.get_device_properties(dev)
                                                .multi_processor_count),
                     "peak_source": f"{src} bf16 burst x{ratio:g} (nominal dense ratio)",
                     "work": "4 d ops per visible (q,k) pair"},
        "e2e": {"value": round(e2e_val, 2), "unit": "TOPS",
                "h2d_bytes_per_step": 3 * elem * 2, "d2h_bytes_per_step": elem * 2},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
    }
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


def oracle_sample(w, heads, rows=None):
    """Run the oracle (emulated path) on the given heads; returns seconds."""
    from oracle import attention as att
    from quantized_attention_quant_b200.workloads import to_numpy32
    q, k, v = (to_numpy32(t) for t in make_qkv(w, heads))
    t0 = time.perf_counter()
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


def cpu_baseline(w, budget_s=12.0):
    rows, pairs = sample_rows(w)
    t = 0.0
    done = 0
    h = 0
    while t < budget_s and h < w.B * w.H:
        t += oracle_sample(w, [(h // w.H, h % w.H)], rows)
        done += pairs
        h += 1
    ops = 4.0 * w.d * done
    desc = (f"{h} head(s), {'all' if rows is None else len(rows)} query rows each, "
            f"emulated quantized path (pre-pass of the sampled heads included)")
    return {"value": round(ops / t / 1e12, 6), "unit": "TOPS", "cores": blas_threads(),
            "kind": "oracle", "sample": desc, "seconds": round(t, 2)}


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


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_sage(args)


if __name__ == "__main__":
    main()
