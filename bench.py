"""Benchmark of the KDA hot path on B200: prefill (chunk forward) and decode.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {ours,reference}]

One step = one kda_chunk_fwd over the prefill workload
"prefill_t8192_h32_d128" (B=1, T=8192, H=32, dk=dv=128, bf16 q/k/v, fp32 g,
beta, zero initial state, final state written).  `value` is whole-job
prefill tokens/s (tokens of the packed T axis, all heads) with inputs resident
in HBM; the inputs (404 MB) are larger than the 126 MB L2, so no flush is
needed between steps.  A second leg times the decode step on
"decode_n256_h32_d128" (256 sequences x 32 heads, fp32 state 512 MiB in
place) and is reported under "decode"; a third times serving decode
(kda_recurrent_steps: 8 tokens per sequence per call, states in a 512-entry
pool picked by slot) under "decode_steps".

Under torchrun (N > 1) every rank runs the same workload on its own GPU
(independent replicas: the hot path has no exchange step), timing is the max
over ranks, and `value` sums all ranks' tokens ("scaling": "weak").

--impl reference times the fp64 CPU oracle (tests' reference implementation)
on the host cores, each step a bounded sample of the same workload (the first
1024 tokens of all 32 heads), reported in the same metric and unit.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KDA tokens/s (prefill chunk fwd, decode step) at 1 B200; % of roofline"
UNIT = "tokens/s"
WORKLOAD = "prefill_t8192_h32_d128"
B, T, H, D = 1, 8192, 32, 128
# algorithmic bytes (bf16 q,k,v,out + fp32 g + fp32 beta per token-head, plus
# the final fp32 state written once per (sequence, head))
PREFILL_BYTES = B * T * H * (3 * D * 2 + D * 4 + 4 + D * 2) + B * H * D * D * 4
DEC_N, DEC_H = 256, 32


def decode_bytes(n):
    """Algorithmic bytes of one decode step for n sequences: the fp32 state
    read and written once, the token's q, k, v, out (bf16), g and beta (fp32)."""
    return n * DEC_H * (2 * D * D * 4 + 3 * D * 2 + D * 4 + 4 + D * 2)


DECODE_BYTES = decode_bytes(DEC_N)
FALLBACK_HBM_GBS = 6650.0

# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) from
# one ncu capture of each kernel on this workload (profiles/), valid only for
# the kernel sources it was taken on: reported as null once they change.
_SRC = os.path.join(ROOT, "gated_delta_rule_88_b200", "csrc")
TRAFFIC = {
    "prefill": {"files": ["chunk_prep.cu", "chunk_chain_tc.cu", "chunk_ws.h", "sm100.cuh", "common.cuh"],
                "sha": "8b788aa77014ac59", "bytes": (336.785152 + 254.092800 + 304.155648 + 49.041920) * 1e6},
    "decode": {"files": ["decode.cu", "common.cuh"], "sha": "4ceac309c0c18d2f",
               "bytes": (547.408128 + 480.674560) * 1e6},
    "decode_steps": {"files": ["decode_pipe.cu", "common.cuh", "sm100.cuh"], "sha": "d9cf376f965488af",
                     "bytes": (621.110016 + 492.918016) * 1e6},
    "backward": {"files": ["recurrent_bwd.cu", "common.cuh"], "sha": "ba9d9318f1b1cd87",
                 "bytes": (2902.812672 + 3861.861120) * 1e6},
    "decode_chunk": {"files": ["decode_chunk.cu", "common.cuh"], "sha": "23a550bc05b00c2b",
                     "bytes": (1210.240000 + 623.093504) * 1e6},
}


def measured_traffic(which):
    import hashlib
    t = TRAFFIC[which]
    m = hashlib.sha256()
    try:
        for f in t["files"]:
            with open(os.path.join(_SRC, f), "rb") as fh:
                m.update(fh.read())
    except OSError:
        return None
    return t["bytes"] if m.hexdigest()[:16] == t["sha"] else None


def measured_peak_hbm():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML (read only)."""

    def __init__(self, index: int, period_s: float = 0.01):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        self.ok = False

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            try:
                uuid = str(torch.cuda.get_device_properties(self.index).uuid)
                self._h = pynvml.nvmlDeviceGetHandleByUUID(
                    uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        except Exception:
            self.ok = False
        return self

    def _run(self):
        nv = self._nv
        names = {
            "gpu_idle": getattr(nv, "nvmlClocksEventReasonGpuIdle", 0x1),
            "sw_power_cap": getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4),
            "hw_slowdown": getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8),
            "sw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
            "hw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
            "hw_power_brake_slowdown": getattr(nv, "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80),
        }
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                get = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
                mask = get(self._h)
                for n, bit in names.items():
                    if mask & bit and n != "gpu_idle":
                        self.reasons.add(n)
            except Exception:
                pass
            time.sleep(self.period)

    def __exit__(self, *a):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        return rank, world, local, dist
    torch.cuda.set_device(0)
    return 0, 1, 0, None


def _coll_device(dist):
    # NCCL reduces device tensors; gloo (the CPU tests of this plumbing) host ones
    return "cuda" if dist.get_backend() == "nccl" else "cpu"


def max_over_ranks(x: float, dist) -> float:
    """Max of a per-rank figure (device time) over all ranks."""
    if dist is None:
        return x
    t = torch.tensor([x], device=_coll_device(dist), dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(dist):
    if dist is not None:
        dist.barrier()
    if torch.cuda.is_available() and torch.cuda.is_initialized():
        torch.cuda.synchronize()


def job_value(units_per_rank: float, world: int, ms: float) -> float:
    """Whole-job throughput: every rank processes the same units (replicas), in
    ms, the max over ranks of the device time."""
    return world * units_per_rank / (ms * 1e-3)


def run_ours(args):
    import gated_delta_rule_88_b200 as kda
    from gated_delta_rule_88_b200 import workloads as W

    rank, world, local, dist = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    inp_cpu = W.named_prefill(WORKLOAD)
    inp = inp_cpu.to(dev)
    out = torch.empty(B, T, H, D, dtype=torch.bfloat16, device=dev)
    sT = torch.empty(B, H, D, D, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.g, inp.beta, None, None, out, sT)

    for _ in range(max(args.warmup, 0)):
        step()
    barrier(dist)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier(dist)
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        barrier(dist)
    ms_local = ev0.elapsed_time(ev1)
    ms = max_over_ranks(ms_local, dist)
    ms_step = ms / args.steps
    assert kda.kda_get_device_error() == 0
    value = job_value(B * T, world, ms_step)
    peak, peak_kind = measured_peak_hbm()
    achieved = PREFILL_BYTES / (ms_step * 1e-3) / 1e9

    # ---- end to end through the public API with host buffers ----
    pin = {n: getattr(inp_cpu, n).pin_memory() for n in ("q", "k", "v", "g", "beta")}
    out_h = torch.empty(B, T, H, D, dtype=torch.bfloat16).pin_memory()
    sT_h = torch.empty(B, H, D, D, dtype=torch.float32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in pin.values())
    d2h = out_h.numel() * out_h.element_size() + sT_h.numel() * sT_h.element_size()

    def e2e_step():
        # the public host-buffer entry point: the copies of each token range
        # overlap the computation of the previous one
        kda.kda_chunk_fwd_host(pin["q"], pin["k"], pin["v"], pin["g"], pin["beta"],
                               out=out_h, final_state=sT_h, device=dev)

    for _ in range(2):
        e2e_step()
    barrier(dist)
    e2e_steps = max(3, min(args.steps, 20))
    ev0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    ev1.record(stream)
    barrier(dist)
    e2e_ms = max_over_ranks(ev0.elapsed_time(ev1), dist) / e2e_steps

    # ---- decode leg (its timed region is sampled for clocks too) ----
    with ClockSampler(local) as clk_dec:
        dec = decode_leg(kda, W, dev, dist, world, args)
        dec_steps = decode_steps_leg(kda, W, dev, dist, world, args)
        dec_chunk = decode_steps_leg(kda, W, dev, dist, world, args, L=CHUNK_L,
                                     flags=kda.KDA_STEPS_CHUNK, kernel="decode_chunk_kernel",
                                     traffic_key="decode_chunk", ring=1)
        bwd = backward_leg(kda, inp, dev, dist, world, args)
        bwd_chunk = backward_leg(kda, inp, dev, dist, world, args, chunked=True)
    clk.samples += clk_dec.samples
    clk.reasons |= clk_dec.reasons

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": B, "T": T, "H": H, "dk": D, "dv": D, "chunk": 64,
                   "initial_state": "zeros (NULL)", "final_state": "written",
                   "l2": "inputs (404 MB) larger than L2 (126 MB); no flush",
                   "parallelism": f"replicas x{world}" if world > 1 else "1 GPU"},
        "roofline": {"bound": "hbm", "kernel": "kda_chunk_fwd (chunk_prep + chunk_chain)",
                     "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_source": peak_kind,
                     "algorithmic_bytes_per_launch": PREFILL_BYTES,
                     "traffic": measured_traffic("prefill")},
        "e2e": {"value": job_value(B * T, world, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms},
        "gpu_launches": 2 * args.steps,
        "clocks": clk.summary(),
        "decode": dec,
        "decode_steps": dec_steps,
        "decode_chunk": dec_chunk,
        "backward": bwd,
        "backward_chunk": bwd_chunk,
    }
    if rank == 0 and world == 1 and not args.no_cpu:
        line["cpu_baseline"] = cpu_baseline(inp_cpu)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def decode_leg(kda, W, dev, dist, world, args):
    n = args.decode_n
    state = torch.empty(n, DEC_H, D, D, dtype=torch.float32, device=dev)
    state.copy_(W.decode_initial_state(n))
    ring = 8
    toks = [tuple(t.to(dev) for t in W.decode_tokens(i, n)) for i in range(ring)]
    out = torch.empty(n, DEC_H, D, dtype=torch.bfloat16, device=dev)
    steps = max(64, args.decode_steps)
    for i in range(max(3, args.warmup)):
        q, k, v, g, b = toks[i % ring]
        kda.kda_recurrent_step(q, k, v, g, b, state, out)
    barrier(dist)
    s = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for i in range(steps):
        q, k, v, g, b = toks[i % ring]
        kda.kda_recurrent_step(q, k, v, g, b, state, out)
    e1.record(s)
    barrier(dist)
    ms = max_over_ranks(e0.elapsed_time(e1), dist) / steps
    peak, kind = measured_peak_hbm()
    nbytes = decode_bytes(n)
    ach = nbytes / (ms * 1e-3) / 1e9
    return {"workload": f"decode_n{n}_h{DEC_H}_d{D}", "value": job_value(n, world, ms),
            "unit": UNIT, "ms_per_step": ms, "steps": steps,
            "l2": f"state ({n * DEC_H * D * D * 4 >> 20} MiB) larger than L2; no flush",
            "roofline": {"bound": "hbm", "kernel": "decode_step_kernel", "achieved": ach,
                         "peak": peak, "unit": "GB/s", "frac": ach / peak, "peak_source": kind,
                         "algorithmic_bytes_per_launch": nbytes,
                         "traffic": measured_traffic("decode") if n == DEC_N else None}}


STEPS_L = 8          # tokens per call, recurrent serving leg
CHUNK_L = 64         # tokens per call, chunk-form serving leg (the mode-switch length)


def steps_bytes(n, L=STEPS_L):
    """Algorithmic bytes of one serving-decode call: n pool states read and
    written once, L tokens' q, k, v, out (bf16), g, beta (fp32) per
    (sequence, head), and the slot indices."""
    return n * DEC_H * (2 * D * D * 4 + L * (3 * D * 2 + D * 4 + 4 + D * 2)) + n * 4


STEPS_BYTES = steps_bytes(DEC_N)


def decode_steps_leg(kda, W, dev, dist, world, args, L=STEPS_L, flags=0,
                     kernel="decode_pipe_kernel", traffic_key="decode_steps", ring=2):
    """Serving decode: L tokens per sequence per call (kda_recurrent_steps,
    with ``flags``) for the n x 32 decode batch (n = 256 by default), states
    in a pool of 2n entries picked by a seeded slot permutation."""
    n = args.decode_n
    pool_n = 2 * n
    pool = torch.empty(pool_n, DEC_H, D, D, dtype=torch.float32, device=dev)
    pool.copy_(W.decode_initial_state(pool_n, DEC_H, D, D))
    gen = torch.Generator().manual_seed(31)
    slots = torch.randperm(pool_n, generator=gen)[:n].to(torch.int32).to(dev)
    toks = []
    for r in range(ring):
        steps_r = [W.decode_tokens(r * L + l, n) for l in range(L)]
        toks.append(tuple(torch.stack([st[i] for st in steps_r], dim=1).contiguous().to(dev)
                          for i in range(5)))
    out = torch.empty(n, L, DEC_H, D, dtype=torch.bfloat16, device=dev)
    calls = max(16, args.decode_steps // 16)
    for i in range(max(3, args.warmup)):
        kda.kda_recurrent_steps(*toks[i % ring], pool, slots, out=out, flags=flags)
    barrier(dist)
    s = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for i in range(calls):
        kda.kda_recurrent_steps(*toks[i % ring], pool, slots, out=out, flags=flags)
    e1.record(s)
    barrier(dist)
    ms = max_over_ranks(e0.elapsed_time(e1), dist) / calls
    peak, kind = measured_peak_hbm()
    nbytes = steps_bytes(n, L)
    ach = nbytes / (ms * 1e-3) / 1e9
    return {"workload": f"decode_steps_n{n}_l{L}_h{DEC_H}_d{D}_pool{pool_n}",
            "flags": flags, "value": job_value(n * L, world, ms), "unit": UNIT,
            "ms_per_call": ms, "calls": calls,
            "l2": f"pool ({pool_n * DEC_H * D * D * 4 >> 20} MiB) larger than L2; no flush",
            "roofline": {"bound": "hbm", "kernel": kernel, "achieved": ach,
                         "peak": peak, "unit": "GB/s", "frac": ach / peak, "peak_source": kind,
                         "algorithmic_bytes_per_launch": nbytes,
                         "traffic": measured_traffic(traffic_key) if n == DEC_N else None}}


# algorithmic bytes of one backward call on the prefill workload: q, k, v,
# do (bf16) + g, beta (fp32) read; dq, dk, dg, dv (fp32) + dbeta written
BWD_BYTES = B * T * H * (4 * D * 2 + D * 4 + 4 + 4 * D * 4 + 4)


def backward_leg(kda, inp, dev, dist, world, args, chunked=False):
    """Training backward on the prefill workload with a seeded output
    gradient; no initial or final state.  chunked: kda_chunk_bwd (tensor
    cores), else kda_recurrent_bwd."""
    gen = torch.Generator().manual_seed(41)
    do = torch.randn(B, T, H, D, generator=gen).to(torch.bfloat16).to(dev)
    fn = kda.kda_chunk_bwd if chunked else kda.kda_recurrent_bwd
    run = lambda: fn(inp.q, inp.k, inp.v, inp.g, inp.beta, do, want_initial_state_grad=False)
    for _ in range(max(1, min(args.warmup, 3))):
        run()
    barrier(dist)
    calls = 3
    s = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(calls):
        run()
    e1.record(s)
    barrier(dist)
    ms = max_over_ranks(e0.elapsed_time(e1), dist) / calls
    peak, kind = measured_peak_hbm()
    ach = BWD_BYTES / (ms * 1e-3) / 1e9
    if chunked:
        bound, kernel, traffic = "hbm", "kda_chunk_bwd (prep, chain, reverse chain, per-chunk pass)", None
    else:
        bound, kernel = "latency (sequential per token)", "recurrent_bwd_kernel"
        traffic = measured_traffic("backward")
    return {"workload": WORKLOAD + "_backward", "value": job_value(B * T, world, ms),
            "unit": UNIT, "ms_per_call": ms, "calls": calls,
            "roofline": {"bound": bound, "kernel": kernel,
                         "achieved": ach, "peak": peak, "unit": "GB/s", "frac": ach / peak,
                         "peak_source": kind, "algorithmic_bytes_per_launch": BWD_BYTES,
                         "traffic": traffic}}


def cpu_baseline(inp_cpu, tokens=None):
    """The fp64 oracle, as it stands, on the host cores."""
    import oracle
    threads = os.cpu_count() or 1
    n = T if tokens is None else tokens
    sl = lambda x: x[:, :n].contiguous()
    oracle.build()
    t0 = time.perf_counter()
    oracle.forward(sl(inp_cpu.q), sl(inp_cpu.k), sl(inp_cpu.v), sl(inp_cpu.g), sl(inp_cpu.beta),
                   None, None, threads=threads)
    dt = time.perf_counter() - t0
    return {"value": B * n / dt, "unit": UNIT, "cores": min(threads, B * H), "kind": "oracle",
            "sample": f"first {n} tokens of all {H} heads of {WORKLOAD} (fp64, token by token), "
                      f"{dt:.2f} s wall"}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from gated_delta_rule_88_b200 import workloads as W
    import oracle
    oracle.build()
    inp = W.named_prefill(WORKLOAD)
    n = 1024
    sl = lambda x: x[:, :n].contiguous()
    q, k, v, g, b = (sl(inp.q), sl(inp.k), sl(inp.v), sl(inp.g), sl(inp.beta))
    threads = os.cpu_count() or 1
    for _ in range(max(args.warmup, 0)):
        oracle.forward(q, k, v, g, b, threads=threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.forward(q, k, v, g, b, threads=threads)
    dt = (time.perf_counter() - t0) / max(args.steps, 1)
    value = B * n / dt
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": B, "T": T, "H": H, "dk": D, "dv": D,
                   "sample_tokens_per_step": n},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": min(threads, H), "kind": "oracle",
                         "sample": f"first {n} tokens of all {H} heads per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--decode-steps", type=int, default=1024)
    ap.add_argument("--decode-n", type=int, default=DEC_N,
                    help="sequences in the decode legs (a smaller case for profiling)")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU-oracle baseline")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
