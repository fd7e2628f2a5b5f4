"""Benchmark of the KDA hot path on B200: prefill (chunk forward) and decode.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {ours,reference}]

One step = one kda_chunk_fwd over the headline prefill workload
"varlen8_h32_d128_resume": 8 packed sequences (lengths drawn uniformly in
[1024, 32768], 146,875 tokens), H=32, dk=dv=128, bf16 q/k/v, fp32 g and beta,
a per-sequence fp32 initial state resumed and the 8 final states written.
`value` is whole-job prefill tokens/s (tokens of the packed T axis, all heads)
with inputs resident in HBM; the inputs (7.2 GB) are far larger than the
126 MB L2, so no flush is needed between steps.  `e2e` is the same workload
through the host-buffer entry point (kda_chunk_fwd_host) from pinned host
memory, copies inside the timed region.

Further legs: the dense prefill workloads "prefill_t8192_h32_d128" and
"prefill_t65536_h32_d128" (each with its own roofline); the decode step on
"decode_n256_h32_d128" (256 sequences x 32 heads, fp32 state 512 MiB in
place); serving decode (kda_recurrent_steps: 8 tokens per call recurrent, 64
tokens per call in the chunk form, states in a 512-entry pool picked by slot);
the training backward (recurrent and chunked) on prefill_t8192_h32_d128.

Under torchrun (N > 1) every rank runs the same workload on its own GPU
(independent replicas: the hot path has no exchange step), timing is the max
over ranks, and `value` sums all ranks' tokens ("scaling": "weak").

--impl reference times the fp64 CPU oracle (tests' reference implementation)
on the host cores, each step a bounded sample of the headline workload (the
first 256 tokens of each of its 8 sequences, all 32 heads), reported in the
same metric and unit.  Under torchrun only rank 0 runs it, on the host's
cores, so its value is one host's throughput whatever N is.
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
WORKLOAD = "varlen8_h32_d128_resume"      # the headline (largest single-GPU config)
DENSE_LEGS = ("prefill_t8192_h32_d128", "prefill_t65536_h32_d128")
H, D, C = 32, 128, 64
# per token-head: bf16 q, k, v, out + fp32 g + fp32 beta
TOKEN_BYTES = 3 * D * 2 + D * 4 + 4 + D * 2
STATE_BYTES = D * D * 4
# FLOPs per chunk-head of the chunk form, triangle-aware (2 per multiply-add):
# A (strict lower) and P (lower) C x C x dk; T = (I + A)^-1 ~C^3/6; W, U with
# the unit-lower T; W S, (q e^G) S and the state update C x dk x dv each;
# P V_new lower C x C x dv
CHUNK_FLOPS = 2 * (C * (C - 1) // 2 * D + C * (C + 1) // 2 * D + C ** 3 // 6
                   + 2 * C * (C + 1) // 2 * D + 3 * C * D * D + C * (C + 1) // 2 * D)


def prefill_bytes(tokens, nseq, initial_state):
    """Algorithmic bytes of one prefill call: every token-head's inputs and
    output once, the final states written, the initial states read if given."""
    return tokens * H * TOKEN_BYTES + nseq * H * STATE_BYTES * (2 if initial_state else 1)


def prefill_flops(lens):
    """Chunk-form FLOPs of one call (partial chunks counted as whole ones)."""
    return sum((n + C - 1) // C for n in lens) * H * CHUNK_FLOPS


DEC_N, DEC_H = 256, 32


def decode_bytes(n):
    """Algorithmic bytes of one decode step for n sequences: the fp32 state
    read and written once, the token's q, k, v, out (bf16), g and beta (fp32)."""
    return n * DEC_H * (2 * D * D * 4 + 3 * D * 2 + D * 4 + 4 + D * 2)


DECODE_BYTES = decode_bytes(DEC_N)
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0

# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) from
# one ncu capture of each kernel on this workload (profiles/), valid only for
# the kernel sources it was taken on: reported as null once they change.
_SRC = os.path.join(ROOT, "gated_delta_rule_88_b200", "csrc")
PREFILL_SRC = ["chunk_prep.cu", "prep_common.cuh", "chunk_chain_tc.cu", "chunk_ws.h", "sm100.cuh",
               "common.cuh"]
TRAFFIC = {
    # prep read + write, chain read + write (ncu, one capture each)
    "prefill_t8192_h32_d128": {"files": PREFILL_SRC, "sha": "36d0ac55854a3ca5",
                               "bytes": 336789760 + 257384192 + 304157696 + 50902784},
    "prefill_t65536_h32_d128": {"files": PREFILL_SRC, "sha": "36d0ac55854a3ca5",
                                "bytes": 2692875264 + 2386116096 + 2452307712 + 521305856},
    "varlen8_h32_d128_resume": {"files": PREFILL_SRC, "sha": "36d0ac55854a3ca5",
                                "bytes": 6036765184 + 5413019136 + 5480518400 + 1200050432},
    # per call: prep, forward chain with images, reverse chain, per-chunk pass
    "backward_chunk": {"files": PREFILL_SRC + ["chunk_chain_bwd.cu", "chunk_bwd.cu"], "sha": "4f22c08865933e43",
                       "bytes": 2832923904},
    # per call from saved intermediates: reverse chain, per-chunk pass
    "backward_chunk_saved": {"files": ['chunk_chain_bwd.cu', 'chunk_bwd.cu', 'prep_common.cuh', 'chunk_ws.h', 'sm100.cuh', 'common.cuh'], "sha": "17f685e0cda4b450",
                             "bytes": 304158720 + 163587072 + 811437312 + 497039360},
    # one launch each at full size, -k <kernel> -c 1 (decode legs: --decode-steps 64)
    "decode": {"files": ["decode.cu", "common.cuh"], "sha": "05d923d8fde4c25f",
               "bytes": 547407616 + 479790080},
    "decode_steps": {"files": ["decode_pipe.cu", "common.cuh", "sm100.cuh"],
                     "sha": "4c819c7229465848", "bytes": 621124352 + 497842176},
    "backward": {"files": ["recurrent_bwd.cu", "common.cuh"], "sha": "0c58bb721f4cdeeb",
                 "bytes": 2902945280 + 3862875392 + 1614867456 + 385818880},
    "decode_chunk": {"files": ["decode_chunk_tc.cu", "decode_chunk.cu", "prep_common.cuh", "common.cuh",
                               "sm100.cuh"], "sha": "4a6e5d9712a95aac", "bytes": 1271683072 + 648224512},
}


def measured_traffic(which):
    import hashlib
    t = TRAFFIC.get(which)
    if not t or not t["sha"]:
        return None
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


def measured_peak_bf16():
    """Dense bf16 tensor peak (TFLOP/s): the burst figure, for a kernel timed
    on its own."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


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


def time_calls(fn, steps, warmup, stream, dist):
    """Device time per call (ms, max over ranks) of `steps` calls after
    `warmup` untimed ones, bracketed by barrier + synchronize."""
    for _ in range(max(warmup, 0)):
        fn()
    barrier(dist)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    barrier(dist)
    return max_over_ranks(e0.elapsed_time(e1), dist) / steps


def prefill_roofline(name, inp, ms):
    """Both sides of the prefill roofline for one call: the algorithmic bytes
    at the measured HBM bandwidth and the chunk-form FLOPs at the measured
    dense bf16 peak; the bound is the slower of the two."""
    lens = seq_lens(inp)
    nbytes = prefill_bytes(sum(lens), len(lens), inp.initial_state is not None)
    flops = prefill_flops(lens)
    hbm, hbm_kind = measured_peak_hbm()
    tc, tc_kind = measured_peak_bf16()
    t_hbm, t_tc = nbytes / (hbm * 1e9), flops / (tc * 1e12)
    ach = nbytes / (ms * 1e-3) / 1e9
    line = {"bound": "hbm" if t_hbm >= t_tc else "tensor",
            "kernel": "kda_chunk_fwd (chunk_prep_tc_kernel + chunk_chain_tc_kernel"
                      + (" + chunk_plan_kernel)" if inp.cu_seqlens is not None else ")"),
            "achieved": ach, "peak": hbm, "unit": "GB/s", "frac": ach / hbm,
            "peak_source": hbm_kind, "algorithmic_bytes_per_launch": nbytes,
            "traffic": measured_traffic(name),
            "tensor_side": {"flops_per_launch": flops, "achieved_tflops": flops / (ms * 1e-3) / 1e12,
                            "peak_tflops": tc, "peak_source": tc_kind,
                            "frac": flops / (ms * 1e-3) / 1e12 / tc,
                            "t_hbm_us": t_hbm * 1e6, "t_tensor_us": t_tc * 1e6}}
    return line


def seq_lens(inp):
    if inp.cu_seqlens is None:
        return [inp.q.shape[1]] * inp.q.shape[0]
    cu = inp.cu_seqlens.cpu().tolist()
    return [cu[i + 1] - cu[i] for i in range(len(cu) - 1)]


def prefill_call(kda, inp, out, sT):
    return lambda: kda.kda_chunk_fwd(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.initial_state,
                                     inp.cu_seqlens, out, sT)


def prefill_leg(kda, W, name, dev, dist, world, args):
    """A dense prefill workload as a leg: device time per call and roofline."""
    inp = W.named_prefill(name).to(dev)
    Bq, Tq = inp.q.shape[:2]
    out = torch.empty(Bq, Tq, H, D, dtype=torch.bfloat16, device=dev)
    sT = torch.empty(inp.num_seqs, H, D, D, dtype=torch.float32, device=dev)
    steps = max(3, min(args.steps, 20))
    ms = time_calls(prefill_call(kda, inp, out, sT), steps, max(3, args.warmup),
                    torch.cuda.current_stream(dev), dist)
    assert kda.kda_get_device_error() == 0
    tokens = Bq * Tq
    gb = tokens * H * TOKEN_BYTES / 1e9
    res = {"workload": name, "value": job_value(tokens, world, ms), "unit": UNIT, "ms_per_call": ms,
           "calls": steps, "B": Bq, "T": Tq, "H": H, "dk": D, "dv": D,
           "initial_state": "zeros (NULL)", "final_state": "written",
           "l2": f"inputs ({gb:.2f} GB) larger than L2 (126 MB); no flush",
           "roofline": prefill_roofline(name, inp, ms)}
    del inp, out, sT
    torch.cuda.empty_cache()
    return res


def run_ours(args):
    import gated_delta_rule_88_b200 as kda
    from gated_delta_rule_88_b200 import workloads as W

    rank, world, local, dist = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)

    if args.only_backward or args.only_decode:
        # profiling: just the chunked backward (then the recurrent one), or
        # just the three decode legs
        if args.only_backward:
            bwd_inp = W.named_prefill(BWD_WORKLOAD).to(dev)
            res = {"backward_chunk": backward_leg(kda, bwd_inp, dev, dist, world, args, chunked=True),
                   "backward_chunk_saved": backward_leg(kda, bwd_inp, dev, dist, world, args,
                                                        saved=True),
                   "backward": backward_leg(kda, bwd_inp, dev, dist, world, args)}
        else:
            res = {"decode": decode_leg(kda, W, dev, dist, world, args),
                   "decode_steps": decode_steps_leg(kda, W, dev, dist, world, args),
                   "decode_chunk": decode_steps_leg(kda, W, dev, dist, world, args, L=CHUNK_L,
                                                    flags=kda.KDA_STEPS_CHUNK,
                                                    kernel="decode_chunk_tc_kernel",
                                                    traffic_key="decode_chunk", ring=1)}
        if rank == 0:
            print(json.dumps(res), flush=True)
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()
        return

    if args.only_prefill:
        # profiling: just the prefill calls of one workload (no legs, no e2e)
        inp = W.named_prefill(args.only_prefill).to(dev)
        lens = seq_lens(inp)
        out = torch.empty(*inp.q.shape[:3], D, dtype=torch.bfloat16, device=dev)
        sT = torch.empty(len(lens), H, D, D, dtype=torch.float32, device=dev)
        ms = time_calls(prefill_call(kda, inp, out, sT), args.steps, args.warmup, stream, dist)
        assert kda.kda_get_device_error() == 0
        if rank == 0:
            print(json.dumps({"workload": args.only_prefill, "ms_per_call": ms,
                              "value": job_value(sum(lens), world, ms), "unit": UNIT,
                              "roofline": prefill_roofline(args.only_prefill, inp, ms)}), flush=True)
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()
        return

    # ---- the dense legs first, so their buffers are gone before the headline's ----
    dense = {name: prefill_leg(kda, W, name, dev, dist, world, args) for name in DENSE_LEGS}

    inp_cpu = W.named_prefill(WORKLOAD)
    inp = inp_cpu.to(dev)
    lens = seq_lens(inp_cpu)
    tokens, nseq = sum(lens), len(lens)
    out = torch.empty(1, tokens, H, D, dtype=torch.bfloat16, device=dev)
    sT = torch.empty(nseq, H, D, D, dtype=torch.float32, device=dev)
    step = prefill_call(kda, inp, out, sT)
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
    ms_step = max_over_ranks(ev0.elapsed_time(ev1), dist) / args.steps
    assert kda.kda_get_device_error() == 0
    value = job_value(tokens, world, ms_step)
    roof = prefill_roofline(WORKLOAD, inp, ms_step)

    # ---- end to end through the public API with host buffers ----
    pin = {n: getattr(inp_cpu, n).pin_memory() for n in ("q", "k", "v", "g", "beta", "initial_state")}
    cu_h = inp_cpu.cu_seqlens.contiguous()
    out_h = torch.empty(1, tokens, H, D, dtype=torch.bfloat16).pin_memory()
    sT_h = torch.empty(nseq, H, D, D, dtype=torch.float32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in pin.values()) + cu_h.numel() * 4
    d2h = out_h.numel() * out_h.element_size() + sT_h.numel() * sT_h.element_size()

    def e2e_step():
        # the public host-buffer entry point: the copies of each token range
        # overlap the computation of the previous one
        kda.kda_chunk_fwd_host(pin["q"], pin["k"], pin["v"], pin["g"], pin["beta"],
                               initial_state=pin["initial_state"], cu_seqlens=cu_h,
                               out=out_h, final_state=sT_h, device=dev)

    e2e_ms = time_calls(e2e_step, max(3, min(args.steps, 10)), 2, stream, dist)
    del inp, out, sT
    torch.cuda.empty_cache()

    # ---- decode and backward legs (their timed regions are sampled for clocks too) ----
    with ClockSampler(local) as clk_dec:
        dec = decode_leg(kda, W, dev, dist, world, args)
        dec_steps = decode_steps_leg(kda, W, dev, dist, world, args)
        dec_chunk = decode_steps_leg(kda, W, dev, dist, world, args, L=CHUNK_L,
                                     flags=kda.KDA_STEPS_CHUNK, kernel="decode_chunk_tc_kernel",
                                     traffic_key="decode_chunk", ring=1)
        bwd_inp = W.named_prefill(BWD_WORKLOAD).to(dev)
        bwd = backward_leg(kda, bwd_inp, dev, dist, world, args)
        bwd_chunk = backward_leg(kda, bwd_inp, dev, dist, world, args, chunked=True)
        bwd_saved = backward_leg(kda, bwd_inp, dev, dist, world, args, saved=True)
        del bwd_inp
    clk.samples += clk_dec.samples
    clk.reasons |= clk_dec.reasons

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "num_seqs": nseq, "seq_lens": lens, "T": tokens, "H": H,
                   "dk": D, "dv": D, "chunk": C,
                   "initial_state": "per sequence, 0.02 N(0,1), resumed",
                   "final_state": "written (8 states)",
                   "l2": f"inputs ({tokens * H * TOKEN_BYTES / 1e9:.2f} GB) larger than L2 (126 MB); no flush",
                   "parallelism": f"replicas x{world}" if world > 1 else "1 GPU"},
        "roofline": roof,
        "e2e": {"value": job_value(tokens, world, e2e_ms), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms, "entry_point": "kda_chunk_fwd_host (pinned host buffers)"},
        "gpu_launches": 3 * args.steps,
        "clocks": clk.summary(),
        "prefill_t8192": dense["prefill_t8192_h32_d128"],
        "prefill_t65536": dense["prefill_t65536_h32_d128"],
        "decode": dec,
        "decode_steps": dec_steps,
        "decode_chunk": dec_chunk,
        "backward": bwd,
        "backward_chunk": bwd_chunk,
        "backward_chunk_saved": bwd_saved,
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


# the backward legs run on the 8192-token dense workload
BWD_WORKLOAD = "prefill_t8192_h32_d128"
BWD_T = 8192
# algorithmic bytes of one backward call: q, k, v, do (bf16) + g, beta (fp32)
# read; dq, dk, dg, dv (fp32) + dbeta written
BWD_BYTES = BWD_T * H * (4 * D * 2 + D * 4 + 4 + 4 * D * 4 + 4)


def backward_leg(kda, inp, dev, dist, world, args, chunked=False, saved=False):
    """Training backward on the 8192-token workload with a seeded output
    gradient; no initial or final state.  chunked: kda_chunk_bwd (tensor
    cores), else kda_recurrent_bwd; saved: kda_chunk_bwd from the
    intermediates of one kda_chunk_fwd_save (whose time is reported too)."""
    gen = torch.Generator().manual_seed(41)
    do = torch.randn(1, BWD_T, H, D, generator=gen).to(torch.bfloat16).to(dev)
    stream = torch.cuda.current_stream(dev)
    extra = {}
    if saved:
        out, _, sv = kda.kda_chunk_fwd_save(inp.q, inp.k, inp.v, inp.g, inp.beta,
                                            output_final_state=False)
        fwd = lambda: kda.kda_chunk_fwd_save(inp.q, inp.k, inp.v, inp.g, inp.beta, out=out,
                                             output_final_state=False, saved=sv)
        extra["forward_save_ms"] = time_calls(fwd, 10, 2, stream, dist)
        run = lambda: kda.kda_chunk_bwd(inp.q, inp.k, inp.v, inp.g, inp.beta, do,
                                        want_initial_state_grad=False, saved=sv)
    else:
        fn = kda.kda_chunk_bwd if chunked else kda.kda_recurrent_bwd
        run = lambda: fn(inp.q, inp.k, inp.v, inp.g, inp.beta, do, want_initial_state_grad=False)
    calls = 3 if not (chunked or saved) else 10
    ms = time_calls(run, calls, max(1, min(args.warmup, 3)), stream, dist)
    assert kda.kda_get_device_error() == 0
    peak, kind = measured_peak_hbm()
    ach = BWD_BYTES / (ms * 1e-3) / 1e9
    if saved:
        bound, kernel = "hbm", "kda_chunk_bwd from saved intermediates (reverse chain, per-chunk pass)"
        traffic = measured_traffic("backward_chunk_saved")
    elif chunked:
        bound, kernel = "hbm", "kda_chunk_bwd (prep, chain, reverse chain, per-chunk pass)"
        traffic = measured_traffic("backward_chunk")
    else:
        bound, kernel = "latency (sequential per token)", "recurrent_bwd_kernel"
        traffic = measured_traffic("backward")
    return {"workload": BWD_WORKLOAD + "_backward", "value": job_value(BWD_T, world, ms),
            "unit": UNIT, "ms_per_call": ms, "calls": calls, **extra,
            "roofline": {"bound": bound, "kernel": kernel,
                         "achieved": ach, "peak": peak, "unit": "GB/s", "frac": ach / peak,
                         "peak_source": kind, "algorithmic_bytes_per_launch": BWD_BYTES,
                         "traffic": traffic}}


def _oracle_sample(inp, per_seq):
    """The first `per_seq` tokens of every sequence of a varlen workload, as a
    packed varlen batch (host tensors)."""
    cu = inp.cu_seqlens.tolist()
    idx = torch.cat([torch.arange(cu[i], cu[i] + min(per_seq, cu[i + 1] - cu[i]))
                     for i in range(len(cu) - 1)])
    lens = [min(per_seq, cu[i + 1] - cu[i]) for i in range(len(cu) - 1)]
    cu_s = torch.zeros(len(lens) + 1, dtype=torch.int32)
    cu_s[1:] = torch.cumsum(torch.tensor(lens), 0).to(torch.int32)
    pick = lambda x: x[:, idx].contiguous()
    return (pick(inp.q), pick(inp.k), pick(inp.v), pick(inp.g), pick(inp.beta),
            inp.initial_state.double(), cu_s, sum(lens))


def cpu_baseline(inp_cpu, per_seq=2048, per_seq_1thread=128):
    """The fp64 oracle, as it stands, on the host cores (all threads, and one
    thread on a smaller sample)."""
    import oracle
    threads = os.cpu_count() or 1
    oracle.build()
    q, k, v, g, b, s0, cu, n = _oracle_sample(inp_cpu, per_seq)
    t0 = time.perf_counter()
    oracle.forward(q, k, v, g, b, s0, cu, threads=threads)
    dt = time.perf_counter() - t0
    q, k, v, g, b, s0, cu, n1 = _oracle_sample(inp_cpu, per_seq_1thread)
    t0 = time.perf_counter()
    oracle.forward(q, k, v, g, b, s0, cu, threads=1)
    dt1 = time.perf_counter() - t0
    nseq = inp_cpu.num_seqs
    return {"value": n / dt, "unit": UNIT, "cores": min(threads, nseq * H), "kind": "oracle",
            "sample": f"first {per_seq} tokens of each of the {nseq} sequences of {WORKLOAD}, "
                      f"all {H} heads, initial states resumed ({n} tokens, fp64, token by token), "
                      f"{dt:.2f} s wall",
            "one_thread": {"value": n1 / dt1, "unit": UNIT, "cores": 1,
                           "sample": f"first {per_seq_1thread} tokens of each sequence, all {H} "
                                     f"heads ({n1} tokens), {dt1:.2f} s wall"}}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from gated_delta_rule_88_b200 import workloads as W
    import oracle
    oracle.build()
    inp = W.named_prefill(WORKLOAD)
    per_seq = 256
    q, k, v, g, b, s0, cu, n = _oracle_sample(inp, per_seq)
    threads = os.cpu_count() or 1
    for _ in range(max(args.warmup, 0)):
        oracle.forward(q, k, v, g, b, s0, cu, threads=threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.forward(q, k, v, g, b, s0, cu, threads=threads)
    dt = (time.perf_counter() - t0) / max(args.steps, 1)
    value = n / dt
    nseq = inp.num_seqs
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "num_seqs": nseq, "H": H, "dk": D, "dv": D,
                   "sample_tokens_per_step": n},
        # rank 0 alone works, on the host's cores: one host's figure at any N
        "host": {"ranks_working": 1, "ranks_launched": world},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": min(threads, nseq * H),
                         "kind": "oracle",
                         "sample": f"first {per_seq} tokens of each of the {nseq} sequences, "
                                   f"all {H} heads, per step"},
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
    ap.add_argument("--only-backward", action="store_true",
                    help="profiling: time only the backward legs (chunked, then recurrent)")
    ap.add_argument("--only-decode", action="store_true",
                    help="profiling: time only the three decode legs")
    ap.add_argument("--only-prefill", metavar="WORKLOAD", default=None,
                    help="profiling: time only kda_chunk_fwd on this named workload "
                         "(e.g. varlen8_h32_d128_resume) and print its line")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
