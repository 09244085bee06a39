#!/usr/bin/env python
"""Benchmark of the KDA hot path on B200: prefill tokens/s and decode steps/s, with roofline.

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]

One step = one kda_chunk_fwd call over the packed variable-length prefill workload (64 sequences
of U{512..32768} tokens, H=64, d=128: about 1.07 M tokens, 105 GB of inputs and outputs resident in
HBM) -- the largest of the prefill workloads that fit one GPU.  Extra rows time the B=1, H=32,
T=8192 prefill and the 1 M-token prefill; the backward and module rows run on the T=8192 workload;
the decode row (kda_decode_step over 256 sequences x 64 heads, 128x128 fp32 states, 512 steps) and
rounds of speculative decode (kda_decode_verify of 4 proposed tokens + kda_decode_commit of the
accepted prefix, same states) are timed in the same run.  Every rank runs its own independent batch
(weak scaling, no collective on the data path); timing is on the device with CUDA events, max over
ranks.  Rank 0 prints one JSON line.

--impl reference times the fp64 CPU oracle (the reference arm of this build) on the host cores.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "KDA prefill tokens/s and decode steps/s on 1 B200; % of roofline"
CHUNK = 64
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0

# DRAM bytes of one prefill launch per kernel (kda_prefill_path: 1 cluster, 2 per-unit), captured on
# the named workload; a prefill row scales it by its own algorithmic bytes (both kernels move
# traffic in proportion to the token-heads and units they process)
PREFILL_TRAFFIC = {
    1: {"workload": "prefill_B1_H32_T8192_d128", "bytes_per_launch": 338915584 + 56528384, "src": "c98d8e5f0ae92cd4"},
    2: {"workload": "saturated_B2_H32_T16384_d128", "bytes_per_launch": 1346526000 + 257653760, "src": "9a662f478223b97e"},
}

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch from one ncu capture of each
# kernel (profiles/ gives the commands), keyed by workload, with the hash of the kernel's sources at
# capture time.  Reported only while the sources are unchanged.
NCU_TRAFFIC = {
    "decode_N256_H64_d128_512steps": {"bytes_per_launch": 1094800000 + 1016000000, "src": "6184bb076c425fa7"},
    # one verify launch plus one commit launch (the fourth round of the captured run; commit's
    # bytes depend on how many sequences accepted at least one token)
    "spec_N256_H64_d128_K4": {"bytes_per_launch": 1158062080 + 49587456 + 930634496 + 830093568,
                              "src": "75fe6eba2414bb31"},
    # kda_chunk_bwd on the prefill workload (ncu prints these two counters to five digits)
    "bwd_prefill_B1_H32_T8192_d128": {"bytes_per_launch": 1.2989e9 + 2.5685e9, "src": "9ec2178bcf630624"},
}


def parse_args():
    p = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="kda", choices=["kda", "reference"])
    p.add_argument("--workload", default="varlen_64seq_U512_32768_H64_d128")
    p.add_argument("--extra-workloads", default="prefill_B1_H32_T8192_d128,long_B1_H32_T1048576_d128")
    p.add_argument("--aux-workload", default="prefill_B1_H32_T8192_d128",
                   help="workload of the backward and module rows")
    p.add_argument("--e2e-steps", type=int, default=3)
    p.add_argument("--decode-steps", type=int, default=512)
    p.add_argument("--spec-rounds", type=int, default=64)
    p.add_argument("--no-decode", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--prefill-path", type=int, default=0, choices=[0, 1, 2],
                   help="prefill kernel: 0 chosen from the shapes, 1 cluster kernel, 2 per-unit kernel")
    return p.parse_args()


# ---- algorithmic work (per (token, head) unless stated) -----------------------------------------

def prefill_bytes(w) -> int:
    per_th = 2 * (3 * w.d_k + w.d_v) + (2 * w.d_v if w.gate else 0) + 4 + 2 * w.d_v
    states = w.num_seqs * w.H * w.d_k * w.d_v * 4
    n_states = (1 if w.init_state != "none" else 0) + (1 if w.final_state else 0)
    return w.total_tokens * w.H * per_th + n_states * states


def prefill_flops(w) -> float:
    C, dk, dv = CHUNK, w.d_k, w.d_v
    per_th = 2.0 * (3 * dk * dv + (C + 1) / 2.0 * (3 * dk + 2 * dv) - dk + C * C / 6.0)
    return w.total_tokens * w.H * per_th


def decode_bytes(dw) -> int:
    per_unit = 2 * dw.d_k * dw.d_v * 4 + 2 * (3 * dw.d_k + 2 * dw.d_v) + 4 + 2 * dw.d_v
    return dw.N * dw.H * per_unit


def spec_bytes(sw, accepted) -> int:
    """Algorithmic bytes of one verify + commit round: verify reads every state and the K tokens'
    inputs and writes the outputs and write vectors; commit reads and writes the states of the
    sequences that accepted at least one token, plus those tokens' k, a and write vectors."""
    units = sw.N * sw.H
    state = sw.d_k * sw.d_v * 4
    per_tok_in = 2 * (3 * sw.d_k + 2 * sw.d_v) + 4
    verify = units * (state + sw.K * (per_tok_in + 2 * sw.d_v + 4 * sw.d_v))
    acc = [int(x) for x in accepted.cpu().tolist()]
    moved = sum(1 for x in acc if x > 0) * sw.H
    commit = moved * 2 * state + sum(acc) * sw.H * (2 * 2 * sw.d_k + 4 * sw.d_v)
    return verify + commit


def decode_flops(dw) -> float:
    return dw.N * dw.H * 7.0 * dw.d_k * dw.d_v


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        m = json.load(open(path))
        return float(m["hbm_gbs"]), float(m["bf16_tflops"]), float(m.get("bf16_tflops_sustained", m["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


# source files each kernel is built from (a DRAM traffic figure is reported only while they are
# unchanged since the ncu capture it came from)
KERNEL_SOURCES = {
    "prefill": ("common.cuh", "mma_frag.cuh", "gate_sigmoid.cuh", "umma.cuh", "prefill_fused.cuh", "prefill_tc.cuh"),
    "prefill_cluster": ("common.cuh", "mma_frag.cuh", "gate_sigmoid.cuh", "umma.cuh", "prefill_fused.cuh"),
    "prefill_unit": ("common.cuh", "mma_frag.cuh", "gate_sigmoid.cuh", "umma.cuh", "prefill_tc.cuh"),
    "decode": ("common.cuh", "decode.cuh"),
    "speculative": ("common.cuh", "decode.cuh", "mma_frag.cuh", "async_copy.cuh", "f32x2.cuh", "speculative.cuh"),
    "backward": ("common.cuh", "decode.cuh", "mma_frag.cuh", "async_copy.cuh", "backward.cuh"),
}


def kernel_source_hash(kernel: str | None = None) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "kda_chunkwise_b200", "csrc")
    names = KERNEL_SOURCES[kernel] if kernel else sorted(os.listdir(csrc))
    for name in names:
        if name.endswith((".cu", ".cuh")):
            h.update(open(os.path.join(csrc, name), "rb").read())
    return h.hexdigest()[:16]


def prefill_traffic(w, path: int):
    """DRAM bytes of one prefill launch on w, scaled from the committed capture of the same kernel."""
    import kda_inputs as KI
    t = PREFILL_TRAFFIC.get(path)
    if not t or t["src"] != kernel_source_hash("prefill_cluster" if path == 1 else "prefill_unit"):
        return None, None
    cw = KI.WORKLOADS[t["workload"]]
    scale = prefill_bytes(w) / prefill_bytes(cw)
    return t["bytes_per_launch"] * scale, t["workload"]


def ncu_traffic(key: str, kernel: str):
    """DRAM bytes (read + write) per launch from the committed ncu capture, if still current."""
    t = NCU_TRAFFIC.get(key)
    return t["bytes_per_launch"] if t and t.get("src") == kernel_source_hash(kernel) else None


# ---- multi-rank plumbing (no data-path collective: every rank runs its own batch) --------------

def rank_workload(w, rank: int):
    """Weak scaling: rank r runs an independent batch of the same workload (seed + r)."""
    return w.replace(seed=w.seed + rank)


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of a per-rank scalar over all ranks (the job finishes when the slowest rank does)."""
    if world == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, ms_max: float) -> float:
    """Units processed by all ranks per second, timed by the slowest rank."""
    return units_per_rank * world / (ms_max * 1e-3)


# ---- clocks sampled during the timed regions (NVML, read-only) -----------------------------------

class ClockSampler:
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device, period_s: float = 0.01):
        self.samples, self.reasons, self.ok = [], 0, False
        self.max_mhz = None
        self._stop = threading.Event()
        self._active = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            import torch
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            try:
                self._h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid).encode())
            except Exception:
                self._h = pynvml.nvmlDeviceGetHandleByUUID("GPU-" + uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            return
        self._t = threading.Thread(target=self._run, args=(period_s,), daemon=True)
        self._t.start()

    def _run(self, period):
        while not self._stop.is_set():
            if self._active.is_set():
                try:
                    self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                    self.reasons |= int(self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h))
                except Exception:
                    pass
            time.sleep(period)

    def active(self, on: bool):
        (self._active.set if on else self._active.clear)()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        self._stop.set()
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


# ---- the reference arm: the fp64 oracle on the host cores -------------------------------------

def host_inputs_f64(inp, heads):
    import numpy as np
    h = lambda t: None if t is None else t[:, heads].detach().cpu().double().numpy()
    S0 = inp.get("initial_state")
    return dict(q=h(inp["q"]), k=h(inp["k"]), v=h(inp["v"]), a=h(inp["a"]), beta=h(inp["beta"]),
                gate=h(inp.get("gate")), A_log=inp["A_log"][heads].cpu().double().numpy(),
                cu=inp["cu_seqlens"].cpu().numpy().astype(np.int64),
                S0=None if S0 is None else S0[:, heads].cpu().double().numpy())


def oracle_step(x, threads):
    import oracle
    oracle.kda_fwd(x["q"], x["k"], x["v"], x["a"], x["beta"], x["A_log"], x["cu"], gate=x["gate"],
                   S0=x["S0"], n_threads=threads)


def oracle_sample(inp, w, target_s: float, threads: int):
    """Pick how many heads (full sequences) one oracle pass covers so it takes about target_s."""
    one = host_inputs_f64(inp, [0])
    t0 = time.perf_counter()
    oracle_step(one, 1)
    per_head = max(time.perf_counter() - t0, 1e-6)
    waves_budget = max(1, int(target_s / per_head))
    heads = max(1, min(w.H, waves_budget * max(1, threads)))
    return list(range(heads)), per_head


def sub_batch(inp, w, max_tokens: int):
    """The first sequences of a packed batch, up to about max_tokens tokens (at least one), on the host."""
    import numpy as np
    import torch
    cu = inp["cu_seqlens"].cpu().numpy().astype(np.int64)
    n = 1
    while n < w.num_seqs and cu[n + 1] <= max_tokens:
        n += 1
    T = int(cu[n])
    sub = {k: (v[:T].cpu() if k in ("q", "k", "v", "a", "beta", "gate") and v is not None else v)
           for k, v in inp.items()}
    sub["cu_seqlens"] = torch.from_numpy(cu[: n + 1].astype(np.int32))
    sub["initial_state"] = None if inp["initial_state"] is None else inp["initial_state"][:n].cpu()
    sub["A_log"] = inp["A_log"].cpu()
    return sub, w.replace(seqlens=tuple(int(x) for x in np.diff(cu[: n + 1])))


def cpu_baseline(inp, w, target_s=15.0, max_tokens=65536):
    """The fp64 oracle on the host cores over a bounded sample of the workload: its first sequences
    (up to max_tokens tokens) and as many heads as take about target_s on all cores; plus the same
    oracle single-threaded on one head of one sequence."""
    threads = len(os.sched_getaffinity(0))
    sub, sw = sub_batch(inp, w, max_tokens)
    heads, _ = oracle_sample(sub, sw, target_s, threads)
    x = host_inputs_f64(sub, heads)
    used = min(threads, len(heads) * sw.num_seqs)
    t0 = time.perf_counter()
    oracle_step(x, used)
    dt = time.perf_counter() - t0
    tokens = sw.total_tokens * len(heads) / w.H
    one, ow = sub_batch(inp, w, 1)
    x1 = host_inputs_f64(one, [0])
    t1 = time.perf_counter()
    oracle_step(x1, 1)
    dt1 = time.perf_counter() - t1
    return {"value": tokens / dt, "unit": "tokens/s", "cores": used, "kind": "oracle",
            "single_thread": {"value": ow.total_tokens / w.H / dt1, "unit": "tokens/s", "cores": 1,
                              "sample": f"1 head x {ow.total_tokens} tokens (one sequence), {dt1:.2f} s"},
            "sample": f"{len(heads)} of {w.H} heads x the first {sw.num_seqs} sequences ({sw.total_tokens} tokens) "
                      f"of {w.name} (fp64 token-by-token recurrence, {dt:.2f} s wall); tokens/s counts whole "
                      f"tokens of all {w.H} heads"}


def run_reference(args):
    import torch

    import kda_inputs as KI
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    w = KI.WORKLOADS[args.workload]
    small = w.replace(seqlens=w.seqlens[:2]) if w.num_seqs > 2 else w
    inp, sw = sub_batch(KI.make_inputs(small, "cpu"), small, 32768)
    threads = len(os.sched_getaffinity(0))
    heads, per_head = oracle_sample(inp, sw, target_s=1.0, threads=threads)
    x = host_inputs_f64(inp, heads)
    used = min(threads, len(heads) * sw.num_seqs)
    for _ in range(args.warmup):
        oracle_step(x, used)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(x, used)
    dt = (time.perf_counter() - t0) / args.steps
    tokens = sw.total_tokens * len(heads) / w.H
    value = tokens / dt
    sample = (f"{len(heads)} of {w.H} heads x the first {sw.num_seqs} sequences ({sw.total_tokens} tokens) "
              f"of {w.name} per step (fp64 oracle; throughput counts whole tokens of all heads)")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.num_seqs, "H": w.H, "T": w.total_tokens,
                   "d_k": w.d_k, "d_v": w.d_v},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": used, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }))
    return 0


# ---- the CUDA arm ------------------------------------------------------------------------------

def time_calls(fn, steps: int, warmup: int, stream, world, dev, barrier, clocks=None):
    """Milliseconds per call of fn (CUDA events on `stream`, after warm-up), max over ranks."""
    import torch
    for _ in range(warmup):
        fn()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if clocks:
        clocks.active(True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    if clocks:
        clocks.active(False)
    barrier()
    return max_over_ranks(e0.elapsed_time(e1) / steps, world, dev)


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=dev)

    import kda_chunkwise_b200 as kda
    import kda_inputs as KI
    if args.prefill_path:
        kda.kda_set_prefill_path(args.prefill_path)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    stream = torch.cuda.current_stream(dev)
    hbm, tf, tf_sus, peak_src = peaks()

    def prefill_setup(w):
        inp = KI.make_inputs(w, dev)
        max_seqlen = max(w.seqlens)
        ws_bytes = kda.kda_chunk_fwd_workspace_size(w.total_tokens, w.num_seqs, max_seqlen, w.H, w.d_k, w.d_v)
        workspace = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
        out = torch.empty((w.total_tokens, w.H, w.d_v), dtype=torch.bfloat16, device=dev)
        S_final = torch.empty((w.num_seqs, w.H, w.d_k, w.d_v), dtype=torch.float32, device=dev)

        def step():
            kda.kda_chunk_fwd(inp["q"], inp["k"], inp["v"], inp["a"], inp["beta"], inp["A_log"],
                              inp["cu_seqlens"], gate=inp["gate"], initial_state=inp["initial_state"],
                              out=out, final_state=S_final, max_seqlen=max_seqlen,
                              workspace=workspace, stream=stream)
        return inp, out, S_final, step

    def prefill_roofline(w, ms):
        bytes_step, flops_step = prefill_bytes(w), prefill_flops(w)
        achieved = bytes_step / (ms * 1e-3) / 1e9
        traffic, captured = prefill_traffic(w, kda.kda_prefill_path(w.num_seqs * w.H, w.d_k, w.d_v))
        return {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                "frac": achieved / hbm, "traffic": traffic,
                "traffic_source": (f"dram__bytes_read.sum + dram__bytes_write.sum of one ncu capture of the same "
                                   f"kernel on {captured} (profiles/), scaled by algorithmic bytes to this "
                                   f"workload; reported while the kernel sources are unchanged since"
                                   if traffic is not None else "no current ncu capture of these kernel sources"),
                "peak_source": f"hbm_gbs of {peak_src}",
                "scope": "one kda_chunk_fwd call (all kernels of the prefill path)",
                "algorithmic_bytes": bytes_step, "algorithmic_flops": flops_step,
                "tensor_frac_of_bf16_peak": flops_step / (ms * 1e-3) / 1e12 / tf}

    # ---- headline: the packed variable-length prefill ----
    w = rank_workload(KI.WORKLOADS[args.workload], rank)
    inp, out, S_final, step = prefill_setup(w)
    clocks = ClockSampler(dev)
    for _ in range(args.warmup):
        step()
    kda.kda_sync_check()
    launches0 = kda.kda_launch_count()
    ms = time_calls(step, args.steps, 0, stream, world, dev, barrier, clocks)
    launches = kda.kda_launch_count() - launches0
    kda.kda_sync_check()
    value = whole_job_rate(w.total_tokens, world, ms)
    bytes_step = prefill_bytes(w)
    roofline = prefill_roofline(w, ms)
    path = kda.kda_prefill_path(w.num_seqs * w.H, w.d_k, w.d_v)
    src_hash = kernel_source_hash()

    # ---- end to end through the public API: kda_chunk_fwd_host on page-locked host tensors (the
    #      copies to and from the device, piece by piece, overlapped with the prefill) ----
    e2e = None
    if not args.no_e2e:
        names = ["q", "k", "v", "a", "beta", "gate", "A_log", "cu_seqlens", "initial_state"]
        host_in = {}
        for n in names:   # straight into page-locked buffers (no pageable intermediate copy)
            if inp[n] is not None:
                host_in[n] = torch.empty(inp[n].shape, dtype=inp[n].dtype, pin_memory=True)
                host_in[n].copy_(inp[n])
        out_h = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        S_h = torch.empty(S_final.shape, dtype=S_final.dtype, pin_memory=True)
        h2d = sum(t.numel() * t.element_size() for t in host_in.values())
        d2h = out_h.numel() * out_h.element_size() + S_h.numel() * S_h.element_size()
        del inp, out, S_final, step
        torch.cuda.empty_cache()
        hbuf = torch.empty(kda.kda_chunk_fwd_host_buffer_size(host_in["cu_seqlens"], w.H, w.d_k, w.d_v, torch.bfloat16),
                           dtype=torch.uint8, device=dev)

        def e2e_step():
            kda.kda_chunk_fwd_host(host_in["q"], host_in["k"], host_in["v"], host_in["a"], host_in["beta"],
                                   host_in["A_log"], host_in["cu_seqlens"], gate=host_in.get("gate"),
                                   initial_state=host_in.get("initial_state"), out=out_h, final_state=S_h,
                                   device_buffer=hbuf, stream=stream)

        ems = time_calls(e2e_step, args.e2e_steps, 1, stream, world, dev, barrier)
        kda.kda_sync_check()
        e2e = {"value": whole_job_rate(w.total_tokens, world, ems), "unit": "tokens/s",
               "ms_per_step": ems, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "steps": args.e2e_steps, "workload": w.name,
               "api": "kda_chunk_fwd_host (2048-token pieces; copies in, prefill, copies out on three streams)"}
        cpu_src = {k: v for k, v in host_in.items()}
        del hbuf, out_h, S_h
        torch.cuda.empty_cache()
    else:
        cpu_src = inp
        del out, S_final, step

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(cpu_src, w)
    del cpu_src
    if not args.no_e2e:
        del host_in
    else:
        del inp
    torch.cuda.empty_cache()

    # ---- extra prefill rows ----
    extra = []
    for name in [x for x in args.extra_workloads.split(",") if x]:
        xw = rank_workload(KI.WORKLOADS[name], rank)
        xinp, xout, xS, xstep = prefill_setup(xw)
        xsteps = 3 if xw.total_tokens * xw.H > 8_000_000 else args.steps
        xms = time_calls(xstep, xsteps, max(3, min(args.warmup, 3)), stream, world, dev, barrier, clocks)
        kda.kda_sync_check()
        extra.append({"workload": xw.name, "value": whole_job_rate(xw.total_tokens, world, xms), "unit": "tokens/s",
                      "ms_per_step": xms, "steps": xsteps,
                      "kernel": "per-unit" if kda.kda_prefill_path(xw.num_seqs * xw.H, xw.d_k, xw.d_v) == 2 else "cluster",
                      "roofline": prefill_roofline(xw, xms)})
        del xinp, xout, xS, xstep
        torch.cuda.empty_cache()

    aw = rank_workload(KI.WORKLOADS[args.aux_workload], rank)
    ainp = KI.make_inputs(aw, dev)
    aout = torch.empty((aw.total_tokens, aw.H, aw.d_v), dtype=torch.bfloat16, device=dev)

    # backward row: kda_chunk_bwd on the aux workload (gradients of every input)
    backward = None
    if not args.no_decode:
        gb = torch.Generator(device=dev).manual_seed(201 + rank)
        dout = torch.randn((aw.total_tokens, aw.H, aw.d_v), generator=gb, device=dev) * 0.1
        dST = torch.randn((aw.num_seqs, aw.H, aw.d_k, aw.d_v), generator=gb, device=dev) * 0.1
        bws = torch.empty(kda.kda_chunk_bwd_workspace_size(aw.total_tokens, aw.num_seqs, aw.H, aw.d_k, aw.d_v),
                          dtype=torch.uint8, device=dev)

        def bstep():
            return kda.kda_chunk_bwd(ainp["q"], ainp["k"], ainp["v"], ainp["a"], ainp["beta"], ainp["A_log"],
                                     ainp["cu_seqlens"], dout, gate=ainp["gate"], initial_state=ainp["initial_state"],
                                     dfinal_state=dST, workspace=bws, stream=stream)

        bms = time_calls(bstep, 3, 1, stream, world, dev, barrier)
        kda.kda_sync_check()
        th = aw.total_tokens * aw.H
        # inputs (as the forward) + dout (fp32) read; dq, dk, da, dv, dgate (fp32), dbeta written;
        # initial state and its gradient, final-state gradient
        bbytes = th * (2 * (3 * aw.d_k + 2 * aw.d_v) + 4 + 4 * aw.d_v + 4 * (3 * aw.d_k + 2 * aw.d_v) + 4) + \
            3 * aw.num_seqs * aw.H * aw.d_k * aw.d_v * 4
        bach = bbytes / (bms * 1e-3) / 1e9
        backward = {"value": whole_job_rate(aw.total_tokens, world, bms), "unit": "tokens/s", "ms_per_step": bms,
                    "workload": aw.name, "scope": "one kda_chunk_bwd call",
                    "roofline": {"bound": "latency (sequential token steps per unit)", "achieved": bach,
                                 "peak": hbm, "unit": "GB/s", "frac": bach / hbm,
                                 "traffic": ncu_traffic("bwd_" + aw.name, "backward"),
                                 "peak_source": f"hbm_gbs of {peak_src}", "algorithmic_bytes": bbytes}}
        del bws
        torch.cuda.empty_cache()
        # the same gradients in chunkwise form (kda_chunk_bwd_chunkwise: four launches, the products
        # on the tensor cores), timed beside the token-level kernel that kda_chunk_bwd runs by default
        cws = torch.empty(kda.kda_chunk_bwd_chunkwise_workspace_size(aw.total_tokens, aw.num_seqs, aw.H, aw.d_k, aw.d_v),
                          dtype=torch.uint8, device=dev)

        def cstep():
            return kda.kda_chunk_bwd(ainp["q"], ainp["k"], ainp["v"], ainp["a"], ainp["beta"], ainp["A_log"],
                                     ainp["cu_seqlens"], dout, gate=ainp["gate"], initial_state=ainp["initial_state"],
                                     dfinal_state=dST, workspace=cws, stream=stream, chunkwise=True)

        cms = time_calls(cstep, 3, 1, stream, world, dev, barrier)
        kda.kda_sync_check()
        backward["chunkwise"] = {"value": whole_job_rate(aw.total_tokens, world, cms), "unit": "tokens/s",
                                 "ms_per_step": cms, "frac_of_hbm_peak": bbytes / (cms * 1e-3) / 1e9 / hbm,
                                 "scope": "one kda_chunk_bwd(chunkwise=True) call: bc_prep, bc_state, bc_dstate, "
                                          "bc_grad"}
        del dout, dST, cws
        torch.cuda.empty_cache()

    # module row: the short convolution of q, k, v (q, k L2-normalised) and the pre-gate
    # normalisation + gate of one fp32 output, on the aux workload's tensors
    module = None
    if not args.no_decode:
        gm = torch.Generator(device=dev).manual_seed(101 + rank)
        cw = torch.randn((aw.H, aw.d_k, 4), generator=gm, device=dev) * 0.5
        nw = torch.rand((aw.d_v,), generator=gm, device=dev) + 0.5
        o32 = torch.randn((aw.total_tokens, aw.H, aw.d_v), generator=gm, device=dev)
        yq, yk, yv = (torch.empty_like(ainp[key]) for key in ("q", "k", "v"))

        def mstep():
            kda.kda_short_conv(ainp["q"], cw, ainp["cu_seqlens"], l2norm=True, out=yq, stream=stream)
            kda.kda_short_conv(ainp["k"], cw, ainp["cu_seqlens"], l2norm=True, out=yk, stream=stream)
            kda.kda_short_conv(ainp["v"], cw, ainp["cu_seqlens"], l2norm=False, out=yv, stream=stream)
            kda.kda_output_norm_gate(o32, ainp["gate"], nw, out=aout, stream=stream)

        mms = time_calls(mstep, args.steps, max(3, args.warmup), stream, world, dev, barrier)
        kda.kda_sync_check()
        th = aw.total_tokens * aw.H
        mbytes = 3 * 2 * th * aw.d_k * 2 + th * aw.d_v * (4 + 2 + 2)   # conv read + write x3; o, gate, out
        mach = mbytes / (mms * 1e-3) / 1e9
        module = {"value": whole_job_rate(aw.total_tokens, world, mms), "unit": "tokens/s", "ms_per_step": mms,
                  "workload": aw.name, "scope": "3 kda_short_conv (width 4) + 1 kda_output_norm_gate",
                  "roofline": {"bound": "hbm", "achieved": mach, "peak": hbm, "unit": "GB/s",
                               "frac": mach / hbm, "traffic": None, "peak_source": f"hbm_gbs of {peak_src}",
                               "algorithmic_bytes": mbytes}}
        del o32, yq, yk, yv
    del ainp, aout
    torch.cuda.empty_cache()

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    # decode row: 512 back-to-back steps over fixed states (each step reads and writes 1.07 GB)
    decode = None
    if not args.no_decode:
        dw = dataclasses.replace(KI.DECODE, seed=KI.DECODE.seed + rank, steps=args.decode_steps)
        d = KI.make_decode_inputs(dw, dev)
        state = d["state"].clone()
        dout = torch.empty((dw.N, dw.H, dw.d_v), dtype=torch.bfloat16, device=dev)

        def dstep(t):
            kda.kda_decode_step(d["q"][t], d["k"][t], d["v"][t], d["a"][t], d["beta"][t],
                                d["A_log"], state, gate=d["gate"][t], out=dout, stream=stream)

        for t in range(max(3, args.warmup)):
            dstep(t % dw.steps)
        state.copy_(d["state"])
        barrier()
        clocks.active(True)
        e0.record(stream)
        for t in range(dw.steps):
            dstep(t)
        e1.record(stream)
        torch.cuda.synchronize()
        clocks.active(False)
        barrier()
        kda.kda_sync_check()
        dms = max_over_ranks(e0.elapsed_time(e1) / dw.steps, world, dev)
        dbytes = decode_bytes(dw)
        dach = dbytes / (dms * 1e-3) / 1e9
        decode = {"value": whole_job_rate(1, world, dms), "unit": "steps/s", "ms_per_step": dms,
                  "workload": dw.name, "tokens_per_s": whole_job_rate(dw.N, world, dms),
                  "roofline": {"bound": "hbm", "achieved": dach, "peak": hbm, "unit": "GB/s",
                               "frac": dach / hbm, "traffic": ncu_traffic(dw.name, "decode"),
                               "peak_source": f"hbm_gbs of {peak_src}",
                               "algorithmic_bytes": dbytes}}
        del d, state, dout
        torch.cuda.empty_cache()

    # speculative decode row: rounds of verify (K proposed tokens) + commit (accepted prefixes)
    spec = None
    if not args.no_decode:
        sw = dataclasses.replace(KI.SPEC, seed=KI.SPEC.seed + rank, rounds=args.spec_rounds)
        d = KI.make_spec_inputs(sw, dev)
        state = d["state"].clone()
        sout = torch.empty((sw.N, sw.K, sw.H, sw.d_v), dtype=torch.bfloat16, device=dev)
        su = torch.empty((sw.N, sw.H, sw.K, sw.d_v), dtype=torch.float32, device=dev)

        def sround(r):
            kda.kda_decode_verify(d["q"][r], d["k"][r], d["v"][r], d["a"][r], d["beta"][r], d["A_log"],
                                  state, gate=d["gate"][r], u=su, out=sout, stream=stream)
            kda.kda_decode_commit(d["k"][r], d["a"][r], d["A_log"], d["accepted"][r], su, state,
                                  stream=stream)

        for r in range(max(3, args.warmup)):
            sround(r % sw.rounds)
        state.copy_(d["state"])
        barrier()
        clocks.active(True)
        e0.record(stream)
        for r in range(sw.rounds):
            sround(r)
        e1.record(stream)
        torch.cuda.synchronize()
        clocks.active(False)
        barrier()
        kda.kda_sync_check()
        sms = max_over_ranks(e0.elapsed_time(e1) / sw.rounds, world, dev)
        sbytes = sum(spec_bytes(sw, d["accepted"][r]) for r in range(sw.rounds)) / sw.rounds
        accepted_per_round = float(d["accepted"].to(torch.float64).sum()) / sw.rounds   # tokens, all heads
        sach = sbytes / (sms * 1e-3) / 1e9
        spec = {"value": whole_job_rate(accepted_per_round, world, sms), "unit": "accepted tokens/s",
                "ms_per_round": sms, "workload": sw.name, "proposed_per_round": sw.N * sw.K,
                "accepted_per_round": accepted_per_round,
                "roofline": {"bound": "hbm", "achieved": sach, "peak": hbm, "unit": "GB/s",
                             "frac": sach / hbm, "traffic": ncu_traffic(sw.name, "speculative"),
                             "peak_source": f"hbm_gbs of {peak_src}",
                             "algorithmic_bytes": int(sbytes),
                             "scope": "one round = kda_decode_verify + kda_decode_commit"}}
        del d, state, sout, su
        torch.cuda.empty_cache()

    clk = clocks.summary()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            # tensor-core operands: tf32 (diagonal Gram blocks), fp16 (off-diagonal Gram blocks and
            # the value path); accumulation, the decay arithmetic and the carried state are fp32
            "dtype": "tf32/fp16 mma, f32 accumulate",
            "data": "synthetic",
            "config": {"workload": w.name, "B": w.num_seqs, "H": w.H, "T": w.total_tokens,
                       "d_k": w.d_k, "d_v": w.d_v, "chunk": CHUNK, "tile": 16,
                       "kernel": "per-unit" if path == 2 else "cluster",
                       "parallelism": f"independent batch per rank x{world}",
                       "l2": f"inputs larger than L2 ({bytes_step / 1e6:.0f} MB per step > 126 MB); no flush"},
            "roofline": roofline, "prefill_rows": extra, "backward": backward, "module": module, "decode": decode,
            "speculative": spec, "e2e": e2e, "cpu_baseline": cpu,
            "gpu_launches": launches, "clocks": clk, "kernel_src": src_hash,
        }
        print(json.dumps(line))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
