#!/usr/bin/env python
"""Benchmark of the gated-delta-rule mixer on B200.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Default workload: one delta-layer prefill, B = 1, T = 4096 tokens, 16 key / 48
value heads, head dim 128 (the headline configuration), metric tokens/s per
layer.  One step = one gdn_prefill call over the whole batch (the conv-state
kernel, then the prefill proper: one overlapped launch of the chunk-parallel
prep and the sequential scan, or the two as separate launches, as the
library's automatic schedule decides), inputs resident in HBM; the L2 is
flushed (256 MiB write) between timed steps and the flush is outside the
timed events.
A secondary line item measures batched decode (256 sequences x 64 steps),
state GB/s.  Under torchrun (N > 1) every rank runs its own batch (weak
scaling, no collective on the data path); the time is the max over ranks.

--impl reference times the fp64 CPU oracle (the correctness reference) on the
host cores instead.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gated_delta_rule_81_b200 import inputs as gin  # noqa: E402

METRIC = "gated-delta prefill tokens/s per layer; decode state GB/s vs B200 HBM peak"

# Algorithmic work per token of a chunk-64 prefill with d = 128 (16 key / 48 value heads):
#   prep kernel: [Q;K]K^T per key head (4 C d) and W = B_W K per value head (2 C d)
#   scan kernel: W S^T, Q S^T, U^T K per value head (6 d^2), U0 = B_U V and P U (4 C d)
def prep_flop_per_token(H_k=16, H_v=48, C=64, d=128):
    return H_k * 4 * C * d + H_v * 2 * C * d          # 1,310,720 at 16/48 heads


def scan_flop_per_token(H_v=48, C=64, d=128):
    return H_v * (6 * d * d + 4 * C * d)              # 6,291,456 at 48 value heads


PREP_FLOP_PER_TOKEN = prep_flop_per_token()
SCAN_FLOP_PER_TOKEN = scan_flop_per_token()
PREFILL_FLOP_PER_TOKEN = PREP_FLOP_PER_TOKEN + SCAN_FLOP_PER_TOKEN     # 7,602,176
PREFILL_BYTES_PER_TOKEN = 20480 + 12288 + 12288 + 192                  # q,k,v + z + out + a,b
DECODE_BYTES_PER_SEQ = 2 * 48 * 128 * 128 * 4                          # fp32 state read + write

# DRAM traffic of one launch from an ncu capture, valid only for the kernel source
# it was taken on (sha256 of the .cu file, first 16 hex digits).
TRAFFIC = {
    (1, "prefill_fused"): {"bytes": 502739968 + 470943744, "sha": "f1c941c89f236f35"},  # ncu, T=4096 16/48, one launch
    (1, "prep"): {"bytes": 87277824 + 383108608, "sha": "f1c941c89f236f35"},
    (1, "scan"): {"bytes": 493164800 + 41825536, "sha": "f1c941c89f236f35"},
    (0, "prep"): {"bytes": 1435904 + 0, "sha": "f1c941c89f236f35"},                  # ncu, T=512 2/6
    (0, "scan"): {"bytes": 7730176 + 0, "sha": "f1c941c89f236f35"},
    (2, "prefill_fused"): {"bytes": 16 * (2214828800 + 1960944128), "sha": "f1c941c89f236f35",
                           "note": "ncu capture of the first 16,384 tokens (fused launch), x16 by tokens"},
    (3, "prep"): {"bytes": round(8.004909618388753 * (306098432 + 1422825216)), "sha": "f1c941c89f236f35",
                 "note": "ncu capture with every packed length scaled to 13,443 tokens in all, x107610/13443"},
    (3, "scan"): {"bytes": round(8.004909618388753 * (1687225856 + 172754176)), "sha": "f1c941c89f236f35",
                 "note": "ncu capture with every packed length scaled to 13,443 tokens in all, x107610/13443"},
}
DECODE_TRAFFIC = {"bytes": 829711104 + 765053696, "sha": "d1cb6c7e2cc2e513"}  # ncu, one step of 256 sequences


def src_sha(name):
    with open(os.path.join(ROOT, "gated_delta_rule_81_b200", "csrc", name), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def decode_traffic():
    """DRAM bytes of one 256-sequence decode launch from the ncu capture, if the source is unchanged."""
    return DECODE_TRAFFIC["bytes"] if DECODE_TRAFFIC["sha"] == src_sha("gdn_decode.cu") else None


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            m = json.load(f)
        return {"hbm_gbs": float(m["hbm_gbs"]), "bf16_tflops": float(m["bf16_tflops"]),
                "bf16_tflops_sustained": float(m.get("bf16_tflops_sustained", m["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ------------------------------------------------------------------ clocks (NVML, sampled during the timed region)


class ClockSampler:
    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, index, period=0.002):
        self.samples, self.reasons, self.period = [], 0, period
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # noqa: BLE001 - clocks are reported as unavailable
            self.max_mhz = None

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def report(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        names = [k for k, bit in self.REASONS.items() if self.reasons & bit and k != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz, "reasons": names,
                "samples": len(self.samples)}


# ------------------------------------------------------------------ distributed plumbing


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
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x, world, device="cuda"):
    if world == 1:
        return x
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard_sequences(lengths, world, rank):
    """Indices of the sequences rank `rank` runs: greedy longest-first onto the
    least-loaded rank (sequences are independent, so no exchange is needed)."""
    loads = [0] * world
    owner = {}
    for i in sorted(range(len(lengths)), key=lambda j: (-lengths[j], j)):
        r = min(range(world), key=lambda k: (loads[k], k))
        owner[i] = r
        loads[r] += lengths[i]
    return [i for i in range(len(lengths)) if owner[i] == rank]


# ------------------------------------------------------------------ workloads


def flush_l2(buf):
    buf.add_(1)  # 256 MiB read + write, more than the 126 MB L2


WORKLOADS = {"prefill4k": 1, "tiny": 0, "fullctx": 2, "varlen": 3}
SCHEDULES = {"auto": 0, "two-launches": 1, "fused": 2}


def case_overrides(args, cfg_id, seed):
    """--tokens: a configuration on a prefix of its tokens (uniform cases) or with every packed
    length scaled to about that total (varlen), the same distributions otherwise."""
    if not getattr(args, "tokens", None):
        return {}
    c = gin.CONFIGS[cfg_id]
    if c["kind"] == "varlen":
        full = gin.varlen_lengths(c["N"], c["len_lo"], c["len_hi"], seed)
        f = args.tokens / sum(full)
        return {"lengths": [max(64, int(n * f)) for n in full]}
    return {"T": args.tokens}


def run_prefill_ours(args, world, rank, dev, pk, cfg_id=1):
    from gated_delta_rule_81_b200 import gdn

    case = gin.prefill_case(cfg_id, seed=rank, **case_overrides(args, cfg_id, rank))
    inp = {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in case["inp"].items()}
    st = case["state_in"].to(dev) if case["state_in"] is not None else None
    varlen = gin.CONFIGS[cfg_id]["kind"] == "varlen"
    N, T_tot = case["N"], case["T_tot"]
    s = gdn.make_inputs(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], inp["z"], inp["conv_w"], inp["A_log"],
                        inp["norm_w"], scale=inp["scale"], schedule=SCHEDULES[args.schedule])
    H_k, H_v = s.H_k, s.H_v
    n_chunks = gdn.chunk_count(case["lengths"])
    ws = torch.empty(gdn.workspace_size(H_k, H_v, N, n_chunks), dtype=torch.uint8, device=dev)
    out = torch.empty(T_tot, H_v, 128, dtype=torch.bfloat16, device=dev)
    S_out = torch.empty(N, H_v, 128, 128, dtype=torch.float32, device=dev)
    C_out = torch.empty(N, 3, (2 * H_k + H_v) * 128, dtype=torch.bfloat16, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(256 * 2**20 // 4, dtype=torch.float32, device=dev).zero_()
    stream = torch.cuda.current_stream()
    cu_dev = case["cu_seqlens"].to(dev)

    def step():
        if varlen:
            gdn.prefill_varlen(s, cu_dev, case["cu_seqlens"], st, None, out=out, state_out=S_out, conv_out=C_out,
                               workspace=ws, err=err)
        else:
            gdn.prefill(s, N, case["lengths"][0], st, None, out=out, state_out=S_out, conv_out=C_out, workspace=ws,
                        err=err)

    for _ in range(args.warmup):
        flush_l2(flush)
        step()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    # per timed step: [step start] helper kernels [lib 0] prep [lib 1] scan [lib 2] [step end]
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
    hooks = []
    with ClockSampler(torch.cuda.current_device()) as clk:
        for ev in evs:
            flush_l2(flush)
            hooks.append(gdn.set_timing_events(s, ev[1:4]))
            ev[0].record(stream)
            step()
            ev[4].record(stream)
        torch.cuda.synchronize()
    gdn.set_timing_events(s, None)
    barrier(world)
    step_ms = [ev[0].elapsed_time(ev[4]) for ev in evs]
    prep_ms = [ev[1].elapsed_time(ev[2]) for ev in evs]
    scan_ms = [ev[2].elapsed_time(ev[3]) for ev in evs]
    total_ms = max_over_ranks(sum(step_ms), world)
    if int(err.item()) != 0:
        raise RuntimeError(f"device error word {int(err.item())}")
    return {"total_ms": total_ms, "step_ms": step_ms, "T": T_tot, "clocks": clk.report(),
            "prefix": bool(getattr(args, "tokens", None)),
            "launches_per_step": 4 if varlen else 3, "case": case, "H_k": H_k, "H_v": H_v, "N": N,
            "kernel_ms": {"prep": statistics.mean(prep_ms), "scan": statistics.mean(scan_ms),
                          "helpers+gaps": statistics.mean(step_ms) - statistics.mean(prep_ms)
                          - statistics.mean(scan_ms)}}


def prefill_roofline(res, cfg_id, pk, ms_per_step):
    """Roofline object of a prefill run: the dominant kernel's algorithmic TFLOP/s from its live
    CUDA-event time (the library's event hook, on the launching stream), against the measured
    bf16 peak; DRAM traffic from the ncu capture of that kernel and workload when the kernel
    source is unchanged since."""
    T = res["T"]
    kt = res["kernel_ms"]
    step_flops = (scan_flop_per_token(res["H_v"]) + prep_flop_per_token(res["H_k"], res["H_v"])) * T
    if kt["prep"] < 0.02:  # one fused launch: the library records its prep/scan split event next to the start
        dom, flops = "prefill_fused", step_flops
        kt = {"prefill_fused": kt["scan"], "helpers+gaps": kt["helpers+gaps"]}
    else:
        dom = "scan" if kt["scan"] >= kt["prep"] else "prep"
        flops = (scan_flop_per_token(res["H_v"]) if dom == "scan" else prep_flop_per_token(res["H_k"], res["H_v"])) * T
    achieved = flops / (kt[dom] * 1e-3) / 1e12
    peak = pk["bf16_tflops"]
    tr = None if res.get("prefix") else TRAFFIC.get((cfg_id, dom))  # (the ncu figures are for the full case)
    traffic = tr["bytes"] if tr and tr.get("sha") == src_sha("gdn_prefill.cu") else None
    return {"kernel": f"{dom}_kernel", "bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "traffic": traffic,
            "traffic_note": tr.get("note") if tr and traffic is not None else None,
            "peak_source": f"{pk['source']} (bf16 burst)",
            "algorithmic_flop_per_launch": flops, "launch_ms": kt[dom],
            "kernel_ms": {k: round(v, 5) for k, v in kt.items()},
            "whole_step": {"achieved": step_flops / (ms_per_step * 1e-3) / 1e12,
                           "frac": step_flops / (ms_per_step * 1e-3) / 1e12 / peak}}


def prefill_secondaries(args, world, rank, dev, pk):
    """The other prefill configurations, each a short run of its own (warm-up, then timed steps
    with the L2 flushed between them), for the record beside the headline."""
    out = []
    for cfg_id, steps in ((0, 20), (2, 3), (3, 5)):
        a = argparse.Namespace(**vars(args))
        a.steps, a.warmup, a.tokens = steps, 3, None
        res = run_prefill_ours(a, world, rank, dev, pk, cfg_id)
        ms = res["total_ms"] / steps
        c = gin.CONFIGS[cfg_id]
        out.append({"workload": c["name"], "metric": "gated-delta prefill tokens/s per layer",
                    "value": world * res["T"] / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms, "steps": steps,
                    "warmup": 3, "sequences": res["N"], "tokens": res["T"],
                    "l2": "flushed between timed steps" + (" (inputs L2-resident: 12 MB)" if cfg_id == 0 else ""),
                    "roofline": prefill_roofline(res, cfg_id, pk, ms), "clocks": res["clocks"],
                    "gpu_launches": res["launches_per_step"] * steps})
        del res
        torch.cuda.empty_cache()
    return out


def run_e2e_prefill(args, world, rank, dev, case):
    """Same workload through the public host-buffer entry point (gdn_prefill_host): every step
    copies its inputs and initial state from pinned host memory to the device, runs the prefill
    and copies the output and final state back to pinned host memory, all inside the timed
    region.  Consecutive steps alternate between two streams, each with its own workspace and
    host output buffers, so that one step's input copies overlap the previous step's compute
    and output copies (the host link is full duplex)."""
    from gated_delta_rule_81_b200 import gdn

    keys = ("q", "k", "v", "a", "b", "z")
    host = {k: case["inp"][k].pin_memory() for k in keys}
    host_state = case["state_in"].pin_memory()
    wts = {k: case["inp"][k].to(dev) for k in ("conv_w", "A_log", "norm_w")}
    T = case["T_tot"]
    H_k, H_v = case["H_k"], case["H_v"]
    s = gdn.make_inputs(host["q"], host["k"], host["v"], host["a"], host["b"], host["z"], wts["conv_w"],
                        wts["A_log"], wts["norm_w"])
    need = gdn.prefill_host_workspace_size(H_k, H_v, 1, T)
    streams = [torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)]
    wss = [torch.empty(need, dtype=torch.uint8, device=dev) for _ in streams]
    outs = [torch.empty(T, H_v, 128, dtype=torch.bfloat16).pin_memory() for _ in streams]
    S_hs = [torch.empty_like(host_state).pin_memory() for _ in streams]
    h2d = sum(t.numel() * t.element_size() for t in host.values()) + host_state.numel() * 4
    d2h = outs[0].numel() * 2 + S_hs[0].numel() * 4
    main = torch.cuda.current_stream()

    def step(i):
        j = i % 2
        gdn.prefill_host(s, 1, T, outs[j], state_in=host_state, state_out=S_hs[j], workspace=wss[j],
                         stream=streams[j])

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(main)
    for st in streams:
        st.wait_event(e0)
    for i in range(args.steps):
        step(i)
    for st in streams:
        done = torch.cuda.Event()
        done.record(st)
        main.wait_event(done)
    e1.record(main)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world)
    return {"value": world * T * args.steps / (ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "api": "gdn_prefill_host, two streams alternating"}


def run_decode_ours(args, dev, steps_per_pass=64, T=1):
    """The decode workload (256 sequences, 64 new tokens each) as 64 / T launches of
    T tokens per sequence.  T = 1 goes through gdn_decode_step; T > 1 through
    gdn_decode_multi with the states in a pool addressed by a permuted slot list."""
    from gated_delta_rule_81_b200 import gdn

    case = gin.decode_case(4)
    N = case["N"]
    state = case["state"].to(dev)
    conv = case["conv_state"].to(dev)
    tok = case["tok"]
    w = {k: v.to(dev) for k, v in case["w"].items()}
    launches = steps_per_pass // T
    if T == 1:
        dtok = {k: tok[k].to(dev) for k in ("q", "k", "v", "a", "b", "z")}
        ins = [gdn.make_inputs(*(dtok[k][i * N:(i + 1) * N] for k in ("q", "k", "v", "a", "b", "z")),
                               w["conv_w"], w["A_log"], w["norm_w"]) for i in range(launches)]
    else:
        # launch i takes steps i*T .. i*T+T-1 of every sequence, sequence-major
        idx = torch.tensor([(i * T + t) * N + n for i in range(launches) for n in range(N) for t in range(T)])
        dtok = {k: tok[k][idx].to(dev) for k in ("q", "k", "v", "a", "b", "z")}
        ins = [gdn.make_inputs(*(dtok[k][i * N * T:(i + 1) * N * T] for k in ("q", "k", "v", "a", "b", "z")),
                               w["conv_w"], w["A_log"], w["norm_w"]) for i in range(launches)]
        slots = torch.randperm(N, generator=torch.Generator().manual_seed(5)).to(torch.int32).to(dev)
    out = torch.empty(N * T, 48, 128, dtype=torch.bfloat16, device=dev)

    def launch(i):
        if T == 1:
            gdn.decode_step(ins[i], N, state, conv, out=out)
        else:
            gdn.decode_multi(ins[i], N, T, state, conv, state_slot=slots, out=out)

    stream = torch.cuda.current_stream()
    for i in range(3):
        launch(i % launches)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(launches):
        launch(i)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    per_launch_s = ms / 1e3 / launches
    gbs = N * DECODE_BYTES_PER_SEQ / per_launch_s / 1e9
    return {"ms_per_launch": ms / launches, "gbs": gbs, "launches": launches, "T": T,
            "tokens_per_s": N * T / per_launch_s}


def run_layer_ours(args, world, rank, dev, pk, T=4096, hidden=5120, H_k=16, H_v=48):
    """One delta-rule layer, y = out_proj(mixer(in_proj(x))), B = 1, T = 4096, hidden 5120,
    16/48 heads, random dense weights (std 1/sqrt(fan_in)); times the three parts with the
    layer's event hook, and cuBLAS (torch.matmul) on the same two projection shapes beside."""
    from gated_delta_rule_81_b200 import gdn

    g = torch.Generator().manual_seed(100 + rank)
    n_in = int(gdn.load().gdn_layer_n_in(H_k, H_v))
    x = torch.randn(T, hidden, generator=g).to(torch.bfloat16).to(dev)
    w_in = (torch.randn(n_in, hidden, generator=g) * hidden ** -0.5).to(torch.bfloat16).to(dev)
    w_out = (torch.randn(hidden, H_v * 128, generator=g) * (H_v * 128) ** -0.5).to(torch.bfloat16).to(dev)
    w = {k: v.to(dev) for k, v in gin.weights(H_k, H_v, seed=rank).items()}
    st = gin.recurrent_state(1, H_v, seed=rank).to(dev)
    L = gdn.make_layer(w_in, w_out, w["conv_w"], w["A_log"], w["norm_w"], H_k, H_v,
                       schedule=SCHEDULES[args.schedule])
    y = torch.empty(T, hidden, dtype=torch.bfloat16, device=dev)
    S = torch.empty(1, H_v, 128, 128, dtype=torch.float32, device=dev)
    ws = torch.empty(gdn.layer_workspace_size(H_k, H_v, 1, T), dtype=torch.uint8, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(256 * 2**20 // 4, dtype=torch.float32, device=dev).zero_()
    stream = torch.cuda.current_stream()

    def step():
        gdn.layer_prefill(L, 1, T, x, st, None, y=y, state_out=S, want_conv=False, workspace=ws, err=err)

    for _ in range(args.warmup):
        flush_l2(flush)
        step()
    torch.cuda.synchronize()
    barrier(world)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    with ClockSampler(torch.cuda.current_device()) as clk:
        for ev in evs:
            flush_l2(flush)
            arr = (ctypes.c_void_p * 4)(*[e.cuda_event or (e.record(stream) or e.cuda_event) for e in ev])
            L.events = ctypes.cast(arr, ctypes.c_void_p)
            step()
        torch.cuda.synchronize()
    L.events = None
    barrier(world)
    if int(err.item()) != 0:
        raise RuntimeError(f"device error word {int(err.item())}")
    parts = {"in_proj": [e[0].elapsed_time(e[1]) for e in evs], "mixer": [e[1].elapsed_time(e[2]) for e in evs],
             "out_proj": [e[2].elapsed_time(e[3]) for e in evs]}
    step_ms = [e[0].elapsed_time(e[3]) for e in evs]
    total_ms = max_over_ranks(sum(step_ms), world)
    # cuBLAS on the same shapes, for comparison
    proj = torch.empty(T, n_in, dtype=torch.bfloat16, device=dev)
    mix = torch.randn(T, H_v * 128, device=dev).to(torch.bfloat16)

    def cublas(fn, reps=10):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        tot = 0.0
        for _ in range(reps):
            flush_l2(flush)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            tot += e0.elapsed_time(e1)
        return tot / reps

    cub = {"in_proj": cublas(lambda: torch.matmul(x, w_in.t(), out=proj)),
           "out_proj": cublas(lambda: torch.matmul(mix, w_out.t(), out=y))}
    flops = {"in_proj": 2 * T * hidden * n_in, "out_proj": 2 * T * H_v * 128 * hidden,
             "mixer": (scan_flop_per_token(H_v) + prep_flop_per_token(H_k, H_v)) * T}
    return {"total_ms": total_ms, "T": T, "parts_ms": {k: statistics.mean(v) for k, v in parts.items()},
            "cublas_ms": cub, "flops": flops, "clocks": clk.report(), "steps": args.steps}


def run_layer_serve_ours(args, world, rank, dev, pk, N=1, T=4096, steps_dec=64, hidden=5120, H_k=16, H_v=48):
    """Prefill -> decode handoff of one delta-rule layer: N prompts of T = 4096 tokens through
    gdn_layer_prefill, then 64 single-token gdn_layer_decode steps that continue in place from
    the prefill's final state and conv buffers (the handoff is the same buffers, no copy).
    Random dense weights (std 1/sqrt(fan_in)); L2 flushed before every timed call."""
    from gated_delta_rule_81_b200 import gdn

    g = torch.Generator().manual_seed(500 + rank)
    n_in = int(gdn.load().gdn_layer_n_in(H_k, H_v))
    C_conv = (2 * H_k + H_v) * 128
    x = torch.randn(N * T, hidden, generator=g).to(torch.bfloat16).to(dev)
    xd = torch.randn(steps_dec, N, hidden, generator=g).to(torch.bfloat16).to(dev)
    w_in = (torch.randn(n_in, hidden, generator=g) * hidden ** -0.5).to(torch.bfloat16).to(dev)
    w_out = (torch.randn(hidden, H_v * 128, generator=g) * (H_v * 128) ** -0.5).to(torch.bfloat16).to(dev)
    w = {k: v.to(dev) for k, v in gin.weights(H_k, H_v, seed=rank).items()}
    L = gdn.make_layer(w_in, w_out, w["conv_w"], w["A_log"], w["norm_w"], H_k, H_v,
                       schedule=SCHEDULES[args.schedule])
    S = torch.empty(N, H_v, 128, 128, dtype=torch.float32, device=dev)
    C = torch.empty(N, 3, C_conv, dtype=torch.bfloat16, device=dev)
    y = torch.empty(N * T, hidden, dtype=torch.bfloat16, device=dev)
    yd = torch.empty(N, hidden, dtype=torch.bfloat16, device=dev)
    ws_p = torch.empty(gdn.layer_workspace_size(H_k, H_v, N, T), dtype=torch.uint8, device=dev)
    ws_d = torch.empty(int(gdn.load().gdn_layer_decode_workspace_size(H_k, H_v, N, 1)), dtype=torch.uint8,
                       device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(256 * 2**20 // 4, dtype=torch.float32, device=dev).zero_()
    stream = torch.cuda.current_stream()

    def hook(ev):
        if ev is None:
            L.events = None
            return None
        arr = (ctypes.c_void_p * 4)(*[e.cuda_event or (e.record(stream) or e.cuda_event) for e in ev])
        L.events = ctypes.cast(arr, ctypes.c_void_p)
        return arr

    def serve(evs_p=None, evs_d=None):
        flush_l2(flush)
        keep = hook(evs_p)
        gdn.layer_prefill(L, N, T, x, None, None, y=y, state_out=S, conv_out=C, workspace=ws_p, err=err)
        for i in range(steps_dec):
            flush_l2(flush)
            keep = hook(evs_d[i] if evs_d else None)
            gdn.layer_decode(L, N, 1, xd[i], S, C, y=yd, workspace=ws_d, err=err)
        hook(None)
        return keep

    for _ in range(max(args.warmup, 1)):
        serve()
    torch.cuda.synchronize()
    barrier(world)
    reps = []
    with ClockSampler(torch.cuda.current_device()) as clk:
        for _ in range(args.steps):
            evs_p = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            evs_d = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps_dec)]
            serve(evs_p, evs_d)
            reps.append((evs_p, evs_d))
        torch.cuda.synchronize()
    barrier(world)
    if int(err.item()) != 0:
        raise RuntimeError(f"device error word {int(err.item())}")
    prefill_ms = [p[0].elapsed_time(p[3]) for p, _ in reps]
    dec = {"in_proj": [], "mixer": [], "out_proj": [], "step": []}
    for _, evs_d in reps:
        for e in evs_d:
            dec["in_proj"].append(e[0].elapsed_time(e[1]))
            dec["mixer"].append(e[1].elapsed_time(e[2]))
            dec["out_proj"].append(e[2].elapsed_time(e[3]))
            dec["step"].append(e[0].elapsed_time(e[3]))
    dec_total = max_over_ranks(sum(dec["step"]), world)
    bytes_step = (n_in * hidden + hidden * H_v * 128) * 2 + N * (2 * H_v * 128 * 128 * 4 + 2 * 3 * C_conv * 2) + \
        N * (hidden * 2 * 2 + n_in * 2 * 2 + H_v * 128 * 2 * 2)
    return {"N": N, "T": T, "steps_dec": steps_dec, "prefill_ms": statistics.mean(prefill_ms),
            "decode_ms": {k: statistics.mean(v) for k, v in dec.items()}, "decode_total_ms": dec_total,
            "bytes_step": bytes_step, "clocks": clk.report(), "steps": args.steps}


def run_attn_layer_ours(args, world, rank, dev, pk, T=4096, hidden=5120):
    """One global-attention layer (24/4 GQA, head dim 256), B = 1, T = 4096, hidden 5120, random
    dense weights (std 1/sqrt(fan_in)); times in_proj, attention (norm + rotary + flash) and
    out_proj with the layer's event hook, and torch's scaled_dot_product_attention (GQA,
    causal) on the same q, k, v shapes beside."""
    from gated_delta_rule_81_b200 import gdn

    g = torch.Generator().manual_seed(200 + rank)
    x = torch.randn(T, hidden, generator=g).to(torch.bfloat16).to(dev)
    w_in = (torch.randn(gdn.ATTN_N_IN, hidden, generator=g) * hidden ** -0.5).to(torch.bfloat16).to(dev)
    w_out = (torch.randn(hidden, 24 * 256, generator=g) * (24 * 256) ** -0.5).to(torch.bfloat16).to(dev)
    qn = (1.0 + 0.1 * torch.randn(256, generator=g)).to(torch.bfloat16).to(dev)
    kn = (1.0 + 0.1 * torch.randn(256, generator=g)).to(torch.bfloat16).to(dev)
    L = gdn.make_attn_layer(w_in, w_out, qn, kn)
    y = torch.empty(T, hidden, dtype=torch.bfloat16, device=dev)
    kc = torch.empty(T, 4, 256, dtype=torch.bfloat16, device=dev)
    vc = torch.empty(T, 4, 256, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(int(gdn.load().gdn_attn_layer_workspace_size(1, T)), dtype=torch.uint8, device=dev)
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(256 * 2**20 // 4, dtype=torch.float32, device=dev).zero_()
    stream = torch.cuda.current_stream()

    def step():
        gdn.attn_layer_prefill(L, 1, T, x, y=y, k_cache=kc, v_cache=vc, workspace=ws, err=err)

    for _ in range(args.warmup):
        flush_l2(flush)
        step()
    torch.cuda.synchronize()
    barrier(world)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    with ClockSampler(torch.cuda.current_device()) as clk:
        for ev in evs:
            flush_l2(flush)
            arr = (ctypes.c_void_p * 4)(*[e.cuda_event or (e.record(stream) or e.cuda_event) for e in ev])
            L.events = ctypes.cast(arr, ctypes.c_void_p)
            step()
        torch.cuda.synchronize()
    L.events = None
    barrier(world)
    if int(err.item()) != 0:
        raise RuntimeError(f"device error word {int(err.item())}")
    parts = {"in_proj": [e[0].elapsed_time(e[1]) for e in evs], "attention": [e[1].elapsed_time(e[2]) for e in evs],
             "out_proj": [e[2].elapsed_time(e[3]) for e in evs]}
    step_ms = [e[0].elapsed_time(e[3]) for e in evs]
    total_ms = max_over_ranks(sum(step_ms), world)
    # torch SDPA on the same shapes (q [1, 24, T, 256], k / v [1, 4, T, 256], causal, GQA)
    q_t = torch.randn(1, 24, T, 256, device=dev).to(torch.bfloat16)
    k_t = torch.randn(1, 4, T, 256, device=dev).to(torch.bfloat16)
    v_t = torch.randn(1, 4, T, 256, device=dev).to(torch.bfloat16)
    sdpa_ms = None
    try:
        for _ in range(3):
            torch.nn.functional.scaled_dot_product_attention(q_t, k_t, v_t, is_causal=True, enable_gqa=True)
        torch.cuda.synchronize()
        tot = 0.0
        for _ in range(10):
            flush_l2(flush)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            torch.nn.functional.scaled_dot_product_attention(q_t, k_t, v_t, is_causal=True, enable_gqa=True)
            e1.record(stream)
            torch.cuda.synchronize()
            tot += e0.elapsed_time(e1)
        sdpa_ms = tot / 10
    except RuntimeError as exc:  # no fused kernel for this shape in the library
        print(f"note: torch SDPA unavailable for the comparison: {exc}", file=sys.stderr)
    n_in = gdn.ATTN_N_IN
    flops = {"in_proj": 2 * T * hidden * n_in, "out_proj": 2 * T * 24 * 256 * hidden,
             "attention": 2 * 2 * 24 * 256 * T * (T + 1) // 2}  # causal QK^T and PV
    return {"total_ms": total_ms, "T": T, "parts_ms": {k: statistics.mean(v) for k, v in parts.items()},
            "sdpa_ms": sdpa_ms, "flops": flops, "clocks": clk.report(), "steps": args.steps}


def run_attn_decode_ours(args, world, rank, dev, pk, N=64, ctx=4096, hidden=5120):
    """One attention-layer decode step for N = 64 sequences whose KV caches hold 4095 rows
    (the step appends row 4096 and attends to all 4096): in_proj GEMM, norm + rotary + cache
    append, split-K attention over the cache, out_proj GEMM.  cache_len is reset before each
    step, outside the timed events."""
    from gated_delta_rule_81_b200 import gdn

    g = torch.Generator().manual_seed(300 + rank)
    x = torch.randn(N, hidden, generator=g).to(torch.bfloat16).to(dev)
    w_in = (torch.randn(gdn.ATTN_N_IN, hidden, generator=g) * hidden ** -0.5).to(torch.bfloat16).to(dev)
    w_out = (torch.randn(hidden, 24 * 256, generator=g) * (24 * 256) ** -0.5).to(torch.bfloat16).to(dev)
    qn = torch.ones(256, dtype=torch.bfloat16, device=dev)
    kc = torch.randn(N, ctx, 4, 256, device=dev).to(torch.bfloat16)
    vc = torch.randn(N, ctx, 4, 256, device=dev).to(torch.bfloat16)
    L = gdn.make_attn_layer(w_in, w_out, qn, qn)
    y = torch.empty(N, hidden, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(int(gdn.load().gdn_attn_decode_workspace_size(N, ctx)), dtype=torch.uint8, device=dev)
    start_len = torch.full((N,), ctx - 1, dtype=torch.int32, device=dev)
    cache_len = start_len.clone()
    err = torch.zeros(1, dtype=torch.int32, device=dev)
    flush = torch.empty(256 * 2**20 // 4, dtype=torch.float32, device=dev).zero_()
    stream = torch.cuda.current_stream()

    def step():
        gdn.attn_layer_decode_step(L, x, kc, vc, cache_len, y=y, workspace=ws, err=err)

    for _ in range(args.warmup):
        cache_len.copy_(start_len)
        flush_l2(flush)
        step()
    torch.cuda.synchronize()
    barrier(world)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    with ClockSampler(torch.cuda.current_device()) as clk:
        for ev in evs:
            cache_len.copy_(start_len)
            flush_l2(flush)
            arr = (ctypes.c_void_p * 4)(*[e.cuda_event or (e.record(stream) or e.cuda_event) for e in ev])
            L.events = ctypes.cast(arr, ctypes.c_void_p)
            step()
        torch.cuda.synchronize()
    L.events = None
    barrier(world)
    if int(err.item()) != 0:
        raise RuntimeError(f"device error word {int(err.item())}")
    parts = {"in_proj": [e[0].elapsed_time(e[1]) for e in evs], "attention": [e[1].elapsed_time(e[2]) for e in evs],
             "out_proj": [e[2].elapsed_time(e[3]) for e in evs]}
    step_ms = [e[0].elapsed_time(e[3]) for e in evs]
    kv_bytes = N * ctx * 4 * 256 * 2 * 2  # K and V rows read by the attention
    return {"total_ms": max_over_ranks(sum(step_ms), world), "parts_ms": {k: statistics.mean(v) for k, v in parts.items()},
            "kv_bytes": kv_bytes, "N": N, "ctx": ctx, "clocks": clk.report(), "steps": args.steps}


# ------------------------------------------------------------------ oracle (CPU) arm


def cpu_oracle_tokens_per_s(min_seconds=10.0, max_reps=8):
    import oracle

    case = gin.prefill_case(1)
    cu = case["cu_seqlens"].tolist()
    oracle.mixer(case["inp"], cu, state_in=case["state_in"], heads=[0], want_conv=False)  # build + warm
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.mixer(case["inp"], cu, state_in=case["state_in"], want_conv=False)
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds or reps >= max_reps:
            break
    return {"value": reps * case["T_tot"] / el, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"full T=4096 layer (48 value heads), fp64, repeated {reps}x ({el:.1f} s)"}


def run_reference(args, world, rank):
    """The fp64 oracle on the host cores (all of them, OpenMP over value heads), one full step
    per timed step: the whole T = 4096, 48-value-head layer, nothing extrapolated."""
    if rank != 0:
        return 0
    import oracle

    case = gin.prefill_case(1)
    cu = case["cu_seqlens"].tolist()
    oracle.mixer(case["inp"], cu, state_in=case["state_in"], heads=[0], want_conv=False)  # build + warm
    for _ in range(args.warmup):
        oracle.mixer(case["inp"], cu, state_in=case["state_in"], want_conv=False)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.mixer(case["inp"], cu, state_in=case["state_in"], want_conv=False)
    el = time.perf_counter() - t0
    s_per_step = el / args.steps
    value = case["T_tot"] / s_per_step
    cfg = {"workload": gin.CONFIGS[1]["name"], "batch": 1, "seq_len": case["T_tot"], "H_k": 16, "H_v": 48,
           "head_dim": 128}
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": s_per_step * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": cfg,
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": f"each step: the whole layer, 48 value heads over T=4096, fp64 "
                                       f"({args.steps} steps in {el:.1f} s)"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ main


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the configurations 0, 2 and 3 that the default line reports beside the headline")
    ap.add_argument("--workload", choices=sorted(WORKLOADS) + ["decode", "layer", "layer_serve", "attn_layer",
                                                              "attn_decode"],
                    default="prefill4k",
                    help="prefill4k (default, the headline line) or another configuration for the record")
    ap.add_argument("--tokens", type=int, default=None,
                    help="prefill workloads: run on a prefix of this many tokens (packed sequences: every "
                         "length scaled to about this total), e.g. for a profiler capture of a smaller case")
    ap.add_argument("--schedule", choices=sorted(SCHEDULES), default="auto",
                    help="prefill launch plan (gdn_inputs.schedule): auto, two-launches, or fused (prep and scan "
                         "overlapped in one launch whenever the scan units fit in half the SMs)")
    ap.add_argument("--serve-seqs", type=int, default=1,
                    help="layer_serve: sequences prefilled and then decoded together")
    ap.add_argument("--attn-seqs", type=int, default=64,
                    help="attn_decode: sequences per step (each with a 4096-row KV cache)")
    ap.add_argument("--decode-tokens", type=int, default=1,
                    help="decode workload: new tokens per sequence per launch (1 .. 8)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        print("note: warm-up raised to 3 steps", file=sys.stderr)
        args.warmup = 3

    world, rank, local = (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
                          int(os.environ.get("LOCAL_RANK", "0")))
    if args.impl == "reference":
        return run_reference(args, world, rank)

    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    from gated_delta_rule_81_b200 import build, gdn

    build.build()
    gdn.load()
    pk = peaks()

    if args.workload == "decode":
        d = run_decode_ours(args, dev, T=args.decode_tokens)
        if rank == 0:
            print(json.dumps({"metric": "decode state GB/s", "value": d["gbs"], "unit": "GB/s", "n_gpus": world,
                              "steps": d["launches"], "warmup": 3, "ms_per_step": d["ms_per_launch"],
                              "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
                              "data": "synthetic",
                              "config": {"workload": gin.CONFIGS[4]["name"], "tokens_per_launch": d["T"],
                                         "state_slots": "permuted pool" if d["T"] > 1 else "slot n",
                                         "tokens_per_s": d["tokens_per_s"]},
                              "roofline": {"bound": "hbm", "achieved": d["gbs"], "peak": pk["hbm_gbs"],
                                           "unit": "GB/s", "frac": d["gbs"] / pk["hbm_gbs"],
                                           "traffic": decode_traffic() if d["T"] == 1 else None},
                              "gpu_launches": d["launches"]}), flush=True)
        return 0
    if args.workload == "attn_decode":
        r = run_attn_decode_ours(args, world, rank, dev, pk, N=args.attn_seqs)
        if rank == 0:
            pm = r["parts_ms"]
            gbs = r["kv_bytes"] / (pm["attention"] * 1e-3) / 1e9
            ms_step = r["total_ms"] / r["steps"]
            print(json.dumps({
                "metric": "attention-layer decode: KV-cache GB/s of the attention segment",
                "value": gbs, "unit": "GB/s", "n_gpus": world, "steps": r["steps"], "warmup": args.warmup,
                "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "f32", "data": "synthetic",
                "config": {"workload": f"attention-decode-{r['N']}seq-ctx4096-hidden5120", "sequences": r["N"],
                           "context": r["ctx"], "tokens_per_s": r["N"] / (ms_step * 1e-3),
                           "l2": "flushed between timed steps"},
                "roofline": {"kernel": "attention decode (norm/rotary + split-K attention + merge)", "bound": "hbm",
                             "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": gbs / pk["hbm_gbs"],
                             "traffic": None, "algorithmic_bytes_per_launch": r["kv_bytes"],
                             "parts_ms": {k: round(v, 5) for k, v in pm.items()}},
                "gpu_launches": 7 * r["steps"], "clocks": r["clocks"]}), flush=True)
        return 0
    if args.workload == "attn_layer":
        r = run_attn_layer_ours(args, world, rank, dev, pk)
        if rank == 0:
            pm = r["parts_ms"]
            tf = {k: r["flops"][k] / (pm[k] * 1e-3) / 1e12 for k in pm}
            ms_step = r["total_ms"] / r["steps"]
            print(json.dumps({
                "metric": "attention-layer prefill tokens/s (in_proj + norm/rotary + flash attention + out_proj)",
                "value": world * r["T"] * r["steps"] / (r["total_ms"] / 1e3), "unit": "tokens/s", "n_gpus": world,
                "steps": r["steps"], "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": "attention-layer-prefill-T4096-hidden5120-24x4x256", "batch": 1,
                           "seq_len": r["T"], "hidden": 5120, "q_heads": 24, "kv_heads": 4, "head_dim": 256,
                           "weights": "random dense, std 1/sqrt(fan_in)", "l2": "flushed between timed steps"},
                "roofline": {"kernel": "attention (norm/rotary + flash_attn_kernel)", "bound": "tensor",
                             "achieved": tf["attention"], "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                             "frac": tf["attention"] / pk["bf16_tflops"], "traffic": None,
                             "peak_source": f"{pk['source']} (bf16 burst)",
                             "algorithmic_flop_per_launch": r["flops"]["attention"],
                             "parts_ms": {k: round(v, 5) for k, v in pm.items()},
                             "parts_tflops": {k: round(v, 1) for k, v in tf.items()}},
                "torch_sdpa": None if r["sdpa_ms"] is None else {
                    "ms": round(r["sdpa_ms"], 5), "tflops": r["flops"]["attention"] / (r["sdpa_ms"] * 1e-3) / 1e12},
                "gpu_launches": 4 * r["steps"], "clocks": r["clocks"]}), flush=True)
        return 0
    if args.workload == "layer_serve":
        r = run_layer_serve_ours(args, world, rank, dev, pk, N=args.serve_seqs)
        if rank == 0:
            dm = r["decode_ms"]
            tok_s = world * r["N"] * r["steps_dec"] * r["steps"] / (r["decode_total_ms"] / 1e3)
            gbs = r["bytes_step"] / (dm["step"] * 1e-3) / 1e9
            print(json.dumps({
                "metric": "delta-layer decode tokens/s after a layer prefill (prefill -> decode handoff)",
                "value": tok_s, "unit": "tokens/s", "n_gpus": world, "steps": r["steps"], "warmup": args.warmup,
                "ms_per_step": r["prefill_ms"] + dm["step"] * r["steps_dec"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": f"delta-layer-serve-{r['N']}seq-prompt{r['T']}-decode{r['steps_dec']}"
                                       f"-hidden5120-16x48", "sequences": r["N"], "prompt": r["T"],
                           "decode_steps": r["steps_dec"], "weights": "random dense, std 1/sqrt(fan_in)",
                           "l2": "flushed before every timed call",
                           "handoff": "decode continues in place on the prefill's state and conv buffers"},
                "prefill_ms": round(r["prefill_ms"], 5),
                "decode_step_ms": {k: round(v, 5) for k, v in dm.items()},
                "roofline": {"kernel": "layer decode step (in_proj GEMM + decode + out_proj GEMM)", "bound": "hbm",
                             "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": gbs / pk["hbm_gbs"],
                             "traffic": None, "algorithmic_bytes_per_step": r["bytes_step"]},
                "gpu_launches": (5 + 3 * r["steps_dec"]) * r["steps"], "clocks": r["clocks"]}), flush=True)
        return 0
    if args.workload == "layer":
        r = run_layer_ours(args, world, rank, dev, pk)
        if rank == 0:
            pm = r["parts_ms"]
            dom = max(pm, key=pm.get)
            achieved = r["flops"][dom] / (pm[dom] * 1e-3) / 1e12
            gemm = {k: {"ms": round(pm[k], 5), "tflops": r["flops"][k] / (pm[k] * 1e-3) / 1e12,
                        "frac_of_peak": r["flops"][k] / (pm[k] * 1e-3) / 1e12 / pk["bf16_tflops"],
                        "cublas_ms": round(r["cublas_ms"][k], 5),
                        "cublas_tflops": r["flops"][k] / (r["cublas_ms"][k] * 1e-3) / 1e12}
                    for k in ("in_proj", "out_proj")}
            ms_step = r["total_ms"] / r["steps"]
            print(json.dumps({
                "metric": "delta-layer prefill tokens/s (in_proj + mixer + out_proj)",
                "value": world * r["T"] * r["steps"] / (r["total_ms"] / 1e3), "unit": "tokens/s", "n_gpus": world,
                "steps": r["steps"], "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": {"workload": "delta-layer-prefill-T4096-hidden5120-16x48", "batch": 1, "seq_len": r["T"],
                           "hidden": 5120, "H_k": 16, "H_v": 48, "weights": "random dense, std 1/sqrt(fan_in)",
                           "l2": "flushed between timed steps"},
                "roofline": {"kernel": dom, "bound": "tensor", "achieved": achieved, "peak": pk["bf16_tflops"],
                             "unit": "TFLOP/s", "frac": achieved / pk["bf16_tflops"], "traffic": None,
                             "peak_source": f"{pk['source']} (bf16 burst)",
                             "parts_ms": {k: round(v, 5) for k, v in pm.items()}},
                "gemm": gemm,
                "gpu_launches": 4 * r["steps"], "clocks": r["clocks"]}), flush=True)
        return 0
    cfg_id = WORKLOADS[args.workload]
    res = run_prefill_ours(args, world, rank, dev, pk, cfg_id)
    T = res["T"]
    total_ms = res["total_ms"]
    value = world * T * args.steps / (total_ms / 1e3)
    ms_per_step = total_ms / args.steps
    roof = prefill_roofline(res, cfg_id, pk, ms_per_step)
    if cfg_id != 1:
        if rank == 0:
            c = gin.CONFIGS[cfg_id]
            print(json.dumps({"metric": "gated-delta prefill tokens/s per layer", "value": value, "unit": "tokens/s",
                              "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                              "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
                              "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                              "config": {"workload": c["name"], "sequences": res["N"], "tokens": T,
                                         "H_k": res["H_k"], "H_v": res["H_v"], "head_dim": 128, "chunk": 64,
                                         "l2": "flushed between timed steps"},
                              "roofline": roof, "gpu_launches": res["launches_per_step"] * args.steps,
                              "clocks": res["clocks"]}), flush=True)
        return 0

    e2e = None if args.no_e2e else run_e2e_prefill(args, world, rank, dev, res["case"])
    decode = None
    if not args.no_decode:
        d = run_decode_ours(args, dev)
        decode = {"workload": gin.CONFIGS[4]["name"], "metric": "decode state GB/s", "value": d["gbs"],
                  "unit": "GB/s", "ms_per_launch": d["ms_per_launch"],
                  "roofline": {"bound": "hbm", "achieved": d["gbs"], "peak": pk["hbm_gbs"], "unit": "GB/s",
                               "frac": d["gbs"] / pk["hbm_gbs"], "traffic": decode_traffic(),
                               "peak_source": pk["source"]}}

    others = None if args.no_secondary else prefill_secondaries(args, world, rank, dev, pk)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_oracle_tokens_per_s()

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": gin.CONFIGS[1]["name"], "batch": 1, "seq_len": T, "H_k": 16, "H_v": 48,
                       "head_dim": 128, "chunk": 64, "state_in": "N(0,0.01) fp32",
                       "l2": "flushed between timed steps (256 MiB write, outside the timed events)",
                       "parallelism": f"dp{world} (independent batch per GPU)"},
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": res["launches_per_step"] * args.steps,
            "clocks": res["clocks"],
            "secondary": decode,
            "secondary_prefill": others,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
