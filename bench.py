"""Benchmark of the GDN-2 recurrence on B200.

One step = one chunked prefill (gdn2_chunk_fwd) of the 48-V-head, d=128 layer
over T=32768 tokens of one sequence (bf16 q,k,v, fp32 per-channel gates,
chunk 64), inputs resident in HBM. The decode workload (B=256 sequences, one
token per step, fp32 states [256,48,128,128]) is timed in the same run and
reported under "decode"; so are the conv + L2 prefill (B=8, T=8192,
"conv_prefill"), the headline prefill with other gate layouts (bf16
logits, "prefill_gate_logits"; alpha and b per QK head, "prefill_qk_gates")
and decode with the conv in the step ("decode_conv").

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload prefill_t32768|prefill_t4096] [--decode-workload decode_b256|decode_b64]
                    [--decode-steps N] [--conv-steps N] [--e2e-steps N] [--logits-steps N]
                    [--qk-gates-steps N] [--decode-conv-steps N]

(--workload prefill_t4096 / --decode-workload decode_b64 are the small cases
the ncu captures run; a count of 0 skips that part.)

Multi-GPU (torchrun, one rank per GPU): every rank runs its own sequence
(independent problems, no data-path collective); value = tokens of all ranks /
max-over-ranks time ("weak" scaling).

--impl reference times the float64 CPU oracle (the only other code path that
computes the recurrence) on the host cores, on a bounded sample of the same
workload.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "prefill tokens/s (48 Vheads x 128^2, T=32K) + % tensor peak; decode HBM GB/s"
PREFILL = "prefill_t32768"
DECODE = "decode_b256"
CONV = "conv_prefill_b8_t8192"
L2_BYTES = 126 * 2**20

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of the prefill
# launches of one T=32768 call, and the hash of the kernel sources they were
# taken on (with other sources the figure is stale and the bench reports
# null). Taken on the T=4096 case (its 2 segments' prep and scan launches,
# 802.4 MB per call, 1.83x its algorithmic bytes) and scaled by the chunk
# count (x8): the slot round trip, which is most of the excess, grows with the
# chunks; the full-size workload is too large for a multi-metric capture.
TRAFFIC_KERNEL_SOURCES = ("delta_rule_linear_gdn_b200/csrc/chunk_tc.cu", "delta_rule_linear_gdn_b200/csrc/tc_prims.cuh")
TRAFFIC = {"sha1": "34f4ca12cb460ea74255900992863d368e16e93a",
           "bytes_per_call": 6419318784}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ------------------------------------------------------------------ accounting

def prefill_bytes(w, gate_mode="full", o_bytes=2, s0=False, gate_bytes=4, qk_gates=False):
    """Algorithmic HBM bytes of one chunk_fwd call: every input read once, every
    output written once (gate_bytes: 4 for fp32 gate values, 2 for bf16 logits;
    qk_gates: alpha and b owned by the QK heads, H_qk of them)."""
    tok = w.B * w.T
    qkb = 2 if w.qkv_dtype == "bf16" else 4
    n = tok * w.H_qk * w.d * qkb * 2 + tok * w.H_v * w.d * qkb
    hg = w.H_qk if qk_gates else w.H_v
    if gate_mode == "full":
        n += tok * (2 * hg + w.H_v) * w.d * gate_bytes
    elif gate_mode == "kda":
        n += tok * hg * (w.d + 1) * gate_bytes
    else:
        n += tok * hg * 2 * gate_bytes
    n += tok * w.H_v * w.d * o_bytes
    n += w.B * w.H_v * w.d * w.d * 4 * (2 if s0 else 1)
    if w.conv:
        n += (2 * w.H_qk * w.d + w.H_v * w.d) * 16
    return n


def prefill_flops(w):
    """Algorithmic FLOPs per call: 6d² + 5Cd per token per value head (state
    products Q̄S, ĒS, K_endᵀU; T and A_qk Gram triangles; A_qk·U; the solve)."""
    return w.B * w.T * w.H_v * (6 * w.d * w.d + 5 * w.chunk * w.d)


def decode_bytes(w, o_bytes=2):
    B, d = w.B, w.d
    state = B * w.H_v * d * d * 4 * 2
    io = B * w.H_qk * d * 2 * 2 + B * w.H_v * d * 2 + B * w.H_v * d * 4 * 3 + B * w.H_v * d * o_bytes
    return state + io


def tc_launches_per_call(w, ws_bytes, dev):
    """Kernel launches of one gdn2_chunk_fwd call of workload w with S_T given
    and the whole sequence in the workspace, by the launcher's rules: the scan
    runs one CTA per (sequence, value head); when that leaves SMs idle and the
    sequence has at least 64 chunks, the call pipelines 2 to 4 segments, else
    it runs one segment; a segment is a prep (with the conv and L2 norm in
    its load when asked for), the exact kernel for strongly decaying chunks
    and a scan. The SIMT path (no workspace) is one launch."""
    if ws_bytes == 0:
        return 1
    import torch
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    scan_ctas = w.B * w.H_v
    nchunks = (w.T + 63) // 64
    if nchunks >= 64 and scan_ctas < sms:
        return 3 * min(4, nchunks // 32)
    return 3


def kernel_sources_sha1():
    h = hashlib.sha1()
    for rel in TRAFFIC_KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def measured_traffic():
    """Per-call DRAM traffic of the prefill kernels if it was captured on the current sources."""
    if TRAFFIC["sha1"] is None or TRAFFIC["sha1"] != kernel_sources_sha1():
        return None
    return TRAFFIC["bytes_per_call"]


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """SM clock and throttle-reason samples during a timed region, read through
    NVML every 5 ms (falls back to `nvidia-smi -lms 50` without the NVML
    bindings). Reads only; no setting of the GPU is touched."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                   "hw_thermal_slowdown": 0x40}

    def __init__(self, cuda_index: int):
        self.cuda_index = cuda_index
        self.proc = None
        self.lines = []
        self.sm = []
        self.mx = None
        self.reasons = set()
        self._t = None
        self._stop = threading.Event()
        self._nvml = None

    def _nvml_loop(self, nv, h):
        get_reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.sm.append(float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)))
                bits = int(get_reasons(h))
                for name, bit in self.REASON_BITS.items():
                    if bits & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            self._stop.wait(0.005)

    def __enter__(self):
        try:
            import pynvml as nv
            import torch
            nv.nvmlInit()
            idx = torch.cuda._get_nvml_device_index(self.cuda_index)
            h = nv.nvmlDeviceGetHandleByIndex(idx)
            self.mx = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            self._nvml = nv
            self._t = threading.Thread(target=self._nvml_loop, args=(nv, h), daemon=True)
            self._t.start()
            return self
        except Exception:
            self._nvml = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.cuda_index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
            # nvidia-smi takes a while to print its first sample: the timed
            # region starts only once it samples (bounded wait)
            t_end = time.time() + 5.0
            while not self.lines and time.time() < t_end and self.proc.poll() is None:
                time.sleep(0.01)
            self.lines.clear()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        self._stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self._t is not None:
            self._t.join(timeout=2)
        if self._nvml is not None:
            try:
                self._nvml.nvmlShutdown()
            except Exception:
                pass

    def summary(self):
        sm, mx, reasons = list(self.sm), self.mx, set(self.reasons)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "source": "nvml" if self._nvml is not None else "nvidia-smi"}


# ------------------------------------------------------------------ reference arm

def cpu_oracle_rate(w, heads, tokens, threads=0, seed=2):
    """Run the float64 oracle on `heads` value heads x `tokens` tokens of workload
    w; return (layer tokens/s, seconds, threads used)."""
    import numpy as np
    import torch
    import oracle
    from dataclasses import replace
    from delta_rule_linear_gdn_b200.inputs import make_inputs

    sub = replace(w, T=tokens, H_v=heads, H_qk=max(1, heads * w.H_qk // w.H_v))
    inp = make_inputs(sub, seed=seed)
    f = lambda t: None if t is None else t.to(torch.float64).numpy()
    args = [f(inp[k]) for k in ("q", "k", "v", "alpha", "b", "w")]
    nthreads = threads or os.cpu_count() or 1
    t0 = time.perf_counter()
    oracle.gdn2_forward(*args, f(inp["S0"]), threads=nthreads)
    dt = time.perf_counter() - t0
    layer_tokens = tokens * heads / w.H_v
    return layer_tokens / dt, dt, min(nthreads, heads)


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from delta_rule_linear_gdn_b200.inputs import workload
    w = workload(PREFILL)
    heads, tokens = w.H_v, 512
    rates = []
    for i in range(args.warmup + args.steps):
        r, dt, used = cpu_oracle_rate(w, heads, tokens)
        if i >= args.warmup:
            rates.append((r, dt))
    total_tok = sum(tokens for _ in rates)
    total_t = sum(dt for _, dt in rates)
    value = total_tok / total_t
    sample = f"{heads} V heads x {tokens} tokens per step of the T=32768 layer (layer tokens = tokens x heads/48)"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total_t / max(1, len(rates)),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_dict(w),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": used, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ rank plumbing

def rank_seed(rank: int) -> int:
    """Seed of a rank's own sequence (independent problems per GPU)."""
    return 2 + 1000 * rank


def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank scalar over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_value(units_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return units_per_rank * world / (ms_max * 1e-3)


def config_dict(w, heads_per_rank=None):
    par = ("independent sequences per GPU" if heads_per_rank is None else
           f"heads split across GPUs: {heads_per_rank[0]} QK / {heads_per_rank[1]} V heads per GPU")
    return {"workload": f"{w.name}: B={w.B} T={w.T} H_qk={w.H_qk} H_v={w.H_v} d={w.d} chunk={w.chunk} "
                        f"{w.qkv_dtype} q,k,v, fp32 per-channel gates, S0=0",
            "global_batch": w.B, "seq_len": w.T, "parallelism": par,
            "l2": f"no flush: each step moves {prefill_bytes(w) / 1e9:.2f} GB (inputs read once, "
                  f"o written once), > 126 MB L2"}


# ------------------------------------------------------------------ our arm

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--e2e-steps", type=int, default=6)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", default=PREFILL, choices=[PREFILL, "prefill_t4096"],
                    help="prefill workload to time (the small one is for profiler captures)")
    ap.add_argument("--decode-workload", default=DECODE, choices=[DECODE, "decode_b64"])
    ap.add_argument("--logits-steps", type=int, default=20,
                    help="timed calls of the T=32768 prefill with bf16 gate logits; 0 skips it")
    ap.add_argument("--qk-gates-steps", type=int, default=20,
                    help="timed calls of the T=32768 prefill with alpha, b per QK head; 0 skips it")
    ap.add_argument("--decode-conv-steps", type=int, default=200,
                    help="timed decode steps with the conv and L2 norm in the step; 0 skips it")
    ap.add_argument("--conv-steps", type=int, default=10,
                    help="timed calls of the conv + L2 workload (B=8, T=8192); 0 skips it")
    ap.add_argument("--tied-steps", type=int, default=20,
                    help="timed calls of the T=32768 prefill with the tied gates of KDA and of Gated DeltaNet")
    ap.add_argument("--t4096-steps", type=int, default=50, help="timed calls of the T=4096 prefill; 0 skips it")
    ap.add_argument("--cp-steps", type=int, default=5,
                    help="with N > 1 ranks: timed calls of the T=32768 sequence split across the ranks "
                         "(context-parallel prefill, strong scaling); 0 skips it")
    ap.add_argument("--split", default="sequences", choices=["sequences", "heads"],
                    help="with N > 1 ranks, what the headline line partitions: whole sequences per rank "
                         "(weak scaling, the default) or the layer's heads (H_qk/N QK heads and the value heads "
                         "that read them per rank, one sequence: strong scaling)")
    ap.add_argument("--heads-steps", type=int, default=20,
                    help="with N > 1 ranks: timed calls of the T=32768 layer with its heads split across the "
                         "ranks (H_qk/N QK heads and the value heads that read them per rank, strong scaling); "
                         "0 skips it")
    ap.add_argument("--bwd-workload", default=CONV, choices=[CONV, "prefill_t4096"],
                    help="backward workload (the small one is for profiler captures)")
    ap.add_argument("--bwd-steps", type=int, default=3,
                    help="timed calls of the backward pass on the B=8, T=8192 training shape; 0 skips it")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist
    from delta_rule_linear_gdn_b200 import gdn2
    from delta_rule_linear_gdn_b200.inputs import make_decode_pool, make_inputs, workload

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    pk = peaks()
    w_layer = workload(args.workload)
    w = w_layer
    heads_split = args.split == "heads" and world > 1
    if heads_split:
        # this rank's block of heads (see delta_rule_linear_gdn_b200/head_parallel.py)
        from dataclasses import replace as _replace
        from delta_rule_linear_gdn_b200.head_parallel import head_shard
        qs, vs = head_shard(w_layer.H_qk, w_layer.H_v, rank, world)
        w = _replace(w_layer, H_qk=qs.stop - qs.start, H_v=vs.stop - vs.start)
    stream = torch.cuda.Stream(device=dev)
    inp = make_inputs(w, seed=rank_seed(rank), device=dev)
    o = torch.empty((w.B, w.T, w.H_v, w.d), dtype=torch.bfloat16, device=dev)
    S_T = torch.empty((w.B, w.H_v, w.d, w.d), dtype=torch.float32, device=dev)
    p = gdn2.make_params(w.B, w.T, w.H_qk, w.H_v, w.d, w.d, chunk=w.chunk)
    ws_bytes = gdn2.chunk_fwd_workspace(p)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    launches_per_call = tc_launches_per_call(w, ws_bytes, dev)

    def prefill_call():
        gdn2.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["b"], inp["w"], None, chunk=w.chunk,
                       o=o, S_T=S_T, workspace=ws, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            prefill_call()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        ev0.record(stream)
        with torch.cuda.stream(stream):
            for _ in range(args.steps):
                prefill_call()
        ev1.record(stream)
        torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    ms = ev0.elapsed_time(ev1) / args.steps
    ms_max = max_over_ranks(ms, dev)
    if heads_split:   # the ranks share one layer's tokens
        tokens_per_step = w.B * w.T
        value = tokens_per_step / (ms_max * 1e-3)
    else:
        tokens_per_step = w.B * w.T * world
        value = weak_value(w.B * w.T, world, ms_max)

    nbytes = prefill_bytes(w)
    flops = prefill_flops(w)
    kernel_s = ms * 1e-3  # one call: the prep and scan launches back to back on one stream
    achieved_gbs = nbytes / kernel_s / 1e9
    tflops = flops / kernel_s / 1e12
    traffic = measured_traffic() if w.name == PREFILL and not heads_split else None
    roofline = {"bound": "hbm", "achieved": achieved_gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": achieved_gbs / pk["hbm_gbs"], "traffic": traffic,
                "peak_source": pk["source"],
                "kernel": "gdn2_chunk_fwd call (chunk_prep_kernel + chunk_scan_kernel per segment)",
                "launches_per_call": launches_per_call, "alg_bytes_per_launch": nbytes,
                "alg_flops_per_launch": flops, "tensor_tflops": tflops, "tensor_frac": tflops / pk["bf16_tflops"]}

    # ---------------------------------------------------------------- decode
    decode = None
    dw = workload(args.decode_workload) if args.decode_steps > 0 else None
    if dw is not None:
        decode = run_decode(args, dw, dev, stream, barrier, pk, world)
    decode_conv = None
    if args.decode_conv_steps > 0:
        decode_conv = run_decode(args, workload(args.decode_workload), dev, stream, barrier, pk, world, conv=True)

    # ---------------------------------------------------------------- conv + L2 fused into the load
    conv = None
    if args.conv_steps > 0:
        conv = run_conv(args, dev, stream, barrier, pk, world)

    # ---------------------------------------------------------------- gates as bf16 logits
    logits = None
    if args.logits_steps > 0:
        logits = run_gate_variant(args.logits_steps, w, dev, stream, barrier, pk, world, gate_logits=True)
    qk_gates = None
    if args.qk_gates_steps > 0:
        qk_gates = run_gate_variant(args.qk_gates_steps, w, dev, stream, barrier, pk, world, qk=True)

    tied = {}
    if args.tied_steps > 0:
        for mode in ("kda", "gdn"):
            tied[mode] = run_gate_variant(args.tied_steps, w, dev, stream, barrier, pk, world, gate_mode=mode)
    t4096 = None
    if args.t4096_steps > 0 and w.name != "prefill_t4096":
        t4096 = run_gate_variant(args.t4096_steps, workload("prefill_t4096"), dev, stream, barrier, pk, world)
    bwd = None
    if args.bwd_steps > 0:
        bwd = run_bwd(args, dev, stream, barrier, pk, world)
    cp_leg = None
    if args.cp_steps > 0 and world > 1:
        cp_leg = run_context_parallel(args, w, dev, stream, barrier, world)
    heads_leg = None
    if args.heads_steps > 0 and world > 1 and w.H_qk % world == 0:
        heads_leg = run_head_split(args, w, dev, stream, barrier, world)

    # ---------------------------------------------------------------- end to end
    e2e = None
    if args.e2e_steps > 0:
        e2e = run_e2e(args, w, inp, o, S_T, ws, dev, stream, barrier, tokens_per_step)

    # ---------------------------------------------------------------- CPU baseline
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        heads, tokens = w.H_v, 8192
        rate, dt, used = cpu_oracle_rate(w, heads, tokens)
        rate1, dt1, _ = cpu_oracle_rate(w, 1, tokens, threads=1)
        cpu = {"value": rate, "unit": "tokens/s", "cores": used, "kind": "oracle",
               "sample": f"{heads} V heads x {tokens} tokens of the T={w.T} layer workload "
                         f"({dt:.1f} s, layer tokens = tokens x heads/{w.H_v})",
               "single_core_value": rate1,
               "single_core_sample": f"1 V head x {tokens} tokens on one thread ({dt1:.1f} s)"}

    clocks = clk.summary()
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True,
            "scaling": "strong" if heads_split else "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": config_dict(w_layer, heads_per_rank=(w.H_qk, w.H_v) if heads_split else None),
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": args.steps * launches_per_call, "clocks": clocks, "decode": decode,
            "conv_prefill": conv, "prefill_gate_logits": logits, "prefill_qk_gates": qk_gates,
            "decode_conv": decode_conv, "prefill_kda": tied.get("kda"), "prefill_gdn": tied.get("gdn"),
            "prefill_t4096": t4096, "backward": bwd, "prefill_context_parallel": cp_leg,
            "prefill_head_split": heads_leg,
        }
        print(json.dumps(line), flush=True)
    return 0


def run_decode(args, dw, dev, stream, barrier, pk, world, conv=False):
    """Consecutive decode steps of B sequences; with ``conv``, each step also
    convolves q, k, v with the three previous inputs (history ping-ponged
    between two buffers) and L2-normalises q, k."""
    import torch
    from delta_rule_linear_gdn_b200 import gdn2
    from delta_rule_linear_gdn_b200.inputs import CONV_STD, make_conv_state, make_decode_pool
    pool = make_decode_pool(dw, pool=16, device=dev)
    S = pool["S0"].clone()
    od = torch.empty((dw.B, dw.H_v, dw.d), dtype=torch.bfloat16, device=dev)
    steps = args.decode_conv_steps if conv else args.decode_steps
    kw = {}
    hist = []
    if conv:
        nch = (2 * dw.H_qk + dw.H_v) * dw.d
        g = torch.Generator(device=dev)
        g.manual_seed(11)
        kw = dict(conv_w=torch.randn((nch, 4), generator=g, device=dev) * CONV_STD, l2norm_qk=True)
        hist = [make_conv_state(dw, seed=12, device=dev), torch.empty((dw.B, 3, nch), dtype=torch.bfloat16,
                                                                       device=dev)]

    def decode_call(i):
        if conv:
            kw["conv_state_in"], kw["conv_state_out"] = hist[i % 2], hist[(i + 1) % 2]
        j = i % 16
        gdn2.decode_step(pool["q"][j], pool["k"][j], pool["v"][j], pool["alpha"][j], pool["b"][j], pool["w"][j],
                         S, o=od, stream=stream, **kw)

    with torch.cuda.stream(stream):
        for i in range(6):
            decode_call(i)
    torch.cuda.synchronize()
    barrier()
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    d0.record(stream)
    with torch.cuda.stream(stream):
        for i in range(steps):
            decode_call(i)
    d1.record(stream)
    torch.cuda.synchronize()
    barrier()
    dms = max_over_ranks(d0.elapsed_time(d1) / steps, dev)
    dbytes = decode_bytes(dw)
    what = ""
    if conv:
        nch = (2 * dw.H_qk + dw.H_v) * dw.d
        dbytes += 2 * dw.B * 3 * nch * 2 + nch * 16      # history in and out (bf16), conv taps
        what = ", depthwise causal conv k=4 (history ping-ponged) and L2 norm of q, k in the step"
    decode = {"workload": f"{dw.name}: B={dw.B} sequences, one token per step, H_qk={dw.H_qk} H_v={dw.H_v} "
                          f"d={dw.d}, fp32 state, bf16 q,k,v,o, {steps} consecutive steps{what}",
              "us_per_step": dms * 1e3, "gbs": dbytes / (dms * 1e-3) / 1e9 * world,
              "roofline": {"bound": "hbm", "achieved": dbytes / (dms * 1e-3) / 1e9, "peak": pk["hbm_gbs"],
                           "unit": "GB/s", "frac": dbytes / (dms * 1e-3) / 1e9 / pk["hbm_gbs"],
                           "traffic": None, "alg_bytes_per_launch": dbytes},
              "tokens_per_s": dw.B * world / (dms * 1e-3)}
    decode["gpu_launches"] = steps
    return decode


def run_conv(args, dev, stream, barrier, pk, world):
    """The B=8, T=8192 workload with the depthwise causal conv on q, k, v and
    the L2 norm of q, k fused into the prep's load (prep, exact kernel and
    scan: three launches per call)."""
    import torch
    from delta_rule_linear_gdn_b200 import gdn2
    from delta_rule_linear_gdn_b200.inputs import make_inputs, workload
    cw = workload(CONV)
    rank = int(os.environ.get("RANK", "0"))
    inp = make_inputs(cw, seed=rank_seed(rank), device=dev)
    o = torch.empty((cw.B, cw.T, cw.H_v, cw.d), dtype=torch.bfloat16, device=dev)
    S_T = torch.empty((cw.B, cw.H_v, cw.d, cw.d), dtype=torch.float32, device=dev)
    p = gdn2.make_params(cw.B, cw.T, cw.H_qk, cw.H_v, cw.d, cw.d, chunk=cw.chunk, l2norm_qk=True,
                         conv_w=inp["conv_w"])
    ws = torch.empty(max(gdn2.chunk_fwd_workspace(p), 1), dtype=torch.uint8, device=dev)

    def call():
        gdn2.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["b"], inp["w"], inp["S0"], chunk=cw.chunk,
                       conv_w=inp["conv_w"], l2norm_qk=True, o=o, S_T=S_T, workspace=ws, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(3):
            call()
    torch.cuda.synchronize()
    barrier()
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(args.conv_steps):
            call()
    c1.record(stream)
    torch.cuda.synchronize()
    barrier()
    cms = max_over_ranks(c0.elapsed_time(c1) / args.conv_steps, dev)
    nbytes = prefill_bytes(cw, s0=True)
    gbs = nbytes / (cms * 1e-3) / 1e9
    return {"workload": f"{cw.name}: B={cw.B} T={cw.T} H_qk={cw.H_qk} H_v={cw.H_v} d={cw.d} chunk={cw.chunk}, "
                        f"depthwise causal conv k=4 on q,k,v and L2 norm of q,k fused into the prep's load, "
                        f"S0 given",
            "ms_per_call": cms, "tokens_per_s": cw.B * cw.T * world / (cms * 1e-3),
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "traffic": None, "alg_bytes_per_launch": nbytes},
            "gpu_launches": 3 * args.conv_steps}


def run_gate_variant(steps, w, dev, stream, barrier, pk, world, gate_logits=False, qk=False, gate_mode="full"):
    """A prefill leg with another gate layout or length: bf16 logits (the
    kernels apply the sigmoid; half the gate bytes), alpha and b owned by the
    QK heads (a third of their bytes at 48 V / 16 QK heads), the tied gates of
    KDA (beta scalar) and Gated DeltaNet (alpha and beta scalar), or another
    workload with the headline's gates."""
    import torch
    from delta_rule_linear_gdn_b200 import gdn2
    from delta_rule_linear_gdn_b200.inputs import make_inputs
    rank = int(os.environ.get("RANK", "0"))
    inp = make_inputs(w, seed=rank_seed(rank), device=dev, gate_logits=gate_logits, gates_per_qk_head=qk,
                      gate_mode=gate_mode)
    o = torch.empty((w.B, w.T, w.H_v, w.d), dtype=torch.bfloat16, device=dev)
    S_T = torch.empty((w.B, w.H_v, w.d, w.d), dtype=torch.float32, device=dev)
    p = gdn2.make_params(w.B, w.T, w.H_qk, w.H_v, w.d, w.d, chunk=w.chunk, gate_logits=gate_logits,
                         gates_per_qk_head=qk, gate_mode=gate_mode)
    ws = torch.empty(max(gdn2.chunk_fwd_workspace(p), 1), dtype=torch.uint8, device=dev)

    def call():
        gdn2.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["b"], inp["w"], None, chunk=w.chunk,
                       o=o, S_T=S_T, workspace=ws, stream=stream, gate_logits=gate_logits, gates_per_qk_head=qk,
                       gate_mode=gate_mode)

    with torch.cuda.stream(stream):
        for _ in range(3):
            call()
    torch.cuda.synchronize()
    barrier()
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(steps):
            call()
    c1.record(stream)
    torch.cuda.synchronize()
    barrier()
    lms = max_over_ranks(c0.elapsed_time(c1) / steps, dev)
    nbytes = prefill_bytes(w, gate_bytes=2 if gate_logits else 4, qk_gates=qk, gate_mode=gate_mode)
    gbs = nbytes / (lms * 1e-3) / 1e9
    tflops = prefill_flops(w) / (lms * 1e-3) / 1e12
    what = ("the gates as bf16 logits (sigmoid in the kernels)" if gate_logits else
            "alpha and b per QK head (shared by its 3 value heads), fp32" if qk else
            "tied gates b = w = beta (KDA): per-channel alpha, scalar beta, fp32" if gate_mode == "kda" else
            "tied gates (Gated DeltaNet): scalar alpha and scalar beta, fp32" if gate_mode == "gdn" else
            "fp32 per-channel gates")
    return {"workload": f"{w.name}: B={w.B} T={w.T} H_qk={w.H_qk} H_v={w.H_v} d={w.d} chunk={w.chunk} with {what}",
            "ms_per_call": lms, "tokens_per_s": w.B * w.T * world / (lms * 1e-3),
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / pk["hbm_gbs"], "traffic": None, "alg_bytes_per_launch": nbytes,
                         "alg_flops_per_launch": prefill_flops(w), "tensor_tflops": tflops,
                         "tensor_frac": tflops / pk["bf16_tflops"]},
            "gpu_launches": steps * tc_launches_per_call(w, gdn2.chunk_fwd_workspace(p), dev)}


def bwd_flops(w):
    """FLOPs of one gdn2_chunk_bwd call, counting its d²-scaled products per
    token and value head: the forward pass's E-bar S and K_endᵀ U (4d²), and in
    the reverse pass E-bar S again (2d²), K_end dS' (2d²), the carried dS
    (Q-barᵀ dO and E-barᵀ dR, 4d²), dQ-bar, dE-bar and dK_end (6d²): 18d²."""
    return w.B * w.T * w.H_v * 18 * w.d * w.d


def alu_peak_tflops(dev):
    """fp32 FMA peak of the CUDA cores: SMs × 128 lanes × 2 FLOP × the maximum
    SM clock (MEASURED_PEAKS' sm_max_mhz, else 1965 MHz)."""
    import torch
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    mhz = 1965.0
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            mhz = float(json.load(f).get("sm_max_mhz", mhz))
    return sms * 128 * 2 * mhz * 1e6 / 1e12


def run_bwd(args, dev, stream, barrier, pk, world):
    """The backward pass (gdn2_chunk_bwd) on the training-shape workload: B=8,
    T=8192, 48 V heads, the recurrence's inputs (unit q, k), nonzero S0,
    upstream gradients of o (bf16) and of S_T (or, for profiler captures, the
    T=4096 layer)."""
    import torch
    from dataclasses import replace
    from delta_rule_linear_gdn_b200 import gdn2
    from delta_rule_linear_gdn_b200.inputs import make_inputs, workload
    rank = int(os.environ.get("RANK", "0"))
    bw = replace(workload(args.bwd_workload), conv=False)
    inp = make_inputs(bw, seed=rank_seed(rank), device=dev)
    g = torch.Generator(device=dev)
    g.manual_seed(21)
    dO = torch.randn((bw.B, bw.T, bw.H_v, bw.d), generator=g, device=dev).to(torch.bfloat16)
    dST = torch.randn((bw.B, bw.H_v, bw.d, bw.d), generator=g, device=dev)
    p = gdn2.make_params(bw.B, bw.T, bw.H_qk, bw.H_v, bw.d, bw.d, chunk=bw.chunk)
    ws = torch.empty(gdn2.chunk_bwd_workspace(p), dtype=torch.uint8, device=dev)

    def call():
        return gdn2.chunk_bwd(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["b"], inp["w"], inp["S0"], dO, dST,
                              workspace=ws, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(3):
            call()
    torch.cuda.synchronize()
    barrier()
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(args.bwd_steps):
            call()
    c1.record(stream)
    torch.cuda.synchronize()
    barrier()
    bms = max_over_ranks(c0.elapsed_time(c1) / args.bwd_steps, dev)
    flops = bwd_flops(bw)
    tf = flops / (bms * 1e-3) / 1e12
    peak = alu_peak_tflops(dev)
    return {"workload": f"{bw.name} recurrence inputs (no conv): B={bw.B} T={bw.T} H_qk={bw.H_qk} H_v={bw.H_v} "
                        f"d={bw.d}, bf16 q,k,v,dO, fp32 per-channel gates, S0 and dS_T given; gradients of "
                        f"q,k,v,alpha,b,w,S0 in fp32",
            "ms_per_call": bms, "tokens_per_s": bw.B * bw.T * world / (bms * 1e-3),
            "roofline": {"bound": "alu", "achieved": tf, "peak": peak, "unit": "TFLOP/s", "frac": tf / peak,
                         "traffic": None, "alg_flops_per_launch": flops,
                         "peak_source": "derived: SMs x 128 fp32 lanes x 2 FLOP x max SM clock"},
            "workspace_bytes": gdn2.chunk_bwd_workspace(p),
            "gpu_launches": args.bwd_steps}


def run_context_parallel(args, w, dev, stream, barrier, world):
    """The headline sequence split across the ranks: rank r runs tokens
    [r·T/N, (r+1)·T/N) and the ranks join through the affine maps of their
    segments (one all-gather); tokens of the one sequence / max-over-ranks
    time ("strong" scaling)."""
    import torch
    from dataclasses import replace
    from delta_rule_linear_gdn_b200 import context_parallel as cp
    from delta_rule_linear_gdn_b200.inputs import make_inputs
    rank = int(os.environ.get("RANK", "0"))
    seg = replace(w, T=w.T // world)
    inp = make_inputs(seg, seed=rank_seed(rank), device=dev)   # this rank's segment

    def call():
        with torch.cuda.stream(stream):
            cp.chunk_fwd_context_parallel(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["b"], inp["w"], None)

    for _ in range(3):
        call()
    torch.cuda.synchronize()
    barrier()
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0.record(stream)
    for _ in range(args.cp_steps):
        call()
    c1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(c0.elapsed_time(c1) / args.cp_steps, dev)
    return {"workload": f"{w.name} split into {world} segments of {seg.T} tokens, one per rank",
            "ms_per_call": ms, "tokens_per_s": w.B * w.T / (ms * 1e-3), "scaling": "strong",
            "gpu_launches": args.cp_steps * (3 * tc_launches_per_call(seg, 1, dev) + world - 1)}


def run_head_split(args, w, dev, stream, barrier, world):
    """The headline layer with its heads split across the ranks: rank r runs
    QK heads [r·H_qk/N, (r+1)·H_qk/N) and the value heads that read them, over
    the whole sequence, with no exchange; tokens of the layer / max-over-ranks
    time ("strong" scaling: the layer is fixed, each rank's share shrinks)."""
    import torch
    from dataclasses import replace
    from delta_rule_linear_gdn_b200 import gdn2
    from delta_rule_linear_gdn_b200.head_parallel import head_shard
    from delta_rule_linear_gdn_b200.inputs import make_inputs
    rank = int(os.environ.get("RANK", "0"))
    qs, vs = head_shard(w.H_qk, w.H_v, rank, world)
    mine = replace(w, H_qk=qs.stop - qs.start, H_v=vs.stop - vs.start)
    inp = make_inputs(mine, seed=rank_seed(rank), device=dev)   # this rank's block of heads
    o = torch.empty((mine.B, mine.T, mine.H_v, mine.d), dtype=torch.bfloat16, device=dev)
    S_T = torch.empty((mine.B, mine.H_v, mine.d, mine.d), dtype=torch.float32, device=dev)
    p = gdn2.make_params(mine.B, mine.T, mine.H_qk, mine.H_v, mine.d, mine.d, chunk=mine.chunk)
    ws_bytes = gdn2.chunk_fwd_workspace(p)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)

    def call():
        gdn2.chunk_fwd(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["b"], inp["w"], None, chunk=mine.chunk,
                       o=o, S_T=S_T, workspace=ws, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(3):
            call()
    torch.cuda.synchronize()
    barrier()
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(args.heads_steps):
            call()
    c1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(c0.elapsed_time(c1) / args.heads_steps, dev)
    return {"workload": f"{w.name} with {mine.H_qk} QK / {mine.H_v} V heads per rank on {world} ranks",
            "ms_per_call": ms, "tokens_per_s": w.B * w.T / (ms * 1e-3), "scaling": "strong",
            "gpu_launches": args.heads_steps * tc_launches_per_call(mine, ws_bytes, dev)}


def run_e2e(args, w, inp, o, S_T, ws, dev, stream, barrier, tokens_per_step):
    """The same prefill through the public call with host buffers: pinned
    host->device copies of each step's inputs, the call, device->host copies
    of its o and S_T, all inside the timed region. Steps are pipelined over
    two buffer sets, as a serving loop would run them: step i+1's inputs
    cross PCIe (on a copy stream) while step i computes and its results come
    back (on a third stream), so the link's two directions overlap."""
    import torch
    from delta_rule_linear_gdn_b200 import gdn2
    host = {k: inp[k].cpu().pin_memory() for k in ("q", "k", "v", "alpha", "b", "w")}
    NB = 2
    dev_in = [{k: torch.empty_like(inp[k]) for k in host} for _ in range(NB)]
    o_dev = [o, torch.empty_like(o)]
    S_dev = [S_T, torch.empty_like(S_T)]
    o_host = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for _ in range(NB)]
    S_host = [torch.empty(S_T.shape, dtype=S_T.dtype).pin_memory() for _ in range(NB)]
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = o_host[0].numel() * o_host[0].element_size() + S_host[0].numel() * S_host[0].element_size()
    up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(NB)]     # inputs of buffer set j landed
    ev_done = [torch.cuda.Event() for _ in range(NB)]   # the call on set j is done (its inputs are free)
    ev_out = [torch.cuda.Event() for _ in range(NB)]    # o, S_T of set j are on the host (free again)

    def e2e_step(i):
        j = i % NB
        with torch.cuda.stream(up):
            if i >= NB:
                up.wait_event(ev_done[j])
            for k_ in host:
                dev_in[j][k_].copy_(host[k_], non_blocking=True)
            ev_in[j].record(up)
        stream.wait_event(ev_in[j])
        if i >= NB:
            stream.wait_event(ev_out[j])
        gdn2.chunk_fwd(dev_in[j]["q"], dev_in[j]["k"], dev_in[j]["v"], dev_in[j]["alpha"], dev_in[j]["b"],
                       dev_in[j]["w"], None, chunk=w.chunk, o=o_dev[j], S_T=S_dev[j], workspace=ws, stream=stream)
        ev_done[j].record(stream)
        with torch.cuda.stream(down):
            down.wait_event(ev_done[j])
            o_host[j].copy_(o_dev[j], non_blocking=True)
            S_host[j].copy_(S_dev[j], non_blocking=True)
            ev_out[j].record(down)

    def run(n):
        for i in range(n):
            e2e_step(i)
        for j in range(min(n, NB)):
            stream.wait_event(ev_out[j])

    run(NB)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    up.wait_event(e0)
    run(args.e2e_steps)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ems = max_over_ranks(e0.elapsed_time(e1) / args.e2e_steps, dev)
    return {"value": tokens_per_step / (ems * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ems, "pipelined": "2 buffer sets, copies on 2 side streams"}


if __name__ == "__main__":
    sys.exit(main())
