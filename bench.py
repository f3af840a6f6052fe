"""Benchmark of the TurboQuant KV-cache path on B200.

One step = one pass of the hot path over one batch: a 64-token bf16 chunk is
appended to every sequence (fused rotate / quantize / pack / append) and one
decode-attention step runs over the packed cache.  Workload (streaming append
+ decode): 16 sequences, contexts uniform in [8192, 65536], 8 kv-heads and 32
query heads of d = 128, mixed 3.5-bit keys and values (64 rotated channels at
4 bits, 64 at 3 bits).  The cache read per step (~570 MB) is larger than L2.

`value` is the packed-KV throughput of the whole step in GB/s: algorithmic
bytes (chunk read + packed rows written + packed cache, queries and outputs
read/written by the decode) over the step time.  Auxiliary measurements of
the other workloads (quantize sweep, prod-mode GQA decode, long-context
asymmetric decode with sink and sparse V, tiny fp32 case) ride along.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

For N > 1 launch with torch.distributed.run: every rank runs its own copy of
the workload (independent sequences, no data exchange: weak scaling); the
time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

N_SEQ, HKV, HQ, D, CHUNK = 16, 8, 32, 128, 64
LEN_LO, LEN_HI = 8192, 65536
ROW_BYTES = 56 + 4  # mixed 3.5-bit code row + fp32 norm, per K or V


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def build_stream_workload(tq, torch, kv_inputs, rank: int, n_steps: int, device, bits: int = 3, params=None):
    """Config: streaming append + decode (mixed rows: bits + 0.5 bits per
    channel, 3.5 by default; `params` replaces the format).  Returns the
    state the step uses."""
    lens = rank_sequence_lengths(kv_inputs, rank)
    if params is None:
        params = tq.Params(bits, bits, mixed_k=1, mixed_v=1, seed=0)
    cap = ((max(lens) + (n_steps + 1) * CHUNK + 63) // 64) * 64
    cache = tq.Cache(params, N_SEQ, HKV, cap, 0, device=device)
    # prefill (untimed): the prefix of each sequence through tq_append
    for s, n in enumerate(lens):
        ids = torch.tensor([s], dtype=torch.int32, device=device)
        done = 0
        while done < n:
            m = min(16384, n - done)
            k = kv_inputs.kv_vectors(m * HKV, D, key=("stream-k", rank, s, done), device=device,
                                     dtype=torch.bfloat16).view(1, m, HKV, D)
            v = kv_inputs.kv_vectors(m * HKV, D, key=("stream-v", rank, s, done), device=device,
                                     dtype=torch.bfloat16).view(1, m, HKV, D)
            tq.tq_append(params, cache, ids, k, v)
            done += m
    torch.cuda.synchronize()
    assert cache.lens.cpu().tolist() == lens
    chunks_k = [kv_inputs.kv_vectors(N_SEQ * CHUNK * HKV, D, key=("chunk-k", rank, i), device=device,
                                     dtype=torch.bfloat16).view(N_SEQ, CHUNK, HKV, D) for i in range(n_steps)]
    chunks_v = [kv_inputs.kv_vectors(N_SEQ * CHUNK * HKV, D, key=("chunk-v", rank, i), device=device,
                                     dtype=torch.bfloat16).view(N_SEQ, CHUNK, HKV, D) for i in range(n_steps)]
    qs = [kv_inputs.queries((N_SEQ, HQ, D), key=("stream-q", rank, i), device=device) for i in range(n_steps)]
    ids = torch.arange(N_SEQ, dtype=torch.int32, device=device)
    ws = tq.decode_workspace(params, N_SEQ, HQ, HKV, cap, device=device)
    out = torch.empty(N_SEQ, HQ, D, dtype=torch.bfloat16, device=device)
    return dict(params=params, cache=cache, lens=lens, cap=cap, ck=chunks_k, cv=chunks_v, qs=qs, ids=ids, ws=ws,
                out=out)


# dram__bytes_read.sum + dram__bytes_write.sum of one decode_kernel launch of
# this workload (one ncu capture: 485.23 MB read, 3.36 MB written), valid for
# the kernel source it was taken on only: reported as null once that changes.
DECODE_TRAFFIC = {"source_sha256": "b1c0097469de345a9d8389441306293cd1e0f4fbf285f65d11e65dd9c7375acb",
                  "bytes": 488584448}


def decode_sources_sha256():
    """sha256 over the decode kernel's sources (tq_decode_common.cuh, then
    tq_attn.cu) with comments and blank lines removed, so that only code
    changes invalidate a captured traffic figure."""
    import hashlib
    import re
    csrc = os.path.join(os.path.dirname(os.path.abspath(__file__)), "online_vector_quantization_b200", "csrc")
    h = hashlib.sha256()
    try:
        for name in ("tq_decode_common.cuh", "tq_attn.cu"):
            with open(os.path.join(csrc, name)) as f:
                text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
            for line in text.splitlines():
                code = re.sub(r"//.*$", "", line).rstrip()
                if code:
                    h.update(code.encode() + b"\n")
    except OSError:
        return None
    return h.hexdigest()


def decode_traffic():
    return DECODE_TRAFFIC["bytes"] if decode_sources_sha256() == DECODE_TRAFFIC["source_sha256"] else None


def max_over_ranks(value: float, dist, device=None) -> float:
    """The largest of one per-rank number over all ranks (every rank calls it,
    in the same order): multi-GPU times are the slowest rank's."""
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_sequence_lengths(kv_inputs, rank: int):
    """The streaming workload's context lengths on one rank: every rank (GPU)
    holds its own 16 sequences (weak scaling, no data shared between ranks)."""
    return kv_inputs.sequence_lengths(N_SEQ, LEN_LO, LEN_HI, key=("stream-lens", rank))


def step_bytes(lens_now):
    append = 2 * N_SEQ * CHUNK * HKV * D * 2 + 2 * N_SEQ * CHUNK * HKV * ROW_BYTES
    decode = sum(HKV * (n + CHUNK) * 2 * ROW_BYTES for n in lens_now) + 2 * N_SEQ * HQ * D * 2
    return append, decode


def run_gpu(args):
    import torch
    import torch.distributed as dist

    import kv_inputs
    import online_vector_quantization_b200 as tq

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", device_id=device, timeout=__import__("datetime").timedelta(seconds=300))
    n_steps = args.warmup + args.steps
    st = build_stream_workload(tq, torch, kv_inputs, rank, n_steps, device)
    params, cache = st["params"], st["cache"]
    stream = torch.cuda.current_stream()

    def step(i, evs=None):
        # on the current stream: the default stream, or the capture stream
        s = torch.cuda.current_stream()
        tq.tq_append(params, cache, st["ids"], st["ck"][i], st["cv"][i], stream=s)
        if evs is not None:
            evs[0].record(s)
        tq.tq_decode_attn(params, st["qs"][i], cache, st["cap"], st["out"], st["ws"], stream=s)
        if evs is not None:
            evs[1].record(s)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    lens_at_timing = [n + args.warmup * CHUNK for n in st["lens"]]
    lens_t = torch.tensor(lens_at_timing, dtype=torch.int32, device=device)
    # The K timed steps are captured once in a CUDA graph (capturing runs
    # nothing) and replayed as one launch.  A second capture of the same steps
    # records timing events around every decode call for the roofline; it is
    # replayed after the timed region (lengths rewound), since an event
    # between the append and the decode call's first kernel holds that kernel
    # until the append has finished (no programmatic overlap).
    d_events = [(torch.cuda.Event(enable_timing=True, external=True), torch.cuda.Event(enable_timing=True, external=True))
                for _ in range(args.steps)]
    # (thread-local capture: a CUDA call from another thread of the process,
    # such as a communication library's watchdog, does not void the capture)
    graph, graph_ev = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    cap_stream = torch.cuda.Stream(device=device)
    with torch.cuda.graph(graph, stream=cap_stream, capture_error_mode="thread_local"):
        for j in range(args.steps):
            step(args.warmup + j)
    with torch.cuda.graph(graph_ev, stream=cap_stream, capture_error_mode="thread_local"):
        for j in range(args.steps):
            step(args.warmup + j, d_events[j])
    torch.cuda.synchronize()
    assert cache.lens.cpu().tolist() == lens_at_timing
    if world > 1:
        dist.barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local)
    sampler.start()
    torch.cuda.synchronize()
    t0.record(stream)
    graph.replay()
    t1.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()

    def rerun(fn):
        cache.lens.copy_(lens_t)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    # the same steps with the decode calls bracketed by events, and issued
    # call by call from the host
    ev_ms = rerun(graph_ev.replay)
    eager_ms = rerun(lambda: [step(args.warmup + j) for j in range(args.steps)])
    del graph, graph_ev
    total_ms = t0.elapsed_time(t1)
    decode_ms = [a.elapsed_time(b) for a, b in d_events]
    if world > 1:
        total_ms = max_over_ranks(total_ms, dist, device)
        eager_ms = max_over_ranks(eager_ms, dist, device)
        ev_ms = max_over_ranks(ev_ms, dist, device)
    append_b, decode_b = 0, 0
    for j in range(args.steps):
        a, d = step_bytes([n + j * CHUNK for n in lens_at_timing])
        append_b += a
        decode_b += d
    ms_per_step = total_ms / args.steps
    value = (append_b + decode_b) * world / (total_ms * 1e-3) / 1e9
    assert int(cache.status.item()) == 0

    # e2e: same step through the public API from pinned host buffers
    e2e = None
    if rank == 0 or world > 1:
        e2e = run_e2e(tq, torch, kv_inputs, args, st, rank, device, world)

    peak, peak_kind = peaks()
    avg_decode_s = sum(decode_ms) / len(decode_ms) * 1e-3
    decode_bytes_per_launch = decode_b / args.steps
    achieved = decode_bytes_per_launch / avg_decode_s / 1e9
    aux = {} if args.no_aux or rank != 0 else run_aux(tq, torch, kv_inputs, device, args)
    cpu = None if (rank != 0 or world > 1 or args.no_cpu) else cpu_baseline_stream(args)
    if rank == 0:
        line = {
            "metric": "decode-attn packed-KV GB/s (streaming append + decode step)",
            "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16-mma/f32-acc", "data": "synthetic",
            "config": {"workload": "streaming append + decode: 16 seqs, ctx U[8192,65536], 64-token bf16 chunk "
                                   "appended (fused rotate/quantize/pack), 1 decode step, mixed 3.5-bit K/V, "
                                   "32 q / 8 kv heads, d=128",
                       "seq_lens": st["lens"], "l2": "inputs larger than L2 (cache read ~570 MB per step)",
                       "tokens_per_s_per_seq": round(1000.0 / ms_per_step, 2),
                       "decode_ms": round(avg_decode_s * 1e3, 4),
                       "launch": "the timed steps captured in one CUDA graph (one replay)",
                       "eager_ms_per_step": round(eager_ms / args.steps, 4),
                       "decode_events_ms_per_step": round(ev_ms / args.steps, 4),
                       "append_plus_decode_bytes_per_step": (append_b + decode_b) // args.steps,
                       "parallelism": f"replicas x{world}"},
            "roofline": {"kernel": "decode_kernel<mixed3.5,mixed3.5> (+qrot, merge)", "bound": "hbm",
                         "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "peak_kind": peak_kind,
                         "bytes_per_launch": int(decode_bytes_per_launch), "traffic": decode_traffic(),
                         "traffic_kernel": "decode_kernel alone (ncu capture)"},
            "clocks": clocks,
            # per step: one append launch (K and V planes of the equal mixed
            # formats together) and the decode call's query rotation, decode
            # kernel and merge
            "gpu_launches": args.steps * 4,
            "e2e": e2e,
            "cpu_baseline": cpu,
            "aux": aux,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_e2e(tq, torch, kv_inputs, args, st, rank, device, world):
    import torch.distributed as dist
    params, cache = st["params"], st["cache"]
    stream = torch.cuda.current_stream()
    hk = [t.cpu().pin_memory() for t in st["ck"][:args.steps]]
    hv = [t.cpu().pin_memory() for t in st["cv"][:args.steps]]
    hq = [t.cpu().pin_memory() for t in st["qs"][:args.steps]]
    hout = [torch.empty(N_SEQ, HQ, D, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    # double-buffered device inputs: the copy stream brings step j's chunk and
    # queries in while the compute stream still decodes step j - 1
    dk = [torch.empty_like(st["ck"][0]) for _ in range(2)]
    dv = [torch.empty_like(st["cv"][0]) for _ in range(2)]
    dq = [torch.empty_like(st["qs"][0]) for _ in range(2)]
    copy_stream = torch.cuda.Stream(device=device)
    copied = [torch.cuda.Event() for _ in range(args.steps)]
    consumed = [torch.cuda.Event() for _ in range(args.steps)]
    # rewind the lengths so the e2e steps see the same contexts as the timed ones
    lens0 = torch.tensor([n + args.warmup * CHUNK for n in st["lens"]], dtype=torch.int32, device=device)
    cache.lens.copy_(lens0)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    def bring_in(j):
        b = j & 1
        with torch.cuda.stream(copy_stream):
            if j >= 2:
                copy_stream.wait_event(consumed[j - 2])  # step j - 2 has read buffer b
            dk[b].copy_(hk[j], non_blocking=True)
            dv[b].copy_(hv[j], non_blocking=True)
            dq[b].copy_(hq[j], non_blocking=True)
            copied[j].record(copy_stream)

    # (1) eager: every call issued from the host loop
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    copy_stream.wait_event(t0)
    bring_in(0)
    for j in range(args.steps):
        b = j & 1
        # the next step's inputs are queued before this step's result copy, so
        # a copy engine shared by both directions never holds them behind it
        if j + 1 < args.steps:
            bring_in(j + 1)
        stream.wait_event(copied[j])
        tq.tq_append(params, cache, st["ids"], dk[b], dv[b], stream=stream)
        tq.tq_decode_attn(params, dq[b], cache, st["cap"], st["out"], st["ws"], stream=stream)
        consumed[j].record(stream)
        hout[b].copy_(st["out"], non_blocking=True)
    t1.record(stream)
    torch.cuda.synchronize()
    eager_ms = t0.elapsed_time(t1)

    # (2) the same calls captured once per step (before the timed region) in a
    # CUDA graph and replayed.  Graph j appends and decodes step j; beside
    # them, on forked branches, it copies step j + 1's inputs in and step
    # j - 1's result out (outputs double-buffered on the device), so neither
    # the copies nor the host's per-call launch work sit on the step's path.
    # One graph per step because every step reads its own pinned host buffers.
    cache.lens.copy_(lens0)
    dout = [st["out"], torch.empty_like(st["out"])]
    cap_stream = torch.cuda.Stream(device=device)
    out_stream = torch.cuda.Stream(device=device)
    graphs = []
    for j in range(args.steps):
        b = j & 1
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap_stream, capture_error_mode="thread_local"):
            # two branches, one per copy direction, so the result copy does
            # not queue behind the input copies
            joins = []
            for active, cs in ((j + 1 < args.steps, copy_stream), (j >= 1, out_stream)):
                if not active:
                    continue
                fork, join = torch.cuda.Event(), torch.cuda.Event()
                fork.record(cap_stream)
                cs.wait_event(fork)
                with torch.cuda.stream(cs):
                    if cs is copy_stream:
                        nb = (j + 1) & 1
                        dk[nb].copy_(hk[j + 1], non_blocking=True)
                        dv[nb].copy_(hv[j + 1], non_blocking=True)
                        dq[nb].copy_(hq[j + 1], non_blocking=True)
                    else:
                        hout[1 - b].copy_(dout[1 - b], non_blocking=True)
                    join.record(cs)
                joins.append(join)
            tq.tq_append(params, cache, st["ids"], dk[b], dv[b], stream=cap_stream)
            tq.tq_decode_attn(params, dq[b], cache, st["cap"], dout[b], st["ws"], stream=cap_stream)
            for join in joins:
                cap_stream.wait_event(join)
        graphs.append(g)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    dk[0].copy_(hk[0], non_blocking=True)
    dv[0].copy_(hv[0], non_blocking=True)
    dq[0].copy_(hq[0], non_blocking=True)
    for g in graphs:
        g.replay()
    last = (args.steps - 1) & 1
    hout[last].copy_(dout[last], non_blocking=True)  # the last step's result
    t1.record(stream)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1)
    assert int(cache.status.item()) == 0
    del graphs
    # the same copies alone (no kernels, each direction on its own stream): how
    # much of the step is PCIe
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0.record(copy_stream)
    out_stream.wait_event(c0)
    for j in range(args.steps):
        b = j & 1
        with torch.cuda.stream(copy_stream):
            dk[b].copy_(hk[j], non_blocking=True)
            dv[b].copy_(hv[j], non_blocking=True)
            dq[b].copy_(hq[j], non_blocking=True)
        with torch.cuda.stream(out_stream):
            hout[b].copy_(st["out"], non_blocking=True)
    done = torch.cuda.Event()
    done.record(out_stream)
    copy_stream.wait_event(done)
    c1.record(copy_stream)
    torch.cuda.synchronize()
    copy_ms = c0.elapsed_time(c1)
    if world > 1:
        ms = max_over_ranks(ms, dist, device)
        copy_ms = max_over_ranks(copy_ms, dist, device)
        eager_ms = max_over_ranks(eager_ms, dist, device)
    total = 0
    for j in range(args.steps):
        a, d = step_bytes([n + (args.warmup + j) * CHUNK for n in st["lens"]])
        total += a + d
    h2d = 2 * N_SEQ * CHUNK * HKV * D * 2 + N_SEQ * HQ * D * 2
    return {"value": round(total * world / (ms * 1e-3) / 1e9, 2), "unit": "GB/s", "ms_per_step": round(ms / args.steps, 4),
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": N_SEQ * HQ * D * 2,
            "copies_alone_ms_per_step": round(copy_ms / args.steps, 4),
            "launch": "one CUDA graph per step of the public calls (captured before the timed region)",
            "eager_ms_per_step": round(eager_ms / args.steps, 4)}


def _flush_l2(torch, buf):
    buf.add_(1)


def _time_call(torch, fn, iters, flush=None):
    """Median device time (ms) of fn over iters calls, L2 flushed between calls.
    A short device-side spin precedes the start event so that the host's
    launch overhead for fn is hidden behind queued GPU work and the interval
    measures fn's kernels only."""
    stream = torch.cuda.current_stream()
    times = []
    for _ in range(iters):
        if flush is not None:
            _flush_l2(torch, flush)
        torch.cuda._sleep(200_000)  # ~0.1 ms of SM clocks
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    return statistics.median(times)


AUX_WORKLOADS = ("quantize-sweep", "prod3-gqa", "k4v3-sink", "tiny", "bf16-sdpa", "fp8-kv", "stream-2.5", "stream-k8v3",
                 "search")


def run_aux(tq, torch, kv_inputs, device, args, only=None, formats=None):
    """The other workloads, measured on the same GPU in the same run.  `only`
    restricts the run to one of AUX_WORKLOADS and `formats` the quantize sweep
    to some of mse1..4, prod1..4 (both for profiling one kernel)."""
    out = {}
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=device)  # 256 MB > L2
    iters = 10
    if only in (None, "quantize-sweep"):
        out["quantize_sweep_1M_bf16"] = _aux_sweep(tq, torch, kv_inputs, device, flush, iters, formats)
    if only in (None, "prod3-gqa"):
        out["decode_prod3_gqa_T32k"] = _aux_prod3(tq, torch, kv_inputs, device, flush, iters)
    if only in (None, "k4v3-sink"):
        out.update(_aux_k4v3(tq, torch, kv_inputs, device, flush, iters))
    if only in (None, "tiny"):
        out["decode_tiny_fp32_T4096"] = _aux_tiny(tq, torch, kv_inputs, device, iters)
    if only in (None, "stream-2.5"):
        out["decode_mixed2.5_stream_shapes"] = _aux_stream25(tq, torch, kv_inputs, device, flush, iters)
    if only in (None, "stream-k8v3"):
        out["decode_k8v3_stream_shapes"] = _aux_stream_k8v3(tq, torch, kv_inputs, device, flush, iters)
    if only in (None, "search"):
        out["ip_search_4M"] = _aux_search(tq, torch, kv_inputs, device, flush, iters, formats)
    if only in (None, "bf16-sdpa"):
        out["bf16_kv_decode_sdpa_stream_shapes"] = _aux_bf16_sdpa(torch, kv_inputs, device, flush, iters)
    if only in (None, "fp8-kv"):
        out["fp8_kv_decode_stream_shapes"] = _aux_fp8_kv(torch, kv_inputs, device, flush, iters)
    return out


def _aux_sweep(tq, torch, kv_inputs, device, flush, iters, formats):
    # quantize sweep: 32 kv-heads x 32768 tokens, bf16 with 4 outlier channels
    n = 32 * 32768
    x = kv_inputs.kv_vectors(n, D, key="sweep", device=device, dtype=torch.bfloat16, outliers=True)
    sweep = {}
    cases = [(mode, name, b, tq.TQ_ROT_HAAR, f"{name}{b}")
             for mode, name in ((tq.TQ_MODE_MSE, "mse"), (tq.TQ_MODE_PROD, "prod")) for b in (1, 2, 3, 4)]
    # the randomized Hadamard rotation in place of the Haar one (same kernels, another Pi)
    cases += [(tq.TQ_MODE_MSE, "mixed", 2, tq.TQ_ROT_HAAR, "mixed2.5"), (tq.TQ_MODE_MSE, "mixed", 3, tq.TQ_ROT_HAAR, "mixed3.5")]
    cases += [(tq.TQ_MODE_MSE, "mse", 3, tq.TQ_ROT_HADAMARD, "mse3_hadamard"),
              (tq.TQ_MODE_PROD, "prod", 3, tq.TQ_ROT_HADAMARD, "prod3_hadamard")]
    # 8-bit codes (256 centroids), the key side of the K8/V3 pair
    cases += [(tq.TQ_MODE_MSE, "mse", 8, tq.TQ_ROT_HAAR, "mse8")]
    for mode, name, b, rot, label in cases:
        if formats and label not in formats:
            continue
        mixed = int(name == "mixed")
        p = tq.Params(b, b if b <= 4 else 3, mode, mode, mixed, mixed, rotation=rot)
        pk = tq.Packed.empty(p, n, tq.TQ_K, device=device)
        ms = _time_call(torch, lambda: tq.tq_quantize(p, x, tq.TQ_K, pk), iters, flush)
        assert p.status() == 0
        cb, qb = p.row_bytes(tq.TQ_K)
        by = n * (D * 2 + cb + 4 + (qb + 4 if qb else 0))
        sweep[label] = {"mvec_per_s": round(n / (ms * 1e-3) / 1e6, 1), "ms": round(ms, 4),
                        "gb_per_s": round(by / (ms * 1e-3) / 1e9, 1)}
    return sweep


def _aux_prod3(tq, torch, kv_inputs, device, flush, iters):
    # GQA decode, prod mode: B=1, 32 q / 8 kv heads, T=32768, K/V 3-bit (2-bit MSE + QJL)
    T = 32768
    p = tq.Params(3, 3, tq.TQ_MODE_PROD, tq.TQ_MODE_PROD)
    cache = tq.Cache(p, 1, 8, T, 0, device=device)
    k = kv_inputs.kv_vectors(T * 8, D, key="c3k", device=device).view(1, T, 8, D)
    v = kv_inputs.kv_vectors(T * 8, D, key="c3v", device=device).view(1, T, 8, D)
    tq.tq_append(p, cache, torch.zeros(1, dtype=torch.int32, device=device), k, v)
    q = kv_inputs.queries((1, 32, D), key="c3q", device=device)
    ws = tq.decode_workspace(p, 1, 32, 8, T, device=device)
    o = torch.empty(1, 32, D, dtype=torch.bfloat16, device=device)
    ms = _time_call(torch, lambda: tq.tq_decode_attn(p, q, cache, T, o, ws), iters, flush)
    by = 8 * T * 2 * (32 + 16 + 8)
    return {"ms": round(ms, 4), "gb_per_s": round(by / (ms * 1e-3) / 1e9, 1), "bytes": by,
            "l2": "flushed between calls"}


def _aux_k4v3(tq, torch, kv_inputs, device, flush, iters):
    # long-context asymmetric: B=4, 64 q / 8 kv, T=131072, sink 128 bf16, K4/V3, sparse V 1e-6
    out = {}
    T = 131072
    p = tq.Params(4, 3)
    cache = tq.Cache(p, 4, 8, T - 128, 128, device=device)
    q = kv_inputs.queries((4, 64, D), key="c4q", device=device)
    for s in range(4):
        ids = torch.tensor([s], dtype=torch.int32, device=device)
        ks, vs = [], []
        for h in range(8):
            kk = kv_inputs.kv_vectors(T, D, key=("c4k", s, h), device=device, dtype=torch.bfloat16)
            kk = kv_inputs.planted_keys(kk, q[s, 8 * h:8 * h + 8], 8, 128, key=("c4p", s, h))
            ks.append(kk)
            vs.append(kv_inputs.kv_vectors(T, D, key=("c4v", s, h), device=device, dtype=torch.bfloat16))
        kt = torch.stack(ks, 1).view(1, T, 8, D)
        vt = torch.stack(vs, 1).view(1, T, 8, D)
        del ks, vs
        for c0 in range(0, T, 32768):
            tq.tq_append(p, cache, ids, kt[:, c0:c0 + 32768].contiguous(), vt[:, c0:c0 + 32768].contiguous())
        del kt, vt
    ws = tq.decode_workspace(p, 4, 64, 8, T, device=device)
    o = torch.empty(4, 64, D, dtype=torch.bfloat16, device=device)
    for thr, name in ((1e-6, "sparse_v"), (0.0, "dense")):
        ms = _time_call(torch, lambda: tq.tq_decode_attn(p, q, cache, T, o, ws, thr), iters, flush)
        by = 4 * 8 * ((T - 128) * (68 + 52) + 128 * 512)
        out[f"decode_k4v3_sink_T128k_{name}"] = {"ms": round(ms, 4), "gb_per_s_dense_equiv": round(by / (ms * 1e-3) / 1e9, 1),
                                                 "dense_bytes": by}
    # what the sparse-V rule dropped in one call (device tallies, untimed)
    stats = torch.zeros(4, dtype=torch.int64, device=device)
    tq.tq_decode_attn(p, q, cache, T, o, ws, 1e-6, sparse_v_stats=stats)
    examined, dropped, tiles, skipped = (int(x) for x in stats.cpu())
    out["decode_k4v3_sink_T128k_sparse_v"].update(
        {"weights_dropped": round(dropped / max(examined, 1), 4), "tiles_skipped": round(skipped / max(tiles, 1), 4),
         "weights_examined": examined, "tiles_examined": tiles})
    # the same cache with peaked queries (x 8): where whole tiles fall below
    # the threshold for every head of the group, sparse V skips their values
    qp = q * 8
    for thr, name in ((1e-6, "sparse_v"), (0.0, "dense")):
        ms = _time_call(torch, lambda: tq.tq_decode_attn(p, qp, cache, T, o, ws, thr), iters, flush)
        by = 4 * 8 * ((T - 128) * (68 + 52) + 128 * 512)
        out[f"decode_k4v3_sink_T128k_peaked_{name}"] = {"ms": round(ms, 4),
                                                        "gb_per_s_dense_equiv": round(by / (ms * 1e-3) / 1e9, 1)}
    stats.zero_()
    tq.tq_decode_attn(p, qp, cache, T, o, ws, 1e-6, sparse_v_stats=stats)
    examined, dropped, tiles, skipped = (int(x) for x in stats.cpu())
    out["decode_k4v3_sink_T128k_peaked_sparse_v"].update(
        {"weights_dropped": round(dropped / max(examined, 1), 4), "tiles_skipped": round(skipped / max(tiles, 1), 4)})
    assert int(cache.status.item()) == 0
    return out


def _aux_stream25(tq, torch, kv_inputs, device, flush, iters):
    """The decode call of the streaming workload (16 sequences, the same
    contexts, 32 q / 8 kv heads) over 2.5-bit rows (64 rotated channels at
    3 bits, 64 at 2: 40-byte code rows)."""
    st = build_stream_workload(tq, torch, kv_inputs, 0, 1, device, bits=2)
    p, cache = st["params"], st["cache"]
    ms = _time_call(torch, lambda: tq.tq_decode_attn(p, st["qs"][0], cache, st["cap"], st["out"], st["ws"]),
                    iters, flush)
    assert int(cache.status.item()) == 0
    row = p.row_bytes(tq.TQ_K)[0] + 4
    by = sum(HKV * n * 2 * row for n in st["lens"]) + 2 * N_SEQ * HQ * D * 2
    out = {"ms": round(ms, 4), "gb_per_s": round(by / (ms * 1e-3) / 1e9, 1), "bytes": by,
           "l2": "flushed between calls"}
    del st, cache
    return out


def _aux_stream_k8v3(tq, torch, kv_inputs, device, flush, iters):
    """The decode call of the streaming workload's shapes with 8-bit keys
    (128-byte code rows, 256 centroids) and 3-bit values (48-byte rows)."""
    st = build_stream_workload(tq, torch, kv_inputs, 0, 1, device, params=tq.Params(8, 3, seed=0))
    p, cache = st["params"], st["cache"]
    ms = _time_call(torch, lambda: tq.tq_decode_attn(p, st["qs"][0], cache, st["cap"], st["out"], st["ws"]),
                    iters, flush)
    assert int(cache.status.item()) == 0
    row = p.row_bytes(tq.TQ_K)[0] + 4 + p.row_bytes(tq.TQ_V)[0] + 4
    by = sum(HKV * n * row for n in st["lens"]) + 2 * N_SEQ * HQ * D * 2
    out = {"ms": round(ms, 4), "gb_per_s": round(by / (ms * 1e-3) / 1e9, 1), "bytes": by,
           "l2": "flushed between calls"}
    del st, cache
    return out


def _aux_search(tq, torch, kv_inputs, device, flush, iters, formats):
    """Inner-product search: a database of 2^22 vectors (d = 128, bf16 with
    lognormal norms and outlier channels, quantized on the GPU), top-10 rows
    for 8 and for 32 bf16 queries; bytes are the packed rows read once per
    group of 8 queries."""
    n = 1 << 22
    x = kv_inputs.kv_vectors(n, D, key="search-db", device=device, dtype=torch.bfloat16, outliers=True)
    out = {}
    ws = tq.search_workspace(device=device)
    for name, bits, mode in (("prod3", 3, tq.TQ_MODE_PROD), ("mse4", 4, tq.TQ_MODE_MSE)):
        if formats and name not in formats:
            continue
        p = tq.Params(bits, bits, mode, mode)
        pk = tq.Packed.empty(p, n, tq.TQ_K, device=device)
        tq.tq_quantize(p, x, tq.TQ_K, pk)
        cb, qb = p.row_bytes(tq.TQ_K)
        row = cb + 4 + (qb + 4 if qb else 0)
        for nq in (8, 32):
            q = kv_inputs.queries((nq, D), key=("search-q", nq), device=device)
            sc = torch.empty(nq, 10, device=device)
            rw = torch.empty(nq, 10, dtype=torch.int64, device=device)
            ms = _time_call(torch, lambda: tq.tq_search(p, tq.TQ_K, pk, n, q, 10, sc, rw, ws), iters, flush)
            by = n * row * ((nq + 7) // 8)
            out[f"{name}_q{nq}_k10"] = {"ms": round(ms, 4), "gb_per_s": round(by / (ms * 1e-3) / 1e9, 1),
                                        "bytes": by, "queries_per_s": round(nq / (ms * 1e-3), 1)}
        assert p.status() == 0
        del pk
    del x
    out["l2"] = "flushed between calls"
    return out


def _aux_tiny(tq, torch, kv_inputs, device, iters):
    # tiny fp32 case: 4096 vectors, b=3, 1 head
    p = tq.Params(3, 3)
    x = kv_inputs.kv_vectors(4096, D, key="c1", device=device)
    cache = tq.Cache(p, 1, 1, 4096, 0, device=device)
    tq.tq_append(p, cache, torch.zeros(1, dtype=torch.int32, device=device), x.view(1, 4096, 1, D), x.view(1, 4096, 1, D))
    q = kv_inputs.queries((1, 1, D), key="c1q", device=device, dtype=torch.float32)
    ws = tq.decode_workspace(p, 1, 1, 1, 4096, device=device)
    o = torch.empty(1, 1, D, dtype=torch.float32, device=device)
    ms = _time_call(torch, lambda: tq.tq_decode_attn(p, q, cache, 4096, o, ws), iters)
    return {"ms": round(ms, 4)}


def _aux_bf16_sdpa(torch, kv_inputs, device, flush, iters):
    """Context for the packed cache: one decode step over an unquantized bf16
    KV cache of the streaming workload's shapes (16 sequences, the same
    contexts, 32 q / 8 kv heads), with PyTorch's fused attention (the fastest
    backend that accepts the shapes), one call per sequence."""
    import torch.nn.functional as F
    from torch.nn.attention import SDPBackend, sdpa_kernel

    lens = kv_inputs.sequence_lengths(N_SEQ, LEN_LO, LEN_HI, key=("stream-lens", 0))
    gen = torch.Generator(device=device).manual_seed(0)
    ks = [torch.randn(1, HKV, n, D, generator=gen, device=device, dtype=torch.bfloat16) for n in lens]
    vs = [torch.randn(1, HKV, n, D, generator=gen, device=device, dtype=torch.bfloat16) for n in lens]
    q = torch.randn(N_SEQ, 1, HQ, 1, D, generator=gen, device=device, dtype=torch.bfloat16)
    by = sum(n * HKV * D * 2 * 2 for n in lens)
    best = None
    for backend in (SDPBackend.CUDNN_ATTENTION, SDPBackend.FLASH_ATTENTION, SDPBackend.EFFICIENT_ATTENTION,
                    SDPBackend.MATH):
        try:
            with sdpa_kernel([backend]):
                def run():
                    for s in range(N_SEQ):
                        F.scaled_dot_product_attention(q[s], ks[s], vs[s], enable_gqa=True)
                run()
                torch.cuda.synchronize()
                ms = _time_call(torch, run, iters, flush)
        except RuntimeError:
            continue
        if best is None or ms < best[1]:
            best = (backend.name, ms)
    if best is None:
        return {"unavailable": "no SDPA backend accepted the shapes"}
    name, ms = best
    return {"backend": name, "ms": round(ms, 4), "gb_per_s": round(by / (ms * 1e-3) / 1e9, 1), "bytes": by,
            "tokens_per_s_per_seq": round(1000.0 / ms, 1), "calls": N_SEQ}


def _aux_fp8_kv(torch, kv_inputs, device, flush, iters):
    """Context for the packed cache: one decode step over an FP8 (e4m3) KV
    cache of the streaming workload's shapes (16 sequences, the same contexts,
    32 q / 8 kv heads), with FlashInfer's decode kernel (one call per
    sequence, the faster of its CUDA-core and tensor-core variants)."""
    try:
        import flashinfer
    except Exception as e:  # pragma: no cover - depends on the image
        return {"unavailable": f"flashinfer import failed: {e}"}
    lens = kv_inputs.sequence_lengths(N_SEQ, LEN_LO, LEN_HI, key=("stream-lens", 0))
    gen = torch.Generator(device=device).manual_seed(0)
    f8 = torch.float8_e4m3fn
    ks = [torch.randn(n, HKV, D, generator=gen, device=device).to(f8) for n in lens]
    vs = [torch.randn(n, HKV, D, generator=gen, device=device).to(f8) for n in lens]
    q = torch.randn(N_SEQ, HQ, D, generator=gen, device=device, dtype=torch.bfloat16)
    by = sum(n * HKV * D * 2 for n in lens)
    best, errors = None, []
    for tc in (False, True):
        try:
            def run():
                for s in range(N_SEQ):
                    flashinfer.single_decode_with_kv_cache(q[s], ks[s], vs[s], use_tensor_cores=tc)
            run()
            torch.cuda.synchronize()
            ms = _time_call(torch, run, iters, flush)
        except Exception as e:
            errors.append(f"use_tensor_cores={tc}: {type(e).__name__}: {str(e)[:200]}")
            continue
        if best is None or ms < best[1]:
            best = (tc, ms)
    if best is None:
        return {"unavailable": "; ".join(errors)}
    tc, ms = best
    return {"backend": f"flashinfer {flashinfer.__version__} single_decode_with_kv_cache "
                       f"(use_tensor_cores={tc})", "ms": round(ms, 4), "gb_per_s": round(by / (ms * 1e-3) / 1e9, 1),
            "bytes": by, "tokens_per_s_per_seq": round(1000.0 / ms, 1), "calls": N_SEQ}


def run_aux_only(args):
    """One auxiliary workload alone (for profiling a kernel): prints its JSON."""
    import torch

    import kv_inputs
    import online_vector_quantization_b200 as tq

    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    formats = set(args.formats.split(",")) if args.formats else None
    out = run_aux(tq, torch, kv_inputs, device, args, only=args.aux_only, formats=formats)
    print(json.dumps({"aux_only": args.aux_only, "aux": out}), flush=True)


# ---------------------------------------------------------------------------
# Oracle timing (CPU baseline / reference arm)
# ---------------------------------------------------------------------------

def _oracle_units(unit_ids):
    """Build oracle state for some (sequence, kv-head) units of the streaming
    workload (untimed) and return a function doing one step on them: quantize
    a 64-token chunk of K and V, append it and decode the unit's 4 query heads.
    Unit u holds a context as long as sequence u mod 16."""
    import numpy as np
    import torch

    import kv_inputs
    from oracle import tq_oracle as o

    lens = kv_inputs.sequence_lengths(N_SEQ, LEN_LO, LEN_HI, key=("stream-lens", 0))
    f = o.Format(3, mixed=True)
    op = o.Params(128, f, f)
    units = []
    for u in unit_ids:
        s = u % N_SEQ
        n = lens[s]
        k = kv_inputs.kv_vectors(n, D, key=("oracle-k", s, u), dtype=torch.bfloat16).double().numpy()
        v = kv_inputs.kv_vectors(n, D, key=("oracle-v", s, u), dtype=torch.bfloat16).double().numpy()
        ck = kv_inputs.kv_vectors(CHUNK, D, key=("oracle-ck", s, u), dtype=torch.bfloat16).double().numpy()
        cv = kv_inputs.kv_vectors(CHUNK, D, key=("oracle-cv", s, u), dtype=torch.bfloat16).double().numpy()
        q = kv_inputs.queries((1, HQ // HKV, D), key=("oracle-q", s, u)).double().numpy()
        cache = o.cache_from_vectors(op, k[None, None], v[None, None], 0)
        units.append((n, ck, cv, q, cache))

    def one_step():
        nbytes = 0
        for n, ck, cv, q, cache in units:
            kr, vr = o.quantize(op, ck, "k"), o.quantize(op, cv, "v")
            c = o.Cache(0)
            c.k_sink[0, 0] = c.v_sink[0, 0] = np.zeros((0, D))
            c.k_rows[0, 0] = o.Packed(np.concatenate([cache.k_rows[0, 0].codes, kr.codes]),
                                      np.concatenate([cache.k_rows[0, 0].norms, kr.norms]), np.zeros((n + CHUNK, 0), np.uint8),
                                      np.zeros(n + CHUNK, np.float32))
            c.v_rows[0, 0] = o.Packed(np.concatenate([cache.v_rows[0, 0].codes, vr.codes]),
                                      np.concatenate([cache.v_rows[0, 0].norms, vr.norms]), np.zeros((n + CHUNK, 0), np.uint8),
                                      np.zeros(n + CHUNK, np.float32))
            o.decode_attention(op, q, c, [n + CHUNK], 1)
            nbytes += 2 * CHUNK * D * 2 + 2 * CHUNK * ROW_BYTES + (n + CHUNK) * 2 * ROW_BYTES + 2 * (HQ // HKV) * D * 2
        return nbytes

    return one_step


_WORKER_STEP = None


def _oracle_worker_init(unit_ids):
    """Pool worker: one BLAS thread per process, then the worker's units."""
    global _WORKER_STEP
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(1)
    except Exception:
        pass
    _WORKER_STEP = _oracle_units(unit_ids)


def _oracle_worker_step(_):
    return _WORKER_STEP()


def _host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


class OraclePool:
    """The oracle over independent units on all host cores: one spawned
    process per core (started before any GPU work of the caller matters, and
    by spawn, never fork), each owning units_per_worker units; a step runs one
    oracle step in every worker at once."""

    def __init__(self, units_per_worker: int, workers: int | None = None):
        import multiprocessing as mp
        # every host core, up to 32 processes (each holds its units' oracle
        # state and a copy of the numpy / torch runtime)
        self.workers = workers or min(_host_cores(), 32)
        self.units = self.workers * units_per_worker
        ctx = mp.get_context("spawn")
        self._pools = []
        # one single-process pool per worker so each gets its own unit ids
        for w in range(self.workers):
            ids = list(range(w * units_per_worker, (w + 1) * units_per_worker))
            self._pools.append(ctx.Pool(1, initializer=_oracle_worker_init, initargs=(ids,)))

    def step(self) -> int:
        res = [p.apply_async(_oracle_worker_step, (0,)) for p in self._pools]
        return sum(r.get() for r in res)

    def close(self):
        for p in self._pools:
            p.terminate()
            p.join()


def cpu_baseline_stream(args, pool=None):
    """The oracle timed on the host: all cores (a spawn process pool over
    independent units) and one thread on one unit."""
    own = pool is None
    if own:
        pool = OraclePool(args.cpu_units)
    pool.step()  # warm-up: every worker has built its units and run once
    t = time.perf_counter()
    nbytes = pool.step()
    dt = time.perf_counter() - t
    workers, units = pool.workers, pool.units
    if own:
        pool.close()
    # one thread, one unit
    try:
        from threadpoolctl import threadpool_limits
        lim = threadpool_limits(1)
    except Exception:
        lim = None
    one = _oracle_units([0])
    one()
    t1 = time.perf_counter()
    b1 = one()
    d1 = time.perf_counter() - t1
    if lim is not None:
        lim.restore_original_limits()
    return {"value": round(nbytes / dt / 1e9, 4), "unit": "GB/s", "cores": workers, "kind": "oracle",
            "sample": f"{units} of {N_SEQ * HKV} (sequence, kv-head) units of the streaming step (64-token append "
                      f"+ 4-head decode each), fp64 numpy oracle, {workers} processes x 1 thread, {dt:.1f} s; "
                      f"the whole step's 128 units would take about {dt * N_SEQ * HKV / units:.1f} s",
            "single_thread": {"value": round(b1 / d1 / 1e9, 5), "unit": "GB/s", "units": 1, "s": round(d1, 2)}}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    pool = OraclePool(args.cpu_units)
    try:
        for _ in range(args.warmup):
            pool.step()
        t = time.perf_counter()
        nbytes = 0
        for _ in range(args.steps):
            nbytes += pool.step()
        dt = time.perf_counter() - t
    finally:
        pool.close()
    value = nbytes / dt / 1e9
    sample = (f"{pool.units} of {N_SEQ * HKV} (sequence, kv-head) units of the streaming step per step "
              f"(64-token append + 4-head decode each), fp64 numpy oracle, {pool.workers} processes x 1 thread")
    line = {"impl": "reference", "metric": "decode-attn packed-KV GB/s (streaming append + decode step)",
            "value": round(value, 4), "unit": "GB/s", "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "streaming append + decode: 16 seqs, ctx U[8192,65536], 64-token bf16 chunk, "
                                   "mixed 3.5-bit K/V, 32 q / 8 kv heads, d=128 (bounded sample)"},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": pool.workers, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="tq", choices=["tq", "reference"])
    ap.add_argument("--no-aux", action="store_true", help="skip the auxiliary workloads")
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle CPU baseline")
    ap.add_argument("--cpu-units", type=int, default=1, help="oracle units per host core (CPU baseline)")
    ap.add_argument("--aux-only", choices=AUX_WORKLOADS, default=None,
                    help="run one auxiliary workload alone and print its numbers (profiling)")
    ap.add_argument("--formats", default=None, help="with --aux-only quantize-sweep: e.g. mse3,prod3")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.aux_only:
        run_aux_only(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
