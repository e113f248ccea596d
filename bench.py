"""Benchmark of one paged decode step: paged_kv_append of one new token per
sequence, then paged_attention_decode over the whole batch.

Default workload: the long-context split-KV layer, the largest single-GPU
shape (batch 4 x 131,072 tokens, 64 q / 8 kv heads, head_dim 128, bf16,
16-token blocks placed at random in a pool of exactly 4 x 8192 blocks, the
first 4 keys of every sequence scaled x4 as attention sinks; 2.15 GB of K and
V per step), seeded synthetic data.  ``--workload`` selects the other shapes
(Llama-3-8B GQA, Llama-2-7B MHA, the shared-prefix ones).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  ``value`` is the KV-read throughput of the
step in GB/s: the K and V bytes of every (block, kv head) tile the step reads
(the algorithmic bytes; tail blocks count whole) divided by the device time
of the step, measured with CUDA events on the launching stream.  Between
timed steps a 256 MiB buffer is written and a second one read (untimed), so
that every step starts with a cold L2 holding no dirty lines.  ``e2e`` is the
same metric through the public API with host buffers: each step's inputs
copied in from pinned memory and its output copied back, pipelined over three
streams as a serving loop runs them (the serial figure is reported beside
it).  With N GPUs each rank runs its own replica (the path needs no exchange
between GPUs) and ``value`` sums the replicas over the slowest rank's time.
``--impl reference`` times the CPU oracle instead, on a bounded sample of the
same workload.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import time
from pathlib import Path

import torch

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

import workloads as W  # noqa: E402
from paged_kv_cache_386_b200 import layout  # noqa: E402

METRIC = "paged decode attention: KV-read GB/s (fraction of HBM peak); tokens/s per layer"
UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0
PROFILE_TRAFFIC = ROOT / "profiles" / "ncu_traffic.json"
KERNEL_SOURCES = ["paged_kv_cache_386_b200/csrc/pkv_kernels.cuh", "paged_kv_cache_386_b200/csrc/pkv_device.cuh",
                  "paged_kv_cache_386_b200/csrc/pkv_api.cu"]

WORKLOADS = {
    "llama3_8b_gqa": (lambda seed, **kw: W.uniform_gqa(seed=seed, **kw),
                      "llama3_8b_gqa: batch 64, 32 q / 8 kv heads, head_dim 128, bf16, block 16, "
                      "context U[128,4096], shuffled pool +10%"),
    "llama2_7b_mha": (lambda seed, **kw: W.lognormal_mha(seed=seed, **kw),
                      "llama2_7b_mha: batch 256, 32 q = 32 kv heads, head_dim 128, fp16, block 16, "
                      "context round(clip(lognormal(ln 300, 1), 1, 2048)), shuffled pool +10%"),
    "shared_prefix_70b": (lambda seed, **kw: W.shared_prefix(seed=seed, **kw),
                          "shared_prefix_70b: 128 seqs, 64 q / 8 kv heads, head_dim 128, bf16, one shared "
                          "2048-token prefix + private suffix U[16,512]"),
    "best_of_8": (lambda seed, **kw: W.best_of_n(seed=seed, **kw),
                  "best_of_8: 16 prompts x 8 samples, 2000-token shared prompt + 100 private tokens, "
                  "64 q / 8 kv heads, head_dim 128, bf16"),
    "long_ctx_128k": (lambda seed, **kw: W.long_context(seed=seed, **kw),
                      "long_ctx_128k: batch 4 x 131072 tokens, 64 q / 8 kv heads, head_dim 128, bf16, "
                      "4 sink keys x4"),
}


def kernel_hash() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        h.update((ROOT / rel).read_bytes())
    return h.hexdigest()[:16]


def measured_hbm_peak() -> tuple[float, str]:
    p = ROOT / "MEASURED_PEAKS.json"
    try:
        d = json.loads(p.read_text())
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled through NVML every
    millisecond in a background thread during the timed region (read-only
    queries; no GPU setting is changed)."""

    def __init__(self, device: torch.device, period_s: float = 0.01, enabled: bool = True):
        self.enabled = enabled
        self.device = device
        self.period = period_s
        self.samples: list[tuple[int, int, int]] = []
        self.error = None

    def _handle(self):
        import pynvml
        pynvml.nvmlInit()
        props = torch.cuda.get_device_properties(self.device)
        bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
        return pynvml, pynvml.nvmlDeviceGetHandleByPciBusId(bus)

    def _run(self):
        try:
            nv, h = self._handle()
            mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            while not self._stop.is_set():
                self.samples.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM), mx,
                                     nv.nvmlDeviceGetCurrentClocksEventReasons(h)))
                self._stop.wait(self.period)
        except Exception as e:  # NVML missing: report no samples
            self.error = repr(e)

    def __enter__(self):
        import threading
        self._stop = threading.Event()
        if not self.enabled:
            self._thread = threading.Thread(target=lambda: None)
            self._thread.start()
            return self
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        self._thread.join(timeout=5)

    def summary(self) -> dict:
        names = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
                 0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}
        reasons = set()
        for _, _, r in self.samples:
            for bit, n in names.items():
                if r & bit:
                    reasons.add(n)
        sm = [c for c, _, _ in self.samples]
        out = {"sm_mhz": statistics.median(sm) if sm else None,
               "sm_max_mhz": self.samples[0][1] if self.samples else None,
               "reasons": sorted(reasons), "samples": len(sm), "source": "nvml"}
        if self.error:
            out["error"] = self.error
        return out


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce_max(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(per_rank_units: float, max_seconds: float, world: int) -> float:
    """Whole-job throughput: the units every replica processed over the slowest
    rank's time (replicas process the same amount of work)."""
    return per_rank_units * world / max_seconds


# ---------------------------------------------------------------------------
# Our arm
# ---------------------------------------------------------------------------

def run_ours(args) -> None:
    import paged_kv_cache_386_b200 as pkv

    world, rank, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)

    make, desc = WORKLOADS[args.workload]
    mq = args.q_len > 1
    if mq and (args.workload != "llama3_8b_gqa" or args.cascade or args.kv != "16-bit"):
        raise SystemExit("--q-len > 1 is measured on llama3_8b_gqa with the 16-bit cache (--workload llama3_8b_gqa)")
    w = (W.uniform_gqa(seed=args.seed, q_len=args.q_len, placement=args.placement) if mq
         else make(args.seed, placement=args.placement))
    if mq:
        desc += f"; {args.q_len} queries per sequence (the last {args.q_len} tokens, causal)"
    es = w.k_cache.element_size()
    int8 = args.kv == "int8"
    if int8 and args.cascade:
        raise SystemExit("--kv int8 and --cascade cannot be combined")
    tr = layout.decode_traffic(w.block_tables, w.context_lens, w.n_q_heads, w.n_kv_heads, w.head_dim, es,
                               kv_int8=int8)
    kv_bytes = tr["kv_unique"]
    # The plain 16-bit decode step runs as one launch, the append fused into
    # the decode (paged_kv_append_and_decode); --separate-append times the
    # two calls instead.
    fused = not (int8 or mq or args.cascade or args.separate_append)
    decode_bytes = tr["total_unique"] + (layout.append_traffic(w.k_new.shape[0], w.n_kv_heads, w.head_dim, es)
                                         if fused else 0)

    # Device copies of the whole problem.
    kc, vc = w.k_cache.to(dev), w.v_cache.to(dev)
    q, k_new, v_new = w.q.to(dev), w.k_new.to(dev), w.v_new.to(dev)
    slots, bt, cl = w.slot_mapping.to(dev), w.block_tables.to(dev), w.context_lens.to(dev)
    out = torch.empty_like(q)
    if int8:
        # The same tokens quantised into the INT8 cache (untimed set-up).
        kv8 = pkv.int8_cache(w.num_blocks, w.n_kv_heads, w.head_dim, device=dev)
        kr, vr, sl = W.cached_token_rows(w)
        pkv.paged_kv_append_int8(kr.to(dev), vr.to(dev), sl.to(dev), kv8)
        del kc, vc, kr, vr
        torch.cuda.synchronize(dev)
    if args.cascade:
        # Shared prefixes attended once per group and kv head, then the suffixes.
        cv = W.cascade_view(w)
        c_pt, c_pl, c_sg, c_bt, c_cl = (t.to(dev) for t in (cv.prefix_block_tables, cv.prefix_lens, cv.seq_group,
                                                             cv.block_tables, cv.context_lens))
        ws = torch.zeros(pkv.paged_attention_cascade_workspace_size(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim,
                                                                    w.dtype), dtype=torch.uint8, device=dev)
    elif mq:
        ws = torch.zeros(pkv.paged_attention_mq_workspace_size(w.batch, args.q_len, w.n_q_heads, w.n_kv_heads,
                                                               w.head_dim, w.dtype), dtype=torch.uint8, device=dev)
    else:
        ws = torch.zeros(pkv.paged_attention_workspace_size(w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim,
                                                            w.dtype), dtype=torch.uint8, device=dev)

    def append(stream_=None):
        if fused:
            return  # inside the decode launch
        if int8:
            pkv.paged_kv_append_int8(k_new, v_new, slots, kv8, stream=stream_)
        else:
            pkv.paged_kv_append(k_new, v_new, slots, kc, vc, stream=stream_)

    def decode(stream_=None):
        if fused:
            pkv.paged_kv_append_and_decode(q, k_new, v_new, slots, kc, vc, bt, cl, w.scale, out=out, workspace=ws,
                                           stream=stream_)
        elif mq:
            pkv.paged_attention_decode_mq(q, kc, vc, bt, cl, w.scale, out=out, workspace=ws, stream=stream_)
        elif int8:
            pkv.paged_attention_decode_int8(q, kv8, bt, cl, w.scale, out=out, workspace=ws, stream=stream_)
        elif args.cascade:
            pkv.paged_attention_decode_cascade(q, kc, vc, c_pt, c_pl, c_sg, c_bt, c_cl, w.scale, out=out,
                                               workspace=ws, stream=stream_)
        else:
            pkv.paged_attention_decode(q, kc, vc, bt, cl, w.scale, out=out, workspace=ws, stream=stream_)
    # L2 flush between steps: write a buffer larger than L2 (126 MB), then
    # read a second one, so that the lines the write left dirty are written
    # back here and not during the timed step (whose reads they would slow).
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_r = torch.zeros(64 << 20, dtype=torch.int32, device=dev)
    flush_sink = torch.empty((), dtype=torch.int64, device=dev)

    def flush_l2(i: int) -> None:
        flush_w.fill_(i & 0xFF)
        torch.sum(flush_r, dim=0, dtype=torch.int64, out=flush_sink)
    stream = torch.cuda.current_stream(dev)

    def step():
        append(stream)
        decode(stream)

    # Warm-up: W steps, continued until 0.3 s have passed so that the SM
    # clock has left its idle state before timing.
    t_warm, warm_steps = time.perf_counter(), 0
    while warm_steps < args.warmup or time.perf_counter() - t_warm < 0.3:
        flush_l2(1)
        step()
        warm_steps += 1
        if warm_steps % 16 == 0:
            torch.cuda.synchronize(dev)
    torch.cuda.synchronize(dev)
    if pkv.pkv_get_device_error(stream) != 0:
        raise RuntimeError("device error flag set during warm-up")

    # The step is captured once as a CUDA graph (append, decode, merge) and
    # replayed, as a serving engine replays its decode step: no host launch
    # gaps between the kernels.  Event-record nodes inside the graph time the
    # whole step and the decode call alone on the launching stream.
    g, launch_note = None, "direct C-ABI calls"
    if not args.no_graph:
        try:
            ev_a, ev_b, ev_c = (torch.cuda.Event(enable_timing=True, external=True) for _ in range(3))
            g = torch.cuda.CUDAGraph()
            cap = torch.cuda.Stream(dev)
            cap.wait_stream(stream)
            with torch.cuda.graph(g, stream=cap):
                ev_a.record()
                append()
                ev_b.record()
                decode()
                ev_c.record()
            stream.wait_stream(cap)
            for _ in range(args.warmup):
                flush_l2(1)
                g.replay()
            torch.cuda.synchronize(dev)
            launch_note = ("CUDA graph of the step (one launch: the append fused into the decode)" if fused
                           else "CUDA graph of the step (append + decode)")
        except Exception as e:  # capture unsupported: time direct calls
            torch.cuda.synchronize(dev)
            g, launch_note = None, f"direct C-ABI calls (graph capture failed: {type(e).__name__})"

    step_ms, decode_ms = [], []
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev, enabled=not args.no_clocks) as clocks:
        t0 = time.perf_counter()
        for i in range(args.steps):
            flush_l2(i)
            if g is not None:
                g.replay()
                ev_c.synchronize()
                step_ms.append(ev_a.elapsed_time(ev_c))
                decode_ms.append(ev_b.elapsed_time(ev_c))
            else:
                a, b, c = (torch.cuda.Event(enable_timing=True) for _ in range(3))
                a.record(stream)
                append(stream)
                b.record(stream)
                decode(stream)
                c.record(stream)
                c.synchronize()
                step_ms.append(a.elapsed_time(c))
                decode_ms.append(b.elapsed_time(c))
        torch.cuda.synchronize(dev)
        wall = time.perf_counter() - t0
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    step_s = sum(step_ms) / 1e3
    max_step_s = reduce_max(step_s, world, dev)
    value = aggregate(kv_bytes, max_step_s / args.steps, world) / 1e9
    tokens_per_s = aggregate(w.batch * args.q_len, max_step_s / args.steps, world)
    dec_avg_s = sum(decode_ms) / len(decode_ms) / 1e3
    achieved = decode_bytes / dec_avg_s / 1e9
    peak, peak_kind = measured_hbm_peak()

    # End to end through the public API with host buffers: pinned host ->
    # device copies of this step's inputs, append + decode, device -> host read
    # of the output, all inside the timed region.
    if args.cascade:
        h_in = [t.pin_memory() for t in (w.q, w.k_new, w.v_new, w.slot_mapping, cv.prefix_block_tables,
                                         cv.prefix_lens, cv.seq_group, cv.block_tables, cv.context_lens)]
        d_in = [q, k_new, v_new, slots, c_pt, c_pl, c_sg, c_bt, c_cl]
    else:
        h_in = [t.pin_memory() for t in (w.q, w.k_new, w.v_new, w.slot_mapping, w.block_tables, w.context_lens)]
        d_in = [q, k_new, v_new, slots, bt, cl]
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in h_in)
    d2h = h_out.numel() * h_out.element_size()

    def e2e_step():
        for d, h in zip(d_in, h_in):
            d.copy_(h, non_blocking=True)
        append(stream)
        decode(stream)
        h_out.copy_(out, non_blocking=True)

    for _ in range(args.warmup):
        flush_l2(1)
        e2e_step()
    torch.cuda.synchronize(dev)
    e2e_ms = []
    for i in range(args.steps):
        flush_l2(i)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        e2e_step()
        b.record(stream)
        b.synchronize()
        e2e_ms.append(a.elapsed_time(b))
    e2e_serial_s = reduce_max(sum(e2e_ms) / 1e3, world, dev)
    e2e_serial_value = aggregate(kv_bytes, e2e_serial_s / args.steps, world) / 1e9

    # The same steps pipelined as a serving loop runs them: three streams and
    # two sets of device buffers, so that the inputs of step i + 1 are copied
    # in and the output of step i - 1 is copied out while step i computes.
    # Every step's copies are inside the timed region (first copy-in to last
    # copy-out).  Each buffer set has its own copy of the KV cache, so that no
    # step finds the previous step's KV in L2 (there is no flush inside this
    # loop).
    # A step's inputs travel as one packed copy (each tensor at a 256-byte
    # aligned offset of one pinned buffer), as a serving loop batches them.
    offs, total = [], 0
    for t in h_in:
        offs.append(total)
        total += (t.numel() * t.element_size() + 255) & ~255
    h_pack = torch.empty(total, dtype=torch.uint8).pin_memory()
    for t, o in zip(h_in, offs):
        h_pack[o:o + t.numel() * t.element_size()].copy_(t.reshape(-1).view(torch.uint8))

    def device_views(buf):
        return [buf[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape) for t, o in zip(h_in, offs)]

    n_sets = 2
    p_sets = [torch.empty(total, dtype=torch.uint8, device=dev) for _ in range(n_sets)]
    d_sets = [device_views(b) for b in p_sets]
    if int8:
        c_sets = [(kv8,)] + [(kv8.clone(),) for _ in range(n_sets - 1)]
    else:
        c_sets = [(kc, vc)] + [(kc.clone(), vc.clone()) for _ in range(n_sets - 1)]
    o_sets = [out] + [torch.empty_like(out) for _ in range(n_sets - 1)]
    h_outs = [h_out] + [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(n_sets - 1)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def append_set(ins, cache, s_):
        if fused:
            return
        if int8:
            pkv.paged_kv_append_int8(ins[1], ins[2], ins[3], cache[0], stream=s_)
        else:
            pkv.paged_kv_append(ins[1], ins[2], ins[3], cache[0], cache[1], stream=s_)

    def decode_set(ins, cache, o, s_):
        q_ = ins[0]
        if fused:
            pkv.paged_kv_append_and_decode(q_, ins[1], ins[2], ins[3], cache[0], cache[1], ins[4], ins[5], w.scale,
                                           out=o, workspace=ws, stream=s_)
        elif args.cascade:
            pkv.paged_attention_decode_cascade(q_, cache[0], cache[1], *ins[4:9], w.scale, out=o, workspace=ws,
                                               stream=s_)
        elif mq:
            pkv.paged_attention_decode_mq(q_, cache[0], cache[1], ins[4], ins[5], w.scale, out=o, workspace=ws,
                                          stream=s_)
        elif int8:
            pkv.paged_attention_decode_int8(q_, cache[0], ins[4], ins[5], w.scale, out=o, workspace=ws, stream=s_)
        else:
            pkv.paged_attention_decode(q_, cache[0], cache[1], ins[4], ins[5], w.scale, out=o, workspace=ws,
                                       stream=s_)

    def run_pipelined(n_steps: int) -> float:
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        comp_done, out_done = [], []
        s_in.wait_stream(stream)
        start.record(s_in)
        for i in range(n_steps):
            k = i % n_sets
            if i >= n_sets:  # buffer set k: step i - n_sets has computed and been copied out
                s_in.wait_event(comp_done[i - n_sets])
                stream.wait_event(out_done[i - n_sets])
            with torch.cuda.stream(s_in):
                p_sets[k].copy_(h_pack, non_blocking=True)
            ev_in = torch.cuda.Event()
            ev_in.record(s_in)
            stream.wait_event(ev_in)
            append_set(d_sets[k], c_sets[k], stream)
            decode_set(d_sets[k], c_sets[k], o_sets[k], stream)
            ev_c = torch.cuda.Event()
            ev_c.record(stream)
            comp_done.append(ev_c)
            s_out.wait_event(ev_c)
            with torch.cuda.stream(s_out):
                h_outs[k].copy_(o_sets[k], non_blocking=True)
            ev_o = torch.cuda.Event()
            ev_o.record(s_out)
            out_done.append(ev_o)
        end.record(s_out)
        end.synchronize()
        stream.wait_stream(s_out)
        return start.elapsed_time(end) / 1e3

    run_pipelined(args.warmup)
    torch.cuda.synchronize(dev)
    e2e_s = reduce_max(run_pipelined(args.steps), world, dev)
    torch.cuda.synchronize(dev)
    e2e_value = aggregate(kv_bytes, e2e_s / args.steps, world) / 1e9
    if pkv.pkv_get_device_error(stream) != 0:
        raise RuntimeError("device error flag set during the timed run")

    traffic = None
    try:
        entries = json.loads(PROFILE_TRAFFIC.read_text())
        for prof in (entries if isinstance(entries, list) else [entries]):
            # The capture is of one exact workload: kernel sources, shape,
            # cache format, seed and placement must all match.
            if (prof.get("kernel_hash") == kernel_hash() and prof.get("workload") == args.workload
                    and prof.get("kv", "16-bit") == ("int8" if int8 else "16-bit") and not args.cascade and not mq
                    and bool(prof.get("fused", False)) == fused
                    and prof.get("seed", 0) == args.seed and prof.get("placement", "shuffle") == args.placement):
                traffic = prof.get("dram_bytes_per_launch")
    except Exception:
        traffic = None

    result = None
    if rank == 0:
        cpu = (cpu_baseline(w, kv_bytes, budget_s=args.cpu_budget)
               if (world == 1 and not args.no_cpu and not int8 and not mq) else None)
        result = {
            "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(max_step_s / args.steps * 1e3, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": ("int8 KV / " if int8 else "") + W.DTYPE_NAMES[w.dtype],
            "data": ("synthetic (seeded N(0,1) q/K/V, random block placement)" if args.placement == "shuffle" else
                     "synthetic (seeded N(0,1) q/K/V, blocks of each sequence consecutive in the pool)"),
            "config": {"workload": desc, "global_batch": w.batch * world, "seq_len": "ragged",
                       "placement": args.placement,
                       "mean_context": round(tr["tokens"] / w.batch, 1), "parallelism": f"replicas x{world}",
                       "l2": "flushed between steps (256 MiB write, then a 256 MiB read that drains its dirty lines; untimed)", "seed": args.seed,
                       "warmup_steps_run": warm_steps,
                       "launch": launch_note,
                       "decode": "cascade (shared prefix once per group)" if args.cascade else "paged decode",
                       "kv_cache": ("INT8 codes + fp32 scale per (token, kv head), one 4224-byte record per "
                                    "(block, kv head)" if int8
                                    else W.DTYPE_NAMES[w.dtype])},
            "tokens_per_s_per_layer": round(tokens_per_s, 1),
            "kv_bytes_per_step": kv_bytes,
            "roofline": {"bound": "hbm",
                         "kernel": ("paged_attention_decode_cascade (pkv_prefix_tc_kernel + pkv_decode_kernel)"
                                    if args.cascade else
                                    "paged_kv_append_and_decode (pkv_decode_kernel, append fused)" if fused else
                                    "paged_attention_decode_int8 (pkv_decode_kernel, INT8)" if int8 else
                                    "paged_attention_decode_mq (pkv_decode_kernel, several queries)" if mq
                                    else "paged_attention_decode (pkv_decode_kernel)"),
                         "achieved": round(achieved, 1), "peak": peak, "peak_kind": peak_kind,
                         "unit": "GB/s", "frac": round(achieved / peak, 4), "traffic": traffic,
                         "algorithmic_bytes_per_launch": decode_bytes,
                         "avg_launch_us": round(dec_avg_s * 1e6, 2),
                         "median_launch_us": round(statistics.median(decode_ms) * 1e3, 2)},
            "cpu_baseline": cpu,
            "e2e": {"value": round(e2e_value, 2), "unit": UNIT, "h2d_bytes_per_step": int(total),
                    "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_s / args.steps * 1e3, 4),
                    "schedule": "pipelined: copy-in (all inputs as one packed copy), compute and copy-out on "
                                "three streams, two buffer sets each with its own KV cache copy, so consecutive "
                                "steps share nothing in L2",
                    "serial_h2d_bytes_per_step": h2d,
                    "serial_value": round(e2e_serial_value, 2),
                    "serial_ms_per_step": round(e2e_serial_s / args.steps * 1e3, 4)},
            "gpu_launches": (3 if args.cascade else 1 if fused else 2) * args.steps,
            "clocks": clocks.summary(),
            "wall_s_timed_loop": round(wall, 4),
        }
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if result is not None:
        print(json.dumps(result), flush=True)


def oracle_units(w) -> list[tuple[int, int]]:
    """The (sequence, kv head) units of a workload, interleaved over the
    sequences: one unit is every query head of one kv head of one sequence,
    the work that reads that sequence's K and V of that kv head once."""
    return [(b, h) for h in range(w.n_kv_heads) for b in range(w.batch)]


def unit_rows(w, units) -> list[tuple[int, int]]:
    g = w.n_q_heads // w.n_kv_heads
    return [(b, h * g + i) for b, h in units for i in range(g)]


def unit_bytes(w, units) -> int:
    """K and V bytes the units read (whole blocks, as the GPU path counts them)."""
    lens = w.lens()
    es = w.k_cache.element_size()
    return sum(layout.blocks_for(lens[b]) * 16 * w.head_dim * es * 2 for b, _ in units)


def oracle_batches(w, cores: int, token_heads: int) -> list[list[tuple[int, int]]]:
    """Consecutive batches of units, each about ``token_heads`` (context tokens
    x query heads) of oracle work and at least one unit."""
    lens = w.lens()
    g = w.n_q_heads // w.n_kv_heads
    out, cur, acc = [], [], 0
    for u in oracle_units(w):
        cur.append(u)
        acc += lens[u[0]] * g
        if acc >= token_heads:
            out.append(cur)
            cur, acc = [], 0
    if cur:
        out.append(cur)
    return out


# fp64 oracle work one host thread does in about a second (context tokens x
# query heads), used to size the samples.
ORACLE_TOKEN_HEADS_PER_S = 250_000


def cpu_baseline(w, kv_bytes: int, budget_s: float = 15.0) -> dict:
    """The oracle (append + fp64 decode) on the host cores, on a bounded
    sample of the same workload: batches of (sequence, kv head) units, each
    about a second of work on all threads, until ``budget_s`` has passed or
    the whole workload is done."""
    import oracle

    cores = oracle.cpu_cores()
    kc, vc = w.k_cache.clone(), w.v_cache.clone()
    t0 = time.perf_counter()
    oracle.kv_append(w.k_new, w.v_new, w.slot_mapping, kc, vc, w.block_size)
    t_total = time.perf_counter() - t0
    done_units, done_bytes = 0, 0
    for units in oracle_batches(w, cores, cores * ORACLE_TOKEN_HEADS_PER_S):
        t0 = time.perf_counter()
        oracle.paged_decode(w.q, kc, vc, w.block_tables, w.context_lens, w.scale, rows=unit_rows(w, units),
                            n_threads=cores)
        t_total += time.perf_counter() - t0
        done_units += len(units)
        done_bytes += unit_bytes(w, units)
        if t_total > budget_s:
            break
    # The same oracle on one thread, a few seconds of it.
    one_units, one_bytes, t_one = 0, 0, 0.0
    for units in oracle_batches(w, 1, ORACLE_TOKEN_HEADS_PER_S):
        t0 = time.perf_counter()
        oracle.paged_decode(w.q, kc, vc, w.block_tables, w.context_lens, w.scale, rows=unit_rows(w, units),
                            n_threads=1)
        t_one += time.perf_counter() - t0
        one_units += len(units)
        one_bytes += unit_bytes(w, units)
        if t_one > min(5.0, budget_s / 3):
            break
    n_all = w.batch * w.n_kv_heads
    return {"value": round(done_bytes / t_total / 1e9, 4), "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"append of all {w.batch} new tokens + fp64 decode of {done_units} of {n_all} "
                      f"(sequence, kv head) units (all their q heads), {t_total:.1f} s on {cores} threads",
            "one_core": {"value": round(one_bytes / t_one / 1e9, 4), "unit": UNIT,
                         "sample": f"fp64 decode of {one_units} (sequence, kv head) units, {t_one:.1f} s "
                                   f"on 1 thread"}}


# ---------------------------------------------------------------------------
# Reference arm: the CPU oracle, as it stands, on the host cores
# ---------------------------------------------------------------------------

def run_reference(args) -> None:
    world, rank, _ = dist_env()
    if rank != 0:
        return
    import oracle

    make, desc = WORKLOADS[args.workload]
    w = make(args.seed, placement=args.placement)
    cores = oracle.cpu_cores()
    # Each step: append of every new token + decode of a fixed sample of
    # (sequence, kv head) units (every q head of each), about a second of
    # work on all threads unless --ref-units asks for more, so that the whole
    # run stays within minutes.
    batches = oracle_batches(w, cores, cores * ORACLE_TOKEN_HEADS_PER_S)
    sample = batches[0] if args.ref_units <= 0 else oracle_units(w)[: args.ref_units]
    rows = unit_rows(w, sample)
    kv_bytes = unit_bytes(w, sample)

    def step():
        kc, vc = w.k_cache, w.v_cache
        oracle.kv_append(w.k_new, w.v_new, w.slot_mapping, kc, vc, w.block_size)
        oracle.paged_decode(w.q, kc, vc, w.block_tables, w.context_lens, w.scale, rows=rows, n_threads=cores)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = kv_bytes * args.steps / dt / 1e9
    sample_desc = (f"append of all {w.batch} new tokens + fp64 decode of {len(sample)} of "
                   f"{w.batch * w.n_kv_heads} (sequence, kv head) units (all their q heads) per step")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) q/K/V, random block placement)",
        "config": {"workload": desc, "global_batch": w.batch, "seq_len": "ragged", "parallelism": "cpu"},
        "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample_desc},
        "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main(argv=None) -> None:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=list(WORKLOADS), default="long_ctx_128k")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--placement", choices=["shuffle", "identity"], default="shuffle",
                    help="physical block placement: a random permutation of the pool, or each sequence's blocks "
                         "consecutive (paged vs contiguous reads with the same kernel)")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU baseline leg")
    ap.add_argument("--no-graph", action="store_true", help="time direct calls instead of a CUDA graph replay")
    ap.add_argument("--separate-append", action="store_true",
                    help="run the step as paged_kv_append + paged_attention_decode (two launches) instead of "
                         "the fused paged_kv_append_and_decode")
    ap.add_argument("--no-clocks", action="store_true", help="do not sample SM clocks during the timed region")
    ap.add_argument("--cascade", action="store_true",
                    help="decode shared-prefix workloads with paged_attention_decode_cascade")
    ap.add_argument("--ref-units", type=int, default=0,
                    help="(sequence, kv head) units per reference-arm step (0: about a second of work)")
    ap.add_argument("--q-len", type=int, default=1,
                    help="queries per sequence (multi-query decode of the last q_len tokens)")
    ap.add_argument("--kv", choices=["16-bit", "int8"], default="16-bit",
                    help="cache format: the workload's 16-bit dtype, or INT8 codes with per-token scales")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
