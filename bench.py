"""Benchmark of the paged-KV decode step on B200.

One step = the whole hot path over one batch: copy-on-write block copies (when
the workload has them), the new-token KV write, and paged decode attention for
every sequence and query head. Inputs are resident in HBM before timing
starts; every workload's KV bytes exceed the 126 MB L2, so the mean step time
is taken without a flush between steps. The line also gives p10 / p50 / p90 of
per-step times, both as they come and with the L2 evicted before every step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload long|gqa|mha|prefix_cow|tiny]
                    [--impl ours|reference] [--block-size BS] [--path auto|simt|tc]

The default workload (the headline line) is long-context decode, the largest
single-GPU configuration (8 sequences of 32K-128K tokens, 64/8 heads, bf16,
block size 32). A default single-GPU run then measures the GQA, MHA and
prefix-sharing configurations with the same keys (`configs`), and the rows
beyond the decode step (`next`): paged vs contiguous placement, the
long-context block-size sweep, a prefill-sized write, block swap, and the
allocator waste simulation.

Under torchrun (N > 1) every rank runs its own independent batch (different
seed) on its own GPU: decode of different sequences needs no exchange, so the
scaling is weak and no collective touches the data path; the step time is the
max over ranks. Rank 0 prints one JSON line.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time
from pathlib import Path

import numpy as np
import torch

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

METRIC = "paged decode: effective KV-read HBM GB/s (% of B200 peak), seq-steps/s"
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="long")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--block-size", type=int, default=0)
    ap.add_argument("--path", default="auto", choices=["auto", "simt", "tc"])
    ap.add_argument("--split", type=int, default=0)
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--pool-blocks", type=int, default=0,
                    help="mha only: pool size in blocks (0 = the workload's 16384)")
    ap.add_argument("--num-seqs", type=int, default=0,
                    help="mha / gqa / long: fewer sequences, for profiling a smaller case")
    ap.add_argument("--no-share-prefixes", action="store_true",
                    help="prefix_cow: read the shared prefix per sequence (pa_decode's "
                         "share_prefixes off)")
    return ap.parse_args()


# pa_decode reads shared prefixes once per group of sequences on workloads
# built with one (prefix_cow), unless --no-share-prefixes
SHARE_PREFIXES = [True]


def share_for(b):
    return bool(SHARE_PREFIXES[0] and "prefix_blocks" in b.meta)


# ---------------------------------------------------------------------------
# distributed plumbing (control path only)
# ---------------------------------------------------------------------------

def dist_setup(n):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """Max of a per-rank time over all ranks (control path only)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int) -> float:
    """Sum of a per-rank count over all ranks (control path only)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def weak_scaling_value(units_all_ranks: float, ms_max: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest
    rank's time."""
    return units_all_ranks / (ms_max * 1e-3)


# ---------------------------------------------------------------------------
# workload
# ---------------------------------------------------------------------------

def make_batch(name, device, rank, block_size, pool_blocks=0, num_seqs=0):
    from paged_kv_cache_339_b200 import workloads as W
    fn = W.FULL[name]
    seed = {"tiny": 1001, "mha": 1002, "gqa": 1003, "prefix_cow": 1004, "long": 1005}[name]
    kw = {"seed": seed + 100 * rank}
    if block_size and name in ("mha", "gqa", "long"):
        kw["block_size"] = block_size
    if pool_blocks and name == "mha":
        kw["num_blocks"] = pool_blocks
    if num_seqs and name in ("mha", "gqa", "long"):
        kw["num_seqs"] = num_seqs
    return fn(device, **kw)


def config_of(b, name, l2_note):
    G = b.num_q_heads // b.num_kv_heads
    lens = b.context_lens.cpu()
    return {
        "workload": b.name, "num_seqs": b.num_seqs, "num_q_heads": b.num_q_heads,
        "num_kv_heads": b.num_kv_heads, "group": G, "head_dim": b.head_dim,
        "block_size": b.block_size, "num_blocks": b.num_blocks,
        "context_len_mean": round(float(lens.float().mean()), 1),
        "context_len_max": int(lens.max()), "cow_pairs": int(b.cow_pairs.shape[0]),
        "kv_bytes_per_step": b.kv_bytes_logical(), "l2": l2_note,
        "share_prefixes": share_for(b),
    }


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    """SM clock and clock-event reasons sampled every ~0.5 ms by a background
    thread through NVML (read-only queries; nothing on the GPU is changed),
    or through `nvidia-smi -lms 100` where NVML is not available. summary()
    keeps the samples taken inside the timed window when there are any."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
            "hw_thermal_slowdown": 0x40}

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.samples = []          # (wall time, sm MHz, reason names)
        self.sm_max = None
        self.window = None
        self.proc = None
        self.out = None
        self._stop = None
        self._thread = None

    def _nvml_loop(self, nv, h):
        while not self._stop.is_set():
            try:
                mhz = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                    nv.nvmlDeviceGetCurrentClocksThrottleReasons
                bits = int(fn(h))
            except Exception:  # noqa: BLE001 - sampling is best effort
                break
            names = [n for n, b in self.BITS.items() if bits & b]
            self.samples.append((time.perf_counter(), mhz, names))
            time.sleep(0.0005)

    def __enter__(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = nv.nvmlDeviceGetHandleByIndex(self.idx)
            self.sm_max = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            self._stop = threading.Event()
            self._thread = threading.Thread(target=self._nvml_loop, args=(nv, h), daemon=True)
            self._thread.start()
        except Exception:  # noqa: BLE001 - fall back to nvidia-smi
            self._thread = None
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}",
                     "--format=csv,noheader,nounits", "-lms", "100"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except OSError:
                self.proc = None
            time.sleep(0.15)
        return self

    def mark(self, t0, t1):
        """Wall-clock bounds of the timed region."""
        self.window = (t0, t1)

    def __exit__(self, *a):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out = ""

    def summary(self):
        if self.samples:
            inside = [x for x in self.samples
                      if self.window and self.window[0] <= x[0] <= self.window[1]]
            use = inside or self.samples
            reasons = sorted({n for _, _, ns in use for n in ns})
            return {"sm_mhz": statistics.median(x[1] for x in use), "sm_max_mhz": self.sm_max,
                    "reasons": reasons, "samples": len(use),
                    "samples_in_timed_region": len(inside), "source": "nvml"}
        if not self.out:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm), "source": "nvidia-smi"}


# ---------------------------------------------------------------------------
# our implementation
# ---------------------------------------------------------------------------

def step_fn(b, ops, out, ws, split, path, stream):
    max_ctx = b.max_context_len
    share = share_for(b)

    def step():
        n = 0
        if b.cow_pairs.numel():
            ops.pa_copy_blocks(b.k_cache, b.v_cache, b.cow_pairs, stream=stream)
            n += 1
        ops.pa_write_kv(b.k_cache, b.v_cache, b.key, b.value, b.slot_mapping, stream=stream)
        ops.pa_decode(out, b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, max_ctx,
                      b.scale, ws, split_tokens=split, path=path, stream=stream,
                      share_prefixes=share)
        return n + 1 + 2 + (1 if share else 0)   # write, plan, (groups,) decode
    return step


def time_device(step, K, W, stream, use_graph, world, clock=None):
    """Device time of K steps (CUDA events on the launching stream)."""
    torch.cuda.synchronize()   # inputs drawn on the default stream are complete
    launches = 0
    with torch.cuda.stream(stream):
        for _ in range(W):
            launches = step()
        torch.cuda.synchronize()
        graph = None
        if use_graph:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=stream):
                step()
            for _ in range(2):
                graph.replay()
            torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        w0 = time.perf_counter()
        e0.record(stream)
        for _ in range(K):
            if graph is not None:
                graph.replay()
            else:
                step()
        e1.record(stream)
        torch.cuda.synchronize()
        w1 = time.perf_counter()
        barrier(world)
    ms = e0.elapsed_time(e1)
    del graph
    if clock is not None:
        clock.mark(w0, w1)
    return ms / K, launches


def device_facts():
    """Name, SM count and L2 size of the GPU the bench ran on."""
    p = torch.cuda.get_device_properties(torch.cuda.current_device())
    return {"name": p.name, "sm_count": p.multi_processor_count,
            "l2_bytes": getattr(p, "L2_cache_size", None),
            "hbm_bytes": p.total_memory}


def l2_flusher():
    """Evicts the L2 by reading a buffer of twice its size (a read leaves no
    dirty lines to write back during the next step)."""
    l2 = getattr(torch.cuda.get_device_properties(torch.cuda.current_device()),
                 "L2_cache_size", 126 << 20) or (126 << 20)
    buf = torch.ones((2 * l2) // 4, dtype=torch.float32, device="cuda")
    sink = torch.empty((), dtype=torch.float32, device="cuda")
    return lambda: torch.sum(buf, 0, out=sink)


def step_times(step, K, stream, use_graph, flush=None):
    """Device time of each of K steps, from a pair of CUDA events around every
    step on the launching stream; `flush`, when given, runs between steps
    outside the events. The step is idempotent (same write, same copies), so
    every repetition does the same work."""
    torch.cuda.synchronize()   # inputs drawn on the default stream are complete
    with torch.cuda.stream(stream):
        graph = None
        if use_graph:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=stream):
                step()
            graph.replay()
        else:
            step()
        torch.cuda.synchronize()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(K)]
        for e_a, e_z in ev:
            if flush is not None:
                flush()
            e_a.record(stream)
            if graph is not None:
                graph.replay()
            else:
                step()
            e_z.record(stream)
        torch.cuda.synchronize()
    del graph
    return [e_a.elapsed_time(e_z) for e_a, e_z in ev]


def percentiles(ms_list, world):
    """p10 / p50 / p90 of per-step times, each the max over ranks."""
    q = np.percentile(np.asarray(ms_list, dtype=np.float64), [10, 50, 90])
    return {k: round(max_over_ranks(float(v), world), 5) for k, v in zip(("p10", "p50", "p90"), q)}


def time_decode_only(b, ops, out, ws, split, path, stream, K, use_graph=True, share=None):
    """Average duration of the decode call alone (plan + main kernels):
    K calls back to back between two events on the launching stream, replayed
    from a CUDA graph like the step, so the device never waits for the host."""
    max_ctx = b.max_context_len
    share = share_for(b) if share is None else share

    def call():
        ops.pa_decode(out, b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens,
                      max_ctx, b.scale, ws, split_tokens=split, path=path, stream=stream,
                      share_prefixes=share)

    torch.cuda.synchronize()   # inputs drawn on the default stream are complete
    with torch.cuda.stream(stream):
        for _ in range(3):
            call()
        torch.cuda.synchronize()
        graph = None
        if use_graph:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=stream):
                call()
            graph.replay()
            torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(K):
            if graph is not None:
                graph.replay()
            else:
                call()
        e1.record(stream)
        torch.cuda.synchronize()
    del graph
    return e0.elapsed_time(e1) / K


STEP_INPUTS = ("q", "key", "value", "slot_mapping", "block_tables", "context_lens", "cow_pairs")


def pack_step_inputs(b):
    """One step's inputs as one host byte buffer, every tensor at a 256-byte
    aligned offset (so one copy moves them all); returns (buffer, offsets)."""
    offs, n = {}, 0
    for k in STEP_INPUTS:
        t = getattr(b, k)
        offs[k] = n
        n += (t.numel() * t.element_size() + 255) // 256 * 256
    host = torch.zeros(max(n, 256), dtype=torch.uint8)
    for k in STEP_INPUTS:
        t = getattr(b, k)
        nb = t.numel() * t.element_size()
        if nb:
            host[offs[k]:offs[k] + nb] = t.contiguous().view(-1).cpu().view(torch.uint8)
    return host, offs


def step_input_views(buf, b, offs):
    """Typed views of a packed buffer (host or device), shaped like b's inputs."""
    out = {}
    for k in STEP_INPUTS:
        t = getattr(b, k)
        nb = t.numel() * t.element_size()
        out[k] = buf[offs[k]:offs[k] + nb].view(t.dtype).view(t.shape)
    return out


def time_e2e(b, ops, ws, split, path, stream, K, W):
    """Same metric through the public API from pinned host memory: every step
    copies its inputs host->device and reads its result back, all inside the
    timed region. The inputs travel as one packed buffer (every tensor at a
    256-byte aligned offset), one copy per step. Two device buffer sets and
    separate upload and download streams pipeline it the way a serving loop
    would: step i+1's inputs go up while step i computes, and step i's result
    comes back while step i+1 computes, both directions of the host link at
    once."""
    host, offs = pack_step_inputs(b)
    host = host.pin_memory()
    raw = [torch.empty_like(host, device="cuda") for _ in range(2)]
    dev = [step_input_views(r, b, offs) for r in raw]
    out = [torch.empty(b.q.shape, dtype=torch.float32, device="cuda") for _ in range(2)]
    out_h = [torch.empty(b.q.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    h2d = host.numel()
    d2h = out_h[0].numel() * 4
    max_ctx = b.max_context_len
    cu, cd = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    up = [ev(), ev()]      # inputs of a slot are on the device
    done = [ev(), ev()]    # the step that used a slot has finished
    back = [ev(), ev()]    # the result of a slot has been read back

    def upload(i):
        sl = i & 1
        with torch.cuda.stream(cu):
            cu.wait_event(done[sl])          # the step two back has released the inputs
            raw[sl].copy_(host, non_blocking=True)
            up[sl].record(cu)

    def compute(i):
        sl, d = i & 1, dev[i & 1]
        with torch.cuda.stream(stream):
            stream.wait_event(up[sl])
            stream.wait_event(back[sl])      # the step two back's result is out
            if d["cow_pairs"].numel():
                ops.pa_copy_blocks(b.k_cache, b.v_cache, d["cow_pairs"], stream=stream)
            ops.pa_write_kv(b.k_cache, b.v_cache, d["key"], d["value"], d["slot_mapping"],
                            stream=stream)
            ops.pa_decode(out[sl], d["q"], b.k_cache, b.v_cache, d["block_tables"],
                          d["context_lens"], max_ctx, b.scale, ws, split_tokens=split,
                          path=path, stream=stream, share_prefixes=share_for(b))
            done[sl].record(stream)

    def download(i):
        sl = i & 1
        with torch.cuda.stream(cd):
            cd.wait_event(done[sl])
            out_h[sl].copy_(out[sl], non_blocking=True)
            back[sl].record(cd)

    def run(n):
        upload(0)
        for i in range(n):
            compute(i)
            if i + 1 < n:
                upload(i + 1)
            download(i)

    torch.cuda.synchronize()   # inputs drawn on the default stream are complete
    for e in done + back:
        e.record(stream)
    run(W)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    cu.wait_event(e0)
    cd.wait_event(e0)
    run(K)
    stream.wait_stream(cu)
    stream.wait_stream(cd)
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / K, h2d, d2h


def time_graph(fn, stream, K):
    """Average device time of fn (captured once in a CUDA graph), K replays
    back to back between two events."""
    torch.cuda.synchronize()   # inputs drawn on the default stream are complete
    with torch.cuda.stream(stream):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn()
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(K):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
    del g
    return e0.elapsed_time(e1) / K


def next_rows(ops, stream, rank):
    """Measurements beyond the decode step: the paged-vs-contiguous cost of the
    block table at block sizes 8, 16 and 32 (same kernel, same lengths, blocks
    adjacent instead of shuffled), a prefill-sized KV write, and block
    swap-out / swap-in between the device pools and pinned host memory."""
    from paged_kv_cache_339_b200 import workloads as W
    res = {}
    for name, mk in (("mha", W.mha), ("gqa", W.gqa)):
        per_bs = {}
        for bs in (8, 16, 32):
            row = {}
            for placement in ("shuffled", "contiguous"):
                b = mk("cuda", seed={"mha": 1002, "gqa": 1003}[name] + 100 * rank,
                       block_size=bs, contiguous=placement == "contiguous")
                B, Hq, D = b.q.shape
                ws = ops.decode_workspace(B, Hq, D, b.max_context_len, b.block_size, 0)
                out = torch.empty((B, Hq, D), dtype=torch.float32, device="cuda")
                ms = time_decode_only(b, ops, out, ws, 0, ops.PA_PATH_AUTO, stream, 20)
                row[placement + "_decode_gbps"] = round(
                    b.kv_bytes_logical() / (ms * 1e-3) / 1e9, 1)
                del b, ws, out
                torch.cuda.empty_cache()
            row["table_cost_pct"] = round(
                100.0 * (1.0 - row["shuffled_decode_gbps"] / row["contiguous_decode_gbps"]), 2)
            per_bs[f"bs{bs}"] = row
        res["paged_vs_contiguous_" + name] = per_bs
    # prefill-sized write: T tokens of the MHA shape. "prompt": 16 prompts of
    # 1024 tokens, each filling its blocks in order (consecutive slots inside
    # a block), blocks taken from a shuffled pool, as the block manager hands
    # them out; "scattered": every token to a random slot of the pool.
    T, H, D, BS, NB = 16384, 32, 128, 16, 2048
    kc = torch.zeros((NB, H, BS, D), dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    key = torch.randn((T, H, D), device="cuda").to(torch.bfloat16)
    val = torch.randn((T, H, D), device="cuda").to(torch.bfloat16)
    g = torch.Generator().manual_seed(1339 + 100 * rank)
    blocks = torch.randperm(NB, generator=g)[:T // BS]
    prompt_slots = (blocks[:, None] * BS + torch.arange(BS)[None, :]).reshape(-1)
    scattered = torch.randperm(NB * BS, generator=g)[:T]
    nbytes = 2 * T * H * D * 2
    peak, _ = measured_peak()
    pw = {"tokens": T, "bytes_written": nbytes}
    for label, sl in (("prompt", prompt_slots), ("scattered", scattered)):
        slots = sl.to(torch.int64).cuda()
        ms = time_graph(lambda: ops.pa_write_kv(kc, vc, key, val, slots, stream=stream),
                        stream, 20)
        pw[label] = {"gbps_written": round(nbytes / (ms * 1e-3) / 1e9, 1),
                     "gbps_read_plus_written": round(2 * nbytes / (ms * 1e-3) / 1e9, 1),
                     "frac_of_measured_peak": round(2 * nbytes / (ms * 1e-3) / 1e9 / peak, 4),
                     "ms": round(ms, 4)}
    res["prefill_write"] = pw
    # swap: P blocks of that pool out to pinned host memory and back
    P = 1024
    hk = torch.empty((P, H, BS, D), dtype=torch.bfloat16, pin_memory=True)
    hv = torch.empty_like(hk, pin_memory=True)
    src = torch.randperm(NB, device="cuda")[:P].to(torch.int64)
    pairs_out = torch.stack([src, torch.arange(P, device="cuda")], 1).contiguous()
    pairs_in = torch.stack([torch.arange(P, device="cuda"), src], 1).contiguous()
    blk = 2 * H * BS * D * 2
    sw = {}
    for label, pairs, d in (("out", pairs_out, ops.PA_SWAP_OUT), ("in", pairs_in, ops.PA_SWAP_IN)):
        with torch.cuda.stream(stream):
            ops.pa_swap_blocks(kc, vc, hk, hv, pairs, d, stream=stream)
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(5):
                ops.pa_swap_blocks(kc, vc, hk, hv, pairs, d, stream=stream)
            e1.record(stream)
            torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / 5
        sw[label + "_gbps"] = round(P * blk / (ms * 1e-3) / 1e9, 1)
    res["swap"] = dict(blocks=P, bytes=P * blk, **sw)
    del kc, vc, key, val, hk, hv
    torch.cuda.empty_cache()
    return res


def uses_tensor_cores(b, path):
    """The decode kernel pa_decode picks for this batch (mirrors its dispatch:
    16-bit KV, head_dim 128, 4..16 query heads per KV head, >= 16 query rows)."""
    G = b.num_q_heads // b.num_kv_heads
    fits = (b.dtype != torch.float32 and b.head_dim == 128 and 4 <= G <= 16
            and b.num_seqs * b.num_q_heads >= 16)
    return path == "tc" or (path == "auto" and fits)


def kernel_source_hash(tensor_cores, groups=False):
    """Hash of the sources of the decode kernels that run (the traffic figure
    is only reported while it was measured on these exact sources); groups:
    the shared-prefix launch (tensor-core kernel) runs too."""
    h = hashlib.sha256()
    csrc = ROOT / "paged_kv_cache_339_b200" / "csrc"
    main = ["pa_decode_tc.cu" if tensor_cores else "pa_decode_simt.cu"]
    if groups and not tensor_cores:
        main.append("pa_decode_tc.cu")
    for name in ["pa_common.cuh"] + main + ["pa_plan_reduce.cu"]:
        h.update((csrc / name).read_bytes())
    return h.hexdigest()[:16]


def traffic_from_profile(workload, kernel_hash):
    """DRAM bytes per launch of the decode kernel from the committed ncu
    summary, if it was taken on the current kernel sources."""
    f = ROOT / "profiles" / "decode_traffic.json"
    if not f.exists():
        return None
    try:
        d = json.loads(f.read_text())
        e = d.get(workload)
        if e and e.get("kernel_source_hash") == kernel_hash:
            return e.get("dram_bytes_per_launch")
    except (ValueError, OSError):
        pass
    return None


def measured_peak():
    f = ROOT / "MEASURED_PEAKS.json"
    try:
        d = json.loads(f.read_text())
        return float(d["hbm_gbs"]), "measured"
    except (OSError, ValueError, KeyError):
        return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------------------
# CPU oracle baseline (bounded sample)
# ---------------------------------------------------------------------------

def oracle_sample(b, seconds, out=None, cache=None):
    """Run the fp64 oracle on (sequence, query head) rows of the batch, in
    order, until about `seconds` of CPU work. Each (sequence, KV head) is
    first copied back and widened to fp64 (not timed; `cache` keeps those
    copies across calls). A row is credited with its share of the KV bytes,
    2 * L * D * e / G, so a whole batch adds up to kv_bytes_logical().
    Returns (KV bytes covered, seconds, rows, sequences touched, threads,
    max-abs error of `out` on those rows or None)."""
    from oracle import ORACLE
    from threadpoolctl import threadpool_info
    BS, D, e = b.block_size, b.head_dim, b.elem_bytes
    G = b.num_q_heads // b.num_kv_heads
    scale = float(np.float32(b.scale))   # the fp32 value the kernels receive
    cache = {} if cache is None else cache
    done_bytes, spent, rows, seqs = 0.0, 0.0, 0, 0
    err = 0.0 if out is not None else None
    stop = False
    for i in range(b.num_seqs):
        L = int(b.context_lens[i])
        nb = (L + BS - 1) // BS
        seqs += 1
        for kv in range(b.num_kv_heads):
            key = (i, kv)
            if key not in cache:
                blk = b.block_tables[i, :nb].long()
                ks = b.k_cache[blk][:, kv:kv + 1].to(torch.float32).cpu().numpy()
                vs = b.v_cache[blk][:, kv:kv + 1].to(torch.float32).cpu().numpy()
                cache[key] = (ORACLE.logical_pool(ks.astype(np.float64)),
                              ORACLE.logical_pool(vs.astype(np.float64)))
            ksub, vsub = cache[key]
            for h in range(kv * G, (kv + 1) * G):
                q = b.q[i, h].to(torch.float32).cpu().numpy().astype(np.float64)
                t0 = time.perf_counter()
                ref = ORACLE.decode_one(q, ksub, vsub, np.arange(nb), L, 0, 1, scale)
                spent += time.perf_counter() - t0
                if out is not None:
                    got = out[i, h].cpu().numpy().astype(np.float64)
                    err = max(err, float(np.max(np.abs(got - ref))))
                done_bytes += 2.0 * L * D * e / G
                rows += 1
                if spent >= seconds:
                    stop = True
                    break
            if stop:
                break
        if stop:
            break
    threads = max([d.get("num_threads", 1) for d in threadpool_info()] + [1])
    return done_bytes, spent, rows, seqs, threads, err


# ---------------------------------------------------------------------------

DTYPE_NAME = {torch.bfloat16: "bf16", torch.float16: "f16", torch.float32: "f32"}
# the other configurations measured, with every key of the headline, in a
# default single-GPU run
OTHER_WORKLOADS = ("long", "gqa", "mha", "prefix_cow")


def measure(name, args, ops, rank, world, local, stream, path, split, steps, cpu_seconds,
            block_size=0, pool_blocks=0, num_seqs=0):
    """One configuration, every figure of the line: the step (copy-on-write
    copies, KV write, decode) timed over `steps` graph replays, the decode
    call alone (roofline), the end-to-end pipeline through pinned host
    memory, per-step percentiles with and without an L2 flush, the clocks
    during the timed region, and, at N = 1 on rank 0, the oracle on a
    bounded sample of the same batch (cpu_baseline and parity)."""
    b = make_batch(name, "cuda", rank, block_size, pool_blocks, num_seqs)
    kv_bytes = b.kv_bytes_logical()
    B, Hq, D = b.q.shape
    ws = ops.decode_workspace(B, Hq, D, b.max_context_len, b.block_size, split)
    out = torch.empty((B, Hq, D), dtype=torch.float32, device="cuda")
    step = step_fn(b, ops, out, ws, split, path, stream)
    W = max(args.warmup, 3)
    use_graph = not args.no_graph

    with ClockSampler(local) as clk:
        ms, per_step = time_device(step, steps, W, stream, use_graph, world, clk)
    ms = max_over_ranks(ms, world)
    torch.cuda.synchronize()
    status = ops.pa_decode_status(ws, stream)
    dec_ms = time_decode_only(b, ops, out, ws, split, path, stream, max(10, steps), use_graph)
    e2e_ms, h2d, d2h = time_e2e(b, ops, ws, split, path, stream, max(5, steps // 2), 3)
    e2e_ms = max_over_ranks(e2e_ms, world)
    hot = percentiles(step_times(step, steps, stream, use_graph), world)
    flushed = percentiles(step_times(step, steps, stream, use_graph, l2_flusher()), world)
    torch.cuda.empty_cache()

    peak, peak_kind = measured_peak()
    kv_bytes_all = sum_over_ranks(kv_bytes, world)
    seqs_all = sum_over_ranks(B, world)
    gbps = weak_scaling_value(kv_bytes_all, ms) / 1e9
    dec_gbps = kv_bytes / (dec_ms * 1e-3) / 1e9
    tc = uses_tensor_cores(b, {ops.PA_PATH_AUTO: "auto", ops.PA_PATH_SIMT: "simt",
                               ops.PA_PATH_TCGEN05: "tc"}[path])
    khash = kernel_source_hash(tc, share_for(b))
    l2_note = (f"inputs larger than L2: {kv_bytes / 1e9:.2f} GB of KV read per step, not "
               "flushed; l2_flushed has per-step times with the L2 evicted before every step")
    if b.cow_pairs.numel():
        l2_note = (f"{kv_bytes / 1e9:.2f} GB of KV read per step (logical), "
                   f"{b.kv_bytes_unique() / 1e9:.2f} GB of distinct slots: the shared prefix "
                   "stays in L2 between siblings; not flushed, l2_flushed has per-step times "
                   "with the L2 evicted before every step")
    res = {
        "metric": METRIC, "value": round(gbps, 1), "unit": "GB/s",
        "ms_per_step": round(ms, 5),
        "dtype": DTYPE_NAME[b.dtype],
        "config": config_of(b, name, l2_note),
        "seq_steps_per_s": round(weak_scaling_value(seqs_all, ms), 1),
        "pct_of_peak": round(100.0 * gbps / world / peak, 2),
        "pct_of_nominal_8tbs": round(100.0 * gbps / world / 8000.0, 2),
        "decode_status": int(status),
        "gpu_launches": per_step * steps,
        "roofline": {
            "bound": "hbm", "kernel": "pa_decode (plan + decode main, merge fused)",
            "decode_kernel": ("tc_decode_kernel (tcgen05)" if tc else "simt_decode_kernel") +
                             (" after the shared-prefix groups' tc_decode_kernel"
                              if share_for(b) else ""),
            "achieved": round(dec_gbps, 1), "peak": peak, "unit": "GB/s",
            "frac": round(dec_gbps / peak, 4), "peak_source": f"{peak_kind} hbm_gbs",
            "algorithmic_bytes_per_launch": kv_bytes,
            "launch_ms": round(dec_ms, 5),
            "traffic": traffic_from_profile(b.name, khash),
            "kernel_source_hash": khash,
        },
        "e2e": {"value": round(weak_scaling_value(kv_bytes_all, e2e_ms) / 1e9, 1), "unit": "GB/s",
                "ms_per_step": round(e2e_ms, 5), "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h)},
        "clocks": clk.summary(),
        "step_ms": dict(mean=round(ms, 5), **hot),
        "l2_flushed": dict(
            note="L2 evicted (a read of 2x its size) before every step, outside the events",
            gbps_at_p50=round(weak_scaling_value(kv_bytes_all, flushed["p50"]) / 1e9, 1),
            **flushed),
    }
    if share_for(b):
        # the same decode call with every sequence reading the prefix itself
        off_ms = time_decode_only(b, ops, out, ws, split, path, stream, max(10, steps),
                                  use_graph, share=False)
        res["prefix_sharing"] = {
            "note": "pa_decode share_prefixes: the common prefix is read once per group of "
                    "up to 16 sequences; decode_gbps_without is the same call with it off",
            "decode_gbps": round(dec_gbps, 1),
            "decode_gbps_without": round(kv_bytes / (off_ms * 1e-3) / 1e9, 1),
            "speedup": round(off_ms / dec_ms, 3),
        }
    if b.cow_pairs.numel():
        # the shared prefix is read by every sibling but crosses HBM once per step
        ub = b.kv_bytes_unique()
        ub_all = sum_over_ranks(ub, world)
        res["unique_bytes"] = {
            "kv_bytes_unique_per_step": ub,
            "gbps_unique": round(weak_scaling_value(ub_all, ms) / 1e9, 1),
            "pct_of_peak_unique": round(100.0 * ub_all / world / (ms * 1e-3) / 1e9 / peak, 2),
            "gbps_unique_l2_flushed": round(weak_scaling_value(ub_all, flushed["p50"]) / 1e9, 1),
            "pct_of_peak_unique_l2_flushed": round(
                100.0 * ub_all / world / (flushed["p50"] * 1e-3) / 1e9 / peak, 2),
        }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # one untimed step on the batch as it is now, so `out` and the oracle
        # see one cache; the pool was drawn on the default stream
        torch.cuda.synchronize()
        step()
        torch.cuda.synchronize()
        nbytes, secs, rows, nseq, threads, err = oracle_sample(b, cpu_seconds, out)
        res["cpu_baseline"] = {
            "value": round(nbytes / secs / 1e9, 4), "unit": "GB/s", "cores": threads,
            "kind": "oracle",
            "sample": f"fp64 NumPy oracle, decode of the first {rows} of "
                      f"{b.num_seqs * b.num_q_heads} (sequence, query head) rows, in order "
                      f"(first {nseq} sequences), {secs:.1f} s",
        }
        tol = 1e-5 if b.dtype == torch.float32 else 2e-3
        res["parity"] = {"max_abs_err": err, "tol": tol, "ok": err <= tol, "rows": rows,
                         "against": "the fp64 oracle, on the cpu_baseline sample's rows"}
    del b, ws, out
    torch.cuda.empty_cache()
    return res


def long_block_size_sweep(ops, stream, rank, steps, use_graph):
    """The long-context workload at block sizes 8, 16 and 32 (same lengths,
    shuffled pool): the step and the decode call alone."""
    from paged_kv_cache_339_b200 import workloads as W
    peak, _ = measured_peak()
    res = {}
    for bs in (8, 16, 32):
        b = W.long_context("cuda", seed=1005 + 100 * rank, block_size=bs)
        B, Hq, D = b.q.shape
        ws = ops.decode_workspace(B, Hq, D, b.max_context_len, b.block_size, 0)
        out = torch.empty((B, Hq, D), dtype=torch.float32, device="cuda")
        st = step_fn(b, ops, out, ws, 0, ops.PA_PATH_AUTO, stream)
        ms, _ = time_device(st, steps, 3, stream, use_graph, 1)
        d = time_decode_only(b, ops, out, ws, 0, ops.PA_PATH_AUTO, stream, steps, use_graph)
        kb = b.kv_bytes_logical()
        res[f"bs{bs}"] = {"step_gbps": round(kb / (ms * 1e-3) / 1e9, 1),
                          "decode_gbps": round(kb / (d * 1e-3) / 1e9, 1),
                          "frac_of_measured_peak": round(kb / (d * 1e-3) / 1e9 / peak, 4),
                          "pct_of_nominal_8tbs": round(100.0 * kb / (d * 1e-3) / 1e9 / 8000.0, 2),
                          "status": ops.pa_decode_status(ws, stream)}
        del b, ws, out, st
        torch.cuda.empty_cache()
    return res


def long_few_sequences(ops, stream, rank, steps, use_graph):
    """The long-context workload with 1, 2, 4 and 8 sequences (block size 32,
    lengths 32K-128K): the decode call alone. Few (sequence, KV head) units
    leave the split plan to spread each sequence over the streams."""
    from paged_kv_cache_339_b200 import workloads as W
    peak, _ = measured_peak()
    res = {}
    for n in (1, 2, 4, 8):
        b = W.long_context("cuda", seed=1005 + 100 * rank, num_seqs=n)
        B, Hq, D = b.q.shape
        ws = ops.decode_workspace(B, Hq, D, b.max_context_len, b.block_size, 0)
        out = torch.empty((B, Hq, D), dtype=torch.float32, device="cuda")
        d = time_decode_only(b, ops, out, ws, 0, ops.PA_PATH_AUTO, stream, steps, use_graph)
        kb = b.kv_bytes_logical()
        res[f"seqs{n}"] = {"kv_bytes": kb,
                           "decode_gbps": round(kb / (d * 1e-3) / 1e9, 1),
                           "frac_of_measured_peak": round(kb / (d * 1e-3) / 1e9 / peak, 4),
                           "status": ops.pa_decode_status(ws, stream)}
        del b, ws, out
        torch.cuda.empty_cache()
    return res


def allocator_waste():
    """Reserved-but-unused fraction of the KV cache under max-length
    contiguous reservation and under paging at block sizes 8 / 16 / 32, over
    one seeded trace of request arrivals and completions (host-side
    bookkeeping only)."""
    from paged_kv_cache_339_b200.block_manager import lifetime_trace, simulate_lifetimes
    trace = lifetime_trace(2000, 4096, seed=1339)
    res = {"trace": "2000 requests, Poisson arrivals 0.5/step, log-normal prompts (mean 256) "
                    "and completions (mean 512), max context 4096, 64 live at most"}
    for bs in (8, 16, 32):
        r = simulate_lifetimes(trace, 4096, bs, max_live=64)
        res[f"bs{bs}"] = {k: (round(v, 5) if isinstance(v, float) else v) for k, v in r.items()
                          if k not in ("requests", "max_context", "max_live", "block_size")}
    return res


def run_ours(args, rank, world, local):
    from paged_kv_cache_339_b200 import build as pa_build
    pa_build.build()
    from paged_kv_cache_339_b200 import ops
    path = {"auto": ops.PA_PATH_AUTO, "simt": ops.PA_PATH_SIMT, "tc": ops.PA_PATH_TCGEN05}[args.path]
    stream = torch.cuda.Stream()
    head = measure(args.workload, args, ops, rank, world, local, stream, path, args.split,
                   args.steps, args.cpu_seconds, args.block_size, args.pool_blocks,
                   args.num_seqs)
    res = {
        "metric": METRIC, "value": head["value"], "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": head["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": head["dtype"],
        "data": "synthetic (seeded N(0,1) K/V/Q, shuffled block placement)",
        "config": head["config"],
    }
    for k, v in head.items():
        res.setdefault(k, v)
    res["device"] = device_facts()
    res["graph"] = not args.no_graph
    if not args.no_secondary and world == 1:
        # the other configurations, each with the headline's keys
        res["configs"] = {}
        for name in OTHER_WORKLOADS:
            if name == args.workload:
                continue
            r = measure(name, args, ops, rank, world, local, stream, ops.PA_PATH_AUTO, 0,
                        max(10, args.steps // 2), args.cpu_seconds / 4)
            res["configs"][r["config"]["workload"]] = r
        res["next"] = next_rows(ops, stream, rank)
        res["next"]["long_block_size_sweep"] = long_block_size_sweep(
            ops, stream, rank, max(10, args.steps // 2), not args.no_graph)
        res["next"]["long_few_sequences"] = long_few_sequences(
            ops, stream, rank, max(10, args.steps // 2), not args.no_graph)
        res["next"]["allocator_waste"] = allocator_waste()
    return res


def run_reference(args, rank, world):
    """The oracle as the reference arm: same workload, bounded sample per step."""
    if rank != 0:
        return None
    b = make_batch(args.workload, "cuda" if torch.cuda.is_available() else "cpu", 0,
                   args.block_size)
    per = max(args.cpu_seconds / max(args.steps, 1), 0.5)
    cache = {}
    for _ in range(min(args.warmup, 1)):
        oracle_sample(b, 0.1, cache=cache)
    tot_b, tot_s, rows, seqs, threads = 0.0, 0.0, 0, 0, 1
    for _ in range(args.steps):
        nb, sec, rows, seqs, threads, _ = oracle_sample(b, per, cache=cache)
        tot_b += nb
        tot_s += sec
    v = tot_b / tot_s / 1e9
    return {
        "metric": METRIC, "value": round(v, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * tot_s / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": config_of(b, args.workload, "host memory"),
        "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": threads,
                         "kind": "oracle",
                         "sample": f"each step: decode of the first {rows} (sequence, query "
                                   f"head) rows (first {seqs} sequences), the fp64 copies of "
                                   "their KV prepared once before timing"},
        "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    args = parse()
    SHARE_PREFIXES[0] = not args.no_share_prefixes
    rank, world, local = dist_setup(args.gpus)
    try:
        if args.impl == "reference":
            res = run_reference(args, rank, world)
        else:
            res = run_ours(args, rank, world, local)
        if rank == 0 and res is not None:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
