"""Benchmark of the paged KV-cache decode path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--block-size BS]
    python bench.py --impl reference ...      # the CPU oracle, timed on the host cores

One step = one decode step of the workload through the whole hot path: for every
layer, the cache write of this step's tokens (reshape_and_cache), paged decode
attention (partition kernel, plus the log-sum-exp reduce when a context spans
several partitions) and, for workloads with shared blocks, the copy-on-write block
copy before the write. The host block manager runs in the end-to-end loop.

Metric: paged decode attention KV-read GB/s = algorithmic K+V bytes the step reads
(sum over layers and sequences of len * Hkv * head_dim * 2 * 2 bytes) / step time;
also decode tokens/s = sequences / step time. Multi-GPU (torchrun): every rank runs
its own replica of the workload (weak scaling, no collective on the data path);
the step time is the maximum over ranks.
"""
from __future__ import annotations

import argparse
import contextlib
import gc
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_kv_cache_320_b200 import synth  # noqa: E402

WORKLOADS = {
    "llama7b_mha": "Llama-7B-shaped MHA decode: B 64, 32/32 heads, d 128, fp16, bs 16, "
                   "lognormal(median 512, sigma 1) clip 16-2048, 32 layers",
    "llama3_8b_gqa": "Llama-3-8B-shaped GQA decode: B 256, 32q/8kv, d 128, bf16, bs 16, "
                     "lognormal(median 1024, sigma 1) clip 8-8192, 1 layer, 256 new tokens",
    "shared_prefix": "shared-prefix parallel sampling: 16 prompts x 8 samples, prefix 1024 "
                     "(refcount 8), suffix U[0,256], 32q/8kv, d 128, bf16, bs 16, 1 layer",
    "long_context": "long-context decode: B 8, U[32768,131072], 64q/8kv, d 128, bf16, 1 layer",
    "shared_prefix_cow": "shared-prefix copy-on-write step: 16 parent prompts of 1024 + u tokens "
                         "(u in [1,255], not a multiple of 16) each forked into 8 samples that "
                         "append one token (128 block copies), then cache write and decode; "
                         "32q/8kv, d 128, bf16, bs 16, 1 layer",
}
METRIC = "paged decode attention KV-read GB/s (% of B200 HBM peak); decode tokens/s"
KERNEL_SOURCES = ["paged_kv_cache_320_b200/csrc/decode_kernels.cuh",
                  "paged_kv_cache_320_b200/csrc/pkv_ptx.cuh"]
STEP_SOURCES = KERNEL_SOURCES + ["paged_kv_cache_320_b200/csrc/step_kernels.cuh"]


def describe(args) -> str:
    """The named workload's description, with any size overridden on the command line."""
    over = [f"{k} {v}" for k, v in (("block_size", getattr(args, "block_size", 0)),
                                    ("layers", getattr(args, "layers", 0)),
                                    ("batch", getattr(args, "batch", 0))) if v]
    text = WORKLOADS[args.workload]
    return text + (f" (run with {', '.join(over)})" if over else "")


def kernel_source_hash(sources=None) -> str:
    h = hashlib.sha256()
    for p in sources or KERNEL_SOURCES:
        h.update(open(os.path.join(ROOT, p), "rb").read())
    return h.hexdigest()[:16]


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def read_traffic(workload, block_size, kernel="paged_decode_partition"):
    """DRAM bytes (read + write) per launch of the decode kernel (the partition kernel,
    or the fused step kernel) from the committed ncu summary for this workload and block
    size, only if it was taken on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", f"{kernel}__{workload}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_hash = re.search(r"kernel_source_sha256:\s*([0-9a-f]+)", text)
    sources = STEP_SOURCES if kernel == "paged_decode_step" else KERNEL_SOURCES
    if not m_hash or m_hash.group(1) != kernel_source_hash(sources):
        return None
    m = re.search(r"traffic_bytes_per_launch\[block_size=%d\]:\s*([0-9]+)" % block_size, text)
    return float(m.group(1)) if m else None


# ----------------------------------------------------------------------------
# clocks sampled during the timed region
# ----------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.lines = []
        target = None
        try:
            import torch
            u = getattr(torch.cuda.get_device_properties(device_index), "uuid", None)
            if u is not None:
                target = "GPU-" + str(u)
        except Exception:
            target = None
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "50"]
        if target:
            cmd += ["-i", target]
        self.cmd = cmd

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(self.cmd, stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------
# the GPU arm
# ----------------------------------------------------------------------------
def algorithmic_bytes(wl):
    """Per layer: K+V bytes (the metric) and the full roofline traffic of the decode
    kernel: K+V + q/out + block-table entries + context lengths."""
    sp = wl.spec
    lens = wl.context_lens.astype(np.int64)
    kv = int(lens.sum()) * sp.num_kv_heads * sp.head_dim * 2 * 2
    qo = wl.num_seqs * sp.num_heads * sp.head_dim * 2 * 2
    tables = int(((lens + sp.block_size - 1) // sp.block_size).sum()) * 4 + wl.num_seqs * 4
    return kv, kv + qo + tables


def cow_arm(args, rank, world, local_rank):
    """The copy-on-write decode step. Each step the block manager forks every parent
    prompt into its samples and appends one token to each sample: the shared, partly
    filled last block is copied for every sample (128 pairs), then copy_blocks ->
    reshape_and_cache -> paged decode. The device-timed step repeats one such step
    (idempotent); the end-to-end step frees the samples, forks and appends again through
    the host block manager every step."""
    import torch
    import paged_kv_cache_320_b200 as pkv

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream(dev)
    cs = synth.make_cow_step(num_layers=1)
    sp = cs.spec
    prompts, samples = len(cs.parent_lens), sp.samples
    B = prompts * samples
    mgr = pkv.BlockManager(cs.num_blocks, sp.block_size, cs.max_blocks_per_seq, cs.initial_order)
    parents = [10_000 + p for p in range(prompts)]
    kids = np.array([p * samples + k for p in range(prompts) for k in range(samples)], np.int64)
    for p, n in zip(parents, cs.parent_lens):
        if mgr.pkv_seq_append(p, int(n))[0] != 0:
            raise RuntimeError("pool too small for the parents")

    kid_parents = np.repeat(np.array(parents, np.int64), samples)
    live = [False]

    def host_step(**outs):
        """Frees the samples (after the first step), forks them again from their parents and
        appends one token to each, exporting their tables in the same call (into the given
        arrays, e.g. views of a pinned buffer, when there are any)."""
        if live[0]:
            st, done = mgr.pkv_seq_free_batch(kids)
            if st != 0:
                raise RuntimeError(f"free failed ({st})")
        st, done = mgr.pkv_seq_fork_batch(kid_parents, kids)
        if st != 0:
            raise RuntimeError(f"fork failed ({st})")
        live[0] = True
        st, done, slots, cows, tables, lens = mgr.pkv_seq_append_tables(kids, 1, **outs)
        if st != 0:
            raise RuntimeError(f"append failed ({st})")
        return slots[:, 0], cows, tables, lens

    dt = synth.torch_dtype(sp.dtype)

    def to_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(dt)

    kc, vc = to_dev(cs.k_cache[0]), to_dev(cs.v_cache[0])
    q, kn, vn = to_dev(cs.q), to_dev(cs.k_new), to_dev(cs.v_new)
    out = torch.empty_like(q)
    kp = torch.tensor([kc.data_ptr()], dtype=torch.int64, device=dev)
    vp = torch.tensor([vc.data_ptr()], dtype=torch.int64, device=dev)
    slots, cows, tables, lens = (x.copy() for x in host_step())
    n_pairs = cows.shape[0]
    max_len = cs.max_blocks_per_seq * sp.block_size
    P = pkv.pkv_decode_partition_size(B, sp.num_heads, sp.num_kv_heads, sp.head_dim,
                                      sp.block_size, max_len, args.partition)
    ws = torch.zeros(max(16, pkv.pkv_decode_workspace_size(
        B, sp.num_heads, sp.num_kv_heads, sp.head_dim, sp.block_size, max_len, P)),
        dtype=torch.uint8, device=dev)
    slots_d = torch.from_numpy(slots).to(dev)
    pairs_d = torch.from_numpy(cows).to(dev)
    bt_d = torch.from_numpy(tables).to(dev)
    lens_d = torch.from_numpy(lens).to(dev)
    dtype_code = pkv.PKV_BF16 if sp.dtype == synth.BF16 else pkv.PKV_F16
    kv_step = int(lens.astype(np.int64).sum()) * sp.num_kv_heads * sp.head_dim * 4
    ev = {"copy": [], "decode": []}

    def step(record=False, s=stream):
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)] if record else None
        if record:
            e[0].record(s)
        pkv.pkv_copy_blocks(kp, vp, pairs_d, sp.num_kv_heads, sp.head_dim, sp.block_size,
                            cs.num_blocks, dtype_code, stream=s)
        pkv.pkv_reshape_and_cache(kn, vn, kc, vc, slots_d, stream=s)
        if record:
            e[1].record(s)
        pkv.pkv_paged_attention_decode(out, q, kc, vc, bt_d, lens_d, max_len, scale=1 / math.sqrt(
            sp.head_dim), partition_size=P, workspace=ws, stream=s)
        if record:
            e[2].record(s)
            ev["copy"].append((e[0], e[1]))
            ev["decode"].append((e[1], e[2]))

    dist = None
    if world > 1:
        import torch.distributed as dist

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        step()
    barrier()
    # per-kernel split from eager steps with events between the launches
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        step(record=True)
    t1.record(stream)
    barrier()
    eager_ms = reduce_max(t0.elapsed_time(t1) / args.steps, dist, dev)
    # the step as a CUDA graph (as the other workloads are timed): `steps` consecutive
    # steps in one graph launched once, so the host cannot leave gaps between them; the
    # one-step graph gives the per-step percentiles
    g_step = record_graph(lambda s: step(s=s), dev, stream)
    for _ in range(args.warmup):
        g_step.replay()
    g_k = record_graph(lambda s: [step(s=s) for _ in range(args.steps)], dev, stream)
    g_k.replay()
    barrier()
    with ClockSampler(local_rank) as clocks:
        barrier()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        g_k.replay()
        t1.record(stream)
        barrier()
    del g_k
    ms_step = reduce_max(t0.elapsed_time(t1) / args.steps, dist, dev)
    percentiles = step_percentiles(g_step.replay, args.steps, stream, dev)
    barrier()
    if pkv.pkv_get_device_status(stream=stream) != 0:
        raise RuntimeError("device status word set during the benchmark")
    copy_us = 1e3 * statistics.mean(a.elapsed_time(b) for a, b in ev["copy"])
    dec_us = 1e3 * statistics.mean(a.elapsed_time(b) for a, b in ev["decode"])
    value, tokens_per_s = weak_scaling_rates(kv_step, B, world, ms_step)
    copy_bytes = n_pairs * 2 * sp.num_kv_heads * sp.block_size * sp.head_dim * 2 * 2

    # end to end: the host block manager frees, re-forks and appends every step (batched
    # calls); two steps in flight with double-buffered inputs and outputs, as in e2e_arm
    NBUF = 2
    pin = dict(pin_memory=True)

    def packed(parts, device=None):
        """One byte buffer holding each (shape, dtype) part at a 256-byte aligned offset,
        and a view of each part: one copy moves all of them."""
        offs, total = [], 0
        for shape, dtp in parts:
            offs.append(total)
            n = int(np.prod(shape)) * torch.empty((), dtype=dtp).element_size()
            total += -(-n // 256) * 256
        buf = (torch.empty(total, dtype=torch.uint8, device=device) if device is not None
               else torch.empty(total, dtype=torch.uint8, **pin))
        views = []
        for (shape, dtp), o in zip(parts, offs):
            n = int(np.prod(shape)) * torch.empty((), dtype=dtp).element_size()
            views.append(buf[o:o + n].view(dtp).view(shape))
        return buf, views

    # this step's query and new K/V rows (one H2D copy), and the host block manager's
    # results (slots, copy-on-write pairs, tables, lengths: one H2D copy)
    act_parts = [(tuple(q.shape), dt), (tuple(kn.shape), dt), (tuple(vn.shape), dt)]
    tab_parts = [((B,), torch.int64), ((B, 2), torch.int32), (tuple(tables.shape), torch.int32),
                 ((B,), torch.int32)]
    act_h, (q_h, kn_h, vn_h) = packed(act_parts)
    q_h.copy_(q.cpu()); kn_h.copy_(kn.cpu()); vn_h.copy_(vn.cpu())
    tab_h = [packed(tab_parts) for _ in range(NBUF)]
    act_e = [packed(act_parts, dev) for _ in range(NBUF)]
    tab_e = [packed(tab_parts, dev) for _ in range(NBUF)]
    out_h = [torch.empty(tuple(q.shape), dtype=dt, **pin) for _ in range(NBUF)]
    out_e = [torch.empty_like(out) for _ in range(NBUF)]

    copy_in = torch.cuda.Stream(dev)
    copy_out = torch.cuda.Stream(dev)

    # The step's three kernels (copy_blocks, cache write, decode), recorded once per buffer
    # set as a CUDA graph; the copies stay on their own streams so that they overlap the
    # other buffer set's kernels.
    def kernels(b):
        def rec(s):
            q_d, kn_d, vn_d = act_e[b][1]
            sl_d, pr_d, bt_dd, ln_d = tab_e[b][1]
            pkv.pkv_copy_blocks(kp, vp, pr_d[:n_pairs], sp.num_kv_heads, sp.head_dim,
                                sp.block_size, cs.num_blocks, dtype_code, stream=s)
            pkv.pkv_reshape_and_cache(kn_d, vn_d, kc, vc, sl_d, stream=s)
            pkv.pkv_paged_attention_decode(out_e[b], q_d, kc, vc, bt_dd, ln_d, max_len,
                                           scale=1 / math.sqrt(sp.head_dim), partition_size=P,
                                           workspace=ws, stream=s)
        return rec

    graphs = [record_graph(kernels(b), dev, stream) for b in range(NBUF)]

    def evs():
        return [torch.cuda.Event() for _ in range(NBUF)]

    ev_h2d, ev_done, ev_d2h = evs(), evs(), evs()
    kstep = [0]

    # the block manager writes slots, pairs, tables and lengths straight into the pinned
    # buffer set of the step
    tab_np = []
    for b in range(NBUF):
        sl_h, pr_h, bt_h, ln_h = tab_h[b][1]
        tab_np.append(dict(slots_out=sl_h.numpy().reshape(B, 1), cows_out=pr_h.numpy(),
                           tables_out=bt_h.numpy(), lens_out=ln_h.numpy()))

    def e2e_step():
        b = kstep[0] % NBUF
        kstep[0] += 1
        ev_h2d[b].synchronize()            # the H2D that last read these host buffers is done
        sl, cw, tb, ln = host_step(**tab_np[b])
        if cw.shape[0] != n_pairs:
            raise RuntimeError("copy-on-write pair count changed")
        copy_in.wait_event(ev_done[b])     # buffer set b's kernels (two steps ago) are done
        with torch.cuda.stream(copy_in):
            act_e[b][0].copy_(act_h, non_blocking=True)
            tab_e[b][0].copy_(tab_h[b][0], non_blocking=True)
        ev_h2d[b].record(copy_in)
        stream.wait_event(ev_h2d[b])
        stream.wait_event(ev_d2h[b])       # out_e[b] has been read back
        with torch.cuda.stream(stream):
            graphs[b].replay()
        ev_done[b].record(stream)
        copy_out.wait_event(ev_done[b])
        with torch.cuda.stream(copy_out):
            out_h[b].copy_(out_e[b], non_blocking=True)
        ev_d2h[b].record(copy_out)

    with host_loop():
        for _ in range(args.warmup):
            e2e_step()
        barrier()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        copy_in.wait_event(a)
        for _ in range(args.steps):
            e2e_step()
        stream.wait_stream(copy_out)
        stream.wait_stream(copy_in)
        b.record(stream)
        barrier()
    e2e_ms = reduce_max(a.elapsed_time(b) / args.steps, dist, dev)
    mgr.close()
    peak, peak_kind = read_peaks()
    h2d = act_h.numel() + tab_h[0][0].numel()   # bytes of the two packed copies
    pmax = max(1, -(-max_len // P))
    return {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": synth.DTYPE_NAMES[sp.dtype], "data": "synthetic",
        "config": {"workload": "shared_prefix_cow", "description": WORKLOADS["shared_prefix_cow"],
                   "num_seqs": B, "copy_pairs_per_step": n_pairs, "partition_size": P,
                   "sum_context_tokens": int(lens.sum()), "kv_bytes_per_step": kv_step,
                   "parallelism": f"replicas x{world}"},
        "tokens_per_s": round(tokens_per_s, 1),
        "pct_of_hbm_peak": round(100 * value / world / peak, 2),
        "timed": "CUDA graph of `steps` consecutive steps (copy_blocks, cache write, decode), "
                 "launched once",
        "step_ms_percentiles": percentiles,
        "eager": {"value": round(weak_scaling_rates(kv_step, B, world, eager_ms)[0], 1),
                  "unit": "GB/s", "ms_per_step": round(eager_ms, 4),
                  "note": "the same steps launched one kernel at a time, with events between "
                          "the launches (the copy / decode split below)"},
        "copy_and_write_us": round(copy_us, 2),
        "copy_blocks_bytes": copy_bytes,
        "decode_us": round(dec_us, 2),
        "clocks": clocks.summary(),
        "e2e": {"value": round(kv_step * world / (e2e_ms * 1e-3) / 1e9, 1), "unit": "GB/s",
                "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(out_h[0].numel() * 2),
                "includes": "host batched frees, forks and appends (copy-on-write pairs) with "
                            "the table export in the same call, written into the pinned buffer; "
                            "pinned H2D (two packed copies: q / k_new / v_new, and "
                            "slots / pairs / tables / lengths), copy_blocks + cache write + "
                            "decode (one CUDA graph per buffer set), D2H; two steps in flight "
                            "(double-buffered inputs and outputs, copies on their own streams); "
                            "Python's garbage collector paused during the loop"},
        "gpu_launches": args.steps * (3 + (1 if pmax > 1 else 0)),
    }


def reduce_max(x, dist, device):
    """Maximum of a per-rank scalar over all ranks (the identity on one process)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_rates(kv_bytes_per_rank_step, seqs_per_rank, world, ms_step):
    """Whole-job rates when every rank runs its own replica for the same step time
    (the slowest rank's): K/V GB/s and decode tokens/s summed over ranks."""
    sec = ms_step * 1e-3
    return kv_bytes_per_rank_step * world / sec / 1e9, seqs_per_rank * world / sec


@contextlib.contextmanager
def host_loop():
    """A latency-bound host loop: Python's cyclic garbage collector runs before it and is
    paused during it (a collection in the middle of a step stalls the launches)."""
    gc.collect()
    gc.disable()
    try:
        yield
    finally:
        gc.enable()


def record_graph(fn, dev, stream):
    """fn(launch_stream)'s launches recorded once as a CUDA graph (captured on a side
    stream that first waits for `stream`)."""
    import torch
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.graph(g, stream=side):
        fn(side)
    stream.wait_stream(side)
    return g


def step_percentiles(run, steps, stream, dev):
    """p10 / p50 / p90 of one step's time (ms): `steps` more steps, each between its own
    CUDA events on `stream` (run after the timed region, on this rank)."""
    import torch
    pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
             for _ in range(max(1, steps))]
    with torch.cuda.stream(stream):
        for a, b in pairs:
            a.record(stream)
            run()
            b.record(stream)
    torch.cuda.synchronize(dev)
    per = sorted(a.elapsed_time(b) for a, b in pairs)

    def q(f):
        return round(per[min(len(per) - 1, int(round(f * (len(per) - 1))))], 4)

    return {"p10": q(0.1), "p50": q(0.5), "p90": q(0.9), "n": len(per),
            "timed": "each step between its own CUDA events, after the timed region"}


def time_replays(g, replays, stream):
    """ms per replay of graph g: `replays` replays between two CUDA events on `stream`
    (the caller synchronises on both sides)."""
    import torch
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        a.record(stream)
        for _ in range(replays):
            g.replay()
        b.record(stream)
    b.synchronize()
    return a.elapsed_time(b) / replays


def gpu_arm(args, rank, world, local_rank, light=False):
    """The device-timed decode step of one workload (every rank its own replica). With
    light, only the step, its dominant kernel and its clocks are timed (no end-to-end leg,
    read probe, memory-utilisation replay or optional legs)."""
    import torch
    import paged_kv_cache_320_b200 as pkv

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    overrides = {}
    if args.block_size:
        overrides["block_size"] = args.block_size
    if args.layers:
        overrides["num_layers"] = args.layers
    if args.batch:
        overrides["batch"] = args.batch
    sp0 = synth.spec(args.workload, **overrides)
    # block tables wide enough, and pool blocks for, the tokens the end-to-end loop appends
    grow = args.steps + args.warmup + 1
    overrides["max_len"] = sp0.max_len + grow + 2 * sp0.block_size
    nseqs = sp0.batch or len(sp0.lens) or sp0.prompts * sp0.samples
    overrides["pool_extra"] = nseqs * (-(-grow // sp0.block_size) + 1)
    # weak scaling: every rank holds its own replica of the same workload
    wl = synth.make_workload(args.workload, values_on="cuda", device=str(dev), **overrides)
    sp = wl.spec
    L = sp.num_layers
    B = wl.num_seqs
    max_len = wl.max_blocks_per_seq * sp.block_size
    P = pkv.pkv_decode_partition_size(B, sp.num_heads, sp.num_kv_heads, sp.head_dim,
                                      sp.block_size, max_len, args.partition)
    pmax = max(1, -(-max_len // P))
    ws_bytes = pkv.pkv_decode_workspace_size(B, sp.num_heads, sp.num_kv_heads, sp.head_dim,
                                             sp.block_size, max_len, P)
    ws = torch.zeros(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    bt = torch.from_numpy(wl.block_tables).to(dev)
    lens = torch.from_numpy(wl.context_lens).to(dev)
    slots = torch.from_numpy(wl.slot_mapping).to(dev)
    outs = [torch.empty_like(wl.q[l]) for l in range(L)]
    stream = torch.cuda.current_stream(dev)
    kv_layer, roof_layer = algorithmic_bytes(wl)
    roof_layer_all = roof_layer
    kv_step = kv_layer * L
    shared = args.decode == "shared"
    if shared:
        if not sp.prompts:
            raise SystemExit("--decode shared needs a workload with shared prefixes")
        starts = torch.arange(0, B + 1, sp.samples, dtype=torch.int32, device=dev)
        prefix = torch.full((sp.prompts,), sp.prefix, dtype=torch.int32, device=dev)
        # the shared-prefix path has its own automatic partition size
        P = pkv.pkv_decode_shared_prefix_partition_size(B, sp.num_heads, sp.num_kv_heads,
                                                        sp.head_dim, sp.block_size, max_len,
                                                        args.partition)
        ws = torch.empty(max(16, pkv.pkv_decode_shared_prefix_workspace_size(
            B, sp.num_heads, sp.num_kv_heads, sp.head_dim, sp.block_size, max_len, P)),
            dtype=torch.uint8, device=dev)
        # unique K/V: each prompt's prefix once per KV head, every private suffix
        uniq = (sp.prompts * sp.prefix + int((wl.context_lens - sp.prefix).sum())) * \
            sp.num_kv_heads * sp.head_dim * 4
        roof_layer = roof_layer - kv_layer + uniq

    fused = args.step == "fused" and not shared   # the shared-prefix decode has its own launches
    if fused:
        ws = torch.zeros(pkv.pkv_decode_step_workspace_size(
            B, sp.num_heads, sp.num_kv_heads, sp.head_dim, sp.block_size, max_len, P),
            dtype=torch.uint8, device=dev)
    # this step's K/V rows as [B, Hkv, D] (one new token per sequence)
    kn3 = [wl.k_new[l].view(B, sp.num_kv_heads, sp.head_dim) for l in range(L)]
    vn3 = [wl.v_new[l].view(B, sp.num_kv_heads, sp.head_dim) for l in range(L)]

    def fused_layer(l, out_t, q_t, kn_t, vn_t, bt_t, lens_t, st):
        pkv.pkv_paged_decode_step(out_t, q_t, kn_t, vn_t, wl.k_cache[l], wl.v_cache[l], bt_t,
                                  lens_t, max_len, ws, scale=wl.scale, partition_size=P,
                                  stream=st)

    def decode(l, out_t, q_t, bt_t, lens_t, st):
        if shared:
            # one plan per step serves every layer (the layers share tables and lengths)
            if l == 0:
                pkv.pkv_shared_prefix_plan(bt_t, lens_t, starts, prefix, sp.num_heads,
                                           sp.num_kv_heads, sp.head_dim, sp.block_size, max_len,
                                           ws, partition_size=P, stream=st)
            pkv.pkv_paged_attention_decode_shared_prefix_planned(
                out_t, q_t, wl.k_cache[l], wl.v_cache[l], bt_t, lens_t, max_len, ws,
                scale=wl.scale, partition_size=P, stream=st)
        else:
            pkv.pkv_paged_attention_decode(out_t, q_t, wl.k_cache[l], wl.v_cache[l], bt_t,
                                           lens_t, max_len, scale=wl.scale, partition_size=P,
                                           workspace=ws, stream=st)

    def step(st):
        for l in range(L):
            if fused:
                # the workload's slot of each sequence is its newest position (len - 1)
                fused_layer(l, outs[l], wl.q[l], kn3[l], vn3[l], bt, lens, st)
            else:
                pkv.pkv_reshape_and_cache(wl.k_new[l], wl.v_new[l], wl.k_cache[l],
                                          wl.v_cache[l], slots, stream=st)
                decode(l, outs[l], wl.q[l], bt, lens, st)

    # The dominant kernel's launches alone (the split entry points): the write-and-decode
    # kernel of the fused step, or the partition kernel; and the merge kernel alone. The
    # step kernel that merges in its own launch is its own call.
    if fused:
        launches_per_layer = pkv.pkv_decode_step_launches(
            B, sp.num_heads, sp.num_kv_heads, sp.head_dim, sp.block_size, max_len, P)
        launches_per_step = L * launches_per_layer
        kernel_key = ("paged_decode_partition_write" if launches_per_layer > 1 or pmax == 1
                      else "paged_decode_step")
    else:
        launches_per_layer = 3 if shared else 2 + (1 if pmax > 1 else 0)
        launches_per_step = (3 * L + 1) if shared else L * launches_per_layer
        kernel_key = "paged_decode_shared" if shared else "paged_decode_partition"
    split = not shared and (not fused or launches_per_layer > 1)

    def kernel_only(st):
        for l in range(L):
            if fused:
                pkv.pkv_paged_decode_step_partitions(outs[l], wl.q[l], kn3[l], vn3[l],
                                                     wl.k_cache[l], wl.v_cache[l], bt, lens,
                                                     max_len, ws, scale=wl.scale,
                                                     partition_size=P, stream=st)
            else:
                pkv.pkv_paged_attention_decode_partitions(outs[l], wl.q[l], wl.k_cache[l],
                                                          wl.v_cache[l], bt, lens, max_len, ws,
                                                          scale=wl.scale, partition_size=P,
                                                          stream=st)

    def merge_only(st):
        for l in range(L):
            pkv.pkv_paged_attention_merge(outs[l], lens, sp.num_kv_heads, sp.block_size,
                                          max_len, ws, partition_size=P, stream=st)

    dist = None
    if world > 1:
        import torch.distributed as dist

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)

    # ---- device-timed region: inputs resident in HBM
    for _ in range(args.warmup):
        step(stream)
    barrier()
    graphs = {}
    g_step = None
    if not args.no_graph:
        # the step's launches (every layer's) recorded as a CUDA graph: the headline timing,
        # as a serving loop runs a decode step; the dominant kernel's and the merge kernel's
        # launches alone in graphs of their own. Each is timed as one graph of `steps`
        # consecutive copies, launched once, so the host cannot leave gaps between steps;
        # the one-step graph gives the per-step percentiles.
        fns = {"step": step}
        if split:
            fns["kernel"] = kernel_only
            if pmax > 1:
                fns["merge"] = merge_only
        g_step = record_graph(step, dev, stream)
        for _ in range(args.warmup):
            g_step.replay()
        for name, fn in fns.items():
            graphs[name] = record_graph(lambda s, fn=fn: [fn(s) for _ in range(args.steps)],
                                        dev, stream)
            graphs[name].replay()   # upload, and one more warm-up pass
        barrier()
    ms = {}
    with ClockSampler(local_rank) as clocks:
        barrier()
        # eager launches (the same steps, one kernel at a time)
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(args.steps):
            step(stream)
        t1.record(stream)
        barrier()
        ms["eager"] = t0.elapsed_time(t1) / args.steps
        for name, g in graphs.items():
            ms[name] = time_replays(g, 1, stream) / args.steps
            barrier()
    percentiles = step_percentiles(g_step.replay if g_step is not None else lambda: step(stream),
                                   args.steps, stream, dev)
    barrier()
    graphs.clear()
    g_step = None
    if pkv.pkv_get_device_status(stream=stream) != 0:
        raise RuntimeError("device status word set during the benchmark")

    def max_over_ranks(x):
        return reduce_max(x, dist, dev)

    ms = {k: max_over_ranks(v) for k, v in ms.items()}
    ms_step = ms.get("step", ms["eager"])
    value, tokens_per_s = weak_scaling_rates(kv_step, B, world, ms_step)
    eager_value, _ = weak_scaling_rates(kv_step, B, world, ms["eager"])
    peak, peak_kind = read_peaks()
    call_us = 1e3 * ms_step / L
    kernel_us = 1e3 * ms["kernel"] / L if "kernel" in ms else call_us
    merge_us = 1e3 * ms["merge"] / L if "merge" in ms else None
    achieved = roof_layer / (kernel_us * 1e-6) / 1e9
    call_achieved = roof_layer / (call_us * 1e-6) / 1e9
    traffic = None if shared else read_traffic(args.workload, sp.block_size, kernel_key)
    if fused:
        call_desc = ("write-and-decode kernel + merge kernel" if launches_per_layer > 1 else
                     "write-and-decode kernel (one partition per context)" if pmax == 1 else
                     "step kernel (cache write, decode and merge in one launch)")
    else:
        call_desc = ("plan (one per step) + shared-prefix decode + merge" if shared else
                     "cache write + partition kernel" + (" + merge kernel" if pmax > 1 else ""))
    roofline = {
        "kernel": f"{kernel_key}_kernel",
        "bound": "hbm",
        "achieved": round(achieved, 1),
        "peak": peak,
        "peak_kind": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
        else "fallback",
        "unit": "GB/s",
        "frac": round(achieved / peak, 4),
        "traffic": traffic,
        "algorithmic_bytes_per_launch": roof_layer,
        "avg_launch_us": round(kernel_us, 2),
        "timed": ("CUDA graph of the kernel's launches alone (all layers), `steps` copies in "
                  "one graph launched once between CUDA events" if "kernel" in ms else
                  "the step's CUDA graph (one launch per layer), `steps` copies launched once"),
        "call_level": {"includes": call_desc, "us_per_layer": round(call_us, 2),
                       "achieved": round(call_achieved, 1),
                       "frac": round(call_achieved / peak, 4)},
    }
    if merge_us is not None:
        roofline["merge_kernel_us"] = round(merge_us, 2)
    if light:
        return {
            "workload": args.workload, "decode": args.decode, "block_size": sp.block_size,
            "layers": L,
            "num_seqs": B, "num_heads": sp.num_heads, "num_kv_heads": sp.num_kv_heads,
            "dtype": synth.DTYPE_NAMES[sp.dtype], "partition_size": P,
            "sum_context_tokens": int(wl.context_lens.sum()), "kv_bytes_per_step": kv_step,
            "value": round(value, 1), "unit": "GB/s", "ms_per_step": round(ms_step, 4),
            "pct_of_hbm_peak": round(100 * value / world / peak, 2),
            "tokens_per_s": round(tokens_per_s, 1),
            "launches_per_layer": launches_per_layer,
            **({"unique_kv_bytes_per_step": (roof_layer - (roof_layer_all - kv_layer)) * L,
                "value_unique": round((roof_layer - (roof_layer_all - kv_layer)) * L * world
                                      / (ms_step * 1e-3) / 1e9, 1),
                "note": "value counts logical K/V bytes (every sequence's whole context); the "
                        "roofline counts the bytes the path must read (each shared prefix once "
                        "per KV head, every private suffix)"} if shared else {}),
            "eager": {"value": round(eager_value, 1), "ms_per_step": round(ms["eager"], 4)},
            "step_ms_percentiles": percentiles,
            "roofline": roofline, "clocks": clocks.summary()}

    roofline["hbm_read_probe_gbs"] = round(hbm_read_probe(dev, stream), 1)
    swap = swap_measurement(wl, dev, stream) if args.swap else None
    mem_mgr = replay_block_manager(wl)
    memory = memory_utilisation(wl, mem_mgr, sp0.max_len)   # the workload's own length cap
    mem_mgr.close()
    prefix_cache = prefix_cache_measurement(sp) if args.prefix_cache else None
    if prefix_cache is not None:
        prefix_cache["decode"] = prefix_cache_decode_measurement(dev, stream, args.steps,
                                                                 args.warmup)

    # ---- end to end: host block manager + pinned host buffers through the public API
    e2e = e2e_arm(args, wl, P, max_len, ws, dev, stream, barrier, max_over_ranks, world, decode,
                  fused_layer if fused else None)

    result = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": synth.DTYPE_NAMES[sp.dtype],
        "data": "synthetic (seeded N(0,1) values, lognormal/uniform lengths, random block placement)",
        "config": {
            "workload": args.workload,
            "description": describe(args),
            "num_seqs": B, "num_heads": sp.num_heads, "num_kv_heads": sp.num_kv_heads,
            "head_dim": sp.head_dim, "block_size": sp.block_size, "layers": L,
            "sum_context_tokens": int(wl.context_lens.sum()),
            "partition_size": P,
            "decode": args.decode,
            "step": "fused" if fused else "separate",
            "timed": "eager launches" if args.no_graph else
                     "CUDA graph of `steps` consecutive steps, launched once",
            "kv_bytes_per_step": kv_step,
            "l2": f"inputs larger than L2: {kv_layer / 1e6:.0f} MB of K/V per layer vs 126 MB L2",
            "parallelism": f"replicas x{world}",
        },
        "tokens_per_s": round(tokens_per_s, 1),
        "pct_of_hbm_peak": round(100 * value / world / peak, 2),
        "pct_of_nominal_8tbs": round(100 * value / world / 8000.0, 2),
        **({"value_unique": round((roof_layer - (roof_layer_all - kv_layer)) * L * world
                                  / (ms_step * 1e-3) / 1e9, 1)} if shared else {}),
        "memory_utilisation": memory,
        "eager": {"value": round(eager_value, 1), "unit": "GB/s",
                  "ms_per_step": round(ms["eager"], 4),
                  "note": "the same steps launched one kernel at a time (no graph)"},
        "step_ms_percentiles": percentiles,
        **({"swap_blocks": swap} if swap else {}),
        **({"prefix_cache": prefix_cache} if prefix_cache else {}),
        "clocks": clocks.summary(),
        "e2e": e2e,
        "gpu_launches": launches_per_step * args.steps,
        "roofline": roofline,
    }
    return result


def replay_block_manager(wl):
    """Rebuild the workload's block tables with the library's block manager seeded
    by the workload's placement permutation: sequences appended in order (shared
    prefix: per prompt, the prefix on the first sample, forks, then each sample's
    suffix). The result must equal the generated tables exactly."""
    import paged_kv_cache_320_b200 as pkv
    sp = wl.spec
    mgr = pkv.BlockManager(wl.num_blocks, sp.block_size, wl.max_blocks_per_seq, wl.perm)

    def append(s, n):
        st, _, cows = mgr.pkv_seq_append(s, n)
        if st != 0 or len(cows):
            raise RuntimeError(f"block manager replay failed ({st})")

    if sp.prompts:
        for p in range(sp.prompts):
            first = p * sp.samples
            append(first, sp.prefix)
            for k in range(1, sp.samples):
                if mgr.pkv_seq_fork(first, first + k) != 0:
                    raise RuntimeError("fork failed")
            for i in range(first, first + sp.samples):
                append(i, int(wl.context_lens[i]) - sp.prefix)
    else:
        for s, n in enumerate(wl.context_lens):
            append(s, int(n))
    st, tables, lens = mgr.pkv_block_tables(np.arange(wl.num_seqs))
    if st != 0 or not np.array_equal(tables, wl.block_tables) or not np.array_equal(
            lens, wl.context_lens):
        raise RuntimeError("block manager replay does not reproduce the workload's tables")
    return mgr


def prefix_cache_measurement(sp, requests=1024, concurrency=128, decode_len=64, seed=11):
    """Host-side prefix caching ("vLLM / PagedAttention — 分页 KV Cache 分析" §2.3, §3.2):
    a stream of requests, each one of the workload's system prompts (its shared-prefix
    length) plus a private question of 32..511 tokens, decoded for decode_len tokens with
    `concurrency` requests live at a time, run once with the cache off and once on.
    Reports the prefill tokens found cached, the blocks held at the peak and the host
    time of admissions (share_prefix + append of the uncached tokens)."""
    import time
    import paged_kv_cache_320_b200 as pkv
    rng = np.random.default_rng(seed)
    prompts = max(sp.prompts, 1)
    prefix = sp.prefix if sp.prompts else 1024
    bs = sp.block_size
    system = [rng.integers(0, 32000, prefix, dtype=np.int32) for _ in range(prompts)]
    reqs = [(int(rng.integers(0, prompts)), rng.integers(0, 32000, int(rng.integers(32, 512)),
                                                          dtype=np.int32))
            for _ in range(requests)]
    max_tokens = prefix + 512 + decode_len
    mb = -(-max_tokens // bs)
    nb = concurrency * mb + prompts * (-(-prefix // bs))
    out = {"requests": requests, "concurrency": concurrency, "decode_tokens": decode_len,
           "prompts": prompts, "prefix_tokens": prefix, "block_size": bs, "num_blocks": nb}
    for on in (0, 1):
        mgr = pkv.BlockManager(nb, bs, mb)
        mgr.pkv_alloc_set_prefix_cache(on)
        live = {}
        nxt = 0
        admit_s = 0.0
        prefill = cached = peak = 0
        while nxt < len(reqs) or live:
            while nxt < len(reqs) and len(live) < concurrency:
                p, q = reqs[nxt]
                toks = np.concatenate([system[p], q])
                t0 = time.perf_counter()
                st, got = mgr.pkv_seq_share_prefix(nxt, toks[:-1])
                st2, _, _ = mgr.pkv_seq_append_tokens(nxt, toks[got:])
                admit_s += time.perf_counter() - t0
                if st or st2:
                    raise RuntimeError(f"prefix-cache admission failed ({st}, {st2})")
                prefill += len(toks)
                cached += got
                live[nxt] = decode_len
                nxt += 1
            peak = max(peak, mgr.pkv_stats()[1])
            for r in list(live):
                if mgr.pkv_seq_append_tokens(r, rng.integers(0, 32000, 1, dtype=np.int32))[0]:
                    raise RuntimeError("prefix-cache decode append failed")
                live[r] -= 1
                if live[r] == 0:
                    mgr.pkv_seq_free(r)
                    del live[r]
        key = "cache_on" if on else "cache_off"
        out[key] = {"prefill_tokens": prefill, "prefill_tokens_cached": cached,
                    "hit_rate": round(cached / prefill, 4), "peak_blocks_held": peak,
                    "admit_us_per_request": round(1e6 * admit_s / len(reqs), 2)}
        mgr.close()
    return out


def prefix_cache_decode_measurement(dev, stream, steps, warmup, requests=128, prompts=4,
                                    prefix=1024, seed=12):
    """Prefix caching feeding the shared-prefix-aware decode: `requests` requests over
    `prompts` system prompts of `prefix` tokens plus private questions of 32..511 tokens
    are admitted through the block manager with the cache on (the later requests of a
    prompt find its blocks), one decode token is appended to each, pkv_prefix_groups
    groups them, and the decode over their tables is timed as CUDA graph replays, plain
    and shared-prefix-aware (Llama-3-8B-shaped heads: 32 query / 8 KV, head_dim 128, bf16,
    block size 16; cache contents random)."""
    import torch
    import paged_kv_cache_320_b200 as pkv
    rng = np.random.default_rng(seed)
    bs, hq, hkv, d = 16, 32, 8, 128
    system = [rng.integers(0, 32000, prefix, dtype=np.int32) for _ in range(prompts)]
    mb = -(-(prefix + 512 + 1) // bs)
    nb = requests * mb
    mgr = pkv.BlockManager(nb, bs, mb)
    mgr.pkv_alloc_set_prefix_cache(1)
    cached = 0
    for r in range(requests):
        toks = np.concatenate([system[r % prompts],
                               rng.integers(0, 32000, int(rng.integers(32, 512)),
                                            dtype=np.int32)])
        st, got = mgr.pkv_seq_share_prefix(r, toks[:-1])
        st2 = mgr.pkv_seq_append_tokens(r, toks[got:])[0]
        st3 = mgr.pkv_seq_append_tokens(r, rng.integers(0, 32000, 1, dtype=np.int32))[0]
        if st or st2 or st3:
            raise RuntimeError("prefix-cache admission failed")
        cached += got
    st, order, gstart, gpre = mgr.pkv_prefix_groups(np.arange(requests))
    st2, tables, lens = mgr.pkv_block_tables(order)
    mgr.close()
    if st or st2:
        raise RuntimeError("prefix groups failed")
    row = hkv * d * 2 * 2
    logical = int(lens.astype(np.int64).sum()) * row
    held = {}
    for t, n in zip(tables, lens):
        for j in range(-(-int(n) // bs)):
            held[int(t[j])] = max(held.get(int(t[j]), 0), min(bs, int(n) - j * bs))
    unique = sum(held.values()) * row
    kc = torch.randn((nb, hkv, bs, d), device=dev).to(torch.bfloat16)
    vc = torch.randn((nb, hkv, bs, d), device=dev).to(torch.bfloat16)
    q = torch.randn((requests, hq, d), device=dev).to(torch.bfloat16)
    out = torch.empty_like(q)
    bt = torch.from_numpy(tables).to(dev)
    ln = torch.from_numpy(lens).to(dev)
    gs = torch.from_numpy(gstart).to(dev)
    gp = torch.from_numpy(gpre).to(dev)
    max_len = mb * bs
    ws_p = torch.zeros(max(16, pkv.pkv_decode_workspace_size(
        requests, hq, hkv, d, bs, max_len,
        pkv.pkv_decode_partition_size(requests, hq, hkv, d, bs, max_len))),
        dtype=torch.uint8, device=dev)
    ws_s = torch.zeros(max(16, pkv.pkv_decode_shared_prefix_workspace_size(
        requests, hq, hkv, d, bs, max_len)), dtype=torch.uint8, device=dev)
    calls = {
        "plain": lambda s: pkv.pkv_paged_attention_decode(out, q, kc, vc, bt, ln, max_len,
                                                          workspace=ws_p, stream=s),
        "shared": lambda s: pkv.pkv_paged_attention_decode_shared_prefix(
            out, q, kc, vc, bt, ln, gs, gp, max_len, workspace=ws_s, stream=s)}
    res = {"requests": requests, "prompts": prompts, "prefix_tokens": prefix,
           "prefill_tokens_cached": cached, "groups": int(len(gstart) - 1),
           "shared_prefix_tokens_per_group": sorted(set(int(x) for x in gpre)),
           "logical_kv_bytes": logical, "unique_kv_bytes": unique}
    for name, fn in calls.items():
        with torch.cuda.stream(stream):
            for _ in range(warmup):
                fn(stream)
        torch.cuda.synchronize(dev)
        g = record_graph(fn, dev, stream)
        for _ in range(warmup):
            g.replay()
        torch.cuda.synchronize(dev)
        ms = time_replays(g, steps, stream)
        del g
        res[name] = {"us": round(ms * 1e3, 2), "logical_gbs": round(logical / (ms * 1e-3) / 1e9, 1),
                     "unique_gbs": round(unique / (ms * 1e-3) / 1e9, 1)}
    if pkv.pkv_get_device_status(stream=stream) != 0:
        raise RuntimeError("device status word set during the prefix-cache decode")
    res["speedup"] = round(res["plain"]["us"] / res["shared"]["us"], 3)
    del kc, vc
    torch.cuda.empty_cache()
    return res


def memory_utilisation(wl, mgr, max_len=None):
    """KV-pool utilisation of the workload's state (\"vLLM / PagedAttention — 分页 KV Cache
    分析\" §4.2: tokens stored / (blocks x page size)): logical tokens over held blocks from
    the block manager (above 1 when blocks are shared), the same with each shared slot
    counted once, and a contiguous pre-allocation of max_len per sequence for contrast."""
    sp = wl.spec
    bs = sp.block_size
    free, held, tokens, util = mgr.pkv_stats()
    lens = wl.context_lens.astype(np.int64)
    slots = []
    for s, n in enumerate(lens):
        nblk = -(-int(n) // bs)
        blocks = wl.block_tables[s, :nblk].astype(np.int64)
        slots.append((blocks[:, None] * bs + np.arange(bs)).reshape(-1)[:int(n)])
    distinct = int(np.unique(np.concatenate(slots)).size) if slots else 0
    max_len = int(max_len or sp.max_len)
    return {"logical": round(util, 4),
            "physical": round(distinct / (held * bs), 4) if held else 0.0,
            "contiguous_prealloc": round(float(lens.sum()) / (len(lens) * max_len), 4),
            "held_blocks": held, "block_size": bs}


def swap_measurement(wl, dev, stream, budget=512 << 20, reps=5):
    """Preemption swap: every block (all layers, K and V) of whole sequences, longest
    first until ~budget bytes, out to pinned host memory and back in with one kernel each
    way; beside it a contiguous pinned copy of the same bytes (what the link gives)."""
    import torch
    import paged_kv_cache_320_b200 as pkv
    sp = wl.spec
    L = sp.num_layers
    tile = sp.num_kv_heads * sp.block_size * sp.head_dim * 2
    per_block = L * 2 * tile
    ids, seqs = [], []
    for s in np.argsort(-wl.context_lens.astype(np.int64), kind="stable"):
        nb = -(-int(wl.context_lens[s]) // sp.block_size)
        if ids and (len(ids) + nb) * per_block > budget:
            break
        ids += [int(b) for b in wl.block_tables[s, :nb]]
        seqs.append(int(s))
    nbytes = len(ids) * per_block
    kp = torch.tensor([t.data_ptr() for t in wl.k_cache], dtype=torch.int64, device=dev)
    vp = torch.tensor([t.data_ptr() for t in wl.v_cache], dtype=torch.int64, device=dev)
    ids_d = torch.tensor(ids, dtype=torch.int32, device=dev)
    host = torch.empty(nbytes // 2, dtype=torch.int16).pin_memory()
    code = pkv.PKV_F16 if sp.dtype == synth.F16 else pkv.PKV_BF16

    def timed(fn):
        fn()
        best = float("inf")
        for _ in range(reps):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            b.synchronize()
            best = min(best, a.elapsed_time(b))
        return nbytes / (best * 1e-3) / 1e9

    swap = lambda to_host: pkv.pkv_swap_blocks(kp, vp, ids_d, host, to_host, sp.num_kv_heads,
                                               sp.head_dim, sp.block_size, wl.num_blocks, code,
                                               stream=stream)
    out_gbs = timed(lambda: swap(1))
    in_gbs = timed(lambda: swap(0))
    # the same swap through a 64 MiB device staging buffer and one large copy per chunk
    staging = torch.empty(64 << 20, dtype=torch.uint8, device=dev)
    staged = lambda to_host: pkv.pkv_swap_blocks_staged(
        kp, vp, ids_d, host, to_host, sp.num_kv_heads, sp.head_dim, sp.block_size,
        wl.num_blocks, code, staging, stream=stream)
    staged_out_gbs = timed(lambda: staged(1))
    staged_in_gbs = timed(lambda: staged(0))
    del staging
    dbuf = torch.empty(nbytes // 2, dtype=torch.int16, device=dev)
    with torch.cuda.stream(stream):
        d2h = timed(lambda: host.copy_(dbuf, non_blocking=True))
        h2d = timed(lambda: dbuf.copy_(host, non_blocking=True))
    return {"sequences": len(seqs), "blocks": len(ids), "bytes": nbytes,
            "out_gbs": round(out_gbs, 1), "in_gbs": round(in_gbs, 1),
            "staged_out_gbs": round(staged_out_gbs, 1), "staged_in_gbs": round(staged_in_gbs, 1),
            "staging_bytes": 64 << 20,
            "contiguous_d2h_gbs": round(d2h, 1), "contiguous_h2d_gbs": round(h2d, 1)}


def hbm_read_probe(dev, stream):
    """Streaming-read bandwidth on this GPU (context for the roofline, not its
    denominator): a 4 GiB fp32 sum, best of 5, timed with CUDA events."""
    import torch
    x = torch.ones(1 << 30, dtype=torch.float32, device=dev)
    best = float("inf")
    for _ in range(6):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        torch.sum(x)
        b.record(stream)
        b.synchronize()
        best = min(best, a.elapsed_time(b))
    del x
    return (1 << 32) / (best * 1e-3) / 1e9


def e2e_arm(args, wl, P, max_len, ws, dev, stream, barrier, max_over_ranks, world, decode,
            fused_layer=None):
    """End to end through the public API, software-pipelined two steps deep. Each step the
    host block manager appends one token to every sequence (one batched call) and its tables
    are exported and sent up (separate kernels), or the device appends and the host
    allocator mirrors it (fused step: tables, lengths and free list stay on the GPU). The
    step's q / k_new / v_new go host->device from pinned memory on a copy stream layer by
    layer, each layer's kernels start once its inputs have landed, and each layer's output
    goes device->host on a second copy stream. Inputs and outputs are double-buffered, so
    step k+1's host work and copies overlap step k's kernels; a buffer set is refilled only
    after the step that used it two steps earlier is done with it. Timed with CUDA events
    from before the first step's host work to the last step's output on the host."""
    import torch
    import paged_kv_cache_320_b200 as pkv

    sp = wl.spec
    L, B, MB = sp.num_layers, wl.num_seqs, wl.max_blocks_per_seq
    fused = fused_layer is not None
    mgr = replay_block_manager(wl)
    ids = np.arange(B, dtype=np.int64)
    NBUF = 2
    pin = dict(pin_memory=True)
    q_h = torch.empty(tuple(wl.q.shape), dtype=wl.q.dtype, **pin)
    q_h.copy_(wl.q.cpu())
    kn_h = torch.empty(tuple(wl.k_new.shape), dtype=wl.k_new.dtype, **pin)
    kn_h.copy_(wl.k_new.cpu())
    vn_h = torch.empty(tuple(wl.v_new.shape), dtype=wl.v_new.dtype, **pin)
    vn_h.copy_(wl.v_new.cpu())
    out_h = [torch.empty(tuple(q_h.shape), dtype=q_h.dtype, **pin) for _ in range(NBUF)]
    slots_h = [torch.empty(B, dtype=torch.int64, **pin) for _ in range(NBUF)]
    bt_h = [torch.empty((B, MB), dtype=torch.int32, **pin) for _ in range(NBUF)]
    lens_h = [torch.empty(B, dtype=torch.int32, **pin) for _ in range(NBUF)]
    q_d = [torch.empty_like(wl.q) for _ in range(NBUF)]
    kn_d = [torch.empty_like(wl.k_new) for _ in range(NBUF)]
    vn_d = [torch.empty_like(wl.v_new) for _ in range(NBUF)]
    out_d = [torch.empty_like(wl.q) for _ in range(NBUF)]
    slots_d = [torch.empty(B, dtype=torch.int64, device=dev) for _ in range(NBUF)]
    bt_d = [torch.empty((B, MB), dtype=torch.int32, device=dev) for _ in range(NBUF)]
    lens_d = [torch.empty(B, dtype=torch.int32, device=dev) for _ in range(NBUF)]
    h2d = q_h.numel() * 2 + kn_h.numel() * 2 + vn_h.numel() * 2
    if not fused:
        h2d += B * 8 + B * MB * 4 + B * 4
    d2h = q_h.numel() * 2
    if fused:
        # resident on the GPU: uploaded once, then advanced by pkv_device_append every step
        st, tables, lens = mgr.pkv_block_tables(ids)
        bt_dev = torch.from_numpy(tables).to(dev)
        lens_dev = torch.from_numpy(lens).to(dev)
        free_d = torch.from_numpy(mgr.pkv_alloc_free_list()).to(dev)
        refc_d = torch.from_numpy(mgr.pkv_alloc_refcounts()).to(dev)
        used_d = torch.zeros(1, dtype=torch.int32, device=dev)
    copy_in = torch.cuda.Stream(dev)
    copy_out = torch.cuda.Stream(dev)
    def ev():
        return [torch.cuda.Event() for _ in range(NBUF)]

    ev_in = [[torch.cuda.Event() for _ in range(L)] for _ in range(NBUF)]
    ev_out = [[torch.cuda.Event() for _ in range(L)] for _ in range(NBUF)]
    ev_tables, ev_step_done, ev_d2h_done = ev(), ev(), ev()
    mirror_lens = mgr.pkv_block_tables(ids)[2].astype(np.int64)
    kv_total = [0]
    k = [0]
    host_s = [0.0]

    def one_step():
        b = k[0] % NBUF
        k[0] += 1
        th = time.perf_counter()
        if fused:
            st, done, sl, cows = mgr.pkv_seq_append_batch(ids, 1)   # host mirror
            if st != 0 or len(cows):
                raise RuntimeError(f"host mirror append failed ({st})")
        else:
            ev_tables[b].synchronize()      # the H2D that last read these host buffers is done
            th = time.perf_counter()
            # appends and table export in one call, written into the pinned buffers
            st, done, sl, cows, tables, lens = mgr.pkv_seq_append_tables(
                ids, 1, slots_out=slots_h[b].numpy().reshape(B, 1), tables_out=bt_h[b].numpy(),
                lens_out=lens_h[b].numpy())
            if st != 0 or len(cows):
                raise RuntimeError(f"append failed ({st}) or needed a copy in an unshared workload")
            host_s[0] += time.perf_counter() - th
            th = None
        if th is not None:
            host_s[0] += time.perf_counter() - th
        mirror_lens[:] += 1
        kv_total[0] += int(mirror_lens.sum()) * sp.num_kv_heads * sp.head_dim * 4 * L
        # buffer set b was last used two steps ago: its kernels must be done before refilling
        copy_in.wait_event(ev_step_done[b])
        if not fused:
            with torch.cuda.stream(copy_in):
                slots_d[b].copy_(slots_h[b], non_blocking=True)
                bt_d[b].copy_(bt_h[b], non_blocking=True)
                lens_d[b].copy_(lens_h[b], non_blocking=True)
            ev_tables[b].record(copy_in)
        else:
            pkv.pkv_device_append(bt_dev, lens_dev, free_d, used_d, wl.num_blocks, max_len,
                                  sp.block_size, block_refcounts=refc_d, stream=stream)
        stream.wait_event(ev_d2h_done[b])   # out_d[b] has been read back
        for l in range(L):
            with torch.cuda.stream(copy_in):
                kn_d[b][l].copy_(kn_h[l], non_blocking=True)
                vn_d[b][l].copy_(vn_h[l], non_blocking=True)
                q_d[b][l].copy_(q_h[l], non_blocking=True)
            ev_in[b][l].record(copy_in)
            stream.wait_event(ev_in[b][l])
            if fused:
                fused_layer(l, out_d[b][l], q_d[b][l],
                            kn_d[b][l].view(B, sp.num_kv_heads, sp.head_dim),
                            vn_d[b][l].view(B, sp.num_kv_heads, sp.head_dim), bt_dev, lens_dev,
                            stream)
            else:
                pkv.pkv_reshape_and_cache(kn_d[b][l], vn_d[b][l], wl.k_cache[l], wl.v_cache[l],
                                          slots_d[b], stream=stream)
                decode(l, out_d[b][l], q_d[b][l], bt_d[b], lens_d[b], stream)
            ev_out[b][l].record(stream)
            copy_out.wait_event(ev_out[b][l])
            with torch.cuda.stream(copy_out):
                out_h[b][l].copy_(out_d[b][l], non_blocking=True)
        ev_step_done[b].record(stream)
        ev_d2h_done[b].record(copy_out)

    with host_loop():
        for _ in range(args.warmup):
            one_step()
        torch.cuda.synchronize(dev)
        barrier()
        kv_total[0] = 0
        host_s[0] = 0.0
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        copy_in.wait_event(t0)
        for _ in range(args.steps):
            one_step()
        stream.wait_stream(copy_out)
        stream.wait_stream(copy_in)
        t1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
    ms = max_over_ranks(t0.elapsed_time(t1)) / args.steps
    if fused:
        # the device's tables and lengths must equal the host allocator's after all steps
        st, tables, lens = mgr.pkv_block_tables(ids)
        if (pkv.pkv_get_device_status(stream=stream) != 0 or
                not np.array_equal(bt_dev.cpu().numpy(), tables) or
                not np.array_equal(lens_dev.cpu().numpy(), lens)):
            raise RuntimeError("device append diverged from the host block manager")
    mgr.close()
    value = kv_total[0] / args.steps * world / (ms * 1e-3) / 1e9
    return {"value": round(value, 1), "unit": "GB/s", "ms_per_step": round(ms, 4),
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "host_block_manager_us_per_step": round(1e6 * host_s[0] / args.steps, 1),
            "includes": ("device append of one token per sequence (tables, lengths and free "
                         "list resident on the GPU; the host allocator mirrors it with one "
                         "batched call), pinned H2D of every layer's q/k_new/v_new, the fused "
                         "step's launches per layer, D2H of every layer's output; two steps in "
                         "flight; Python's garbage collector paused during the loop"
                         if fused else
                         "host block-manager append and table export (one call, into the pinned "
                         "buffers), pinned H2D of slots/tables/lengths and every layer's q/k_new/v_new, all "
                         "layers' kernels, D2H of every layer's output; two steps in flight "
                         "(double-buffered inputs and outputs); Python's garbage collector "
                         "paused during the loop")}


# ----------------------------------------------------------------------------
# the CPU oracle (baseline leg and reference arm)
# ----------------------------------------------------------------------------
def oracle_sample(workload, block_size, nseq, seed=0):
    """Host copies of a sample of the workload for the C oracle: the lengths and
    layout of the first ``nseq`` sequences of layer 0, values drawn with numpy."""
    if workload == "shared_prefix_cow":
        workload = "shared_prefix"          # same shapes and lengths
    overrides = {"block_size": block_size} if block_size else {}
    wl = synth.make_workload(workload, values_on="none", **overrides)
    sp = wl.spec
    bs = sp.block_size
    lens = wl.context_lens[:nseq].copy()
    nblk = [-(-int(n) // bs) for n in lens]
    nb = sum(nblk)
    rng = np.random.default_rng(sp.seed + 77 + seed)
    kc = synth.round_to_bits(rng.standard_normal((nb, sp.num_kv_heads, bs, sp.head_dim),
                                                 dtype=np.float32), sp.dtype)
    vc = synth.round_to_bits(rng.standard_normal((nb, sp.num_kv_heads, bs, sp.head_dim),
                                                 dtype=np.float32), sp.dtype)
    q = synth.round_to_bits(rng.standard_normal((nseq, sp.num_heads, sp.head_dim),
                                                dtype=np.float32), sp.dtype)
    kn = synth.round_to_bits(rng.standard_normal((nseq, sp.num_kv_heads, sp.head_dim),
                                                 dtype=np.float32), sp.dtype)
    vn = synth.round_to_bits(rng.standard_normal((nseq, sp.num_kv_heads, sp.head_dim),
                                                 dtype=np.float32), sp.dtype)
    bt = np.full((nseq, max(nblk)), -1, np.int32)
    order = rng.permutation(nb).astype(np.int32)
    off = 0
    for s in range(nseq):
        bt[s, :nblk[s]] = order[off:off + nblk[s]]
        off += nblk[s]
    last = lens.astype(np.int64) - 1
    slots = bt[np.arange(nseq), last // bs].astype(np.int64) * bs + last % bs
    kv = int(lens.astype(np.int64).sum()) * sp.num_kv_heads * sp.head_dim * 4
    return dict(spec=sp, q=q, kc=kc, vc=vc, kn=kn, vn=vn, bt=bt, lens=lens, slots=slots, kv=kv,
                scale=1.0 / math.sqrt(sp.head_dim))


def oracle_step(smp, nthreads=0):
    from oracle import c_oracle
    kc, vc = c_oracle.reshape_and_cache(smp["kn"], smp["vn"], smp["kc"], smp["vc"], smp["slots"])
    c_oracle.paged_decode_attention(smp["q"], kc, vc, smp["bt"], smp["lens"], smp["scale"],
                                    smp["spec"].dtype, nthreads=nthreads)


def pick_nseq(workload, block_size):
    return {"llama7b_mha": 16, "llama3_8b_gqa": 32, "shared_prefix": 16,
            "shared_prefix_cow": 16, "long_context": 1}[workload]


def cpu_baseline(args):
    from oracle import c_oracle
    nseq = pick_nseq(args.workload, args.block_size)
    smp = oracle_sample(args.workload, args.block_size, nseq)
    oracle_step(smp)                       # warm-up
    t0 = time.perf_counter()
    n = 0
    while True:
        oracle_step(smp)
        n += 1
        if time.perf_counter() - t0 >= args.cpu_seconds:
            break
    dt = (time.perf_counter() - t0) / n
    # the same sample on one core, for a fraction of the time
    t1 = time.perf_counter()
    n1 = 0
    while True:
        oracle_step(smp, nthreads=1)
        n1 += 1
        if time.perf_counter() - t1 >= max(1.0, args.cpu_seconds / 4):
            break
    dt1 = (time.perf_counter() - t1) / n1
    return {"value": round(smp["kv"] / dt / 1e9, 3), "unit": "GB/s",
            "cores": c_oracle.num_threads(), "kind": "oracle",
            "value_one_core": round(smp["kv"] / dt1 / 1e9, 4),
            "sample": f"layer 0, first {nseq} sequences ({int(smp['lens'].sum())} context tokens) "
                      f"of the workload: cache write + attention in the plain-C fp64 oracle, "
                      f"{n} repetitions over {args.cpu_seconds:.0f}+ s"}


def reference_arm(args, rank):
    if rank != 0:
        return None
    from oracle import c_oracle
    c_oracle.build()
    nseq = pick_nseq(args.workload, args.block_size)
    smp = oracle_sample(args.workload, args.block_size, nseq)
    for _ in range(args.warmup):
        oracle_step(smp)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(smp)
    dt = (time.perf_counter() - t0) / args.steps
    value = smp["kv"] / dt / 1e9
    sp = smp["spec"]
    sample = (f"each step: layer 0, first {nseq} sequences ({int(smp['lens'].sum())} context "
              f"tokens) of the workload, cache write + attention, plain-C fp64 oracle")
    return {
        "impl": "reference",
        "metric": METRIC, "value": round(value, 3), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "description": describe(args),
                   "block_size": sp.block_size},
        "tokens_per_s": round(nseq / dt, 2),
        "cpu_baseline": {"value": round(value, 3), "unit": "GB/s", "kind": "oracle",
                         "cores": c_oracle.num_threads(), "sample": sample},
        "e2e": {"value": round(value, 3), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# (workload, block size, decode, layers): the Llama-3-8B-shaped GQA and long-context
# workloads with the plain decode, and the shared-prefix workload with the shared-prefix-aware
# decode over 8 layers (one plan per step serves them all)
CONFIG_WORKLOADS = [("llama3_8b_gqa", 16, "plain", 0), ("long_context", 8, "plain", 0),
                    ("long_context", 16, "plain", 0), ("long_context", 32, "plain", 0),
                    ("shared_prefix", 16, "shared", 8)]


def run_configs(args, local_rank):
    """The other decode workloads at their own sizes, each timed like the headline
    workload: the step as CUDA graph replays, `steps` timed after `warmup`, its dominant
    kernel alone, clocks sampled during its timed region; then the copy-on-write step
    (copy_blocks, cache write, decode) with its end-to-end loop."""
    import torch
    out = {}
    for workload, bs, decode, layers in CONFIG_WORKLOADS:
        sub = argparse.Namespace(**vars(args))
        sub.workload, sub.block_size, sub.layers, sub.batch = workload, bs, layers, 0
        sub.decode, sub.swap, sub.prefix_cache, sub.partition = decode, False, False, 0
        key = f"{workload}_bs{bs}" + (f"_{decode}_decode_{layers}_layers" if decode != "plain"
                                      else "")
        out[key] = gpu_arm(sub, 0, 1, local_rank, light=True)
        torch.cuda.empty_cache()
    sub = argparse.Namespace(**vars(args))
    sub.workload, sub.block_size, sub.layers, sub.batch, sub.partition = \
        "shared_prefix_cow", 0, 0, 0, 0
    out["shared_prefix_cow_bs16"] = cow_arm(sub, 0, 1, local_rank)
    torch.cuda.empty_cache()
    return out


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1,
                    help="GPUs of this node, one process each (started here under "
                         "torch.distributed.run unless already launched by it)")
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="llama7b_mha", choices=sorted(WORKLOADS))
    ap.add_argument("--block-size", type=int, default=0)
    ap.add_argument("--layers", type=int, default=0, help="override the workload's layer count")
    ap.add_argument("--partition", type=int, default=0, help="decode partition size (0 = auto)")
    ap.add_argument("--swap", action="store_true",
                    help="also time pkv_swap_blocks (preemption) against a contiguous copy")
    ap.add_argument("--no-graph", action="store_true",
                    help="time eager launches only (by default the device step is recorded once "
                         "as a CUDA graph and the replays are timed)")
    ap.add_argument("--prefix-cache", action="store_true",
                    help="also replay a request stream through the block manager's prefix cache")
    ap.add_argument("--step", default="fused", choices=["separate", "fused"],
                    help="fused (default): the block-table update on the device and the cache "
                         "write folded into the decode launch (partitions merged in the same "
                         "launch or by the reduce kernel); separate: cache-write, decode and "
                         "reduce launches with host-built tables")
    ap.add_argument("--decode", default="plain", choices=["plain", "shared"],
                    help="shared: the shared-prefix-aware decode (shared-prefix workload)")
    ap.add_argument("--batch", type=int, default=0,
                    help="override the sequence count of a length-distribution workload")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-workload `configs` lines of the default run")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    if args.gpus < 1:
        raise SystemExit("--gpus must be at least 1")
    return args


def free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def launch_command(argv, nproc, port, script=None):
    """torch.distributed.run over `nproc` local processes (one per GPU), rendezvous on
    127.0.0.1, each running `script` (this file) with the same arguments."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
            f"--nproc-per-node={nproc}", "--master-addr", "127.0.0.1", "--master-port", str(port),
            script or os.path.abspath(__file__), *argv]


def rank_env():
    """(rank, world size, local rank) from the launcher's environment (1 process if unset)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def run_ranks(args, arm, backend="nccl"):
    """This process's part of the run: with several ranks, a process group over the
    launcher's rendezvous (short timeout), then arm(args, rank, world, local_rank) (every
    rank its own replica; the arm takes the max over ranks of its times), then a closing
    barrier. Returns the arm's result on rank 0, None elsewhere."""
    rank, world, local_rank = rank_env()
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but {world} process(es) were launched")
    dist = None
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local_rank)
            kw["device_id"] = torch.device("cuda", local_rank)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    res = arm(args, rank, world, local_rank)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return res if rank == 0 else None


def main(argv=None):
    argv = sys.argv[1:] if argv is None else list(argv)
    args = parse_args(argv)
    rank, world, local_rank = rank_env()

    if args.impl == "reference":
        res = reference_arm(args, rank)
        if res is not None:
            print(json.dumps(res), flush=True)
        return 0

    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        # one process per GPU: start them under torch.distributed.run with these arguments
        return subprocess.call(launch_command(argv, args.gpus, free_port()))

    # the default line (one GPU, the headline workload at its own sizes) also carries the
    # other workloads, the copy-on-write step, the swap and the prefix-cache legs
    full = (world == 1 and not args.no_configs and args.workload == "llama7b_mha"
            and args.decode == "plain" and not args.block_size and not args.layers
            and not args.batch and not args.partition)
    if full:
        args.swap = args.prefix_cache = True
    arm = cow_arm if args.workload == "shared_prefix_cow" else gpu_arm
    res = run_ranks(args, arm)
    if res is None:
        return 0
    if full:
        res["configs"] = run_configs(args, local_rank)
    if world == 1 and not args.no_cpu_baseline and args.workload != "shared_prefix_cow":
        res["cpu_baseline"] = cpu_baseline(args)
    print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
