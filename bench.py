"""Benchmark of one verify step (paged KV-append of the candidates, then paged tree attention) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Prints one JSON line on rank 0. A step is the whole hot path over one batch of seeded synthetic input:
paged_kv_append writes every candidate's K/V into its cache slot, then paged_tree_attention attends
all candidates over their paged prefixes. Inputs are resident in HBM when the timed region starts;
the KV cache (0.6 - 1.5 GB) is larger than the 126 MB L2, so L2 is not flushed between steps.

value        = algorithmic bytes of the step / device time per step, summed over ranks (GB/s):
               attention reads K and V of every key once plus Q, writes O; append reads and writes
               each appended K/V row.
e2e          = the same metric through the public Python API with the step's per-call inputs
               (q, k_new, v_new, tables, lengths, masks, slots) copied host->device from pinned memory
               and the output copied back, every step; the KV cache is device-resident state. The
               copies run on their own streams with two buffer sets, so step k's transfers overlap the
               kernels of steps k - 1 and k + 1.
roofline     = the attention kernel alone: its algorithmic bytes / its mean launch time (CUDA events on
               its stream) against the measured HBM copy bandwidth.
cpu_baseline = the CPU oracle (fp64 NumPy) timed on a bounded sample of the same workload.

With torchrun (N > 1) every rank runs an independent batch (its own seed) on its own GPU: the path
needs no exchange between sequences, so there is no collective on the data path ("weak" scaling);
the only collectives are a barrier and the max-over-ranks of the timings.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from paged_kv_cache_tree_b200 import workloads as wl  # noqa: E402

METRIC = "paged tree-attn KV GB/s & % of B200 HBM peak; candidate-tokens/s vs CPU oracle"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
DEFAULT_WORKLOAD = "long"
# the other full-size workloads, each measured in the same run under "per_config"
PER_CONFIG = ("decode", "chain", "tree", "long")
CLOCK_WINDOW_S = 1.5
KERNEL_SOURCES = ("device_common.cuh", "verify_mma.cuh", "verify_mma.cu", "verify_tc.cuh", "verify_tc.cu",
                  "combine.cu")


def time_at_roofline(bytes_moved: float, flops: float, bw_gbs: float, tflops: float):
    """Seconds a step needs at a bandwidth (GB/s, 1e9) and a compute peak (TFLOP/s, 1e12): (io, compute)."""
    return bytes_moved / (bw_gbs * 1e9), flops / (tflops * 1e12)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        p = os.path.join(ROOT, "paged_kv_cache_tree_b200", "csrc", name)
        if os.path.exists(p):
            with open(p, "rb") as f:
                h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str):
    """DRAM bytes per attention launch from a committed ncu summary, if it matches the current kernel."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d.get(workload)
        if e and e.get("kernel_hash") == kernel_source_hash():
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap,clocks.mem,temperature.gpu,temperature.memory")

    def __init__(self, device_index: int):
        self.proc = None
        try:
            props = torch.cuda.get_device_properties(device_index)
            bus = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={bus}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except Exception:
            self.proc.kill()
            return None
        sm, smax, reasons, mem, power, tgpu, tmem = [], [], set(), [], [], [], []
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
            for lst, i in ((power, 2), (mem, 8), (tgpu, 9), (tmem, 10)):
                try:
                    lst.append(float(parts[i]))
                except (ValueError, IndexError):
                    pass
        if not sm:
            return None
        rec = {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "samples": len(sm),
               "reasons": sorted(reasons)}
        if mem:
            rec["mem_mhz"] = statistics.median(mem)
        if power:
            rec["power_w"] = statistics.median(power)
        if tgpu:
            rec["temp_gpu_c_max"] = max(tgpu)
        if tmem:
            rec["temp_mem_c_max"] = max(tmem)
        return rec


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        backend = "nccl" if args.impl == "ours" else "gloo"
        if args.impl == "ours":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif args.impl == "ours":
        torch.cuda.set_device(0)
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist

    device = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def launch_kernels(launches: int, fused: bool) -> str:
    """What one paged_tree_attention_append call launched, from the library's own count."""
    if fused:
        return "the verify kernel with the append inside" + (" + the combine kernel" if launches == 2 else "")
    return "the append kernel + the verify kernel" + (" + the combine kernel" if launches == 3 else "")


def step_bytes(w) -> int:
    return w.kv_bytes() + w.qo_bytes() + w.append_bytes()


# --------------------------------------------------------------------------------------------- CPU oracle
def oracle_sample(w, budget_s: float):
    """Time the oracle (append + attention) on the first sequences of ``w`` until about ``budget_s``.

    Returns (bytes, candidate tokens, seconds, description) of the sample it ran.
    """
    import numpy as np

    import oracle

    bits = dict(q=wl.to_numpy_bits(w.q), kc=wl.to_numpy_bits(w.k_cache), vc=wl.to_numpy_bits(w.v_cache),
                kn=wl.to_numpy_bits(w.k_new), vn=wl.to_numpy_bits(w.v_new))
    masks = wl.as_uint32(w.tree_mask)
    bt, ctx, nc, so = w.block_tables.numpy(), w.context_lens.numpy(), w.num_candidates.numpy(), w.slot_offsets.numpy()
    done_b, spent, nbytes, ncand = 0, 0.0, 0, 0
    for b in range(w.B):
        sl = slice(b, b + 1)
        t0 = time.perf_counter()
        # the append oracle returns a new cache; give it a cache holding just this sequence's blocks
        blocks = bt[b, : (int(ctx[b]) + w.bs - 1) // w.bs]
        sub_bt = np.arange(len(blocks), dtype=np.int32)[None, :]
        sub_k, sub_v = oracle.paged_kv_append(bits["kn"][sl], bits["vn"][sl], sub_bt, so[sl],
                                              bits["kc"][blocks], bits["vc"][blocks])
        oracle.paged_tree_attention(bits["q"][sl], sub_k, sub_v, sub_bt, ctx[sl], nc[sl], masks[sl], w.scale, w.dtype)
        spent += time.perf_counter() - t0
        done_b += 1
        L = int(ctx[b])
        nbytes += L * w.Hkv * w.D * 4 + 2 * w.C * w.Hq * w.D * 2 + 4 * int(nc[b]) * w.Hkv * w.D * 2
        ncand += int(nc[b])
        if spent >= budget_s:
            break
    return nbytes, ncand, spent, f"{done_b} of {w.B} sequences (all their KV heads and candidates), append + attention"


def host_cores() -> dict:
    """Host CPU counts: all logical CPUs, the ones this process may run on, and the BLAS pool."""
    try:
        aff = len(os.sched_getaffinity(0))
    except Exception:
        aff = os.cpu_count() or 1
    return {"host_cpus": os.cpu_count() or 1, "affinity_cpus": aff, "blas_threads": blas_threads()}


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info

        n = [int(i.get("num_threads", 1)) for i in threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return 1


# --------------------------------------------------------------------------------------------- arms
def run_reference(args, world, rank):
    if rank != 0:
        return None
    w = wl.make_workload(args.workload, seed=None, fill="zero")
    # size each step so that warmup + steps fit in about 90 s of CPU time
    per_step_budget = max(0.02, 90.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        oracle_sample(w, per_step_budget)
    tot_bytes, tot_cand, tot_s, desc = 0, 0, 0.0, ""
    for _ in range(args.steps):
        nb, ncnd, s, desc = oracle_sample(w, per_step_budget)
        tot_bytes += nb
        tot_cand += ncnd
        tot_s += s
    gbs = tot_bytes / tot_s / 1e9
    hc = host_cores()
    cores = hc["blas_threads"]
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_s / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.WORKLOAD_DESCRIPTIONS[args.workload], "name": args.workload,
                   "l2": "not applicable (host)"},
        "candidate_tokens_per_s": tot_cand / tot_s,
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"each step: {desc}", **hc},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    return line


def measure_accept(taco, w, d, dev, stream, args):
    """The step after the verify, timed on its own: argmax of the target's logits over the vocabulary,
    greedy acceptance, and the compaction append of the accepted candidates' K/V. The logits
    ([B, C + 1, 128256], 5-70 MB) fit in L2, so L2 is flushed before each timed iteration by reading a
    256 MB buffer (a read leaves clean lines: a write would make the next kernel pay for writing back
    L2's dirty lines); each launch is timed with CUDA events on its stream."""
    a = wl.make_accept_inputs(w)
    logits = a.target_logits.to(dev)
    tokens = a.tokens.to(dev)
    amax = torch.empty(w.B, w.C + 1, dtype=torch.int32, device=dev)
    flush = torch.ones(64 << 20, dtype=torch.float32, device=dev)
    steps = max(10, min(args.steps, 200))
    t_arg, t_acc, t_app = [], [], []
    acc_len = None
    for it in range(args.warmup + steps):
        flush.sum()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        ev[0].record(stream)
        taco.logits_argmax(logits, out=amax, stream=stream)
        ev[1].record(stream)
        acc_len, path, bonus, slots = taco.tree_greedy_accept(amax, tokens, d.parents, d.num_candidates,
                                                              d.context_lens, stream=stream)
        ev[2].record(stream)
        taco.paged_kv_append(d.k_new, d.v_new, d.block_tables, slots, d.k_cache, d.v_cache, stream=stream)
        ev[3].record(stream)
        torch.cuda.synchronize(dev)
        if it >= args.warmup:
            t_arg.append(ev[0].elapsed_time(ev[1]))
            t_acc.append(ev[1].elapsed_time(ev[2]))
            t_app.append(ev[2].elapsed_time(ev[3]))
    taco.check_device(stream)
    # the argmax alone, back to back over copies of the logits that together exceed L2 (each launch
    # reads a copy the previous launches evicted): no flush and no event pair per launch. The launches
    # are replayed from a CUDA graph, so the host's per-call cost does not pace them.
    del flush
    n_copies = max(2, min(64, -(-(256 << 20) // a.logits_bytes())))
    copies = [logits.clone() for _ in range(n_copies)]
    graph = torch.cuda.CUDAGraph()
    torch.cuda.synchronize(dev)
    with torch.cuda.graph(graph):
        cap = torch.cuda.current_stream(dev)
        for c in copies:
            taco.logits_argmax(c, out=amax, stream=cap)
    t_b2b = []
    for it in range(args.warmup + max(5, min(args.steps, 50))):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            graph.replay()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        if it >= args.warmup:
            t_b2b.append(e0.elapsed_time(e1) / n_copies)
    del graph, copies
    med = lambda x: statistics.median(x)
    arg_bytes = a.logits_bytes() + amax.numel() * 4
    return {
        "vocab": a.vocab, "logits_bytes": a.logits_bytes(),
        "argmax_us": 1e3 * med(t_b2b), "argmax_us_single_launch": 1e3 * med(t_arg),
        "argmax_timing": f"argmax_us: {n_copies} launches back to back (one CUDA graph) over copies of the logits "
                         "totalling more than L2, per launch; argmax_us_single_launch: one launch after an L2 flush",
        "accept_us": 1e3 * med(t_acc), "compaction_append_us": 1e3 * med(t_app),
        "argmax_roofline": {"bound": "hbm", "achieved": arg_bytes / (med(t_b2b) * 1e-3) / 1e9, "unit": "GB/s",
                            "traffic": None},
        "mean_accept_len": float(acc_len.float().mean().item()),
        "tokens_per_step": float(acc_len.float().sum().item()) + w.B,
        "l2": "flushed before each iteration (256 MB read)",
        "inputs": "seeded synthetic logits with a planted maximum per row; candidate hits with p = 0.7",
    }


def measure_append(taco, w, d, dev, stream, args):
    """Step A1 on its own: paged_kv_append of the step's candidates into their slots, timed with CUDA
    events on its stream (median of 50 launches). Bytes = read + write of every appended row
    (2 tensors x 2 x rows x Hkv x D x elt); the rows are a few hundred kB, so the call is launch-bound."""
    n = 50
    ts = []
    for it in range(args.warmup + n):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        taco.paged_kv_append(d.k_new, d.v_new, d.block_tables, d.slot_offsets, d.k_cache, d.v_cache, stream=stream)
        e1.record(stream)
        if it >= args.warmup:
            ts.append((e0, e1))
    torch.cuda.synchronize(dev)
    taco.check_device(stream)
    us = 1e3 * statistics.median(a.elapsed_time(b) for a, b in ts)
    rows = int((w.slot_offsets >= 0).sum().item())
    nbytes = 2 * 2 * rows * w.Hkv * w.D * 2
    return {"rows": rows, "bytes": nbytes, "us": us, "GBps": nbytes / (us * 1e-6) / 1e9, "launches": n}


def measure_kv8(taco, w, d, dev, stream, args):
    """The same verify step over 8-bit (e4m3) K/V caches with per-KV-head scales: the quantising append
    of the candidates' rows, then the attention. Caches are seeded random codes drawn on the device with
    the workload's block layout (larger than L2, no flush); each launch is timed with CUDA events on its
    stream. Narrow tiles run the mma.sync kernel (codes widened in registers), wide ones the tcgen05
    kernel (each tile widened once to f16 in shared memory)."""
    c8 = wl.make_e4m3_cache(d)
    out = torch.empty_like(d.q)
    steps = max(10, min(args.steps, 500))
    t_app, t_att = [], []
    for it in range(args.warmup + steps):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        ev[0].record(stream)
        taco.paged_kv_append_e4m3(d.k_new, d.v_new, d.block_tables, d.slot_offsets, c8.k_scale, c8.v_scale,
                                  c8.k_cache, c8.v_cache, stream=stream)
        ev[1].record(stream)
        taco.paged_tree_attention_e4m3(d.q, c8.k_cache, c8.v_cache, c8.k_scale, c8.v_scale, d.block_tables,
                                       d.context_lens, d.num_candidates, d.tree_mask, w.scale, out=out,
                                       stream=stream)
        ev[2].record(stream)
        if it >= args.warmup:
            t_app.append((ev[0], ev[1]))
            t_att.append((ev[1], ev[2]))
    torch.cuda.synchronize(dev)
    taco.check_device(stream)
    # the one-call form (paged_tree_attention_append_e4m3): the append fused into the verify on narrow
    # units, else the append kernel and then the verify, which reads all but the appended slots early
    t_call = []
    for it in range(args.warmup + steps):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        ev[0].record(stream)
        taco.paged_tree_attention_e4m3(d.q, c8.k_cache, c8.v_cache, c8.k_scale, c8.v_scale, d.block_tables,
                                       d.context_lens, d.num_candidates, d.tree_mask, w.scale, out=out,
                                       k_new=d.k_new, v_new=d.v_new, stream=stream)
        ev[1].record(stream)
        if it >= args.warmup:
            t_call.append((ev[0], ev[1]))
    torch.cuda.synchronize(dev)
    taco.check_device(stream)
    call_launches = taco.last_call_launches()
    app_ms = statistics.median(a.elapsed_time(b) for a, b in t_app)
    att_ms = statistics.median(a.elapsed_time(b) for a, b in t_att)
    call_ms = statistics.median(a.elapsed_time(b) for a, b in t_call)
    att_bytes = wl.kv8_attention_bytes(w)
    step_b = att_bytes + wl.kv8_append_bytes(w)
    del c8
    return {
        "kv_dtype": "e4m3 codes, float32 scale per KV head", "q_dtype": w.dtype,
        "attention_bytes": att_bytes, "append_bytes": wl.kv8_append_bytes(w),
        "attention_us": 1e3 * att_ms, "append_us": 1e3 * app_ms,
        "attention_GBps": att_bytes / (att_ms * 1e-3) / 1e9,
        "step_GBps": step_b / ((att_ms + app_ms) * 1e-3) / 1e9,
        "call_us": 1e3 * call_ms, "call_GBps": step_b / (call_ms * 1e-3) / 1e9, "call_launches": call_launches,
        "candidate_tokens_per_s": w.candidate_tokens() / (call_ms * 1e-3),
        "steps": steps, "l2": "caches larger than L2, no flush",
        "caches": "seeded random e4m3 codes drawn on the device (sign, mantissa uniform; exponent field "
                  "mostly 9..14), scales U[0.004, 0.012]",
    }


def measure_prefix(taco, dev, stream, args):
    """Prefix-tree KV lookup for prefill, timed on its own: 256 cached sequences (about 0.9 M tokens,
    34 k distinct full blocks of 16 tokens) inserted in one call into a fresh table, then 64 prompts
    (about 176 k tokens, each a prefix of a cached sequence plus a divergent tail) looked up in one
    call. The table and node arrays (about 6 MB) stay in L2, so the lookup is latency-bound (one warp
    walks each prompt's blocks); no L2 flush. Launches timed with CUDA events on their stream."""
    pi = wl.make_prefix_inputs()
    d = pi.to(dev)
    cap = 1 << max(2, (2 * pi.num_blocks - 1).bit_length())
    steps = max(10, min(args.steps, 200))
    t_ins = []
    for it in range(11):  # the first insert warms up and is not counted; the median of the other 10
        cache = taco.PrefixCache(pi.num_blocks, pi.bs, cap, device=dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        cache.insert(d.cached_tokens, d.cached_starts, d.cached_tables, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        if it > 0:
            t_ins.append(e0.elapsed_time(e1))
    out_b = torch.empty((d.prompt_starts.numel() - 1, pi.max_blocks), dtype=torch.int32, device=dev)
    out_m = torch.empty((d.prompt_starts.numel() - 1,), dtype=torch.int32, device=dev)
    t_lk = []
    for it in range(args.warmup + steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        cache.lookup(d.prompts, d.prompt_starts, pi.max_blocks, out_blocks=out_b, out_matched=out_m, stream=stream)
        e1.record(stream)
        if it >= args.warmup:
            t_lk.append((e0, e1))
    torch.cuda.synchronize(dev)
    taco.check_device(stream)
    lk_ms = statistics.median(a.elapsed_time(b) for a, b in t_lk)
    matched = int(out_m.sum().item())
    n_prompts = d.prompt_starts.numel() - 1
    return {
        "cached_sequences": int(d.cached_starts.numel() - 1), "cached_tokens": int(pi.cached_tokens.numel()),
        "prompts": n_prompts, "prompt_tokens": pi.prompt_tokens(), "block_size": pi.bs,
        "matched_blocks": matched, "matched_token_frac": matched * pi.bs / max(1, pi.prompt_tokens()),
        "lookup_us": 1e3 * lk_ms, "prompts_per_s": n_prompts / (lk_ms * 1e-3),
        "prompt_tokens_per_s": pi.prompt_tokens() / (lk_ms * 1e-3),
        "insert_one_call_us": 1e3 * statistics.median(t_ins), "table_slots": cap,
        "bound": "latency (table and nodes L2-resident; a warp's probes depend on its scan)",
    }


def measure_lookahead(taco, dev, stream, args):
    """Batched Lookahead Cache, timed on its own: candidate forests (C = 16, copy_len U[1, 8], contexts of
    up to 4 tokens) for 64 sequences with 0.5-4 k-token phrase-structured histories against a 37 k-token
    global cache; then the copy_len update. The histories and the cache (about 0.8 MB) stay in L2, and
    each CTA's passes over them end in a sequential trie insertion, so the step is latency-bound. Launches
    timed with CUDA events on their stream; no L2 flush."""
    li = wl.make_lookahead_inputs()
    d = li.to(dev)
    steps = max(10, min(args.steps, 200))
    t = []
    for it in range(args.warmup + steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        tok, par, num = taco.lookahead_propose(d.history, d.hist_starts, d.global_tokens, d.copy_len, li.max_match,
                                               li.C, stream=stream)
        e1.record(stream)
        if it >= args.warmup:
            t.append((e0, e1))
    hit = torch.full((d.copy_len.numel(),), 0.5, dtype=torch.float32, device=dev)
    cl = d.copy_len.clone()
    acc = torch.div(num, 2, rounding_mode="floor").to(torch.int32)
    for _ in range(3):   # warm-up: the first launch of a kernel includes loading it
        taco.lookahead_update_copy_len(acc, num, hit, cl, copy_max=8, stream=stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    taco.lookahead_update_copy_len(acc, num, hit, cl, copy_max=8, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    taco.check_device(stream)
    ms = statistics.median(a.elapsed_time(b) for a, b in t)
    B = li.copy_len.numel()
    return {
        "sequences": B, "history_tokens": int(li.history.numel()), "global_tokens": int(li.global_tokens.numel()),
        "max_candidates": li.C, "max_match": li.max_match, "propose_us": 1e3 * ms,
        "sequences_per_s": B / (ms * 1e-3), "candidates_proposed": int(num.sum().item()),
        "copy_len_update_us": 1e3 * e0.elapsed_time(e1),
        "bound": "latency (inputs L2-resident; per-sequence trie insertion is sequential)",
    }


def sustain(step, seconds: float, dev) -> int:
    """Run `step` back to back for about `seconds` (untimed), so that clock samples see the kernel under
    load for longer than one nvidia-smi period. Returns the number of steps run."""
    n, t0 = 0, time.perf_counter()
    while time.perf_counter() - t0 < seconds:
        for _ in range(50):
            step()
        torch.cuda.synchronize(dev)
        n += 50
    return n


def measure_config(taco, name, world, rank, dev, stream, args, peak, peak_kind):
    """One full-size workload's verify step (paged_tree_attention_append), timed on its own with CUDA events
    on its stream: 200 steps after the warm-up, max over ranks, then an untimed window of the same step
    for the clock record; plus the step over e4m3 caches where that kernel exists."""
    w = wl.make_workload(name, seed=1000 + wl.WORKLOADS[name]["k"] + 7919 * rank, fill="zero")
    d = w.to(dev)
    out = torch.empty_like(d.q)
    nbytes = step_bytes(w)
    fused = w.G * w.C <= 16

    def step(ev_pair=None):
        if ev_pair is not None:
            ev_pair[0].record(stream)
        taco.paged_tree_attention_append(d.q, d.k_new, d.v_new, d.k_cache, d.v_cache, d.block_tables, d.context_lens,
                                         d.num_candidates, d.tree_mask, w.scale, out=out, stream=stream)
        if ev_pair is not None:
            ev_pair[1].record(stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    launches = taco.last_call_launches()
    n = 200
    pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev.index) if rank == 0 else None
    barrier(world)
    torch.cuda.synchronize(dev)
    t0.record(stream)
    for k in range(n):
        step(pairs[k])
    t1.record(stream)
    torch.cuda.synchronize(dev)
    sustain(step, CLOCK_WINDOW_S, dev)
    clocks = sampler.stop() if sampler else None
    barrier(world)
    taco.check_device(stream)
    ms_per_step = max_over_ranks(t0.elapsed_time(t1) / n, world)
    launch_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in pairs) / n, world)
    achieved = nbytes / (launch_ms * 1e-3) / 1e9
    accept = measure_accept(taco, w, d, dev, stream, args)
    accept["argmax_roofline"]["peak"] = peak
    accept["argmax_roofline"]["frac"] = accept["argmax_roofline"]["achieved"] / peak
    append = measure_append(taco, w, d, dev, stream, args)
    kv8 = measure_kv8(taco, w, d, dev, stream, args)
    if kv8 is not None:
        kv8["attention_frac"] = kv8["attention_GBps"] / peak
        kv8["traffic"] = recorded_traffic(f"{name}_e4m3")
        kv8["attention_speedup_vs_16bit"] = launch_ms / (kv8["attention_us"] * 1e-3)
        kv8["call_frac"] = kv8["call_GBps"] / peak
        kv8["call_speedup_vs_16bit"] = launch_ms / (kv8["call_us"] * 1e-3)
    res = {
        "workload": wl.WORKLOAD_DESCRIPTIONS[name], "steps": n,
        "value": world * nbytes / (ms_per_step * 1e-3) / 1e9, "unit": "GB/s", "ms_per_step": ms_per_step,
        "step_bytes": nbytes, "candidate_tokens_per_step": w.candidate_tokens(),
        "candidate_tokens_per_s": world * w.candidate_tokens() / (ms_per_step * 1e-3),
        "candidate_tokens_per_s_at_roofline": world * w.candidate_tokens() * peak * 1e9 / nbytes,
        "hbm_frac_of_nominal_8tbs": nbytes / (ms_per_step * 1e-3) / 1e9 / NOMINAL_HBM_GBS,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": recorded_traffic(name), "algorithmic_bytes": nbytes, "launch_ms": launch_ms,
                     "peak_source": f"{peak_kind} hbm_gbs",
                     "kernel": "paged_tree_attention_append (append fused into the verify)" if fused else
                               "paged_tree_attention_append (append kernel, then the verify)"},
        "gpu_launches": launches * n,
        "launch_kernels": launch_kernels(launches, fused),
        "clocks": clocks,
        "accept": accept,
        "append": append,
        "kv8": kv8,
    }
    del d, out
    torch.cuda.empty_cache()
    return res


def run_ours(args, world, rank, local):
    import paged_kv_cache_tree_b200 as taco

    taco.load()
    dev = torch.device("cuda", local if world > 1 else 0)
    w = wl.make_workload(args.workload, seed=1000 + wl.WORKLOADS[args.workload]["k"] + 7919 * rank, fill="zero")
    d = w.to(dev)
    out = torch.empty_like(d.q)
    stream = torch.cuda.current_stream(dev)
    nbytes = step_bytes(w)
    attn_bytes = w.kv_bytes() + w.qo_bytes()

    # one step = the candidates' KV-append and the verify attention, through the fused entry point
    # (append inside the verify kernel for narrow units, the append kernel first otherwise); the
    # events bracket the whole call, so the attention roofline below counts the append's bytes too;
    # a call is one to three launches (see launch_kernels below), counted by the library itself
    fused = w.G * w.C <= 16

    def step(ev_pair=None):
        if ev_pair is not None:
            ev_pair[0].record(stream)
        taco.paged_tree_attention_append(d.q, d.k_new, d.v_new, d.k_cache, d.v_cache, d.block_tables, d.context_lens,
                                         d.num_candidates, d.tree_mask, w.scale, out=out, stream=stream)
        if ev_pair is not None:
            ev_pair[1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    taco.check_device(stream)
    launches_per_step = taco.last_call_launches()

    pairs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t_start, t_stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(dev.index) if rank == 0 else None
    barrier(world)
    torch.cuda.synchronize(dev)
    t_start.record(stream)
    for k in range(args.steps):
        step(pairs[k])
    t_stop.record(stream)
    torch.cuda.synchronize(dev)
    # the timed region is shorter than one nvidia-smi sample: keep the same step running, untimed, for
    # a while longer so that the clock record covers the kernel under load
    sustained_steps = sustain(step, CLOCK_WINDOW_S, dev)
    clocks = sampler.stop() if sampler else None
    if clocks is not None:
        clocks["window"] = (f"the timed region plus {sustained_steps} more steps of the same call right after it "
                            f"(untimed, about {CLOCK_WINDOW_S} s)")
    barrier(world)
    taco.check_device(stream)
    region_ms = t_start.elapsed_time(t_stop)
    attn_ms = sum(a.elapsed_time(b) for a, b in pairs) / args.steps
    region_ms = max_over_ranks(region_ms, world)
    attn_ms = max_over_ranks(attn_ms, world)
    ms_per_step = region_ms / args.steps
    value = world * nbytes / (ms_per_step * 1e-3) / 1e9

    # ---- end to end through the public API with host buffers. Two sets of buffers: step k's inputs
    # are copied host->device on one stream and its output device->host on another, overlapping the
    # kernels of the neighbouring steps on the compute stream; events order every buffer's reuse.
    host_keys = ("q", "k_new", "v_new", "block_tables", "context_lens", "num_candidates", "tree_mask")
    hosts = [{k: getattr(w, k).pin_memory() for k in host_keys} for _ in range(2)]
    dev_in = [{k: torch.empty_like(v, device=dev) for k, v in hosts[0].items()} for _ in range(2)]
    out_dev = [torch.empty_like(d.q) for _ in range(2)]
    out_host = [torch.empty(w.q.shape, dtype=w.q.dtype).pin_memory() for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in hosts[0].values())
    d2h = out_host[0].numel() * out_host[0].element_size()
    s_h2d = torch.cuda.Stream(dev)
    s_d2h = torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]     # inputs of the slot landed
    ev_used = [torch.cuda.Event() for _ in range(2)]   # the slot's kernels finished
    ev_out = [torch.cuda.Event() for _ in range(2)]    # the slot's output is on the host

    def e2e_step(k):
        j = k % 2
        with torch.cuda.stream(s_h2d):
            s_h2d.wait_event(ev_used[j])               # step k - 2 no longer reads these inputs
            for key, v in hosts[j].items():
                dev_in[j][key].copy_(v, non_blocking=True)
            ev_in[j].record(s_h2d)
        stream.wait_event(ev_in[j])
        stream.wait_event(ev_out[j])                   # step k - 2's output has left this buffer
        di = dev_in[j]
        taco.paged_tree_attention_append(di["q"], di["k_new"], di["v_new"], d.k_cache, d.v_cache, di["block_tables"],
                                         di["context_lens"], di["num_candidates"], di["tree_mask"], w.scale,
                                         out=out_dev[j], stream=stream)
        ev_used[j].record(stream)
        with torch.cuda.stream(s_d2h):
            s_d2h.wait_event(ev_used[j])
            out_host[j].copy_(out_dev[j], non_blocking=True)
            ev_out[j].record(s_d2h)

    for k in range(args.warmup):
        e2e_step(k)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    e0.record(stream)
    s_h2d.wait_event(e0)
    for k in range(args.steps):
        e2e_step(k)
    stream.wait_event(ev_out[(args.steps - 1) % 2])
    stream.wait_event(ev_out[(args.steps - 2) % 2] if args.steps > 1 else ev_out[(args.steps - 1) % 2])
    e1.record(stream)
    torch.cuda.synchronize(dev)
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    taco.check_device(stream)
    e2e_value = world * nbytes / (e2e_ms * 1e-3) / 1e9

    accept = measure_accept(taco, w, d, dev, stream, args)
    append = measure_append(taco, w, d, dev, stream, args)
    kv8 = measure_kv8(taco, w, d, dev, stream, args)
    prefix = measure_prefix(taco, dev, stream, args)
    lookahead = measure_lookahead(taco, dev, stream, args)
    del d, out, dev_in, out_dev
    torch.cuda.empty_cache()
    peak, peak_kind = measured_peaks()
    per_config = {}
    if not args.no_per_config:
        for name in PER_CONFIG:
            if name != args.workload:
                per_config[name] = measure_config(taco, name, world, rank, dev, stream, args, peak, peak_kind)

    if rank != 0:
        return None
    achieved = nbytes / (attn_ms * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic (seeded N(0,1) values, seeded block tables)",
        "config": {"workload": wl.WORKLOAD_DESCRIPTIONS[args.workload], "name": args.workload,
                   "step_bytes": nbytes, "attention_bytes": attn_bytes, "append_bytes": w.append_bytes(),
                   "candidate_tokens_per_step": w.candidate_tokens(),
                   "l2": "inputs larger than L2 (KV cache > 126 MB), no flush", "parallelism": f"dp{world} (independent batches)"},
        "candidate_tokens_per_s": world * w.candidate_tokens() / (ms_per_step * 1e-3),
        # the same rate at the roofline: every step's bytes moved at the measured copy bandwidth
        "candidate_tokens_per_s_at_roofline": world * w.candidate_tokens() * measured_peaks()[0] * 1e9 / nbytes,
        "hbm_frac_of_measured": value / world / peak,
        "hbm_frac_of_nominal_8tbs": value / world / NOMINAL_HBM_GBS,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": recorded_traffic(args.workload),
                     "kernel": "paged_tree_attention_append (append fused into the verify)" if fused else
                               "paged_tree_attention_append (append kernel, then the verify)",
                     "algorithmic_bytes": nbytes, "peak_source": f"{peak_kind} hbm_gbs",
                     "launch_ms": attn_ms},
        "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms},
        "gpu_launches": launches_per_step * args.steps,
        "launch_kernels": launch_kernels(launches_per_step, fused),
        "clocks": clocks,
        "accept": accept,
        "append": append,
        "kv8": kv8,
        "prefix_cache": prefix,
        "lookahead_cache": lookahead,
        "per_config": per_config,
    }
    if not args.no_per_config:
        # the headline workload's own entry, from the timed region above
        per_config[args.workload] = {
            "workload": wl.WORKLOAD_DESCRIPTIONS[args.workload], "steps": args.steps, "value": value, "unit": "GB/s",
            "ms_per_step": ms_per_step, "step_bytes": nbytes, "candidate_tokens_per_step": w.candidate_tokens(),
            "candidate_tokens_per_s": line["candidate_tokens_per_s"],
            "candidate_tokens_per_s_at_roofline": line["candidate_tokens_per_s_at_roofline"],
            "hbm_frac_of_nominal_8tbs": line["hbm_frac_of_nominal_8tbs"], "roofline": line["roofline"],
            "gpu_launches": line["gpu_launches"], "clocks": clocks, "kv8": kv8, "headline": True}
        line["per_config"] = {k: per_config[k] for k in PER_CONFIG if k in per_config}
    if kv8 is not None:
        kv8["attention_frac"] = kv8["attention_GBps"] / peak
        kv8["traffic"] = recorded_traffic(f"{args.workload}_e4m3")
        kv8["attention_speedup_vs_16bit"] = attn_ms / (kv8["attention_us"] * 1e-3)
        kv8["call_frac"] = kv8["call_GBps"] / peak
        kv8["call_speedup_vs_16bit"] = attn_ms / (kv8["call_us"] * 1e-3)
    accept["argmax_roofline"]["peak"] = peak
    accept["argmax_roofline"]["frac"] = accept["argmax_roofline"]["achieved"] / peak
    if world == 1 and not args.no_cpu_baseline:
        nb, ncnd, secs, desc = oracle_sample(w, args.cpu_budget)
        hc = host_cores()
        line["cpu_baseline"] = {"value": nb / secs / 1e9, "unit": "GB/s", "cores": hc["blas_threads"],
                                "kind": "oracle", "sample": f"{desc}; {secs:.1f} s",
                                "candidate_tokens_per_s": ncnd / secs, **hc}
    return line


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(wl.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle time for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true", help="skip the other workloads' per_config entries")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            line = run_reference(args, world, rank)
        else:
            line = run_ours(args, world, rank, local)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
