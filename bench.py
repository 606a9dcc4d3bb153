#!/usr/bin/env python
"""Benchmark of the tree-verify hot path on B200.

One step = one pass of the whole hot path over one batch: jf_build_tree on the step's draft logits
(best-first tree of `budget` nodes), jf_tree_attention of every tree node over the paged KV cache
(prefix + the tree the step just built), jf_accept of the built tree against the target logits.  The
default workload is the largest single-GPU one: the Qwen3-30B-A3B attention shape (32 q / 4 kv heads),
batch 4, 32768-token prefixes, 256-node trees.  Metric: tree nodes verified per second (whole job),
with the attention kernel's achieved TFLOP/s and HBM GB/s against the measured B200 peaks.

After the step, the same line carries `legs`: the other workloads' calls timed alone -- tree attention
on the Qwen3-8B shape (256 nodes, 4096 prefix), on the serving batch (16 sequences, 64-node trees,
prefixes U[1024, 8192]) and on the tiny case (latency), and the tree build and the accept walk at batch
8 over the full 151936-token vocabulary -- each against its own roofline.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl jf|reference] [--workload qwen3_30b_a3b]

N > 1 is launched with torchrun: every rank verifies its own independent batch (weak scaling, no
collective on the data path); the step time is the max over ranks.  `--impl reference` times the CPU
oracle (the deliberately slow, obviously correct float64 restatement of the method) on a bounded
sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOADS = {
    # name: (batch, q heads, kv heads, prefix, budget, topk, max_depth, vocab, draft depths)
    "qwen3_8b": dict(batch=1, hq=32, hkv=8, prefix=4096, budget=256, topk=4, max_depth=16, vocab=151936, depths=16),
    "qwen3_30b_a3b": dict(batch=4, hq=32, hkv=4, prefix=32768, budget=256, topk=4, max_depth=16, vocab=151936,
                          depths=16),
    # serving: per-sequence prefix lengths uniform in [1024, 8192], all pages of the batch interleaved in one pool
    "serving": dict(batch=16, hq=32, hkv=8, prefix=(1024, 8192), budget=64, topk=4, max_depth=12, vocab=151936,
                    depths=16),
}
HEAD_DIM = 128
PAGE = 16
L2_FLUSH_BYTES = 256 << 20
# kernels launched per step: row statistics, best-first expansion, attention, split combine, accept
LAUNCHES_PER_STEP = 5
ROPE_THETA = 1.0e6  # rotary base of the tree K/V append timed beside the step
DEFAULT_WORKLOAD = "qwen3_30b_a3b"
# Kernel sources whose hash gates the recorded DRAM traffic below.
ATTN_SOURCES = ("tree_verify_attention_jf_b200/csrc/tree_attention.cu", "tree_verify_attention_jf_b200/csrc/jf_device.cuh",
                "tree_verify_attention_jf_b200/csrc/jf_internal.h")
# DRAM traffic of one tree_attention_kernel launch per workload (dram__bytes_read.sum + dram__bytes_write.sum of an
# ncu capture of that workload), valid only for the kernel sources it was taken on: the roofline reports null once
# any of them has changed.  Keys: bench workloads and legs.
ATTN_TRAFFIC = {
    "qwen3_30b_a3b": dict(bytes=331_310_080 + 21_271_040, source_sha256="c77f7b6b23b3b21b197d8eb90cb4a50a49a0de2978c769ccc8fa8f3d5d042b79"),
    "qwen3_8b": dict(bytes=20_044_032 + 33_792, source_sha256="c77f7b6b23b3b21b197d8eb90cb4a50a49a0de2978c769ccc8fa8f3d5d042b79"),
    "serving": dict(bytes=298_682_624 + 17_449_216, source_sha256="c77f7b6b23b3b21b197d8eb90cb4a50a49a0de2978c769ccc8fa8f3d5d042b79"),
}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]), bf16_sus=float(d["bf16_tflops_sustained"]),
                    src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


# ----------------------------------------------------------------------------------------------
# Inputs (seeded, synthetic; shapes of the pages' Qwen3 workloads)
# ----------------------------------------------------------------------------------------------
def prefix_lengths(cfg, rng):
    """Per-sequence prefix lengths: fixed, or uniform over a (low, high) range."""
    B, pr = cfg["batch"], cfg["prefix"]
    if isinstance(pr, tuple):
        return [int(x) for x in rng.integers(pr[0], pr[1] + 1, size=B)]
    return [int(pr)] * B


def make_inputs(cfg, seed):
    from tree_verify_attention_jf_b200 import synth

    B, N = cfg["batch"], cfg["budget"]
    rng = np.random.default_rng(seed)
    x, roots = synth.draft_logits(seed, B, cfg["depths"], cfg["vocab"])
    prefix = prefix_lengths(cfg, rng)
    pages_per_seq = [(P + N + PAGE - 1) // PAGE for P in prefix]
    bt, num_pages = synth.page_pool(rng, pages_per_seq, interleave=True)
    q = rng.standard_normal((B * N, cfg["hq"], HEAD_DIM), dtype=np.float32) * np.float32(0.5)
    kv_shape = (num_pages, PAGE, cfg["hkv"], HEAD_DIM)
    return dict(draft=x, roots=roots, q=q, kv_shape=kv_shape, block_table=bt, prefix=np.array(prefix, np.int32),
                offsets=(np.arange(B + 1) * N).astype(np.int32))


def attention_sources_digest():
    import hashlib
    h = hashlib.sha256()
    for rel in ATTN_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def attention_traffic(workload):
    """Per-launch DRAM bytes of the attention kernel recorded from an ncu capture of this workload, if the
    kernel sources are still the ones that were profiled; else None."""
    rec = ATTN_TRAFFIC.get(workload)
    if rec is None:
        return None
    return rec["bytes"] if attention_sources_digest() == rec["source_sha256"] else None


# Workloads whose attention is bandwidth-bound (arithmetic intensity at or below the ridge) are graded
# against HBM bandwidth, the others against the dense bf16 tensor peak.
HBM_BOUND = {"serving"}


def roofline(workload, tflops, gbs, pk, flops, nbytes):
    common = {"kernel": "jf_tree_attention: tree_attention_kernel then combine_kernel, timed together",
              "traffic": attention_traffic(workload), "traffic_scope": "one tree_attention_kernel launch",
              "algorithmic_flops": flops, "algorithmic_bytes": nbytes}
    if workload in HBM_BOUND:
        return dict(common, bound="hbm", achieved=gbs, peak=pk["hbm"], unit="GB/s", frac=gbs / pk["hbm"],
                    peak_source=pk["src"] + " HBM copy", tensor_achieved_tflops=tflops,
                    tensor_frac=tflops / pk["bf16"])
    return dict(common, bound="tensor", achieved=tflops, peak=pk["bf16"], unit="TFLOP/s", frac=tflops / pk["bf16"],
                peak_source=pk["src"] + " bf16 burst", hbm_achieved_gbs=gbs, hbm_frac=gbs / pk["hbm"])


def rank_seed(rank):
    """Every rank verifies its own independent seeded batch (weak scaling)."""
    return 1000 + rank


def job_nodes_per_sec(batch, budget, world, step_ms):
    """Whole-job throughput: all ranks' tree nodes over the max-over-ranks step time."""
    return batch * budget * world / (step_ms * 1e-3)


def visible_pairs(parent, prefix):
    """sum over nodes of |visible set| = P + depth(node) (node with parent -1 has depth 1)."""
    tot = 0
    for b in range(parent.shape[0]):
        d = np.zeros(parent.shape[1], dtype=np.int64)
        for i in range(parent.shape[1]):
            p = parent[b, i]
            d[i] = 1 if p < 0 else d[p] + 1
        tot += int(prefix[b]) * parent.shape[1] + int(d.sum())
    return tot


def visible_pairs_ragged(parent, offsets, prefix):
    """visible_pairs for trees of different sizes: parent int [T] local indices, offsets [B+1]."""
    return sum(visible_pairs(np.asarray(parent[offsets[b]:offsets[b + 1]])[None], [prefix[b]])
               for b in range(len(prefix)))


def attention_work(nodes, hq, hkv, prefix, pairs):
    """Algorithmic work of one tree-attention call: 4*d flops per visible (query head, key) pair; bytes = the K/V of
    every sequence's P + N slots read once per kv head, q read and out written once, and the metadata (block
    table rows in use, parent, prefix length and offsets)."""
    flops = 4.0 * HEAD_DIM * hq * pairs
    kv = sum(hkv * (P + n) * HEAD_DIM * 2 * 2 for P, n in zip(prefix, nodes))
    qo = 2 * sum(nodes) * hq * HEAD_DIM * 2
    meta = sum(4 * ((P + n + PAGE - 1) // PAGE) + 4 * n + 12 for P, n in zip(prefix, nodes))
    return flops, kv + qo + meta


class ClockSampler:
    def __init__(self, uuid, out_path):
        self.proc = None
        self.path = out_path
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.fh = open(out_path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={uuid if str(uuid).startswith('GPU-') else 'GPU-' + str(uuid)}", f"--query-gpu={q}", "--format=csv,noheader",
                                          "-lms", "100"], stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return dict(sm_mhz=None, sm_max_mhz=None, reasons=["unsampled"])
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1].split()[0]))
                smax.append(float(f[2].split()[0]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return dict(sm_mhz=None, sm_max_mhz=None, reasons=["unsampled"])
        return dict(sm_mhz=statistics.median(sm), sm_max_mhz=max(smax), reasons=sorted(reasons), samples=len(sm))


class NvmlSampler:
    """SM clock and clock-event reasons read through NVML every ~0.2 ms by a background thread, so that a timed
    region of a few milliseconds still yields samples under load (reads only; no setting is changed).  Falls
    back to the nvidia-smi sampler when NVML is unavailable."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4))

    def __init__(self, uuid, out_path):
        import threading
        self.fallback = None
        self.sm, self.bits = [], []
        try:
            import pynvml
            pynvml.nvmlInit()
            u = str(uuid)
            self.h = pynvml.nvmlDeviceGetHandleByUUID(u if u.startswith("GPU-") else "GPU-" + u)
            self.smax = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.nv = pynvml
        except Exception:
            self.fallback = ClockSampler(uuid, out_path)
            time.sleep(0.3)  # nvidia-smi's first sample
            return
        self.stop_flag = threading.Event()
        self.running = threading.Event()
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()
        self.running.wait(timeout=2.0)  # the thread polls before the timed region starts; only later samples count
        self.sm, self.bits = [], []

    def _run(self):
        nv = self.nv
        while not self.stop_flag.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                break
            self.sm.append(sm)
            self.bits.append(bits)
            self.running.set()
            time.sleep(0.0002)

    def stop(self):
        if self.fallback is not None:
            return self.fallback.stop()
        self.stop_flag.set()
        self.thread.join(timeout=5)
        if not self.sm:
            return dict(sm_mhz=None, sm_max_mhz=None, reasons=["unsampled"])
        reasons = sorted({n for b in self.bits for n, m in self.REASONS if b & m})
        return dict(sm_mhz=statistics.median(self.sm), sm_max_mhz=self.smax, reasons=reasons, samples=len(self.sm),
                    source="nvml")


# ----------------------------------------------------------------------------------------------
# CPU oracle leg (cpu_baseline and --impl reference)
# ----------------------------------------------------------------------------------------------
def oracle_step_rate(cfg, seed, budget_s=15.0, max_steps=40, warmup=0):
    """Times the oracle over whole steps (build + attention + accept) of the same workload: `warmup` untimed
    steps, then steps until about `budget_s` seconds of CPU work or `max_steps` steps; returns (nodes/s, steps
    timed, seconds, threads)."""
    from oracle.accept import accept as o_accept
    from oracle.build_tree import build_tree as o_build
    from oracle.tree_attention import tree_attention
    from tree_verify_attention_jf_b200 import synth

    inp = make_inputs(cfg, seed)
    B, N = cfg["batch"], cfg["budget"]
    rng = np.random.default_rng(seed + 1)
    k = synth.bf16_round(rng.standard_normal(inp["kv_shape"], dtype=np.float32) * np.float32(0.5))
    v = synth.bf16_round(rng.standard_normal(inp["kv_shape"], dtype=np.float32) * np.float32(0.5))
    q = synth.bf16_round(inp["q"])
    tree = o_build(inp["draft"], inp["roots"], cfg["topk"], N, cfg["max_depth"])
    tgt, _ = synth.target_logits_with_path(seed + 2, tree["parent"], tree["token"], cfg["vocab"])

    def one_step():
        t = o_build(inp["draft"], inp["roots"], cfg["topk"], N, cfg["max_depth"])
        tree_attention(q, k, v, inp["block_table"], inp["prefix"], inp["offsets"], t["parent"].reshape(-1),
                       1.0 / np.sqrt(HEAD_DIM), cfg["hkv"])
        o_accept(t["token"], t["parent"], tgt, cfg["max_depth"])

    for _ in range(warmup):
        one_step()
    steps, t0 = 0, time.perf_counter()
    while True:
        one_step()
        steps += 1
        el = time.perf_counter() - t0
        if el >= budget_s or steps >= max_steps:
            break
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        threads = os.cpu_count() or 1
    return B * N * steps / el, steps, el, threads


# ----------------------------------------------------------------------------------------------
# GPU leg
# ----------------------------------------------------------------------------------------------
def graph_timer(args, stream, flush):
    """Times a callable captured once in a CUDA graph: `steps` replays, each after a 256 MiB write that
    flushes L2 (outside the events), CUDA events on the launching stream.  Returns the per-replay ms."""
    import torch

    def capture(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, capture_error_mode="thread_local"):
            fn()
        return g

    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]

    def timed(g, reps=None):
        for _ in range(3):
            g.replay()
        ms = []
        for _ in range(reps or args.steps):
            flush.zero_()
            ev[0].record(stream)
            g.replay()
            ev[1].record(stream)
            ev[1].synchronize()
            ms.append(ev[0].elapsed_time(ev[1]))
        return ms

    return capture, timed


FP8_SCALES = (1.0 / 128, 1.0 / 64)  # K and V cache scales of the 8-bit legs (N(0, 0.5) values -> codes in +-448)


def attention_leg(name, args, device, capture, timed, pk, fp8=False):
    """Tree attention alone on one of the seeded attention workloads (the inputs the parity tests use); with
    fp8, over the same cache stored as 8-bit E4M3 codes (jf_tree_attention_fp8)."""
    import torch

    from tree_verify_attention_jf_b200 import api, synth, workloads

    inp = workloads.attention_workload(name)
    bf = lambda a: synth.to_bf16_tensor(a).to(device)
    i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)
    q = bf(inp.q)
    if fp8:
        kc = torch.from_numpy(synth.e4m3_cache(inp.k_cache, FP8_SCALES[0])).to(device)
        vc = torch.from_numpy(synth.e4m3_cache(inp.v_cache, FP8_SCALES[1])).to(device)
    else:
        kc, vc = bf(inp.k_cache), bf(inp.v_cache)
    bt, pl, offs, par = i32(inp.block_table), i32(inp.prefix_lens), i32(inp.tree_offsets), i32(inp.parent)
    out = torch.empty_like(q)
    ws = api.AttentionWorkspace(torch.device(device))

    def call():
        if fp8:
            api.tree_attention_fp8(q, kc, vc, FP8_SCALES[0], FP8_SCALES[1], bt, pl, offs, par, inp.sm_scale, out=out,
                                   workspace=ws)
        else:
            api.tree_attention(q, kc, vc, bt, pl, offs, par, inp.sm_scale, out=out, workspace=ws)

    call()
    torch.cuda.synchronize()
    g = capture(call)
    ms = statistics.mean(timed(g))
    del g
    offs_h = [int(x) for x in inp.tree_offsets]
    nodes = [offs_h[b + 1] - offs_h[b] for b in range(inp.batch)]
    prefix = [int(x) for x in inp.prefix_lens]
    pairs = visible_pairs_ragged(inp.parent, offs_h, prefix)
    flops, nbytes = attention_work(nodes, inp.num_q_heads, inp.num_kv_heads, prefix, pairs)
    if fp8:  # the cache's bytes are halved (one byte per element)
        nbytes -= sum(inp.num_kv_heads * (P + n) * HEAD_DIM * 2 for P, n in zip(prefix, nodes))
    tflops = flops / (ms * 1e-3) / 1e12
    gbs = nbytes / (ms * 1e-3) / 1e9
    leg = {"call": "jf_tree_attention_fp8" if fp8 else "jf_tree_attention", "ms": ms, "nodes": sum(nodes), "nodes_per_s": sum(nodes) / (ms * 1e-3),
           "batch": inp.batch, "q_heads": inp.num_q_heads, "kv_heads": inp.num_kv_heads,
           "prefix": prefix if len(prefix) <= 4 else f"{min(prefix)}..{max(prefix)} (mean {statistics.mean(prefix):.0f})",
           "algorithmic_flops": flops, "algorithmic_bytes": nbytes, "tflops": tflops, "gbs": gbs,
           "tensor_frac": tflops / pk["bf16"], "hbm_frac": gbs / pk["hbm"],
           "traffic": attention_traffic(name + ("_fp8" if fp8 else ""))}
    if fp8:
        leg["cache"] = f"E4M3 codes, k_scale {FP8_SCALES[0]}, v_scale {FP8_SCALES[1]}"
    if name in HBM_BOUND:
        leg.update(bound="hbm", frac=gbs / pk["hbm"])
    elif name == "tiny":
        leg.update(bound="latency", latency_us=ms * 1e3)
    else:
        leg.update(bound="tensor", frac=tflops / pk["bf16"])
    return leg


def build_accept_leg(args, device, capture, timed, pk):
    """Tree build and accept walk at batch 8 over the full vocabulary: draft logits fp32 [8, 16, 151936] with a
    planted Zipf-peaked head per row, top-4, budget 256, max depth 16; target logits fp32 [8, 256, 151936] that
    agree with the built tree along a seeded path of length U{1..16}."""
    import torch

    from tree_verify_attention_jf_b200 import api, synth, workloads

    c = workloads.BUILD
    B, depths, V, topk, budget, max_depth = (c["batch"], c["depths"], c["vocab"], c["topk"], c["budget"],
                                             c["max_depth"])
    x_np, roots_np = workloads.build_inputs()
    x = torch.from_numpy(x_np).to(device)
    roots = torch.from_numpy(roots_np).to(device)
    ws = api.build_tree_workspace(B, depths, V, topk, device)
    tree = api.build_tree(x, roots, topk, budget, max_depth, workspace=ws)
    torch.cuda.synchronize()
    par, tok = tree["parent"].cpu().numpy(), tree["token"].cpu().numpy()
    tgt_np, paths = synth.target_logits_with_path(workloads.SEEDS["build_accept"] + 100, par, tok, V)
    tgt = torch.from_numpy(tgt_np).to(device)
    del tgt_np
    acc = dict(accepted_len=torch.empty(B, dtype=torch.int32, device=device),
               path=torch.empty(B, max_depth + 1, dtype=torch.int32, device=device),
               bonus=torch.empty(B, dtype=torch.int32, device=device))

    def build():
        api.build_tree(x, roots, topk, budget, max_depth, workspace=ws, out=tree)

    def accept():
        api.accept(tree["token"], tree["parent"], tgt, max_depth, out=acc)

    build()
    accept()
    torch.cuda.synchronize()
    got = acc["accepted_len"].cpu().tolist()
    if got != [len(p) - 1 for p in paths]:
        raise RuntimeError(f"accept leg: accepted lengths {got} != planted {[len(p) - 1 for p in paths]}")
    gb, ga = capture(build), capture(accept)
    build_ms = statistics.mean(timed(gb))
    accept_ms = statistics.mean(timed(ga))
    del gb, ga
    build_bytes = B * depths * V * 4
    accept_bytes = sum((a + 1) * V * 4 for a in got)  # one target row per node on the walk
    return {
        "build_tree": {"call": "jf_build_tree", "batch": B, "vocab": V, "depths": depths, "topk": topk,
                       "budget": budget, "ms": build_ms, "algorithmic_bytes": build_bytes,
                       "gbs": build_bytes / (build_ms * 1e-3) / 1e9,
                       "hbm_frac": build_bytes / (build_ms * 1e-3) / 1e9 / pk["hbm"],
                       "nodes_per_s": B * budget / (build_ms * 1e-3), "bound": "hbm"},
        "accept": {"call": "jf_accept", "batch": B, "vocab": V, "nodes": budget, "accepted_len": got, "ms": accept_ms,
                   "algorithmic_bytes": accept_bytes, "gbs": accept_bytes / (accept_ms * 1e-3) / 1e9,
                   "hbm_frac": accept_bytes / (accept_ms * 1e-3) / 1e9 / pk["hbm"],
                   "nodes_per_s": B * budget / (accept_ms * 1e-3), "bound": "latency (dependent argmax chain)"},
    }


def frontier_leg(args, device, flush, pk, batch=8, width=32, topk=4, budget=256, max_depth=16, rounds_before=4):
    """jf_expand_frontier (per-node draft logits) at batch 8 over the full vocabulary: one round in the middle of a
    256-node tree (after `rounds_before` rounds, a frontier of `width` nodes), timed from the same saved state each
    time.  Algorithmic bytes: the frontier rows read once (F x V x 4 per sequence)."""
    import torch

    from tree_verify_attention_jf_b200 import api, synth

    V = synth.VOCAB
    roots = torch.arange(1, batch + 1, dtype=torch.int32, device=device)
    tree = api.FrontierTree(batch, budget, topk, device)
    gen = torch.Generator(device=device).manual_seed(77)
    # the draft head's rows for one round: N(0, 2^2) logits (the same random rows every round; each node's own
    # top-k still comes from the row of its frontier position)
    logits = torch.randn((batch, width, V), generator=gen, device=device) * 2.0
    ws = api.expand_frontier_workspace(batch, width, V, device)
    for _ in range(rounds_before):
        api.expand_frontier(logits, roots, tree, max_depth, width, workspace=ws)
    torch.cuda.synchronize()
    nodes = tree.num_nodes.cpu().tolist()
    fb = tree.frontier_begin.cpu().tolist()
    saved = [t.clone() for t in (tree.parent, tree.token, tree.depth, tree.score, tree.num_nodes,
                                 tree.frontier_begin, tree.state)]

    def restore():
        for dst, src in zip((tree.parent, tree.token, tree.depth, tree.score, tree.num_nodes, tree.frontier_begin,
                             tree.state), saved):
            dst.copy_(src)

    stream = torch.cuda.current_stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="thread_local"):
        api.expand_frontier(logits, roots, tree, max_depth, width, workspace=ws)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    ms = []
    for it in range(args.steps + 3):
        restore()
        flush.zero_()
        ev[0].record(stream)
        g.replay()
        ev[1].record(stream)
        ev[1].synchronize()
        if it >= 3:
            ms.append(ev[0].elapsed_time(ev[1]))
    del g
    t = statistics.mean(ms)
    rows = [n - f for n, f in zip(nodes, fb)]
    nbytes = sum(rows) * V * 4
    added = [a - n for a, n in zip(tree.num_nodes.cpu().tolist(), nodes)]
    return {"call": "jf_expand_frontier", "batch": batch, "vocab": V, "topk": topk, "budget": budget,
            "width": width, "round": rounds_before + 1, "frontier_rows": rows, "nodes_added": added, "ms": t,
            "algorithmic_bytes": nbytes, "gbs": nbytes / (t * 1e-3) / 1e9,
            "hbm_frac": nbytes / (t * 1e-3) / 1e9 / pk["hbm"], "nodes_per_s": sum(added) / (t * 1e-3),
            "bound": "hbm", "timing": "CUDA graph replay from the saved state, L2 flushed (row statistics + expansion)"}


def run_gpu(args, cfg, rank, world, device):
    import torch

    from tree_verify_attention_jf_b200 import api, synth

    torch.cuda.set_device(device)
    seed = rank_seed(rank)
    inp = make_inputs(cfg, seed)
    B, N, V = cfg["batch"], cfg["budget"], cfg["vocab"]
    gen = torch.Generator(device=device).manual_seed(seed)
    kc = (torch.randn(inp["kv_shape"], generator=gen, device=device) * 0.5).to(torch.bfloat16)
    vc = (torch.randn(inp["kv_shape"], generator=gen, device=device) * 0.5).to(torch.bfloat16)
    i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)
    draft_h = torch.from_numpy(inp["draft"]).pin_memory()
    roots = i32(inp["roots"])
    q_h = torch.from_numpy(inp["q"]).to(torch.bfloat16).pin_memory()
    draft = draft_h.to(device)
    q = q_h.to(device)
    bt, prefix, offs = i32(inp["block_table"]), i32(inp["prefix"]), i32(inp["offsets"])
    out = torch.empty_like(q)
    ws_attn = api.AttentionWorkspace(torch.device(device))
    ws_build = api.build_tree_workspace(B, cfg["depths"], V, cfg["topk"], device)
    tree = api.build_tree(draft, roots, cfg["topk"], N, cfg["max_depth"], workspace=ws_build)
    torch.cuda.synchronize()
    par_h, tok_h = tree["parent"].cpu().numpy(), tree["token"].cpu().numpy()
    # Target logits that agree with this tree along a seeded path (the tree is fixed by the seeded draft
    # logits; it is read back once, outside any timed region, only to plant the path).
    tgt_np, paths = synth.target_logits_with_path(seed + 2, par_h, tok_h, V)
    tgt_h = torch.from_numpy(tgt_np).pin_memory()
    tgt = tgt_h.to(device)
    del tgt_np
    acc_out = dict(accepted_len=torch.empty(B, dtype=torch.int32, device=device),
                   path=torch.empty(B, cfg["max_depth"] + 1, dtype=torch.int32, device=device),
                   bonus=torch.empty(B, dtype=torch.int32, device=device))
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    capture, timed = graph_timer(args, stream, flush)

    def build():
        api.build_tree(draft, roots, cfg["topk"], N, cfg["max_depth"], workspace=ws_build, out=tree)

    def attention():
        api.tree_attention(q, kc, vc, bt, prefix, offs, tree["parent"].view(-1), 1.0 / np.sqrt(HEAD_DIM), out=out,
                           workspace=ws_attn)

    def accept():
        api.accept(tree["token"], tree["parent"], tgt, cfg["max_depth"], out=acc_out)

    def step():
        build()
        attention()
        accept()

    # the next row after the step: commit the accepted path's K/V into the cache (timed on its own; it rewrites
    # a few slots of kc/vc in place, which changes no timing)
    new_prefix = torch.empty_like(prefix)

    def commit():
        api.commit_kv(kc, vc, bt, prefix, offs, acc_out["path"], acc_out["accepted_len"], new_prefix_lens=new_prefix)

    # and the row before attention: the tree tokens' K/V (synthetic projections) written into the cache with rotary
    # positions, q rotated in place (timed on its own)
    k_new = (torch.randn((B * N, cfg["hkv"], HEAD_DIM), generator=gen, device=device) * 0.5).to(torch.bfloat16)
    v_new = (torch.randn((B * N, cfg["hkv"], HEAD_DIM), generator=gen, device=device) * 0.5).to(torch.bfloat16)

    def append():
        api.tree_kv_append(k_new, v_new, kc, vc, bt, prefix, offs, tree["depth"].view(-1), ROPE_THETA, q=q)

    # eager warm-up (loads the library, sets kernel attributes), then one CUDA graph per timed region:
    # the whole step, and each of its three calls alone for the per-kernel times
    step()
    torch.cuda.synchronize()
    graphs = {name: capture(fn) for name, fn in (("step", step), ("build_tree", build), ("tree_attention", attention),
                                                 ("accept", accept), ("commit_kv", commit),
                                                 ("tree_kv_append", append))}
    for _ in range(args.warmup):
        graphs["step"].replay()
    torch.cuda.synchronize()
    expect_len = [len(p) - 1 for p in paths]
    got_len = acc_out["accepted_len"].cpu().tolist()
    if got_len != expect_len:
        raise RuntimeError(f"accepted lengths {got_len} != planted {expect_len}")

    # ---- timed region: K graph replays of the whole step, L2 flushed between steps (outside the events)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    barrier(world)
    torch.cuda.synchronize()
    import tempfile
    clocks_dir = args.clocks_dir or tempfile.gettempdir()
    sampler = NvmlSampler(torch.cuda.get_device_properties(device).uuid,
                          os.path.join(clocks_dir, f"jf_clocks_r{rank}.csv"))
    step_ms = []
    for _ in range(args.steps):
        flush.zero_()
        ev[0].record(stream)
        graphs["step"].replay()
        ev[1].record(stream)
        ev[1].synchronize()
        step_ms.append(ev[0].elapsed_time(ev[1]))
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop()
    # then each call alone, for the per-kernel times
    build_ms = timed(graphs["build_tree"])
    attn_ms = timed(graphs["tree_attention"])
    accept_ms = timed(graphs["accept"])
    commit_ms = timed(graphs["commit_kv"])
    append_ms = timed(graphs["tree_kv_append"])
    torch.cuda.synchronize()
    del graphs

    # ---- e2e: the same step through the public API with host buffers; H2D of the step's inputs
    # (draft logits, tree queries, target logits) from pinned memory and D2H of its result inside
    res_h = torch.empty(B * (cfg["max_depth"] + 3), dtype=torch.int32).pin_memory()
    e2e_ms = []
    e_s, e_e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_e2e = max(3, min(args.steps, 20))
    for _ in range(n_e2e):
        flush.zero_()
        e_s.record(stream)
        draft.copy_(draft_h, non_blocking=True)
        q.copy_(q_h, non_blocking=True)
        tgt.copy_(tgt_h, non_blocking=True)
        step()
        res = torch.cat([acc_out["accepted_len"], acc_out["bonus"], acc_out["path"].view(-1)])
        res_h.copy_(res, non_blocking=True)
        e_e.record(stream)
        e_e.synchronize()
        e2e_ms.append(e_s.elapsed_time(e_e))
    h2d = draft_h.numel() * 4 + q_h.numel() * 2 + tgt_h.numel() * 4
    d2h = res_h.numel() * 4
    r = dict(step_ms=step_ms, attn_ms=attn_ms, build_ms=build_ms, accept_ms=accept_ms, commit_ms=commit_ms,
             append_ms=append_ms, clocks=clocks, accepted=acc_out["accepted_len"].cpu().tolist(),
             e2e_ms=e2e_ms, h2d=h2d, d2h=d2h, parent=par_h, prefix=inp["prefix"])
    del tgt, tgt_h, draft, q, kc, vc, k_new, v_new
    torch.cuda.empty_cache()

    # ---- the other workloads' calls, each alone (rank 0 of a single-GPU run only)
    if world == 1 and not args.no_legs:
        pk = peaks()
        legs = {}
        for name in ("qwen3_8b", "serving", "tiny"):
            if name != args.workload:
                legs[name] = attention_leg(name, args, device, capture, timed, pk)
                torch.cuda.empty_cache()
        # the serving batch over an 8-bit (E4M3) cache: half the cache bytes
        legs["serving_fp8"] = attention_leg("serving", args, device, capture, timed, pk, fp8=True)
        torch.cuda.empty_cache()
        legs.update(build_accept_leg(args, device, capture, timed, pk))
        torch.cuda.empty_cache()
        legs["expand_frontier"] = frontier_leg(args, device, flush, pk)
        torch.cuda.empty_cache()
        r["legs"] = legs
    return r


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world, device):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="jf", choices=["jf", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-legs", action="store_true", help="skip the other workloads' calls timed after the step")
    ap.add_argument("--clocks-dir", default=None, help="where the nvidia-smi clock samples of the timed region go "
                    "(default: the system temporary directory)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    cfg = WORKLOADS[args.workload]
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    metric = "tree nodes verified/sec"
    config = {"workload": f"{args.workload}_tree_verify", "batch": cfg["batch"], "q_heads": cfg["hq"],
              "kv_heads": cfg["hkv"], "head_dim": HEAD_DIM,
              "prefix": (f"U[{cfg['prefix'][0]},{cfg['prefix'][1]}]" if isinstance(cfg["prefix"], tuple)
                         else cfg["prefix"]), "page_size": PAGE,
              "budget": cfg["budget"], "topk": cfg["topk"], "max_depth": cfg["max_depth"], "vocab": cfg["vocab"],
              "step": "build_tree + tree_attention (one layer) + accept", "parallelism": f"replicas{world}",
              "l2": "flushed between steps (256 MiB write outside the timed events)",
              "launch": "one CUDA graph per step (host launch overhead outside the device timing)"}

    if args.impl == "reference":
        if rank != 0:
            return
        # each step is the oracle over one sequence of the workload (the whole workload when B = 1), so that
        # the whole --steps K --warmup W run stays within minutes; exactly K steps are timed after W
        sample_cfg = dict(cfg, batch=1)
        rate, steps, el, threads = oracle_step_rate(sample_cfg, rank_seed(0), budget_s=float("inf"),
                                                    max_steps=args.steps, warmup=args.warmup)
        what = "whole step(s)" if cfg["batch"] == 1 else f"step(s) of one sequence of the {cfg['batch']}"
        line = {"impl": "reference", "metric": metric, "value": rate, "unit": "nodes/s", "n_gpus": args.gpus,
                "steps": steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
                "config": config,
                "cpu_baseline": {"value": rate, "unit": "nodes/s", "cores": threads, "kind": "oracle",
                                 "sample": f"{steps} timed {what} (build + attention + accept) after "
                                           f"{args.warmup} untimed, {el:.1f} s"},
                "e2e": {"value": rate, "unit": "nodes/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    import torch
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    device = f"cuda:{local}"
    r = run_gpu(args, cfg, rank, world, device)
    mean_step = statistics.mean(r["step_ms"])
    step_ms = max_over_ranks(mean_step, world, device)
    e2e_step = max_over_ranks(statistics.mean(r["e2e_ms"]), world, device)
    attn_ms = statistics.mean(r["attn_ms"])
    B, N = cfg["batch"], cfg["budget"]
    pk = peaks()
    prefixes = [int(x) for x in r["prefix"]]
    pairs = visible_pairs(r["parent"], prefixes)
    flops, nbytes = attention_work([N] * B, cfg["hq"], cfg["hkv"], prefixes, pairs)
    tflops = flops / (attn_ms * 1e-3) / 1e12
    gbs = nbytes / (attn_ms * 1e-3) / 1e9
    shares = {"build_tree": statistics.mean(r["build_ms"]) / mean_step,
              "tree_attention": attn_ms / mean_step, "accept": statistics.mean(r["accept_ms"]) / mean_step}
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    if rank != 0:
        return
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        # a bounded sample: whole steps of one sequence of the workload for about 15 s of CPU work
        sample_cfg = dict(cfg, batch=1)
        rate, steps, el, threads = oracle_step_rate(sample_cfg, rank_seed(0))
        what = "whole step(s)" if cfg["batch"] == 1 else f"step(s) of one sequence of the {cfg['batch']}"
        cpu = {"value": rate, "unit": "nodes/s", "cores": threads, "kind": "oracle",
               "sample": f"{steps} {what} of the same workload (build + attention + accept), {el:.1f} s"}
    line = {
        "metric": metric, "value": job_nodes_per_sec(B, N, world, step_ms), "unit": "nodes/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded)", "config": config,
        "roofline": roofline(args.workload, tflops, gbs, pk, flops, nbytes),
        "kernel_ms": {"build_tree": statistics.mean(r["build_ms"]), "tree_attention": attn_ms,
                      "accept": statistics.mean(r["accept_ms"])},
        # the next rows, outside the step: jf_commit_kv of the accepted path (2 * L * Hkv * 256 bytes moved per
        # sequence, read and written once) and the tree K/V append (k_new, v_new read and written, q read and
        # written, bf16)
        "next_rows": {"commit_kv_ms": statistics.mean(r["commit_ms"]), "accepted_len": r["accepted"],
                      "commit_bytes": sum(2 * 2 * a * cfg["hkv"] * HEAD_DIM * 2 for a in r["accepted"]),
                      "tree_kv_append_ms": statistics.mean(r["append_ms"]),
                      "tree_kv_append_bytes": B * N * (4 * cfg["hkv"] + 2 * cfg["hq"]) * HEAD_DIM * 2},
        "time_share": shares,
        "legs": r.get("legs"),
        "e2e": {"value": job_nodes_per_sec(B, N, world, e2e_step), "unit": "nodes/s", "h2d_bytes_per_step": r["h2d"],
                "d2h_bytes_per_step": r["d2h"]},
        "gpu_launches": LAUNCHES_PER_STEP * args.steps,
        "clocks": r["clocks"],
        "cpu_baseline": cpu,
    }
    print(json.dumps(line))


if __name__ == "__main__":
    main()
