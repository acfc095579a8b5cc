#!/usr/bin/env python
"""Per-denoise-step block-diffusion attention benchmark (FlashBlock / LoSA).

Workload: the dLLM configuration (bf16, batch 1, 32 heads MHA, d=128, frozen
prefix of 32768 tokens, block of 32 tokens denoised over 32 steps, Poisson(2)
row updates per step, tau=4), synthetic and seeded. One bench step is one
whole block: 32 denoise steps of attention (prefix partial when needed,
block partial, merge). Inputs are resident in HBM before timing; L2 is flushed
between denoise steps, outside the timed events: a 256 MiB write, then a read of
another 256 MiB buffer, so the write's dirty lines are written back before the
timed step rather than during it.

Modes, each timed over the same K blocks:
  reuse  FlashBlock threshold reuse (tau=4) through fb_step: the headline value
  dense  tau = 0 through fb_step: the prefix partial recomputed every step and
         merged with the in-block partial (dense block-diffusion attention);
         the prefix call alone (fb_prefix_attn) is also timed, for its GB/s
  losa   LoSA (4 active rows, top-256 of 2048 pages) through fb_step
  sparse_residual  FlashBlock + sparse attention (20% of pages per kv head,
         residual of the rest cached, tau=4) through fb_step
  block_commit     fb_block_commit of one block's rows (into a separate cache)

value = microseconds per denoise step of the whole job (max over ranks of the
device time / denoise steps of all ranks). With N GPUs every rank runs its own
replica (weak scaling; the path has no exchange step).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "µs per denoise-step attention & prefix HBM GB/s (dense vs reuse vs LoSA)"
UNIT = "µs"
WORKLOAD = ("dllm: bf16, batch 1, 32 heads MHA, head_dim 128, prefix 32768 tokens, block 32, "
            "32 denoise steps per block, Poisson(2) updates, tau 4; LoSA 4 active rows, top-256 pages")
FLUSH_BYTES = 256 << 20
LOSA_ACTIVE, LOSA_TOPK = 4, 256
SR_DENSITY_PCT = 20  # sparse-residual mode: selected pages per kv head, percent
ORACLE_HEADS = 4  # oracle sample: this many of the 32 heads, scaled to all heads
BASELINE_HEADS, BASELINE_BLOCKS = 8, 2  # CPU baseline sample of our arm (about 10 s)


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20, help="timed blocks of 32 denoise steps")
    p.add_argument("--warmup", type=int, default=3, help="untimed blocks before timing")
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--mode", choices=["all", "reuse", "dense", "losa", "sparse_residual",
                                      "prefix", "block", "losa_step", "sr_step"],
                   default="all",
                   help="all: the contract line; reuse/dense/losa/sparse_residual: time only "
                   "that mode; prefix/block/losa_step/sr_step: run only that call eagerly, untimed "
                   "(for profilers)")
    p.add_argument("--sweep", action="store_true",
                   help="long-context sweep instead of the contract line: dense vs reuse per "
                   "denoise step over prefixes of 32k..800k tokens (one JSON line per length)")
    p.add_argument("--workload", choices=["dllm", "tiny", "gqa", "video", "losa"],
                   default="dllm", help="dllm is the contract workload; the others are for "
                   "the per-configuration table")
    return p.parse_args()


# ---------------------------------------------------------------------------
# distributed plumbing (one process per GPU; only barriers and a MAX reduce)
# ---------------------------------------------------------------------------
def dist_init(n_gpus):
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    import torch
    import torch.distributed as dist
    if world > 1:
        dist.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def max_over_ranks(x, world):
    """Maximum of a per-rank host value over all ranks (NCCL reduces device
    tensors; gloo, used by the CPU tests, host tensors)."""
    import torch
    import torch.distributed as dist
    if world == 1:
        return x
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        # raw samples: FB_CLOCKS_DIR if set, else the temporary directory
        import tempfile
        out_dir = os.environ.get("FB_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(out_dir, f"clocks_gpu{gpu_index}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        load = [r for r in rows if r[2] > 250.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in load for i in range(4) if r[3][i].lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in load),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows), "samples_under_load": len(load)}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
# Sources of the kernels the dllm prefix call launches (split-KV attention and
# combine); a traffic record is valid only for the sources it was taken on.
PREFIX_KERNEL_SOURCES = ("attn.cuh", "common.cuh")


def kernel_source_hash():
    h = hashlib.sha256()
    d = os.path.join(ROOT, "block_diffusion_attention_fb_b200", "csrc")
    for name in PREFIX_KERNEL_SOURCES:
        with open(os.path.join(d, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def profiled_traffic():
    """dram bytes per launch of the prefix call from the committed ncu summary,
    if it was taken on the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", "prefix_attn_dllm_traffic.txt")
    if not os.path.exists(path):
        return None
    kv = {}
    for line in open(path):
        if ":" in line and not line.startswith("#"):
            k, v = line.split(":", 1)
            kv[k.strip()] = v.strip()
    if kv.get("kernel_sources_sha256_16") != kernel_source_hash():
        return None
    try:
        return int(kv["dram_bytes_per_call"])
    except (KeyError, ValueError):
        return None


def measured_peaks():
    """HBM copy bandwidth and bf16 GEMM throughput measured on this machine's
    B200s (MEASURED_PEAKS.json), else the earlier measurement's fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    out = {"gbs": 6650.0, "tflops": 1590.0, "kind": "fallback"}
    if os.path.exists(path):
        try:
            j = json.load(open(path))
            out = {"gbs": float(j["hbm_gbs"]), "tflops": float(j["bf16_tflops"]),
                   "kind": "measured"}
        except (ValueError, KeyError):
            pass
    out["ridge"] = out["tflops"] * 1e12 / (out["gbs"] * 1e9)
    return out


def run_ours(args, rank, world, local):
    import torch

    import block_diffusion_attention_fb_b200 as fb
    from block_diffusion_attention_fb_b200.runtime import BlockAttention, HostBlockPipeline
    from workloads import make_workload
    from workloads.torch_io import prefix_tensors, to_torch

    fb.load_library()
    wl = make_workload(args.workload)
    sp = wl.spec
    S = sp.steps
    dt = sp.dtype
    t = prefix_tensors(wl.prefix, dt)
    kv = fb.KV(t["k"], t["v"], seq_len=t["seq_len"], page_table=t["page_table"],
               page_size=t["page_size"], max_seq_len=t["max_seq_len"])
    steps = list(wl.steps())
    dq = [to_torch(x.q, dt) for x in steps]
    dk = [to_torch(x.k_in, dt) for x in steps]
    dv = [to_torch(x.v_in, dt) for x in steps]
    hq = [to_torch(x.q, dt, "cpu", pin=True) for x in steps]
    hk = [to_torch(x.k_in, dt, "cpu", pin=True) for x in steps]
    hv = [to_torch(x.v_in, dt, "cpu", pin=True) for x in steps]
    ms = [x.m_updated.tolist() for x in steps]
    batch, B, Hq, d = sp.batch, sp.block, sp.n_heads_q, sp.head_dim
    A = torch.zeros(batch, B, Hq, d, device="cuda")
    L = torch.zeros(batch, B, Hq, device="cuda")
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    flush_rd = torch.zeros(FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    def flush_l2():
        flush.zero_()
        flush_rd.max()

    if sp.gamma is not None:
        reuse = BlockAttention(kv, B, Hq, "per_head", gamma=sp.gamma)
        reuse_desc = f"FlashBlock per-head reuse (gamma={sp.gamma})"
    else:
        tau = sp.tau if sp.tau is not None else 4  # the losa spec states no tau
        reuse = BlockAttention(kv, B, Hq, "threshold", tau=tau)
        reuse_desc = f"FlashBlock threshold reuse (tau={tau})"
    # dense baseline: the same controller with tau = 0 (recompute every step)
    dense = BlockAttention(kv, B, Hq, "threshold", tau=0)
    n_act = sp.n_active or LOSA_ACTIVE
    topk = sp.topk_pages or LOSA_TOPK
    losa = BlockAttention(kv, B, Hq, "losa", n_active=n_act, topk_pages=topk)
    # FlashBlock + sparse residual: 20% page density (the pages pair FlashBlock
    # with SparseD at 20-40%); supported up to 64 stacked rows per kv head
    sr_topk = max(1, -(-kv.n_pages * SR_DENSITY_PCT // 100))
    sr_tau = sp.tau if sp.tau is not None else 4
    sres = (BlockAttention(kv, B, Hq, "sparse_residual", tau=sr_tau, topk_pages=sr_topk)
            if B * (Hq // sp.n_heads_kv) <= 64 else None)
    # block commit: a separate contiguous cache with room for every timed
    # commit (the commit reads only the block rows, so its content is not needed)
    commit = None
    if wl.prefix.page_table is None:
        n_commits = max(1, args.warmup) + args.steps
        cap = int(wl.prefix.max_seq_len) + n_commits * S * B
        ck = torch.empty(batch * cap, sp.n_heads_kv, d, dtype=dk[0].dtype, device="cuda")
        cv = torch.empty_like(ck)
        clen = torch.from_numpy(wl.prefix.seq_len.astype("int32")).cuda()
        ckv = fb.KV(ck, cv, seq_len=clen, page_table=None, page_size=t["page_size"],
                    max_seq_len=cap)
        cmin = torch.empty(batch, ckv.n_pages, sp.n_heads_kv, d, dtype=dk[0].dtype, device="cuda")
        cmax = torch.empty_like(cmin)
        commit = {"kv": ckv, "min": cmin, "max": cmax,
                  "len": wl.prefix.seq_len.astype("int32").copy()}
    a_out = torch.zeros(batch, B, Hq, d, device="cuda")
    l_out = torch.zeros(batch, B, Hq, device="cuda")
    a_in = torch.zeros_like(a_out)
    l_in = torch.zeros_like(l_out)
    ws = torch.empty(fb.fb_workspace_size(kv, B, Hq), dtype=torch.uint8, device="cuda")

    def ev():
        return torch.cuda.Event(enable_timing=True)

    def reuse_step(s):
        if s == 0:
            reuse.reset()
        reuse.step(dq[s], dk[s], dv[s], A, L, m_updated=ms[s])

    def prefix_call(s):
        fb.fb_prefix_attn(dq[s], kv, a_out, l_out, ws)

    def dense_step(s):
        if s == 0:
            dense.reset()
        dense.step(dq[s], dk[s], dv[s], A, L, m_updated=ms[s])

    def losa_step(s):
        if s == 0:
            losa.reset()
        losa.step(dq[s], dk[s], dv[s], A, L)

    def sres_step(s):
        if s == 0:
            sres.reset()
        sres.step(dq[s], dk[s], dv[s], A, L, m_updated=ms[s])

    def commit_call(s):
        fb.fb_block_commit(commit["kv"], commit["len"], dk[s], dv[s], commit["min"], commit["max"])
        commit["len"] += B


    # end to end: each step's q/k/v packed in pinned host memory, A_full/L_full
    # returned to pinned host memory, copies overlapped with attention on their
    # own streams (runtime.HostBlockPipeline), one CUDA graph per block
    e2e_blk = (BlockAttention(kv, B, Hq, "per_head", gamma=sp.gamma) if sp.gamma is not None
               else BlockAttention(kv, B, Hq, "threshold",
                                   tau=sp.tau if sp.tau is not None else 4))
    pipe = HostBlockPipeline(e2e_blk, dq[0].dtype, depth=3)
    host_in = [pipe.pack_inputs(hq[s], hk[s], hv[s]) for s in range(S)]
    host_out = [pipe.new_output() for _ in range(S)]

    def e2e_block():
        pipe.enqueue_block(host_in, host_out, ms)

    K, W = args.steps, args.warmup
    if args.mode in ("prefix", "block", "losa_step", "sr_step"):  # eager, for profilers
        if args.mode == "sr_step" and sres is None:
            raise SystemExit("sr_step: the sparse-residual mode takes at most 64 stacked rows "
                             "per kv head")
        for _ in range(W + K):
            for s in range(S):
                flush_l2()
                if args.mode == "prefix":
                    prefix_call(s)
                elif args.mode == "block":
                    fb.fb_block_attn(dq[s], dk[s], dv[s], a_in, l_in)
                elif args.mode == "losa_step":
                    losa_step(s)
                else:
                    sres_step(s)
        torch.cuda.synchronize()
        fb.fb_device_status()
        if rank == 0:
            print(json.dumps({"mode": args.mode, "calls": (W + K) * S}))
        return
    # warm-up of every path (eager, untimed): also sets kernel attributes
    for _ in range(max(1, W)):
        for s in range(S):
            reuse_step(s)
            prefix_call(s)
            dense_step(s)
            losa_step(s)
            if sres is not None:
                sres_step(s)
            if commit is not None:
                commit_call(s)
        e2e_block()
    torch.cuda.synchronize()

    # one CUDA graph per denoise step: the host decisions (tau, LoSA step
    # index) are taken at capture, as a sampler picks a pre-captured variant
    def capture(fn):
        graphs = []
        for s in range(S):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                fn(s)
            graphs.append(g)
        return graphs

    n0 = fb.fb_kernel_launches()
    g_reuse = capture(reuse_step)
    launches_per_block = fb.fb_kernel_launches() - n0
    g_prefix = capture(prefix_call)
    g_dense = capture(dense_step)
    g_losa = capture(losa_step)
    g_e2e = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_e2e):
        e2e_block()
    g_sres = capture(sres_step) if sres is not None else None
    rec = sum(1 for s in range(S) if s == 0 or (sp.gamma is None and ms[s][0] >= reuse.policy.tau))

    def timed(graph_lists, n_blocks, timed_flag=True):
        """Replays n_blocks blocks; returns device ms of each graph list's steps."""
        pairs = [[] for _ in graph_lists]
        stream = torch.cuda.current_stream()
        for _ in range(n_blocks):
            for s in range(S):
                flush_l2()
                for gi, gl in enumerate(graph_lists):
                    e0, e1 = ev(), ev()
                    e0.record(stream)
                    gl[s].replay()
                    e1.record(stream)
                    pairs[gi].append((e0, e1))
        torch.cuda.synchronize()
        return [sum(a.elapsed_time(b) for a, b in p) for p in pairs], pairs

    def eager(fn, n_blocks):
        pairs = []
        stream = torch.cuda.current_stream()
        for _ in range(n_blocks):
            for s in range(S):
                flush_l2()
                e0, e1 = ev(), ev()
                e0.record(stream)
                fn(s)
                e1.record(stream)
                pairs.append((e0, e1))
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in pairs)

    def back_to_back_time(fn, n_blocks):
        stream = torch.cuda.current_stream()
        flush_l2()  # also gives the host a head start on enqueueing
        e0, e1 = ev(), ev()
        e0.record(stream)
        for _ in range(n_blocks):
            for s in range(S):
                fn(s)
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    for gl in (g_reuse, g_losa):
        timed([gl], 1)
    timed([g_prefix], 1)
    timed([g_dense], 1)
    if args.mode != "all":
        lists = {"reuse": [g_reuse], "dense": [g_dense], "losa": [g_losa],
                 "sparse_residual": [g_sres]}[args.mode]
        barrier(world)
        tot, _ = timed(lists, K)
        barrier(world)
        if rank == 0:
            print(json.dumps({"mode": args.mode, "us_per_step": sum(tot) * 1000 / (K * S)}))
        return

    clocks = ClockSampler(local)
    barrier(world)
    clocks.start()
    barrier(world)
    (t_reuse,), _ = timed([g_reuse], K)
    barrier(world)
    (t_dense,), _ = timed([g_dense], K)
    barrier(world)
    (t_prefix,), _ = timed([g_prefix], K)
    barrier(world)
    (t_losa,), _ = timed([g_losa], K)
    barrier(world)
    t_sres = timed([g_sres], K)[0][0] if g_sres is not None else None
    barrier(world)
    # block commit: one call per denoise step's block rows, eager, L2 flushed before
    t_commit = eager(commit_call, K) if commit is not None else None
    barrier(world)
    # one whole block per timed iteration, L2 flushed between blocks
    e2e_pairs = []
    for _ in range(K):
        flush_l2()
        e0, e1 = ev(), ev()
        e0.record()
        g_e2e.replay()
        e1.record()
        e2e_pairs.append((e0, e1))
    torch.cuda.synchronize()
    t_e2e = sum(a.elapsed_time(b) for a, b in e2e_pairs)
    barrier(world)
    # the roofline of the dominant kernel call, the dense prefix partial
    kv_bytes = 2 * int(wl.prefix.seq_len.sum()) * sp.n_heads_kv * d * (2 if dt == "bf16" else 4)
    io_bytes = batch * B * Hq * d * (2 if dt == "bf16" else 4) + batch * B * Hq * (d + 1) * 4
    alg_bytes = kv_bytes + io_bytes
    flops = 4.0 * int(wl.prefix.seq_len.sum()) * B * Hq * d
    peaks = measured_peaks()
    # bound by arithmetic intensity against the measured ridge point
    # (bf16 TFLOP/s over HBM GB/s, about 250 flop per byte)
    tensor_bound = flops / alg_bytes > peaks["ridge"] and dt == "bf16"
    # the roofline's kernel time: the prefix call launched eagerly (attention
    # kernel + split combine), an L2 flush before each call outside the events
    # (the flush keeps the stream busy while the host enqueues, so the events
    # bracket device work only), against the burst peaks. An HBM-bound call
    # whose K/V is at least twice the L2 also runs back to back between one
    # pair of events (each call evicts what the previous one left, so none
    # starts warm), which leaves out the first-access cost after a flush; that
    # time is the one reported. Tensor-bound calls keep the per-call figure: run
    # back to back they settle under the power cap, which the burst GEMM peak
    # they are compared with does not.
    t_prefix_flushed = eager(prefix_call, K)
    l2_bytes = int(getattr(torch.cuda.get_device_properties(0), "L2_cache_size", 0)) or (126 << 20)
    back_to_back = kv_bytes >= 2 * l2_bytes and not tensor_bound
    t_prefix_kernel = back_to_back_time(prefix_call, K) if back_to_back else t_prefix_flushed
    barrier(world)
    clk = clocks.stop()

    # Quality of the cheap modes against dense attention on the same block
    # (reported, not asserted: the pages give no number to hold it to). One
    # untimed block per mode; A_full compared per denoise step.
    def collect(step_fn):
        outs = []
        for s in range(S):
            step_fn(s)
            outs.append(A.clone())
        return outs

    def dense_full(s):
        prefix_call(s)
        fb.fb_block_attn(dq[s], dk[s], dv[s], a_in, l_in)
        fb.fb_merge(a_out, l_out, a_in, l_in, A, L)

    ref_outs = collect(dense_full)
    quality = {}
    for qname, fn in (("reuse", reuse_step), ("losa", losa_step),
                      ("sparse_residual", sres_step if sres is not None else None)):
        if fn is None:
            continue
        outs = collect(fn)
        diffs = [(o - r).abs() for o, r in zip(outs, ref_outs)]
        quality[qname] = {"max_abs_vs_dense": round(max(float(x.max()) for x in diffs), 5),
                          "mean_abs_vs_dense": round(sum(float(x.mean()) for x in diffs) / S, 6)}
    torch.cuda.synchronize()
    fb.fb_device_status()

    n_steps_all = K * S * world
    t_reuse_max = max_over_ranks(t_reuse, world)
    t_dense_max = max_over_ranks(t_dense, world)
    t_losa_max = max_over_ranks(t_losa, world)
    t_sres_max = max_over_ranks(t_sres, world) if t_sres is not None else None
    t_commit_max = max_over_ranks(t_commit, world) if t_commit is not None else None
    t_e2e_max = max_over_ranks(t_e2e, world)
    us = lambda ms_total: ms_total * 1000.0 / n_steps_all  # noqa: E731

    prefix_avg_ms = t_prefix / (K * S)
    kernel_avg_ms = max_over_ranks(t_prefix_kernel, world) / (K * S)
    flushed_avg_ms = max_over_ranks(t_prefix_flushed, world) / (K * S)  # every rank joins
    achieved = alg_bytes / (prefix_avg_ms * 1e-3) / 1e9
    if tensor_bound:
        k_ach, k_peak, k_unit = flops / (kernel_avg_ms * 1e-3) / 1e12, peaks["tflops"], "TFLOP/s"
    else:
        k_ach, k_peak, k_unit = alg_bytes / (kernel_avg_ms * 1e-3) / 1e9, peaks["gbs"], "GB/s"
    traffic = profiled_traffic() if args.workload == "dllm" else None
    if rank != 0:
        return
    line = {
        "metric": METRIC,
        "value": round(us(t_reuse_max), 3),
        "unit": UNIT,
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": round(t_reuse_max / K, 4),
        "higher_is_better": False,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": dt,
        "data": "synthetic (seeded generator; no model weights or datasets)",
        "config": {
            "workload": WORKLOAD if args.workload == "dllm" else args.workload,
            "global_batch": world * batch,
            "seq_len": int(wl.prefix.max_seq_len),
            "block": B,
            "denoise_steps_per_bench_step": S,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "flushed between denoise steps (256 MiB write, then 256 MiB read of another buffer; outside the timed events)",
            "value_mode": f"reuse: {reuse_desc} through fb_step, one CUDA graph per denoise step",
        },
        "modes": {
            "reuse": {"us_per_step": round(us(t_reuse_max), 3),
                      "prefix_recomputes_per_block": rec if sp.gamma is None else None},
            "dense": {"us_per_step": round(us(t_dense_max), 3),
                      "via": "fb_step with tau=0: prefix partial every step, merge fused "
                             "into the in-block kernel",
                      "prefix_call_us": round(prefix_avg_ms * 1000, 3),
                      "prefix_gbs": round(achieved, 1),
                      "prefix_tflops": round(flops / (prefix_avg_ms * 1e-3) / 1e12, 1)},
            "sparse_residual": ({"us_per_step": round(us(t_sres_max), 3), "tau": sr_tau,
                                 "topk_pages": sr_topk, "of_pages": kv.n_pages}
                                if t_sres_max is not None else None),
            "block_commit": ({"us_per_call": round(us(t_commit_max), 3),
                              "bytes_per_call": 2 * batch * B * sp.n_heads_kv * d * dk[0].element_size()}
                             if t_commit_max is not None else None),
            "losa": {"us_per_step": round(us(t_losa_max), 3), "n_active": n_act,
                     "topk_pages": topk},
        },
        "quality": quality,
        "tokens_per_s": round(world * K * batch * B / (t_reuse_max * 1e-3), 1),
        # context, not a target: the pages' own dense-vs-FlashBlock figures (end to
        # end in a model, hardware not stated) beside this run's per-step ratio
        "context": {
            "dense_over_reuse_attention_time": round(t_dense_max / t_reuse_max, 2),
            "pages": "FlashBlock vs dense block diffusion: up to 1.6x lower attention time, "
                     "up to 1.44x token throughput (312 -> 451 tokens/s); hardware not stated",
        },
        "roofline": {
            "bound": "tensor" if tensor_bound else "hbm",
            "kernel": "fb_prefix_attn (split-KV attention + combine), dense prefix, eager launch",
            "kernel_us": round(kernel_avg_ms * 1000, 3),
            "timing": (f"{K * S} calls back to back between two events (inputs "
                       f"{kv_bytes / l2_bytes:.1f}x the L2, no flush)" if back_to_back
                       else "L2 flushed before each call, outside the events"),
            "kernel_us_l2_flushed_each_call": round(flushed_avg_ms * 1000, 3),
            "achieved": round(k_ach, 1),
            "peak": k_peak,
            "peak_kind": peaks["kind"] + (" (cuBLAS bf16 GEMM, burst)" if tensor_bound
                                          else " (copy bandwidth, burst)"),
            "unit": k_unit,
            "frac": round(k_ach / k_peak, 4),
            "algorithmic_bytes_per_call": alg_bytes,
            "algorithmic_flops_per_call": flops,
            "traffic": traffic,
        },
        "e2e": {
            "value": round(us(t_e2e_max), 3),
            "unit": UNIT,
            "h2d_bytes_per_step": pipe.in_bytes * S,
            "d2h_bytes_per_step": pipe.out_floats * 4 * S,
            "bytes_counted_per": f"bench step (one block of {S} denoise steps)",
            "api": "runtime.HostBlockPipeline over fb_step (the reuse controller): every "
                   "denoise step's q/k/v copied in from pinned host memory and A_full/L_full "
                   "copied back, copies overlapped with attention on two copy streams, one "
                   "CUDA graph per block, L2 flushed between blocks",
        },
        "gpu_launches": int(launches_per_block * K),
        "clocks": clk,
    }
    if world == 1 and not args.no_cpu_baseline and args.workload == "dllm":
        line["cpu_baseline"] = oracle_baseline(wl)
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# oracle on the host cores (the reference arm and the CPU baseline)
# ---------------------------------------------------------------------------
class _HeadSlice:
    """The first n heads of a prefix cache (a bounded sample of the workload)."""

    def __init__(self, prefix, n):
        self.k = prefix.k[:, :n]
        self.v = prefix.v[:, :n]
        self.seq_len = prefix.seq_len
        self.page_table = prefix.page_table
        self.page_size = prefix.page_size
        self.max_seq_len = prefix.max_seq_len


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max(int(i.get("num_threads", 1)) for i in threadpool_info()) or 1
    except Exception:
        return os.cpu_count() or 1


def oracle_blocks(wl, blocks, steps_cache=None, n=ORACLE_HEADS):
    """Wall-clock seconds of `blocks` oracle blocks (threshold reuse) on the
    first n heads, scaled to all heads."""
    from oracle.controllers import ThresholdController
    sp = wl.spec
    sub = _HeadSlice(wl.prefix, n)
    steps = steps_cache if steps_cache is not None else list(wl.steps())
    total = 0.0
    for _ in range(blocks):
        ctl = ThresholdController(sub, sp.dtype, sp.tau)
        t0 = time.perf_counter()
        for st in steps:
            ctl.step(st.step, st.q[:, :, :n], st.k_in[:, :, :n], st.v_in[:, :, :n], st.m_updated)
        total += time.perf_counter() - t0
    return total * (sp.n_heads_q / n)


def oracle_baseline(wl, blocks=BASELINE_BLOCKS, n=BASELINE_HEADS):
    secs = oracle_blocks(wl, blocks, n=n)
    per_step_us = secs * 1e6 / (blocks * wl.spec.steps)
    return {"value": round(per_step_us, 1), "unit": UNIT, "cores": blas_threads(),
            "kind": "oracle",
            "sample": f"{blocks} block(s) of {wl.spec.steps} denoise steps, threshold reuse "
                      f"(tau={wl.spec.tau}), {n} of {wl.spec.n_heads_q} heads, time "
                      f"scaled by {wl.spec.n_heads_q // n} to all heads; float64 numpy"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    from workloads import make_workload
    wl = make_workload("dllm")
    steps = list(wl.steps())
    oracle_blocks(wl, args.warmup, steps)
    secs = oracle_blocks(wl, args.steps, steps)
    value = secs * 1e6 / (args.steps * wl.spec.steps)
    cpu = {"value": round(value, 1), "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
           "sample": f"each bench step: one block of {wl.spec.steps} denoise steps of the oracle "
                     f"(threshold reuse, tau={wl.spec.tau}) on {ORACLE_HEADS} of "
                     f"{wl.spec.n_heads_q} heads, scaled to all heads"}
    line = {"metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(secs * 1000 / args.steps, 3), "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "global_batch": 1, "seq_len": 32768,
                       "parallelism": "host cores"},
            "impl": "reference", "cpu_baseline": cpu,
            "e2e": {"value": round(value, 1), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


SWEEP_LENGTHS = (32768, 65536, 131072, 262144, 524288, 819200)


def run_sweep(args, rank, world):
    """Per-denoise-step attention at growing context, dllm head configuration
    (32 heads MHA, d=128, block 32, tau=4 schedule of the dllm steps): the dense
    prefix call, the dense step and the FlashBlock reuse step, each a CUDA graph
    per denoise step with the L2 flushed before it; prefixes drawn on the GPU
    (workloads.long_context)."""
    import torch

    import block_diffusion_attention_fb_b200 as fb
    from block_diffusion_attention_fb_b200.runtime import BlockAttention
    from workloads import make_workload
    from workloads.long_context import long_prefix
    from workloads.torch_io import to_torch

    fb.load_library()
    wl = make_workload("dllm", prefix_min=16, prefix_max=16)
    sp = wl.spec
    steps = list(wl.steps())
    S, B, Hq, d = sp.steps, sp.block, sp.n_heads_q, sp.head_dim
    dq = [to_torch(x.q, "bf16") for x in steps]
    dk = [to_torch(x.k_in, "bf16") for x in steps]
    dv = [to_torch(x.v_in, "bf16") for x in steps]
    ms = [x.m_updated.tolist() for x in steps]
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    flush_rd = torch.zeros(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
    A = torch.zeros(1, B, Hq, d, device="cuda")
    L = torch.zeros(1, B, Hq, device="cuda")
    peaks = measured_peaks()
    K, W = args.steps, max(1, args.warmup)
    for n_tok in SWEEP_LENGTHS:
        k, v, _ = long_prefix(n_tok, sp.n_heads_kv, d, seed=2000 + n_tok)
        seq_len = torch.tensor([n_tok], dtype=torch.int32, device="cuda")
        kv = fb.KV(k, v, seq_len=seq_len, page_table=None, page_size=16, max_seq_len=n_tok)
        reuse = BlockAttention(kv, B, Hq, "threshold", tau=sp.tau)
        dense = BlockAttention(kv, B, Hq, "threshold", tau=0)

        def run(blk):
            def step(s):
                if s == 0:
                    blk.reset()
                blk.step(dq[s], dk[s], dv[s], A, L, m_updated=ms[s])
            return step

        graphs = {}
        for name, blk in (("reuse", reuse), ("dense", dense)):
            fn = run(blk)
            for _ in range(W):
                for s in range(S):
                    fn(s)
            torch.cuda.synchronize()
            gl = []
            for s in range(S):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    fn(s)
                gl.append(g)
            graphs[name] = gl
        tot = {}
        for name, gl in graphs.items():
            pairs = []
            for _ in range(K):
                for s in range(S):
                    flush.zero_()
                    flush_rd.max()
                    e0 = torch.cuda.Event(enable_timing=True)
                    e1 = torch.cuda.Event(enable_timing=True)
                    e0.record()
                    gl[s].replay()
                    e1.record()
                    pairs.append((e0, e1))
            torch.cuda.synchronize()
            tot[name] = sum(a.elapsed_time(b) for a, b in pairs) * 1000 / (K * S)
        kv_bytes = 2 * n_tok * sp.n_heads_kv * d * 2
        line = {"sweep": "long_context", "prefix_tokens": n_tok,
                "config": "dllm heads: 32 MHA, head_dim 128, block 32, 32 denoise steps, "
                          "tau 4 schedule; prefix drawn on the GPU",
                "dense_us_per_step": round(tot["dense"], 2),
                "reuse_us_per_step": round(tot["reuse"], 2),
                "reuse_speedup": round(tot["dense"] / tot["reuse"], 3),
                "prefix_recomputes_per_block": sum(1 for s in range(S) if s == 0 or ms[s][0] >= sp.tau),
                "dense_step_kv_gbs": round(kv_bytes / (tot["dense"] * 1e-6) / 1e9, 1),
                "dense_step_kv_frac_of_hbm": round(kv_bytes / (tot["dense"] * 1e-6) / 1e9 /
                                                   peaks["gbs"], 4)}
        if rank == 0:
            print(json.dumps(line), flush=True)
        del graphs, reuse, dense, kv, k, v
        torch.cuda.empty_cache()


def main():
    args = parse_args()
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        run_reference(args, rank, world)
        return
    rank, world, local = dist_init(args.gpus)
    try:
        if args.sweep:
            run_sweep(args, rank, world)
        else:
            run_ours(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
