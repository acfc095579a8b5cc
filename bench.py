#!/usr/bin/env python
"""Per-denoise-step block-diffusion attention benchmark (FlashBlock / LoSA).

Headline workload: the dLLM configuration (bf16, batch 1, 32 heads MHA, d=128,
frozen prefix of 32768 tokens, block of 32 tokens denoised over 32 steps,
Poisson(2) row updates per step, tau=4), synthetic and seeded. One bench step
is one whole block: 32 denoise steps of attention (prefix partial when needed,
block partial, merge). Inputs are resident in HBM before timing; L2 is flushed
between denoise steps, outside the timed events: a 256 MiB write, then a read
of another 256 MiB buffer, so the write's dirty lines are written back before
the timed step rather than during it.

The default run measures all five workloads the same way (tiny, dllm, gqa,
video, losa; the line's "configs" key) and the packed-row comparison of
BlockBatch-style branches (the line's "varlen" key); --workload W times one.

Modes of every workload, each timed over the same K blocks:
  reuse  FlashBlock reuse through fb_step (threshold tau, or per-head gamma for
         video): the headline value for dllm
  dense  tau = 0 through fb_step: the prefix partial recomputed every step and
         merged with the in-block partial (dense block-diffusion attention);
         the prefix call alone (fb_prefix_attn) is also timed for the roofline
  losa   LoSA (active rows, top-k pages) through fb_step; its selection and
         gather also timed apart, with the union sizes and byte rates
  sparse_residual  FlashBlock + sparse attention (20% of pages per kv head,
         residual of the rest cached) through fb_step
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
CPU_BASELINE_BLOCKS = 6  # sample steps of the CPU baseline in our arm (about 10 s)


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20, help="timed blocks of 32 denoise steps")
    p.add_argument("--warmup", type=int, default=3, help="untimed blocks before timing")
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--mode", choices=["all", "prefix", "block", "losa_step", "sr_step"],
                   default="all",
                   help="all: the contract line; prefix/block/losa_step/sr_step: run only that "
                   "call eagerly, untimed, L2 flushed before each (for profilers)")
    p.add_argument("--sweep", action="store_true",
                   help="long-context sweep instead of the contract line: dense vs reuse per "
                   "denoise step over prefixes of 32k..800k tokens (one JSON line per length)")
    p.add_argument("--workload", choices=["dllm", "tiny", "gqa", "video", "losa"],
                   default=None, help="time this workload alone (it becomes the line's "
                   "headline); default: all five, dllm as the headline, plus the packed-row "
                   "(BlockBatch branches) comparison")
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


class _Flush:
    """L2 flush between timed regions: a 256 MiB write, then a read of another
    256 MiB buffer, so the write's dirty lines leave L2 before the next region."""

    def __init__(self):
        import torch
        self.w = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device="cuda")
        self.r = torch.zeros(FLUSH_BYTES, dtype=torch.uint8, device="cuda")

    def __call__(self):
        self.w.zero_()
        self.r.max()


def _ev():
    import torch
    return torch.cuda.Event(enable_timing=True)


def _eager_ms(fn, calls, flush):
    """Summed device ms of fn(i) for i in calls, L2 flushed before each call
    outside the events (the flush keeps the stream busy while the host
    enqueues, so the events bracket device work only)."""
    import torch
    pairs = []
    stream = torch.cuda.current_stream()
    for i in calls:
        flush()
        e0, e1 = _ev(), _ev()
        e0.record(stream)
        fn(i)
        e1.record(stream)
        pairs.append((e0, e1))
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in pairs)


class Rig:
    """Device inputs, controllers and step functions of one workload."""

    def __init__(self, name, args, with_e2e=False, with_commit=True):
        import torch

        import block_diffusion_attention_fb_b200 as fb
        from block_diffusion_attention_fb_b200.runtime import BlockAttention, HostBlockPipeline
        from workloads import make_workload
        from workloads.torch_io import prefix_tensors, to_torch

        self.name = name
        self.fb = fb
        wl = make_workload(name)
        self.wl, self.sp = wl, wl.spec
        sp = self.sp
        self.S, self.dt = sp.steps, sp.dtype
        dt = self.dt
        t = prefix_tensors(wl.prefix, dt)
        self.kv = kv = fb.KV(t["k"], t["v"], seq_len=t["seq_len"], page_table=t["page_table"],
                             page_size=t["page_size"], max_seq_len=t["max_seq_len"])
        steps = list(wl.steps())
        self.dq = [to_torch(x.q, dt) for x in steps]
        self.dk = [to_torch(x.k_in, dt) for x in steps]
        self.dv = [to_torch(x.v_in, dt) for x in steps]
        self.ms = [x.m_updated.tolist() for x in steps]
        batch, B, Hq, d = sp.batch, sp.block, sp.n_heads_q, sp.head_dim
        self.batch, self.B, self.Hq, self.d = batch, B, Hq, d
        self.esz = 2 if dt == "bf16" else 4
        self.A = torch.zeros(batch, B, Hq, d, device="cuda")
        self.L = torch.zeros(batch, B, Hq, device="cuda")
        if sp.gamma is not None:
            self.reuse = BlockAttention(kv, B, Hq, "per_head", gamma=sp.gamma)
            self.reuse_desc = f"FlashBlock per-head reuse (gamma={sp.gamma})"
        else:
            tau = sp.tau if sp.tau is not None else 4  # the losa spec states no tau
            self.reuse = BlockAttention(kv, B, Hq, "threshold", tau=tau)
            self.reuse_desc = f"FlashBlock threshold reuse (tau={tau})"
        # dense baseline: the same controller with tau = 0 (recompute every step)
        self.dense = BlockAttention(kv, B, Hq, "threshold", tau=0)
        self.n_act = sp.n_active or LOSA_ACTIVE
        self.topk = sp.topk_pages or LOSA_TOPK
        self.losa = BlockAttention(kv, B, Hq, "losa", n_active=self.n_act, topk_pages=self.topk)
        # FlashBlock + sparse residual: 20% page density (the pages pair FlashBlock
        # with SparseD at 20-40%)
        self.sr_topk = max(1, -(-kv.n_pages * SR_DENSITY_PCT // 100))
        self.sr_tau = sp.tau if sp.tau is not None else 4
        self.sres = BlockAttention(kv, B, Hq, "sparse_residual", tau=self.sr_tau,
                                   topk_pages=self.sr_topk)
        # block commit: a separate contiguous cache with room for every timed
        # commit (the commit reads only the block rows, so its content is not needed)
        self.commit = None
        if with_commit and wl.prefix.page_table is None:
            n_commits = max(1, args.warmup) + args.steps
            cap = int(wl.prefix.max_seq_len) + n_commits * self.S * B
            ck = torch.empty(batch * cap, sp.n_heads_kv, d, dtype=self.dk[0].dtype, device="cuda")
            cv = torch.empty_like(ck)
            clen = torch.from_numpy(wl.prefix.seq_len.astype("int32")).cuda()
            ckv = fb.KV(ck, cv, seq_len=clen, page_table=None, page_size=t["page_size"],
                        max_seq_len=cap)
            cmin = torch.empty(batch, ckv.n_pages, sp.n_heads_kv, d, dtype=self.dk[0].dtype,
                               device="cuda")
            self.commit = {"kv": ckv, "min": cmin, "max": torch.empty_like(cmin),
                           "len": wl.prefix.seq_len.astype("int32").copy()}
        self.a_out = torch.zeros(batch, B, Hq, d, device="cuda")
        self.l_out = torch.zeros(batch, B, Hq, device="cuda")
        self.a_in = torch.zeros_like(self.a_out)
        self.l_in = torch.zeros_like(self.l_out)
        self.ws = torch.empty(fb.fb_workspace_size(kv, B, Hq), dtype=torch.uint8, device="cuda")
        self.pipe = None
        if with_e2e:
            # end to end: each step's q/k/v packed in pinned host memory, A_full/L_full
            # returned to pinned host memory, copies overlapped with attention on their
            # own streams (runtime.HostBlockPipeline), one CUDA graph per block
            hq = [to_torch(x.q, dt, "cpu", pin=True) for x in steps]
            hk = [to_torch(x.k_in, dt, "cpu", pin=True) for x in steps]
            hv = [to_torch(x.v_in, dt, "cpu", pin=True) for x in steps]
            e2e_blk = (BlockAttention(kv, B, Hq, "per_head", gamma=sp.gamma)
                       if sp.gamma is not None
                       else BlockAttention(kv, B, Hq, "threshold",
                                           tau=sp.tau if sp.tau is not None else 4))
            self.pipe = HostBlockPipeline(e2e_blk, self.dq[0].dtype, depth=3)
            self.host_in = [self.pipe.pack_inputs(hq[s], hk[s], hv[s]) for s in range(self.S)]
            self.host_out = [self.pipe.new_output() for _ in range(self.S)]

    # -- one denoise step of each mode ------------------------------------------
    def reuse_step(self, s):
        if s == 0:
            self.reuse.reset()
        self.reuse.step(self.dq[s], self.dk[s], self.dv[s], self.A, self.L, m_updated=self.ms[s])

    def prefix_call(self, s):
        self.fb.fb_prefix_attn(self.dq[s], self.kv, self.a_out, self.l_out, self.ws)

    def block_call(self, s):
        self.fb.fb_block_attn(self.dq[s], self.dk[s], self.dv[s], self.a_in, self.l_in)

    def dense_step(self, s):
        if s == 0:
            self.dense.reset()
        self.dense.step(self.dq[s], self.dk[s], self.dv[s], self.A, self.L, m_updated=self.ms[s])

    def losa_step(self, s):
        if s == 0:
            self.losa.reset()
        self.losa.step(self.dq[s], self.dk[s], self.dv[s], self.A, self.L)

    def sres_step(self, s):
        if s == 0:
            self.sres.reset()
        self.sres.step(self.dq[s], self.dk[s], self.dv[s], self.A, self.L, m_updated=self.ms[s])

    def commit_call(self, s):
        c = self.commit
        self.fb.fb_block_commit(c["kv"], c["len"], self.dk[s], self.dv[s], c["min"], c["max"])
        c["len"] += self.B

    def e2e_block(self):
        self.pipe.enqueue_block(self.host_in, self.host_out, self.ms)

    def dense_full(self, s):
        """Dense attention with three separate calls (prefix, block, merge)."""
        self.prefix_call(s)
        self.block_call(s)
        self.fb.fb_merge(self.a_out, self.l_out, self.a_in, self.l_in, self.A, self.L)

    # -- LoSA bookkeeping ----------------------------------------------------------
    def max_union(self):
        G = self.Hq // self.sp.n_heads_kv
        return min(min(self.n_act, self.B) * G * self.topk, self.kv.n_pages)

    def losa_select_call(self, s):
        t, blk = self.losa.t, self.losa
        self.fb.losa_select(self.dq[s], self.dq[s - 1], blk.page_min, blk.page_max, self.kv,
                            self.n_act, self.topk, t["active_rows"], t["union_bitmap"],
                            t["union_list"], t["union_count"], blk.workspace,
                            row_scores=t["row_scores"])

    def losa_gather_call(self, s):
        t, blk = self.losa.t, self.losa
        self.fb.losa_gather(self.dq[s], t["active_rows"], self.n_act, t["union_list"],
                            t["union_count"], self.kv, blk.a_out, blk.l_out, blk.workspace,
                            max_union=self.max_union())


def _capture(torch, fn, S):
    graphs = []
    for s in range(S):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            fn(s)
        graphs.append(g)
    return graphs


def _replay_ms(torch, graphs, n_blocks, flush):
    """Summed device ms of n_blocks replays of a block's per-step graphs, L2
    flushed before every denoise step outside the events."""
    pairs = []
    stream = torch.cuda.current_stream()
    for _ in range(n_blocks):
        for g in graphs:
            flush()
            e0, e1 = _ev(), _ev()
            e0.record(stream)
            g.replay()
            e1.record(stream)
            pairs.append((e0, e1))
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in pairs)


def _back_to_back_ms(torch, fn, n_blocks, S, flush):
    stream = torch.cuda.current_stream()
    flush()  # also gives the host a head start on enqueueing
    e0, e1 = _ev(), _ev()
    e0.record(stream)
    for _ in range(n_blocks):
        for s in range(S):
            fn(s)
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


def measure_workload(rig, args, world, flush, headline=False):
    """Times every mode of one workload over args.steps blocks (max over ranks)
    and returns its summary: per-mode µs per denoise step, the roofline of the
    dense prefix call, LoSA's union sizes and byte rates, quality against dense."""
    import torch
    fb = rig.fb
    S, K, W = rig.S, args.steps, args.warmup
    sp, kv = rig.sp, rig.kv
    # warm-up of every path (eager, untimed): also sets kernel attributes
    for _ in range(max(1, W)):
        for s in range(S):
            rig.reuse_step(s)
            rig.prefix_call(s)
            rig.dense_step(s)
            rig.losa_step(s)
            if rig.sres is not None:
                rig.sres_step(s)
            if rig.commit is not None:
                rig.commit_call(s)
        if rig.pipe is not None:
            rig.e2e_block()
    torch.cuda.synchronize()
    # one CUDA graph per denoise step: the host decisions (tau, LoSA step index)
    # are taken at capture, as a sampler picks a pre-captured variant
    n0 = fb.fb_kernel_launches()
    g_reuse = _capture(torch, rig.reuse_step, S)
    launches_per_block = fb.fb_kernel_launches() - n0
    g_dense = _capture(torch, rig.dense_step, S)
    g_losa = _capture(torch, rig.losa_step, S)
    g_sres = _capture(torch, rig.sres_step, S) if rig.sres is not None else None
    g_e2e = None
    if rig.pipe is not None:
        g_e2e = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_e2e):
            rig.e2e_block()
    for gl in (g_reuse, g_dense, g_losa) + ((g_sres,) if g_sres else ()):
        _replay_ms(torch, gl, 1, flush)
    out = {}
    barrier(world)
    out["reuse"] = max_over_ranks(_replay_ms(torch, g_reuse, K, flush), world)
    barrier(world)
    out["dense"] = max_over_ranks(_replay_ms(torch, g_dense, K, flush), world)
    barrier(world)
    out["losa"] = max_over_ranks(_replay_ms(torch, g_losa, K, flush), world)
    barrier(world)
    t = _replay_ms(torch, g_sres, K, flush) if g_sres is not None else -1.0
    out["sres"] = max_over_ranks(t, world)
    barrier(world)
    t = _eager_ms(rig.commit_call, [s for _ in range(K) for s in range(S)], flush) \
        if rig.commit is not None else -1.0
    out["commit"] = max_over_ranks(t, world)
    barrier(world)
    if g_e2e is not None:
        # one whole block per timed iteration, L2 flushed between blocks
        pairs = []
        for _ in range(K):
            flush()
            e0, e1 = _ev(), _ev()
            e0.record()
            g_e2e.replay()
            e1.record()
            pairs.append((e0, e1))
        torch.cuda.synchronize()
        out["e2e"] = max_over_ranks(sum(a.elapsed_time(b) for a, b in pairs), world)
        barrier(world)

    # roofline of the dense prefix call (attention kernel + split combine)
    B, Hq, d, esz = rig.B, rig.Hq, rig.d, rig.esz
    n_tok = int(rig.wl.prefix.seq_len.sum())
    kv_bytes = 2 * n_tok * sp.n_heads_kv * d * esz
    io_bytes = rig.batch * B * Hq * d * esz + rig.batch * B * Hq * (d + 1) * 4
    alg_bytes = kv_bytes + io_bytes
    flops = 4.0 * n_tok * B * Hq * d
    peaks = measured_peaks()
    # bound by arithmetic intensity against the measured ridge point
    # (bf16 TFLOP/s over HBM GB/s, about 250 flop per byte)
    tensor_bound = flops / alg_bytes > peaks["ridge"] and rig.dt == "bf16"
    # The roofline's kernel time: the prefix call launched eagerly, an L2 flush
    # before each call outside the events, against the burst peaks. An
    # HBM-bound call whose K/V is at least twice the L2 also runs back to back
    # between one pair of events (each call evicts what the previous one left,
    # so none starts warm); that time is the one reported. Tensor-bound calls
    # keep the per-call figure: run back to back they settle under the power
    # cap, which the burst GEMM peak they are compared with does not.
    calls = [s for _ in range(K) for s in range(S)]
    t_flushed = max_over_ranks(_eager_ms(rig.prefix_call, calls, flush), world)
    l2_bytes = int(getattr(torch.cuda.get_device_properties(0), "L2_cache_size", 0)) or (126 << 20)
    back_to_back = kv_bytes >= 2 * l2_bytes and not tensor_bound
    t_kernel = (max_over_ranks(_back_to_back_ms(torch, rig.prefix_call, K, S, flush), world)
                if back_to_back else t_flushed)
    barrier(world)
    kernel_ms = t_kernel / (K * S)
    flushed_ms = t_flushed / (K * S)
    if tensor_bound:
        k_ach, k_peak, k_unit = flops / (kernel_ms * 1e-3) / 1e12, peaks["tflops"], "TFLOP/s"
    else:
        k_ach, k_peak, k_unit = alg_bytes / (kernel_ms * 1e-3) / 1e9, peaks["gbs"], "GB/s"
    roof = {
        "bound": "tensor" if tensor_bound else "hbm",
        "kernel": "fb_prefix_attn (split-KV attention + combine), dense prefix, eager launch",
        "kernel_us": round(kernel_ms * 1000, 3),
        "timing": (f"{K * S} calls back to back between two events (inputs "
                   f"{kv_bytes / l2_bytes:.1f}x the L2, no flush)" if back_to_back
                   else "L2 flushed before each call, outside the events"),
        "kernel_us_l2_flushed_each_call": round(flushed_ms * 1000, 3),
        "achieved": round(k_ach, 1),
        "peak": k_peak,
        "peak_kind": peaks["kind"] + (" (cuBLAS bf16 GEMM, burst)" if tensor_bound
                                      else " (copy bandwidth, burst)"),
        "unit": k_unit,
        "frac": round(k_ach / k_peak, 4),
        "algorithmic_bytes_per_call": alg_bytes,
        "algorithmic_flops_per_call": flops,
        "traffic": profiled_traffic() if rig.name == "dllm" else None,
    }

    # in-block partial of a long block (the video frame): tensor roofline
    block_roof = None
    if B > 64:
        t_blk = max_over_ranks(_eager_ms(rig.block_call, calls, flush), world)
        blk_ms = t_blk / (K * S)
        bflops = 4.0 * rig.batch * B * B * Hq * d
        block_roof = {"bound": "tensor", "kernel": "fb_block_attn (in-block partial), eager",
                      "kernel_us": round(blk_ms * 1000, 3),
                      "achieved": round(bflops / (blk_ms * 1e-3) / 1e12, 1),
                      "peak": peaks["tflops"], "unit": "TFLOP/s",
                      "frac": round(bflops / (blk_ms * 1e-3) / 1e12 / peaks["tflops"], 4),
                      "algorithmic_flops_per_call": bflops}

    # LoSA: the selection (locality score, page scores, top-k, union) and the
    # gather timed apart, eagerly, with the union sizes they produced
    losa_steps = [s for _ in range(max(1, K // 4)) for s in range(1, S)]
    t_sel = t_gat = 0.0
    counts = []
    pairs_s, pairs_g = [], []
    stream = torch.cuda.current_stream()
    for s in losa_steps:
        flush()
        e0, e1 = _ev(), _ev()
        e0.record(stream)
        rig.losa_select_call(s)
        e1.record(stream)
        flush()
        e2, e3 = _ev(), _ev()
        e2.record(stream)
        rig.losa_gather_call(s)
        e3.record(stream)
        pairs_s.append((e0, e1))
        pairs_g.append((e2, e3))
        counts.append(rig.losa.t["union_count"].clone())
    torch.cuda.synchronize()
    t_sel = max_over_ranks(sum(a.elapsed_time(b) for a, b in pairs_s), world) / len(losa_steps)
    t_gat = max_over_ranks(sum(a.elapsed_time(b) for a, b in pairs_g), world) / len(losa_steps)
    cnt = torch.stack(counts).double()  # [calls, batch, Hkv]
    P = kv.c.page_size
    n_pages_total = sum(-(-int(n) // P) for n in rig.wl.prefix.seq_len)
    sum_bytes = 2 * n_pages_total * sp.n_heads_kv * d * esz  # page min and max
    union_bytes = float(cnt.sum(dim=(1, 2)).mean()) * P * d * esz * 2  # K and V of the union
    n_act = min(rig.n_act, B)
    gather_io = rig.batch * n_act * Hq * (d * esz + (d + 1) * 4)
    sel_io = 2 * rig.batch * B * Hq * d * esz  # q_cur and q_prev
    step_block_io = rig.batch * B * (Hq + 2 * sp.n_heads_kv) * d * esz + \
        2 * rig.batch * B * Hq * (d + 1) * 4
    losa_step_bytes = sum_bytes + sel_io + union_bytes + gather_io + step_block_io
    losa_us = out["losa"] * 1000 / (K * S)
    losa_info = {
        "n_active": rig.n_act, "topk_pages": rig.topk, "pages_per_sequence": kv.n_pages,
        "union_pages_per_kv_head": {"mean": round(float(cnt.mean()), 1),
                                    "max": int(cnt.max()), "min": int(cnt.min())},
        "select_us": round(t_sel * 1000, 3),
        "select_summary_bytes": sum_bytes,
        "select_gbs": round((sum_bytes + sel_io) / (t_sel * 1e-3) / 1e9, 1),
        "gather_us": round(t_gat * 1000, 3),
        "gather_union_bytes": int(union_bytes),
        "gather_gbs": round((union_bytes + gather_io) / (t_gat * 1e-3) / 1e9, 1),
        "step_algorithmic_bytes": int(losa_step_bytes),
        "step_gbs": round(losa_step_bytes / (losa_us * 1e-6) / 1e9, 1),
        "step_frac_of_hbm": round(losa_step_bytes / (losa_us * 1e-6) / 1e9 / peaks["gbs"], 4),
        "timing": "selection and gather eager, L2 flushed before each call; step from the "
                  "graph replays (step 0 of a block is dense, so the step figure includes it)",
    }

    # Quality of the cheap modes against dense attention on the same block
    # (reported, not asserted: the pages give no number to hold it to). One
    # untimed block per mode, run in lockstep with the three-call dense path.
    quality = {}
    A_ref = torch.empty_like(rig.A)
    for qname, fn in (("reuse", rig.reuse_step), ("losa", rig.losa_step),
                      ("sparse_residual", rig.sres_step if rig.sres is not None else None)):
        if fn is None:
            continue
        mx, mean = 0.0, 0.0
        for s in range(S):
            rig.dense_full(s)
            A_ref.copy_(rig.A)
            fn(s)
            diff = (rig.A - A_ref).abs()
            mx = max(mx, float(diff.max()))
            mean += float(diff.mean()) / S
        quality[qname] = {"max_abs_vs_dense": round(mx, 5), "mean_abs_vs_dense": round(mean, 6)}
    torch.cuda.synchronize()
    fb.fb_device_status()
    del g_reuse, g_dense, g_losa, g_sres

    n_steps_all = K * S * world
    us = lambda ms_total: round(ms_total * 1000.0 / n_steps_all, 3)  # noqa: E731
    rec = sum(1 for s in range(S) if s == 0 or (sp.gamma is None and
                                                 rig.ms[s][0] >= rig.reuse.policy.tau))
    summary = {
        "workload": rig.name,
        "dtype": rig.dt,
        "shape": {"batch": rig.batch, "heads_q": Hq, "heads_kv": sp.n_heads_kv, "head_dim": d,
                  "block": B, "denoise_steps": S,
                  "prefix_tokens": [int(rig.wl.prefix.seq_len.min()),
                                    int(rig.wl.prefix.seq_len.max())],
                  "paged": rig.wl.prefix.page_table is not None},
        "reuse_us_per_step": us(out["reuse"]),
        "reuse_mode": rig.reuse_desc,
        "prefix_recomputes_per_block": rec if sp.gamma is None else None,
        "dense_us_per_step": us(out["dense"]),
        "losa_us_per_step": us(out["losa"]),
        "sparse_residual_us_per_step": us(out["sres"]) if out["sres"] >= 0 else None,
        "block_commit_us_per_call": us(out["commit"]) if out["commit"] >= 0 else None,
        "tokens_per_s_reuse": round(world * K * rig.batch * B / (out["reuse"] * 1e-3), 1),
        "dense_over_reuse": round(out["dense"] / out["reuse"], 2),
        "dense_over_losa": round(out["dense"] / out["losa"], 2),
        "roofline": roof,
        "in_block_roofline": block_roof,
        "losa": losa_info,
        "quality": quality,
    }
    extra = {"launches_per_block": launches_per_block, "raw": out}
    return summary, extra


def _branch_kv(fb, kv, b):
    """Sequence b of a paged cache as a batch of one (views of the same pool)."""
    return fb.KV(kv.k, kv.v, seq_len=kv.seq_len[b:b + 1], page_table=kv.page_table[b:b + 1],
                 page_size=kv.c.page_size, max_seq_len=kv.c.max_seq_len)


def measure_varlen(args, world, flush):
    """Packed rows (BlockBatch branches): blocks of 4..128 rows of one request,
    sharing its paged prefix, denoised together. Per denoise step: all branches
    in one packed launch per kernel (fb_step_varlen) against one fb_step per
    branch, both with the threshold reuse; and the dense (tau = 0) packed step."""
    import torch

    import block_diffusion_attention_fb_b200 as fb
    from block_diffusion_attention_fb_b200.runtime import BlockAttention, VarlenBlockAttention
    from workloads.torch_io import prefix_tensors, to_torch
    from workloads.varlen import BLOCKBATCH_ROWS, make_varlen_workload

    rows = BLOCKBATCH_ROWS
    wl = make_varlen_workload("gqa", rows, shared_prefix=True, prefix_min=VARLEN_PREFIX,
                              prefix_max=VARLEN_PREFIX, steps=VARLEN_STEPS)
    sp = wl.spec
    S, K, W = sp.steps, args.steps, args.warmup
    dt = sp.dtype
    t = prefix_tensors(wl.prefix, dt)
    kv = fb.KV(t["k"], t["v"], seq_len=t["seq_len"], page_table=t["page_table"],
               page_size=t["page_size"], max_seq_len=t["max_seq_len"])
    steps = list(wl.steps())
    dq = [to_torch(x.q, dt) for x in steps]
    dk = [to_torch(x.k_in, dt) for x in steps]
    dv = [to_torch(x.v_in, dt) for x in steps]
    ms = [x.m_updated.tolist() for x in steps]
    Hq, d, T = sp.n_heads_q, sp.head_dim, wl.total
    A = torch.zeros(T, Hq, d, device="cuda")
    L = torch.zeros(T, Hq, device="cuda")
    packed = VarlenBlockAttention(kv, wl.cu, Hq, tau=sp.tau)
    packed_dense = VarlenBlockAttention(kv, wl.cu, Hq, tau=0)
    sep = [BlockAttention(_branch_kv(fb, kv, b), r, Hq, "threshold", tau=sp.tau)
           for b, r in enumerate(rows)]
    cu = [int(x) for x in wl.cu]
    # per-branch views of the packed buffers ([1, B_b, H, d])
    qv = [[x[cu[b]:cu[b + 1]].unsqueeze(0) for b in range(len(rows))] for x in dq]
    kvv = [[x[cu[b]:cu[b + 1]].unsqueeze(0) for b in range(len(rows))] for x in dk]
    vvv = [[x[cu[b]:cu[b + 1]].unsqueeze(0) for b in range(len(rows))] for x in dv]
    Av = [A[cu[b]:cu[b + 1]].unsqueeze(0) for b in range(len(rows))]
    Lv = [L[cu[b]:cu[b + 1]].unsqueeze(0) for b in range(len(rows))]

    def packed_step(blk):
        def f(s):
            if s == 0:
                blk.reset()
            blk.step(dq[s], dk[s], dv[s], A, L, m_updated=ms[s])
        return f

    def separate_step(s):
        for b, blk in enumerate(sep):
            if s == 0:
                blk.reset()
            blk.step(qv[s][b], kvv[s][b], vvv[s][b], Av[b], Lv[b], m_updated=[ms[s][b]])

    fns = {"packed": packed_step(packed), "packed_dense": packed_step(packed_dense),
           "one_call_per_branch": separate_step}
    for _ in range(max(1, W)):
        for s in range(S):
            for f in fns.values():
                f(s)
    torch.cuda.synchronize()
    graphs = {k: _capture(torch, f, S) for k, f in fns.items()}
    res = {}
    for k, g in graphs.items():
        _replay_ms(torch, g, 1, flush)
        barrier(world)
        res[k] = max_over_ranks(_replay_ms(torch, g, K, flush), world) * 1000 / (K * S)
        barrier(world)
    fb.fb_device_status()
    del graphs
    return {
        "workload": f"BlockBatch-style branches: blocks of {list(rows)} rows of one request "
                    f"packed into {T} rows, one shared paged prefix of {VARLEN_PREFIX} tokens, "
                    f"GQA 32/8 heads, head_dim 128, bf16, {S} denoise steps, Poisson(3) "
                    f"updates per branch, tau {sp.tau}",
        "packed_reuse_us_per_step": round(res["packed"], 3),
        "one_call_per_branch_reuse_us_per_step": round(res["one_call_per_branch"], 3),
        "packed_dense_us_per_step": round(res["packed_dense"], 3),
        "packing_speedup": round(res["one_call_per_branch"] / res["packed"], 3),
    }


HEADLINE = "dllm"
CONFIG_ORDER = ("dllm", "tiny", "gqa", "video", "losa")
VARLEN_PREFIX, VARLEN_STEPS = 32768, 32


def run_profile_mode(args, rank):
    """--mode prefix/block/losa_step/sr_step: one call kind, eager and untimed,
    for profilers (ncu's launch list and captures)."""
    import torch
    name = args.workload or HEADLINE
    rig = Rig(name, args, with_commit=False)
    flush = _Flush()
    fn = {"prefix": rig.prefix_call, "block": rig.block_call, "losa_step": rig.losa_step,
          "sr_step": lambda s: rig.sres_step(s)}[args.mode]
    for _ in range(args.warmup + args.steps):
        for s in range(rig.S):
            flush()
            fn(s)
    torch.cuda.synchronize()
    rig.fb.fb_device_status()
    if rank == 0:
        print(json.dumps({"mode": args.mode, "workload": name,
                          "calls": (args.warmup + args.steps) * rig.S}))


def run_ours(args, rank, world, local):
    import torch

    import block_diffusion_attention_fb_b200 as fb

    fb.load_library()
    if args.mode in ("prefix", "block", "losa_step", "sr_step"):
        run_profile_mode(args, rank)
        return
    names = [args.workload] if args.workload else list(CONFIG_ORDER)
    flush = _Flush()
    clocks = ClockSampler(local)
    barrier(world)
    clocks.start()
    barrier(world)
    configs, extras, e2e_info = {}, {}, None
    for name in names:
        rig = Rig(name, args, with_e2e=(name == names[0]))
        summary, extra = measure_workload(rig, args, world, flush, headline=(name == names[0]))
        configs[name], extras[name] = summary, extra
        if rig.pipe is not None:
            e2e_info = {"in": rig.pipe.in_bytes * rig.S, "out": rig.pipe.out_floats * 4 * rig.S,
                        "S": rig.S}
        del rig
        torch.cuda.empty_cache()
    varlen = measure_varlen(args, world, flush) if not args.workload else None
    barrier(world)
    clk = clocks.stop()
    if rank != 0:
        return
    head = names[0]
    hs, hx = configs[head], extras[head]
    K, S = args.steps, hs["shape"]["denoise_steps"]
    n_steps_all = K * S * world
    raw = hx["raw"]
    line = {
        "metric": METRIC,
        "value": hs["reuse_us_per_step"],
        "unit": UNIT,
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(raw["reuse"] / K, 4),
        "higher_is_better": False,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": hs["dtype"],
        "data": "synthetic (seeded generator; no model weights or datasets)",
        "config": {
            "workload": WORKLOAD if head == "dllm" else head,
            "global_batch": world * hs["shape"]["batch"],
            "seq_len": hs["shape"]["prefix_tokens"][1],
            "block": hs["shape"]["block"],
            "denoise_steps_per_bench_step": S,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "l2": "flushed between denoise steps (256 MiB write, then 256 MiB read of another "
                  "buffer; outside the timed events)",
            "value_mode": f"reuse: {hs['reuse_mode']} through fb_step, one CUDA graph per "
                          "denoise step",
        },
        "modes": {
            "reuse": {"us_per_step": hs["reuse_us_per_step"],
                      "prefix_recomputes_per_block": hs["prefix_recomputes_per_block"]},
            "dense": {"us_per_step": hs["dense_us_per_step"],
                      "via": "fb_step with tau=0: prefix partial every step, merge fused into "
                             "the in-block kernel",
                      "prefix_call_us": hs["roofline"]["kernel_us_l2_flushed_each_call"]},
            "losa": {"us_per_step": hs["losa_us_per_step"], "n_active": hs["losa"]["n_active"],
                     "topk_pages": hs["losa"]["topk_pages"],
                     "union_pages_per_kv_head": hs["losa"]["union_pages_per_kv_head"],
                     "step_gbs": hs["losa"]["step_gbs"]},
            "sparse_residual": ({"us_per_step": hs["sparse_residual_us_per_step"],
                                 "topk_pages_pct": SR_DENSITY_PCT}
                                if hs["sparse_residual_us_per_step"] is not None else None),
            "block_commit": ({"us_per_call": hs["block_commit_us_per_call"]}
                             if hs["block_commit_us_per_call"] is not None else None),
        },
        "quality": hs["quality"],
        "tokens_per_s": hs["tokens_per_s_reuse"],
        # context, not a target: the pages' own dense-vs-FlashBlock figures (end to
        # end in a model, hardware not stated) beside this run's per-step ratio
        "context": {
            "dense_over_reuse_attention_time": hs["dense_over_reuse"],
            "pages": "FlashBlock vs dense block diffusion: up to 1.6x lower attention time, "
                     "up to 1.44x token throughput (312 -> 451 tokens/s); LoSA vs dense: "
                     "4.14x (RTX A6000), 3.67x (RTX 5090); hardware of the FlashBlock "
                     "figures not stated",
        },
        "roofline": hs["roofline"],
        "e2e": {
            "value": round(raw["e2e"] * 1000.0 / n_steps_all, 3),
            "unit": UNIT,
            "h2d_bytes_per_step": e2e_info["in"],
            "d2h_bytes_per_step": e2e_info["out"],
            "bytes_counted_per": f"bench step (one block of {S} denoise steps)",
            "api": "runtime.HostBlockPipeline over fb_step (the reuse controller): every "
                   "denoise step's q/k/v copied in from pinned host memory and A_full/L_full "
                   "copied back, copies overlapped with attention on two copy streams, one "
                   "CUDA graph per block, L2 flushed between blocks",
        },
        "gpu_launches": int(hx["launches_per_block"] * K),
        "clocks": clk,
        "configs": configs,
        "varlen": varlen,
    }
    if world == 1 and not args.no_cpu_baseline and head == "dllm":
        line["cpu_baseline"] = oracle_baseline()
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


# One sample definition for the CPU baseline and the reference arm: a sample
# step is one whole dllm block (32 denoise steps, threshold reuse, tau 4) of
# the oracle on the first ORACLE_HEADS of the 32 heads. Heads are independent
# and cost the same, so the per-denoise-step figure scales by 32 / ORACLE_HEADS;
# the measured seconds are reported as they are.
ORACLE_HEADS = 8


def oracle_sample_seconds(wl, steps, n=ORACLE_HEADS):
    """Wall-clock seconds of one sample step (one block on n heads)."""
    from oracle.controllers import ThresholdController
    sp = wl.spec
    sub = _HeadSlice(wl.prefix, n)
    ctl = ThresholdController(sub, sp.dtype, sp.tau)
    t0 = time.perf_counter()
    for st in steps:
        ctl.step(st.step, st.q[:, :, :n], st.k_in[:, :, :n], st.v_in[:, :, :n], st.m_updated)
    return time.perf_counter() - t0


def _sample_desc(wl, blocks):
    sp = wl.spec
    return (f"{blocks} sample step(s), each one block of {sp.steps} denoise steps of the oracle "
            f"(threshold reuse, tau={sp.tau}) on {ORACLE_HEADS} of {sp.n_heads_q} heads; "
            f"us per denoise step scaled by {sp.n_heads_q // ORACLE_HEADS} to all heads; "
            f"float64 numpy")


def oracle_baseline(blocks=CPU_BASELINE_BLOCKS):
    """The oracle on the host cores (the reported CPU baseline of our arm), with
    the BLAS thread pool as it stands and again limited to one thread."""
    from workloads import make_workload
    wl = make_workload("dllm")
    steps = list(wl.steps())
    scale = wl.spec.n_heads_q / ORACLE_HEADS
    secs = sum(oracle_sample_seconds(wl, steps) for _ in range(blocks))
    per_step_us = secs * 1e6 * scale / (blocks * wl.spec.steps)
    out = {"value": round(per_step_us, 1), "unit": UNIT, "cores": blas_threads(),
           "kind": "oracle", "sample": _sample_desc(wl, blocks),
           "measured_seconds": round(secs, 3)}
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(1):
            s1 = oracle_sample_seconds(wl, steps)
        out["single_thread"] = {"value": round(s1 * 1e6 * scale / wl.spec.steps, 1),
                                "unit": UNIT, "cores": 1, "sample": _sample_desc(wl, 1),
                                "measured_seconds": round(s1, 3)}
    except ImportError:
        out["single_thread"] = None
    return out


def run_reference(args, rank, world):
    """The reference arm: the oracle, as it stands, on the host cores (rank 0
    only). Each bench step is one sample step; ms_per_step is the measured
    sample time, value the per-denoise-step figure scaled to all heads."""
    if rank != 0:
        return
    from workloads import make_workload
    wl = make_workload("dllm")
    sp = wl.spec
    steps = list(wl.steps())
    for _ in range(args.warmup):
        oracle_sample_seconds(wl, steps)
    secs = sum(oracle_sample_seconds(wl, steps) for _ in range(args.steps))
    scale = sp.n_heads_q / ORACLE_HEADS
    value = secs * 1e6 * scale / (args.steps * sp.steps)
    cpu = {"value": round(value, 1), "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
           "sample": _sample_desc(wl, args.steps)}
    line = {"metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(secs * 1000 / args.steps, 3),
            "ms_per_step_is": f"measured seconds of one sample step ({ORACLE_HEADS} of "
                              f"{sp.n_heads_q} heads); value scales by "
                              f"{sp.n_heads_q // ORACLE_HEADS} to all heads",
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "global_batch": 1, "seq_len": 32768,
                       "block": sp.block, "denoise_steps_per_bench_step": sp.steps,
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
