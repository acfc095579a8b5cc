"""Helpers shared by the GPU parity tests: device copies of workload arrays,
and the comparison against the oracle with the stated tolerances.

Tolerances (GPU vs float64 oracle on the same inputs):
  bf16 inputs, fp32 accumulation: max-abs 2e-2 and mean-abs 2e-3 on A;
  fp32 inputs: max-abs 1e-4 on A; L (log normaliser): max-abs 1e-3.
Integer results (active rows, page unions, masks) must match exactly.
"""

from __future__ import annotations

import numpy as np
import torch

from workloads.torch_io import prefix_tensors, to_torch

TOL = {"bf16": (2e-2, 2e-3), "f32": (1e-4, 1e-4)}
TOL_L = 1e-3


def dev(arr, dtype):
    return to_torch(arr, dtype, "cuda")


def make_kv(prefix, dtype):
    import block_diffusion_attention_fb_b200 as fb
    t = prefix_tensors(prefix, dtype, "cuda")
    kv = fb.KV(t["k"], t["v"], seq_len=t["seq_len"], page_table=t["page_table"],
               page_size=t["page_size"], max_seq_len=t["max_seq_len"])
    return kv


def assert_close_A(got, want, dtype, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - want)
    mx, mean = TOL[dtype]
    assert err.max() <= mx, f"{what}: max-abs {err.max():.3e} > {mx}"
    assert err.mean() <= mean, f"{what}: mean-abs {err.mean():.3e} > {mean}"
    return float(err.max()), float(err.mean())


def assert_close_L(got, want, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape
    both_inf = np.isneginf(got) & np.isneginf(want)
    assert np.array_equal(np.isneginf(got), np.isneginf(want)), f"{what}: -inf pattern differs"
    err = np.abs(np.where(both_inf, 0.0, got) - np.where(both_inf, 0.0, want))
    assert err.max() <= TOL_L, f"{what}: L max-abs {err.max():.3e} > {TOL_L}"
    return float(err.max())


def cpu(t):
    return t.detach().cpu().numpy()


def sync():
    torch.cuda.synchronize()
