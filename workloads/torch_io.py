"""Moves workload arrays (numpy storage: float32 or bf16 bit patterns) into
torch tensors on a device, bit for bit. No arithmetic on the values."""

from __future__ import annotations

import numpy as np
import torch


def to_torch(arr: np.ndarray, dtype: str, device="cuda", pin: bool = False) -> torch.Tensor:
    if dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32))
    if device == "cpu":
        return t.pin_memory() if pin else t
    return t.to(device)


def prefix_tensors(prefix, dtype: str, device="cuda") -> dict:
    """The prefix cache on the device: k, v, seq_len, page_table (or None)."""
    out = {
        "k": to_torch(prefix.k, dtype, device),
        "v": to_torch(prefix.v, dtype, device),
        "seq_len": torch.from_numpy(prefix.seq_len.astype(np.int32)).to(device),
        "page_table": None,
        "page_size": prefix.page_size,
        "max_seq_len": prefix.max_seq_len,
    }
    if prefix.page_table is not None:
        out["page_table"] = torch.from_numpy(prefix.page_table.astype(np.int32)).to(device)
    return out
