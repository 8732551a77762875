"""Move seeded host inputs (numpy, from :mod:`.inputs`) onto the GPU as library descriptors.

Pure data movement: bf16 arrays arrive as uint16 bit patterns and are reinterpreted, never
converted, so the device sees exactly the bytes the oracle reads.
"""
from __future__ import annotations

from typing import Optional

import numpy as np
import torch

from . import inputs as gen
from .sdattn import KVCache, Queries


def tensor(a: np.ndarray, dtype: str, device="cuda", pin: bool = False) -> torch.Tensor:
    """numpy array in the KV storage type -> torch tensor (bf16 reinterpreted from uint16)."""
    a = np.ascontiguousarray(a)
    if dtype == gen.BF16:
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(a.astype(np.float32, copy=False))
    if pin:
        return t.pin_memory()
    return t.to(device)


def int32(a, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)


def kv_cache(w: gen.AttnWorkload, kv_len: Optional[np.ndarray] = None, device="cuda",
             k: Optional[torch.Tensor] = None, v: Optional[torch.Tensor] = None) -> KVCache:
    """Library cache over workload ``w`` (verify lengths unless ``kv_len`` is given).

    ``k`` / ``v`` may pass tensors already on the device (shared between several caches)."""
    lens = w.kv_len_verify if kv_len is None else kv_len
    k = tensor(w.k, w.dtype, device) if k is None else k
    v = tensor(w.v, w.dtype, device) if v is None else v
    bt = int32(w.block_table, device) if w.paged else None
    return KVCache(k, v, int32(lens, device), block_table=bt)


def queries(q: np.ndarray, q_start: np.ndarray, dtype: str, max_kv_len: int, device="cuda",
            softmax_scale: float = 0.0) -> Queries:
    qs = np.asarray(q_start, dtype=np.int32)
    max_rows = int(np.max(np.diff(qs))) if len(qs) > 1 else 1
    return Queries(tensor(q, dtype, device), int32(qs, device), max(max_rows, 1), int(max_kv_len),
                   softmax_scale=softmax_scale)


def draft_queries(w: gen.AttnWorkload, step: int, device="cuda") -> Queries:
    """One query row per sequence for draft step ``step`` (kv_len = ctx + step + 1)."""
    q = w.q_draft[step]
    qs = np.arange(w.n_seq + 1, dtype=np.int32)
    return queries(q, qs, w.dtype, int(w.kv_len_draft(step).max()), device)


def verify_queries(w: gen.AttnWorkload, device="cuda") -> Queries:
    return queries(w.q_verify, w.q_verify_start, w.dtype, int(w.kv_len_verify.max()), device)


def to_numpy_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)
