"""Upload of the seeded synthetic workloads to device memory, slice by slice.

Each (batch, head) slice is drawn on the host, rounded to bf16 and copied into
a preallocated device tensor, so a 32K- or 128K-token workload never exists
whole in host memory. The values equal those of ``workloads.prefill_inputs``
and ``workloads.decode_inputs`` for the same slices.
"""
from __future__ import annotations

from typing import Dict

import numpy as np
import torch

from . import workloads as W


def _put(dst: torch.Tensor, x: np.ndarray, dtype=torch.bfloat16):
    dst.copy_(torch.from_numpy(np.ascontiguousarray(x)).to(dtype), non_blocking=False)


def prefill_to_device(w: W.Workload, device="cuda", with_do=None) -> Dict[str, torch.Tensor]:
    B, Hq, Hkv, N, d, NB = w.batch, w.n_q_heads, w.n_kv_heads, w.seq_len, w.head_dim, w.n_blocks
    with_do = w.backward if with_do is None else with_do
    bf = torch.bfloat16
    out = dict(q=torch.empty((B, Hq, N, d), dtype=bf, device=device),
               k=torch.empty((B, Hkv, N, d), dtype=bf, device=device),
               v=torch.empty((B, Hkv, N, d), dtype=bf, device=device),
               s=torch.empty((B, Hkv, NB, NB), dtype=torch.float32, device=device))
    if with_do:
        out["do"] = torch.empty((B, Hq, N, d), dtype=bf, device=device)
    for b in range(B):
        for hq in range(Hq):
            _put(out["q"][b, hq], W.q_slice(w, b, hq))
            if with_do:
                _put(out["do"][b, hq], W.do_slice(w, b, hq))
        for h in range(Hkv):
            _put(out["k"][b, h], W.k_slice(w, b, h))
            _put(out["v"][b, h], W.v_slice(w, b, h))
            _put(out["s"][b, h], W.s_slice(w, b, h), torch.float32)
    return out


def decode_to_device(w: W.Workload, device="cuda", cache_len=None) -> Dict[str, torch.Tensor]:
    B, Hq, Hkv, L, d, NB = w.batch, w.n_q_heads, w.n_kv_heads, w.seq_len, w.head_dim, w.n_blocks
    bf = torch.bfloat16
    out = dict(q=torch.empty((B, Hq, d), dtype=bf, device=device),
               k=torch.empty((B, Hkv, L, d), dtype=bf, device=device),
               v=torch.empty((B, Hkv, L, d), dtype=bf, device=device),
               s=torch.empty((B, Hkv, NB), dtype=torch.float32, device=device))
    for b in range(B):
        for hq in range(Hq):
            _put(out["q"][b, hq], W.q_slice(w, b, hq))
        for h in range(Hkv):
            _put(out["k"][b, h], W.k_slice(w, b, h))
            _put(out["v"][b, h], W.v_slice(w, b, h))
            _put(out["s"][b, h], W.s_slice(w, b, h), torch.float32)
    cl = W.cache_lens(w) if cache_len is None else np.asarray(cache_len, dtype=np.int32)
    out["cache_len"] = torch.from_numpy(cl).to(device)
    return out
