"""Seeded synthetic workloads with the shapes of the SAS experiments.

The pages train and evaluate on datasets and checkpoints that are not available
here (OpenR1-Math, GPQA-Diamond, LongBench, RULER and the Qwen3 / Llama-3.1
weights). These generators stand in for them. They reproduce the shapes that
matter to the kernels: block size 64, Top-K budgets of 16 to 64 blocks, GQA
head grouping and sequence lengths from 1K to 128K.

Every tensor is drawn per (tensor, batch, head) slice from its own
``numpy.random.SeedSequence``. Any slice can therefore be regenerated alone,
and a parity test on one KV head of a 32K or 128K workload does not have to
build the whole tensor on the host.

Values are drawn in fp32 and rounded to bf16 with round-to-nearest-even. The
rounded values are what both sides consume. ``*_bits`` arrays hold the raw
bf16 bit patterns (uint16), and ``*`` arrays hold the same values widened to
fp32.

Normal distributions are written N(mean, variance): ``s ~ N(0, 2)`` has
standard deviation sqrt(2).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, List, Optional, Sequence

import numpy as np

BLOCK = 64

# tensor ids used in the per-slice seed sequences
_T_Q, _T_K, _T_V, _T_DO, _T_S, _T_HH_U, _T_HH_POS, _T_S_NOISE = range(8)


# --------------------------------------------------------------------------
# bf16 rounding (round to nearest, ties to even), on the raw fp32 bits
# --------------------------------------------------------------------------
def bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 array -> uint16 bf16 bit patterns, round-to-nearest-even."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        r[nan] = 0x7FC0
    return r


def bits_to_f32(b: np.ndarray) -> np.ndarray:
    """uint16 bf16 bit patterns -> fp32 values (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """fp32 -> fp32 holding the nearest bf16 value."""
    return bits_to_f32(bf16_bits(x))


def _rng(seed: int, tensor: int, *ids: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tensor, *ids])))


def _normal(seed: int, tensor: int, ids: Sequence[int], shape, std: float = 1.0) -> np.ndarray:
    g = _rng(seed, tensor, *ids)
    x = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


# --------------------------------------------------------------------------
# workload descriptions
# --------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str  # "prefill" (fwd [+ bwd]) or "decode"
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    seq_len: int  # prefill: N; decode: KV-cache capacity Lmax
    top_k: int
    seed: int
    backward: bool = True
    s_var: float = 2.0
    heavy_hitters: bool = False
    cache_len: Optional[int] = None  # decode: tokens in the cache, new token included
    block: int = BLOCK

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def n_blocks(self) -> int:
        return self.seq_len // self.block

    def describe(self) -> str:
        return (f"{self.name}: B{self.batch} H{self.n_q_heads}/{self.n_kv_heads} d{self.head_dim} "
                f"{'L' if self.kind == 'decode' else 'N'}{self.seq_len} K{self.top_k}")


WORKLOADS: Dict[str, Workload] = {
    # small case, every tensor checkable by the fp64 oracle in seconds
    "tiny": Workload("tiny", "prefill", 1, 2, 2, 64, 1024, 4, seed=0),
    # Qwen3-4B-shaped training prefill (fwd + bwd incl. ds)
    "qwen3_4b_train_32k": Workload("qwen3_4b_train_32k", "prefill", 1, 32, 8, 128, 32768, 32, seed=1),
    # single-token decode, split-K over the selected blocks
    "decode_b16_32k": Workload("decode_b16_32k", "decode", 16, 32, 8, 128, 32768, 16, seed=2,
                               backward=False, cache_len=32768),
    # Llama-3.1-8B-shaped long prefill, forward only, planted heavy hitters
    "llama31_8b_fwd_128k": Workload("llama31_8b_fwd_128k", "prefill", 1, 32, 8, 128, 131072, 64, seed=3,
                                    backward=False, heavy_hitters=True),
}


def sweep_workloads() -> List[Workload]:
    """Qwen3-14B-shaped budget x length sweep (40/8 heads, d 128, fwd + bwd)."""
    out = []
    i = 0
    for k in (16, 32, 64):
        for n in (8192, 32768, 65536):
            out.append(Workload(f"qwen3_14b_k{k}_n{n}", "prefill", 1, 40, 8, 128, n, k, seed=10 + i))
            i += 1
    return out


for _w in sweep_workloads():
    WORKLOADS[_w.name] = _w


# --------------------------------------------------------------------------
# generators
# --------------------------------------------------------------------------
def _hh_unit(w: Workload, b: int, h: int) -> np.ndarray:
    u = _normal(w.seed, _T_HH_U, (b, h), (w.head_dim,)).astype(np.float64)
    return (u / np.linalg.norm(u)).astype(np.float32)


def _hh_positions(w: Workload, b: int, h: int) -> np.ndarray:
    g = _rng(w.seed, _T_HH_POS, b, h)
    n_hh = max(1, int(round(0.01 * w.seq_len)))
    return np.sort(g.choice(w.seq_len, size=n_hh, replace=False))


def q_slice(w: Workload, b: int, hq: int) -> np.ndarray:
    """bf16-rounded fp32 [N, d] (prefill) or [d] (decode) for query head hq."""
    n = 1 if w.kind == "decode" else w.seq_len
    x = _normal(w.seed, _T_Q, (b, hq), (n, w.head_dim))
    if w.heavy_hitters:
        x += 4.0 * _hh_unit(w, b, hq // w.group)[None, :]
    x = bf16_round(x)
    return x[0] if w.kind == "decode" else x


def k_slice(w: Workload, b: int, h: int) -> np.ndarray:
    x = _normal(w.seed, _T_K, (b, h), (w.seq_len, w.head_dim))
    if w.heavy_hitters:
        x[_hh_positions(w, b, h)] += 4.0 * _hh_unit(w, b, h)[None, :]
    return bf16_round(x)


def v_slice(w: Workload, b: int, h: int) -> np.ndarray:
    return bf16_round(_normal(w.seed, _T_V, (b, h), (w.seq_len, w.head_dim)))


def do_slice(w: Workload, b: int, hq: int) -> np.ndarray:
    return bf16_round(_normal(w.seed, _T_DO, (b, hq), (w.seq_len, w.head_dim)))


def s_slice(w: Workload, b: int, h: int) -> np.ndarray:
    """Block scores for one (batch, KV head): [NQB, NKB] (prefill) or [NKB] (decode), fp32.

    Entries with m >= t (prefill) or m >= current block (decode) are drawn too
    but carry no meaning; every consumer must ignore them.
    """
    nb = w.n_blocks
    if w.kind == "decode":
        return _normal(w.seed, _T_S, (b, h), (nb,), std=math.sqrt(w.s_var))
    if not w.heavy_hitters:
        return _normal(w.seed, _T_S, (b, h), (nb, nb), std=math.sqrt(w.s_var))
    # structured scores: a block-mean proxy of q.k plus N(0, 0.5) noise
    k = k_slice(w, b, h).astype(np.float64)
    kbar = k.reshape(nb, w.block, w.head_dim).mean(axis=1)  # [NKB, d]
    qbar = np.zeros((nb, w.head_dim))
    for g in range(w.group):
        qbar += q_slice(w, b, h * w.group + g).astype(np.float64).reshape(nb, w.block, w.head_dim).mean(axis=1)
    qbar /= w.group
    s = qbar @ kbar.T / math.sqrt(w.head_dim)
    s += _normal(w.seed, _T_S_NOISE, (b, h), (nb, nb), std=math.sqrt(0.5))
    return s.astype(np.float32)


def cache_lens(w: Workload) -> np.ndarray:
    assert w.kind == "decode"
    return np.full((w.batch,), w.cache_len if w.cache_len is not None else w.seq_len, dtype=np.int32)


def prefill_inputs(w: Workload, kv_heads: Optional[Sequence[int]] = None, batches: Optional[Sequence[int]] = None,
                   with_do: Optional[bool] = None) -> Dict[str, np.ndarray]:
    """fp32 (bf16-valued) inputs of a prefill workload.

    With ``kv_heads`` (and/or ``batches``) given, only those KV heads and their
    query-head groups are generated; the values equal the corresponding
    slices of the full tensors.
    """
    assert w.kind == "prefill"
    hs = list(range(w.n_kv_heads)) if kv_heads is None else list(kv_heads)
    bs = list(range(w.batch)) if batches is None else list(batches)
    with_do = w.backward if with_do is None else with_do
    G = w.group
    q = np.stack([np.stack([q_slice(w, b, h * G + g) for h in hs for g in range(G)]) for b in bs])
    k = np.stack([np.stack([k_slice(w, b, h) for h in hs]) for b in bs])
    v = np.stack([np.stack([v_slice(w, b, h) for h in hs]) for b in bs])
    s = np.stack([np.stack([s_slice(w, b, h) for h in hs]) for b in bs])
    out = dict(q=q, k=k, v=v, s=s)
    if with_do:
        out["do"] = np.stack([np.stack([do_slice(w, b, h * G + g) for h in hs for g in range(G)]) for b in bs])
    return out


def decode_inputs(w: Workload, cache_len: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """fp32 (bf16-valued) inputs of a decode workload.

    q [B, Hq, d]; k, v caches [B, Hkv, Lmax, d]; s [B, Hkv, NKB]; cache_len [B].
    """
    assert w.kind == "decode"
    B, Hq, Hkv = w.batch, w.n_q_heads, w.n_kv_heads
    q = np.stack([np.stack([q_slice(w, b, h) for h in range(Hq)]) for b in range(B)])
    k = np.stack([np.stack([k_slice(w, b, h) for h in range(Hkv)]) for b in range(B)])
    v = np.stack([np.stack([v_slice(w, b, h) for h in range(Hkv)]) for b in range(B)])
    s = np.stack([np.stack([s_slice(w, b, h) for h in range(Hkv)]) for b in range(B)])
    cl = cache_lens(w) if cache_len is None else np.asarray(cache_len, dtype=np.int32)
    return dict(q=q, k=k, v=v, s=s, cache_len=cl)


def custom(name: str = "custom", kind: str = "prefill", **kw) -> Workload:
    """A workload with explicit sizes (tests use it for ragged and edge cases)."""
    return Workload(name=name, kind=kind, **kw)
