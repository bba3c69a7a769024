"""Python binding of the SAS gated block-sparse attention library (B200, sm_100a).

A thin ctypes layer over ``libsas_b200.so``. Every function named like a C
entry point marshals torch tensors into device pointers and calls the C
function. All computation runs in the library's CUDA kernels, and nothing
here falls back to PyTorch or the CPU. Importing this package fails loudly
when the library has not been built (``python -m learned_block_sparse_warp_b200.build``).

The entry points and their contracts are those of include/sas.h:
``sas_topk_select``, ``sas_gate_lse``, ``sas_fwd``, ``sas_bwd``
(+ ``sas_bwd_workspace_size``), ``sas_decode``, ``sas_decode_combine``,
``sas_get_device_error``.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

__all__ = [
    "SAS_GATE_LOG_SOFTMAX", "SAS_GATE_NONE", "SAS_GATE_LOG_SIGMOID", "SAS_GATE_LOGIT",
    "SAS_GATE_SOFTMAX_OUTSIDE", "SasError", "Params", "lib",
    "sas_topk_select", "sas_gate_lse", "sas_fwd", "sas_bwd_workspace_size", "sas_bwd_workspace_size_min", "sas_bwd",
    "sas_decode",
    "sas_decode_combine", "sas_decode_paged", "sas_decode_noalloc", "sas_get_device_error", "sas_status_string",
    "sas_version",
    "DecodeGraph", "sas_selftest_wait_timeout", "sas_block_mean_keys", "sas_decode_select_scored",
    "decode_step_scored", "sas_train_steps_host", "empty_device_slot", "sas_decode_fused", "sas_decode_fused_paged",
    "decode_step_fused",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsas_b200.so")

SAS_GATE_LOG_SOFTMAX = 0
SAS_GATE_NONE = 1
SAS_GATE_LOG_SIGMOID = 2  # ablation: log g = log σ(s)
SAS_GATE_LOGIT = 3  # ablation: log g = s
SAS_GATE_SOFTMAX_OUTSIDE = 4  # ablation: g = softmax(s) weights the values after the softmax
STATUS = {0: "SAS_OK", 1: "SAS_ERR_INVALID_ARG", 2: "SAS_ERR_UNSUPPORTED", 3: "SAS_ERR_WORKSPACE",
          4: "SAS_ERR_CUDA", 5: "SAS_ERR_TIMEOUT", 6: "SAS_ERR_DEVICE_INDEX"}
BLOCK = 64


class SasError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn} failed: {sas_status_string(code)}")


class sas_host_step(ctypes.Structure):
    """Mirror of ``sas_host_step``: one training step's host buffers."""
    _fields_ = [(n, ctypes.c_void_p) for n in ("q", "k", "v", "s", "dO", "o", "lse_o", "dq", "dk", "dv", "ds")]


class sas_device_slot(ctypes.Structure):
    """Mirror of ``sas_device_slot``: one set of device buffers for a step."""
    _fields_ = [(n, ctypes.c_void_p) for n in ("q", "k", "v", "dO", "o", "dq", "dk", "dv", "s", "lse_s", "lse_o",
                                                "ds", "idx", "ws")] + [("ws_bytes", ctypes.c_size_t)]


class sas_params(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int), ("n_q_heads", ctypes.c_int), ("n_kv_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int), ("seq_len", ctypes.c_int), ("block", ctypes.c_int),
        ("top_k", ctypes.c_int), ("softmax_scale", ctypes.c_float), ("gate_mode", ctypes.c_int),
    ]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m learned_block_sparse_warp_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(sas_params)
    vp, sz = ctypes.c_void_p, ctypes.c_size_t
    sig = {
        "sas_topk_select": [P, vp, vp, vp, vp, vp],
        "sas_gate_lse": [P, vp, vp, vp, vp],
        "sas_fwd": [P, vp, vp, vp, vp, vp, vp, vp, vp, vp],
        "sas_bwd_workspace_size": [P, ctypes.POINTER(sz)],
        "sas_bwd_workspace_size_min": [P, ctypes.POINTER(sz)],
        "sas_bwd": [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp],
        "sas_decode": [P, vp, vp, vp, vp, vp, vp, vp, ctypes.c_int, vp, vp, vp],
        "sas_decode_paged": [P, vp, vp, vp, ctypes.c_int, vp, vp, vp, vp, vp, ctypes.c_int, vp, vp, vp],
        "sas_decode_combine": [P, ctypes.c_int, vp, vp, vp, vp, vp],
        "sas_get_device_error": [vp, ctypes.POINTER(ctypes.c_int)],
        "sas_decode_noalloc": [P, vp, vp, vp, vp, vp, vp, vp, vp],
        "sas_decode_fused": [P, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp],
        "sas_decode_fused_paged": [P, vp, vp, vp, ctypes.c_int, vp, vp, vp, vp, vp, vp, vp, vp],
        "sas_selftest_wait_timeout": [vp],
        "sas_block_mean_keys": [P, vp, vp, vp, vp],
        "sas_decode_select_scored": [P, vp, vp, vp, vp, vp, vp, vp],
        "sas_train_steps_host": [P, ctypes.c_int, ctypes.POINTER(sas_host_step), ctypes.POINTER(sas_device_slot), vp],
    }
    for name, args in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    L.sas_status_string.argtypes = [ctypes.c_int]
    L.sas_status_string.restype = ctypes.c_char_p
    L.sas_version.argtypes = []
    L.sas_version.restype = ctypes.c_int
    return L


lib = _load()


def sas_status_string(code: int) -> str:
    return lib.sas_status_string(int(code)).decode()


def sas_version() -> int:
    return int(lib.sas_version())


@dataclass
class Params:
    """Mirror of ``sas_params``. ``seq_len`` is N for prefill and Lmax for decode."""
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    seq_len: int
    top_k: int
    block: int = BLOCK
    softmax_scale: float = 0.0
    gate_mode: int = SAS_GATE_LOG_SOFTMAX

    @property
    def n_blocks(self) -> int:
        return self.seq_len // self.block

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    def c(self) -> sas_params:
        return sas_params(self.batch, self.n_q_heads, self.n_kv_heads, self.head_dim, self.seq_len, self.block,
                          self.top_k, float(self.softmax_scale), int(self.gate_mode))


def _ptr(t: Optional[torch.Tensor], dtype: Optional[torch.dtype] = None, shape=None, name: str = "?"):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name}: expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name}: expected {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _check(fn: str, code: int):
    if code != 0:
        raise SasError(fn, code)


def _shapes(p: Params, decode: bool):
    B, Hq, Hkv, d, NB, K = p.batch, p.n_q_heads, p.n_kv_heads, p.head_dim, p.n_blocks, p.top_k
    if decode:
        return dict(s=(B, Hkv, NB), idx=(B, Hkv, K), lse_s=(B, Hkv))
    return dict(s=(B, Hkv, NB, NB), idx=(B, Hkv, NB, K), lse_s=(B, Hkv, NB), q=(B, Hq, p.seq_len, d),
                kv=(B, Hkv, p.seq_len, d), lse_o=(B, Hq, p.seq_len))


bf16, f32, i32 = torch.bfloat16, torch.float32, torch.int32


def sas_topk_select(p: Params, s: torch.Tensor, idx: torch.Tensor, lse_s: Optional[torch.Tensor] = None,
                    cache_len: Optional[torch.Tensor] = None, stream=None) -> None:
    sh = _shapes(p, cache_len is not None)
    _check("sas_topk_select", lib.sas_topk_select(
        ctypes.byref(p.c()), _ptr(s, f32, sh["s"], "s"), _ptr(cache_len, i32, (p.batch,), "cache_len"),
        _ptr(idx, i32, sh["idx"], "idx"), _ptr(lse_s, f32, sh["lse_s"], "lse_s"), _stream(stream)))


def sas_gate_lse(p: Params, s: torch.Tensor, lse_s: torch.Tensor, cache_len: Optional[torch.Tensor] = None,
                 stream=None) -> None:
    sh = _shapes(p, cache_len is not None)
    _check("sas_gate_lse", lib.sas_gate_lse(
        ctypes.byref(p.c()), _ptr(s, f32, sh["s"], "s"), _ptr(cache_len, i32, (p.batch,), "cache_len"),
        _ptr(lse_s, f32, sh["lse_s"], "lse_s"), _stream(stream)))


def sas_fwd(p: Params, q, k, v, s, idx, lse_s, o, lse_o=None, stream=None) -> None:
    sh = _shapes(p, False)
    _check("sas_fwd", lib.sas_fwd(
        ctypes.byref(p.c()), _ptr(q, bf16, sh["q"], "q"), _ptr(k, bf16, sh["kv"], "k"), _ptr(v, bf16, sh["kv"], "v"),
        _ptr(s, f32, sh["s"], "s"), _ptr(idx, i32, sh["idx"], "idx"), _ptr(lse_s, f32, sh["lse_s"], "lse_s"),
        _ptr(o, bf16, sh["q"], "o"), _ptr(lse_o, f32, sh["lse_o"], "lse_o"), _stream(stream)))


def sas_bwd_workspace_size(p: Params) -> int:
    n = ctypes.c_size_t(0)
    _check("sas_bwd_workspace_size", lib.sas_bwd_workspace_size(ctypes.byref(p.c()), ctypes.byref(n)))
    return int(n.value)


def sas_bwd_workspace_size_min(p: Params) -> int:
    n = ctypes.c_size_t(0)
    _check("sas_bwd_workspace_size_min", lib.sas_bwd_workspace_size_min(ctypes.byref(p.c()), ctypes.byref(n)))
    return int(n.value)


def sas_bwd(p: Params, q, k, v, o, dO, s, idx, lse_s, lse_o, dq, dk, dv, ds, ws: torch.Tensor, stream=None) -> None:
    sh = _shapes(p, False)
    _check("sas_bwd", lib.sas_bwd(
        ctypes.byref(p.c()), _ptr(q, bf16, sh["q"], "q"), _ptr(k, bf16, sh["kv"], "k"), _ptr(v, bf16, sh["kv"], "v"),
        _ptr(o, bf16, sh["q"], "o"), _ptr(dO, bf16, sh["q"], "dO"), _ptr(s, f32, sh["s"], "s"),
        _ptr(idx, i32, sh["idx"], "idx"), _ptr(lse_s, f32, sh["lse_s"], "lse_s"),
        _ptr(lse_o, f32, sh["lse_o"], "lse_o"), _ptr(dq, bf16, sh["q"], "dq"), _ptr(dk, bf16, sh["kv"], "dk"),
        _ptr(dv, bf16, sh["kv"], "dv"), _ptr(ds, f32, sh["s"], "ds"), _ptr(ws, None, None, "ws"),
        ctypes.c_size_t(ws.numel() * ws.element_size()), _stream(stream)))


def sas_decode(p: Params, q, kc, vc, cache_len, s, idx, lse_s, n_split: int, o_part, lse_part, stream=None) -> None:
    B, Hq, Hkv, d = p.batch, p.n_q_heads, p.n_kv_heads, p.head_dim
    sh = _shapes(p, True)
    _check("sas_decode", lib.sas_decode(
        ctypes.byref(p.c()), _ptr(q, bf16, (B, Hq, d), "q"), _ptr(kc, bf16, (B, Hkv, p.seq_len, d), "kc"),
        _ptr(vc, bf16, (B, Hkv, p.seq_len, d), "vc"), _ptr(cache_len, i32, (B,), "cache_len"),
        _ptr(s, f32, sh["s"], "s"), _ptr(idx, i32, sh["idx"], "idx"), _ptr(lse_s, f32, sh["lse_s"], "lse_s"),
        int(n_split), _ptr(o_part, f32, (B, Hq, n_split, d), "o_part"),
        _ptr(lse_part, f32, (B, Hq, n_split), "lse_part"), _stream(stream)))


def sas_decode_paged(p: Params, q, k_pages, v_pages, block_table, cache_len, s, idx, lse_s, n_split: int, o_part,
                     lse_part, stream=None) -> None:
    """sas_decode over a paged cache: k_pages/v_pages [n_pages, Hkv, 64, d], block_table int32 [B, NKB]."""
    B, Hq, Hkv, d = p.batch, p.n_q_heads, p.n_kv_heads, p.head_dim
    n_pages = int(k_pages.shape[0]) if k_pages is not None else 0
    sh = _shapes(p, True)
    _check("sas_decode_paged", lib.sas_decode_paged(
        ctypes.byref(p.c()), _ptr(q, bf16, (B, Hq, d), "q"), _ptr(k_pages, bf16, (n_pages, Hkv, p.block, d), "k_pages"),
        _ptr(v_pages, bf16, (n_pages, Hkv, p.block, d), "v_pages"), n_pages,
        _ptr(block_table, i32, (B, p.n_blocks), "block_table"), _ptr(cache_len, i32, (B,), "cache_len"),
        _ptr(s, f32, sh["s"], "s"), _ptr(idx, i32, sh["idx"], "idx"), _ptr(lse_s, f32, sh["lse_s"], "lse_s"),
        int(n_split), _ptr(o_part, f32, (B, Hq, n_split, d), "o_part"),
        _ptr(lse_part, f32, (B, Hq, n_split), "lse_part"), _stream(stream)))


def sas_decode_combine(p: Params, n_split: int, o_part, lse_part, o, lse_o=None, stream=None) -> None:
    B, Hq, d = p.batch, p.n_q_heads, p.head_dim
    _check("sas_decode_combine", lib.sas_decode_combine(
        ctypes.byref(p.c()), int(n_split), _ptr(o_part, f32, (B, Hq, n_split, d), "o_part"),
        _ptr(lse_part, f32, (B, Hq, n_split), "lse_part"), _ptr(o, bf16, (B, Hq, d), "o"),
        _ptr(lse_o, f32, (B, Hq), "lse_o"), _stream(stream)))


def sas_decode_noalloc(p: Params, q, kc, vc, cache_len, s, o, lse_o=None, stream=None) -> None:
    """Whole decode step with the library's fixed device scratch (see include/sas.h)."""
    B, Hq, Hkv, d = p.batch, p.n_q_heads, p.n_kv_heads, p.head_dim
    _check("sas_decode_noalloc", lib.sas_decode_noalloc(
        ctypes.byref(p.c()), _ptr(q, bf16, (B, Hq, d), "q"), _ptr(kc, bf16, (B, Hkv, p.seq_len, d), "kc"),
        _ptr(vc, bf16, (B, Hkv, p.seq_len, d), "vc"), _ptr(cache_len, i32, (B,), "cache_len"),
        _ptr(s, f32, (B, Hkv, p.n_blocks), "s"), _ptr(o, bf16, (B, Hq, d), "o"), _ptr(lse_o, f32, (B, Hq), "lse_o"),
        _stream(stream)))


def sas_decode_fused(p: Params, q, kc, vc, cache_len, s, o, idx=None, lse_s=None, lse_o=None, stream=None) -> None:
    """Whole decode step in one launch: select, attention, merge (idx, lse_s and lse_o are optional outputs)."""
    B, Hq, Hkv, d = p.batch, p.n_q_heads, p.n_kv_heads, p.head_dim
    sh = _shapes(p, True)
    _check("sas_decode_fused", lib.sas_decode_fused(
        ctypes.byref(p.c()), _ptr(q, bf16, (B, Hq, d), "q"), _ptr(kc, bf16, (B, Hkv, p.seq_len, d), "kc"),
        _ptr(vc, bf16, (B, Hkv, p.seq_len, d), "vc"), _ptr(cache_len, i32, (B,), "cache_len"),
        _ptr(s, f32, sh["s"], "s"), _ptr(idx, i32, sh["idx"], "idx"), _ptr(lse_s, f32, sh["lse_s"], "lse_s"),
        _ptr(o, bf16, (B, Hq, d), "o"), _ptr(lse_o, f32, (B, Hq), "lse_o"), _stream(stream)))


def sas_decode_fused_paged(p: Params, q, k_pages, v_pages, block_table, cache_len, s, o, idx=None, lse_s=None,
                           lse_o=None, stream=None) -> None:
    """sas_decode_fused over a paged cache: k_pages/v_pages [n_pages, Hkv, 64, d], block_table int32 [B, NKB]."""
    B, Hq, Hkv, d = p.batch, p.n_q_heads, p.n_kv_heads, p.head_dim
    n_pages = int(k_pages.shape[0]) if k_pages is not None else 0
    sh = _shapes(p, True)
    _check("sas_decode_fused_paged", lib.sas_decode_fused_paged(
        ctypes.byref(p.c()), _ptr(q, bf16, (B, Hq, d), "q"), _ptr(k_pages, bf16, (n_pages, Hkv, p.block, d), "k_pages"),
        _ptr(v_pages, bf16, (n_pages, Hkv, p.block, d), "v_pages"), n_pages,
        _ptr(block_table, i32, (B, p.n_blocks), "block_table"), _ptr(cache_len, i32, (B,), "cache_len"),
        _ptr(s, f32, sh["s"], "s"), _ptr(idx, i32, sh["idx"], "idx"), _ptr(lse_s, f32, sh["lse_s"], "lse_s"),
        _ptr(o, bf16, (B, Hq, d), "o"), _ptr(lse_o, f32, (B, Hq), "lse_o"), _stream(stream)))


def sas_block_mean_keys(p: Params, k, kmean, cache_len=None, stream=None) -> None:
    """k̄[b, h, m] = mean of block m's 64 keys (bf16). With cache_len, only each sequence's just-completed block."""
    B, Hkv, d = p.batch, p.n_kv_heads, p.head_dim
    _check("sas_block_mean_keys", lib.sas_block_mean_keys(
        ctypes.byref(p.c()), _ptr(k, bf16, (B, Hkv, p.seq_len, d), "k"), _ptr(cache_len, i32, (B,), "cache_len"),
        _ptr(kmean, bf16, (B, Hkv, p.n_blocks, d), "kmean"), _stream(stream)))


def sas_decode_select_scored(p: Params, q, kmean, cache_len, s, idx, lse_s=None, stream=None) -> None:
    """Selector scores from block-mean keys (written to s for m < c) and their decode-form Top-K, fused."""
    B, Hq, Hkv, d = p.batch, p.n_q_heads, p.n_kv_heads, p.head_dim
    sh = _shapes(p, True)
    _check("sas_decode_select_scored", lib.sas_decode_select_scored(
        ctypes.byref(p.c()), _ptr(q, bf16, (B, Hq, d), "q"), _ptr(kmean, bf16, (B, Hkv, p.n_blocks, d), "kmean"),
        _ptr(cache_len, i32, (B,), "cache_len"), _ptr(s, f32, sh["s"], "s"), _ptr(idx, i32, sh["idx"], "idx"),
        _ptr(lse_s, f32, sh["lse_s"], "lse_s"), _stream(stream)))


def _host_ptr(t: Optional[torch.Tensor], dtype, shape, name: str):
    if t is None:
        return None
    if t.is_cuda:
        raise ValueError(f"{name}: expected a host tensor (pinned memory lets the copies overlap)")
    if not t.is_contiguous() or t.dtype != dtype or tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected a contiguous {dtype} tensor of shape {tuple(shape)}")
    return t.data_ptr()


def sas_train_steps_host(p: Params, steps, slots, stream=None) -> None:
    """Training steps end to end from host memory (see include/sas.h): step i runs on slots[i % 2],
    with the upload of step i + 1 and the download of step i - 1 overlapping step i's kernels.

    steps: list of dicts of host tensors with keys q, k, v, s, do (inputs) and o, lse_o, dq, dk, dv,
    ds (outputs; lse_o and ds may be missing). slots: one or two dicts from ``empty_device_slot``.
    Asynchronous on ``stream``."""
    B, Hq, Hkv, N, d, NB = p.batch, p.n_q_heads, p.n_kv_heads, p.seq_len, p.head_dim, p.n_blocks
    qs, kvs, ss, ls = (B, Hq, N, d), (B, Hkv, N, d), (B, Hkv, NB, NB), (B, Hq, N)
    hs = (sas_host_step * len(steps))()
    for i, st in enumerate(steps):
        hs[i] = sas_host_step(
            _host_ptr(st["q"], bf16, qs, "q"), _host_ptr(st["k"], bf16, kvs, "k"), _host_ptr(st["v"], bf16, kvs, "v"),
            _host_ptr(st["s"], f32, ss, "s"), _host_ptr(st["do"], bf16, qs, "do"), _host_ptr(st["o"], bf16, qs, "o"),
            _host_ptr(st.get("lse_o"), f32, ls, "lse_o"), _host_ptr(st["dq"], bf16, qs, "dq"),
            _host_ptr(st["dk"], bf16, kvs, "dk"), _host_ptr(st["dv"], bf16, kvs, "dv"),
            _host_ptr(st.get("ds"), f32, ss, "ds"))
    K = p.top_k
    slot_layout = dict(q=(bf16, qs), k=(bf16, kvs), v=(bf16, kvs), do=(bf16, qs), o=(bf16, qs), dq=(bf16, qs),
                       dk=(bf16, kvs), dv=(bf16, kvs), s=(f32, ss), lse_s=(f32, (B, Hkv, NB)), lse_o=(f32, ls),
                       ds=(f32, ss), idx=(i32, (B, Hkv, NB, K)), ws=(torch.uint8, None))
    ds_ = (sas_device_slot * 2)()
    for k, sl in enumerate(slots[:2]):
        ptr = {n: (_ptr(sl[n], dt, shp, f"slots[{k}].{n}").value if sl.get(n) is not None else None)
               for n, (dt, shp) in slot_layout.items()}
        ds_[k] = sas_device_slot(ptr["q"], ptr["k"], ptr["v"], ptr["do"], ptr["o"], ptr["dq"], ptr["dk"], ptr["dv"],
                                 ptr["s"], ptr["lse_s"], ptr["lse_o"], ptr["ds"], ptr["idx"], ptr["ws"],
                                 sl["ws"].numel() if sl.get("ws") is not None else 0)
    _check("sas_train_steps_host", lib.sas_train_steps_host(ctypes.byref(p.c()), len(steps), hs, ds_,
                                                            _stream(stream)))


def sas_selftest_wait_timeout(stream=None) -> None:
    """One bounded wait that runs out (about a second); sas_get_device_error then reads SAS_ERR_TIMEOUT."""
    _check("sas_selftest_wait_timeout", lib.sas_selftest_wait_timeout(_stream(stream)))


def sas_get_device_error(stream=None) -> int:
    code = ctypes.c_int(0)
    _check("sas_get_device_error", lib.sas_get_device_error(_stream(stream), ctypes.byref(code)))
    return int(code.value)


# ---------------------------------------------------------------------------
# Allocation helpers (device memory comes from PyTorch)
# ---------------------------------------------------------------------------
def empty_prefill_outputs(p: Params, device="cuda", backward: bool = True) -> dict:
    B, Hq, Hkv, N, d, NB, K = p.batch, p.n_q_heads, p.n_kv_heads, p.seq_len, p.head_dim, p.n_blocks, p.top_k
    out = dict(
        idx=torch.empty((B, Hkv, NB, K), dtype=i32, device=device),
        lse_s=torch.empty((B, Hkv, NB), dtype=f32, device=device),
        o=torch.empty((B, Hq, N, d), dtype=bf16, device=device),
        lse_o=torch.empty((B, Hq, N), dtype=f32, device=device),
    )
    if backward:
        out.update(
            dq=torch.empty((B, Hq, N, d), dtype=bf16, device=device),
            dk=torch.empty((B, Hkv, N, d), dtype=bf16, device=device),
            dv=torch.empty((B, Hkv, N, d), dtype=bf16, device=device),
            ds=torch.empty((B, Hkv, NB, NB), dtype=f32, device=device),
            ws=torch.empty((sas_bwd_workspace_size(p),), dtype=torch.uint8, device=device),
        )
    return out


def empty_device_slot(p: Params, device="cuda") -> dict:
    """Device buffers of one training step for ``sas_train_steps_host``: inputs, outputs, idx, lse_s, workspace."""
    B, Hq, Hkv, N, d, NB = p.batch, p.n_q_heads, p.n_kv_heads, p.seq_len, p.head_dim, p.n_blocks
    slot = dict(q=torch.empty((B, Hq, N, d), dtype=bf16, device=device),
                k=torch.empty((B, Hkv, N, d), dtype=bf16, device=device),
                v=torch.empty((B, Hkv, N, d), dtype=bf16, device=device),
                s=torch.empty((B, Hkv, NB, NB), dtype=f32, device=device),
                do=torch.empty((B, Hq, N, d), dtype=bf16, device=device))
    slot.update(empty_prefill_outputs(p, device=device, backward=True))
    return slot


def empty_decode_outputs(p: Params, n_split: int, device="cuda") -> dict:
    B, Hq, Hkv, d, K = p.batch, p.n_q_heads, p.n_kv_heads, p.head_dim, p.top_k
    return dict(
        idx=torch.empty((B, Hkv, K), dtype=i32, device=device),
        lse_s=torch.empty((B, Hkv), dtype=f32, device=device),
        o_part=torch.empty((B, Hq, n_split, d), dtype=f32, device=device),
        lse_part=torch.empty((B, Hq, n_split), dtype=f32, device=device),
        o=torch.empty((B, Hq, d), dtype=bf16, device=device),
        lse_o=torch.empty((B, Hq), dtype=f32, device=device),
    )


def prefill_step(p: Params, q, k, v, s, dO, out: dict, backward: bool = True, stream=None) -> None:
    """One pass of the training hot path: select + LSE, forward, backward with ds."""
    sas_topk_select(p, s, out["idx"], out["lse_s"], stream=stream)
    sas_fwd(p, q, k, v, s, out["idx"], out["lse_s"], out["o"], out["lse_o"], stream=stream)
    if backward:
        sas_bwd(p, q, k, v, out["o"], dO, s, out["idx"], out["lse_s"], out["lse_o"], out["dq"], out["dk"], out["dv"],
                out["ds"], out["ws"], stream=stream)


def decode_step_paged(p: Params, q, k_pages, v_pages, block_table, cache_len, s, n_split: int, out: dict,
                      stream=None) -> None:
    """One decode step over a paged KV cache: select, split-K attention through the block table, merge."""
    sas_topk_select(p, s, out["idx"], out["lse_s"], cache_len=cache_len, stream=stream)
    sas_decode_paged(p, q, k_pages, v_pages, block_table, cache_len, s, out["idx"], out["lse_s"], n_split,
                     out["o_part"], out["lse_part"], stream=stream)
    sas_decode_combine(p, n_split, out["o_part"], out["lse_part"], out["o"], out["lse_o"], stream=stream)


def decode_step(p: Params, q, kc, vc, cache_len, s, n_split: int, out: dict, stream=None) -> None:
    """One decode step: Top-K select (decode form), split-K attention, LSE merge."""
    sas_topk_select(p, s, out["idx"], out["lse_s"], cache_len=cache_len, stream=stream)
    sas_decode(p, q, kc, vc, cache_len, s, out["idx"], out["lse_s"], n_split, out["o_part"], out["lse_part"],
               stream=stream)
    sas_decode_combine(p, n_split, out["o_part"], out["lse_part"], out["o"], out["lse_o"], stream=stream)


def decode_step_fused(p: Params, q, kc, vc, cache_len, s, out: dict, stream=None) -> None:
    """One decode step in one launch (select, attention, merge); fills out["o"], out["lse_o"], out["idx"] and
    out["lse_s"] when present."""
    sas_decode_fused(p, q, kc, vc, cache_len, s, out["o"], idx=out.get("idx"), lse_s=out.get("lse_s"),
                     lse_o=out.get("lse_o"), stream=stream)


def decode_step_scored(p: Params, q, kc, vc, kmean, cache_len, s, n_split: int, out: dict, stream=None) -> None:
    """A decode step that scores its own history: update the block means of any block the newest token
    completed, score and select in one launch (s is written), split-K attention, merge."""
    sas_block_mean_keys(p, kc, kmean, cache_len=cache_len, stream=stream)
    sas_decode_select_scored(p, q, kmean, cache_len, s, out["idx"], out["lse_s"], stream=stream)
    sas_decode(p, q, kc, vc, cache_len, s, out["idx"], out["lse_s"], n_split, out["o_part"], out["lse_part"],
               stream=stream)
    sas_decode_combine(p, n_split, out["o_part"], out["lse_part"], out["o"], out["lse_o"], stream=stream)


class DecodeGraph:
    """A decode step (select, split-K, merge) captured once as a CUDA graph.

    The graph records the buffers' addresses, so a serving loop writes the
    next step's query, scores and cache lengths into the same tensors and
    calls ``replay()``. One replay is three kernel launches with no host work
    between them. The three kernels are chained by programmatic dependent
    launch, so each one's launch overlaps the tail of the one before. With
    ``fused=True`` a replay is the single launch of sas_decode_fused.
    """

    def __init__(self, p: Params, q, kc, vc, cache_len, s, n_split: int, out: dict, stream=None, kmean=None,
                 fused: bool = False):
        # with kmean, the step scores its own history (decode_step_scored) and s is an output; with fused, the
        # step is the single launch of sas_decode_fused (n_split is then unused)
        if fused and kmean is None:
            self.step, self.args = decode_step_fused, (p, q, kc, vc, cache_len, s, out)
        elif kmean is None:
            self.step, self.args = decode_step, (p, q, kc, vc, cache_len, s, n_split, out)
        else:
            self.step, self.args = decode_step_scored, (p, q, kc, vc, kmean, cache_len, s, n_split, out)
        side = torch.cuda.Stream() if stream is None else stream
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):  # first call outside capture: kernel attributes get set here
            self.step(*self.args, stream=side)
        torch.cuda.current_stream().wait_stream(side)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, stream=side, capture_error_mode="thread_local"):
            self.step(*self.args, stream=side)

    def replay(self) -> None:
        self.graph.replay()
