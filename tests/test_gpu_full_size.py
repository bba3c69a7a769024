"""GPU parity at the benchmark workloads' full sizes.

The GPU runs the whole workload exactly as bench.py launches it. The fp64
oracle then checks what it can finish in seconds to a minute:
* Top-K index sets and LSE(s) of every row of every head, bit-exact and to
  1e-4 respectively;
* the forward on sampled query blocks of one KV head (all of its query heads);
* the backward on one whole KV head (dq of its query heads, dk, dv, ds);
* decode on sampled sequences, at full and ragged cache lengths;
* properties that hold at any size: each ds row sums to zero, ds is zero on
  and above the diagonal, and every o and dq value is finite.
"""
import numpy as np
import pytest
import torch

import oracle.sas_oracle as O
from synth import workloads as W
from synth.device import decode_to_device, prefill_to_device
from tests.parity_util import TOL_L, TOL_LSE_S, TOL_O, TOL_REL, assert_idx_equal, host, max_abs, rel_fro

pytestmark = pytest.mark.gpu


def _sas():
    import learned_block_sparse_warp_b200 as sas
    return sas


def _params(sas, w, gate):
    return sas.Params(batch=w.batch, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, head_dim=w.head_dim,
                      seq_len=w.seq_len, top_k=w.top_k, gate_mode=gate)


def _check_select_all_heads(w, s_dev, idx_dev, lse_dev):
    s = s_dev.cpu().numpy().astype(np.float64)
    ref_idx, ref_lse = O.prefill_select(s, w.top_k)
    assert_idx_equal(idx_dev.cpu().numpy(), ref_idx)
    got = host(lse_dev)
    assert np.all(np.isneginf(got[:, :, 0]))
    assert max_abs(got[:, :, 1:], ref_lse[:, :, 1:]) < TOL_LSE_S
    return ref_idx


def _run_prefill_full(w, gate, h_check, t_sample, backward):
    sas = _sas()
    p = _params(sas, w, gate)
    x = prefill_to_device(w, with_do=backward)
    out = sas.empty_prefill_outputs(p, backward=backward)
    sas.prefill_step(p, x["q"], x["k"], x["v"], x["s"], x.get("do"), out, backward=backward)
    torch.cuda.synchronize()
    assert sas.sas_get_device_error() == 0
    ref_idx = _check_select_all_heads(w, x["s"], out["idx"], out["lse_s"])
    assert torch.isfinite(out["o"].float()).all()
    G = w.group
    hs = slice(h_check * G, (h_check + 1) * G)
    xo = W.prefill_inputs(w, kv_heads=[h_check], with_do=backward)
    idx_h = ref_idx[:, h_check:h_check + 1]
    o, L = O.forward(xo["q"], xo["k"], xo["v"], xo["s"], idx_h, gate_mode=gate, t_list=t_sample)
    rows = np.concatenate([np.arange(64 * t, 64 * t + 64) for t in t_sample])
    got_o = host(out["o"][:, hs])
    got_L = host(out["lse_o"][:, hs])
    assert max_abs(got_o[:, :, rows], o[:, :, rows]) < TOL_O
    assert max_abs(got_L[:, :, rows], L[:, :, rows]) < TOL_L
    if not backward:
        return
    assert torch.isfinite(out["dq"].float()).all()
    dq, dk, dv, ds, _ = O.backward(xo["q"], xo["k"], xo["v"], xo["s"], idx_h, xo["do"], gate_mode=gate)
    errs = {"dq": rel_fro(host(out["dq"][:, hs]), dq), "dk": rel_fro(host(out["dk"][:, h_check:h_check + 1]), dk),
            "dv": rel_fro(host(out["dv"][:, h_check:h_check + 1]), dv)}
    ds_all = host(out["ds"])
    if gate == O.GATE_LOG_SOFTMAX:
        errs["ds"] = rel_fro(ds_all[:, h_check:h_check + 1], ds)
        # any size: each row sums to zero; nothing on or above the diagonal
        assert np.abs(ds_all.sum(-1)).max() < 1e-3 * max(1.0, np.abs(ds_all).max())
        iu = np.triu_indices(w.n_blocks)
        assert np.all(ds_all[..., iu[0], iu[1]] == 0)
    else:
        assert np.all(ds_all == 0)
    assert all(e < TOL_REL for e in errs.values()), errs


def test_qwen3_4b_train_32k_full_size():
    w = W.WORKLOADS["qwen3_4b_train_32k"]
    _run_prefill_full(w, O.GATE_LOG_SOFTMAX, h_check=5, t_sample=[0, 1, 2, 31, 32, 33, 200, 511], backward=True)


def test_qwen3_14b_gqa5_8k_full_size():
    w = W.WORKLOADS["qwen3_14b_k16_n8192"]
    _run_prefill_full(w, O.GATE_LOG_SOFTMAX, h_check=7, t_sample=[0, 15, 16, 17, 127], backward=True)


def test_llama31_8b_fwd_128k_full_size():
    w = W.WORKLOADS["llama31_8b_fwd_128k"]
    _run_prefill_full(w, O.GATE_LOG_SOFTMAX, h_check=2, t_sample=[0, 1, 63, 64, 65, 1024, 2047], backward=False)


@pytest.mark.parametrize("ragged", [False, True])
def test_decode_b16_32k_full_size(ragged):
    sas = _sas()
    w = W.WORKLOADS["decode_b16_32k"]
    cl = None
    if ragged:
        cl = np.array([32768, 1, 30001, 16385, 64, 65, 4097, 32767, 12345, 99, 31000, 2048, 2049, 777, 20000, 5],
                      dtype=np.int32)
    x = decode_to_device(w, cache_len=cl)
    p = _params(sas, w, sas.SAS_GATE_NONE)
    n_split = w.top_k + 1
    out = sas.empty_decode_outputs(p, n_split)
    sas.decode_step(p, x["q"], x["k"], x["v"], x["cache_len"], x["s"], n_split, out)
    torch.cuda.synchronize()
    assert sas.sas_get_device_error() == 0
    cls = x["cache_len"].cpu().numpy()
    s = x["s"].cpu().numpy().astype(np.float64)
    ref_idx, ref_lse = O.decode_select(s, cls, w.top_k)
    assert_idx_equal(out["idx"].cpu().numpy(), ref_idx)
    for b in (0, 9, 15):
        q = np.stack([W.q_slice(w, b, hq) for hq in range(w.n_q_heads)])[None]
        kc = np.stack([W.k_slice(w, b, h) for h in range(w.n_kv_heads)])[None]
        vc = np.stack([W.v_slice(w, b, h) for h in range(w.n_kv_heads)])[None]
        ref = O.decode(q, kc, vc, cls[b:b + 1], s[b:b + 1], w.top_k, n_split=n_split)
        assert max_abs(host(out["o"][b:b + 1]), ref["o"]) < TOL_O
        assert max_abs(host(out["lse_o"][b:b + 1]), ref["lse"]) < TOL_L
        lp = host(out["lse_part"][b:b + 1])
        fin = np.isfinite(ref["lse_part"])
        assert np.array_equal(np.isfinite(lp), fin)
        assert max_abs(host(out["o_part"][b:b + 1]), ref["o_part"]) < TOL_O
