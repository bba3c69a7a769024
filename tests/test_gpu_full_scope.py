"""Full scope and large K: index lists longer than 256 blocks.

With K >= t every query block attends to its whole causal history, each block
weighted by its softmax-normalised gate. The sequence here has 320 blocks, so
the block lists, the reverse index of the backward and the ds chain all hold
more than 256 entries per row.
- K = 320 (every history block), log-softmax gate: the whole backward
  (dq, dk, dv, ds) against the fp64 oracle.
- K = 320 without a gate, and K = 300 (a real Top-K past 256 slots): the
  forward and dq on sampled query blocks, and the ds rows of those blocks.
  Each of these depends on its own query block only.
"""
import numpy as np
import pytest
import torch

import oracle.sas_oracle as O
from synth import workloads as W
from tests.parity_util import TOL_L, TOL_O, TOL_REL, assert_idx_equal, bf16_dev, f32_dev, host, max_abs, rel_fro

pytestmark = pytest.mark.gpu

NB = 320
N = NB * 64


def _run(K, gate, Hq, Hkv, seed):
    import learned_block_sparse_warp_b200 as sas
    w = W.custom("full_scope", batch=1, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=128, seq_len=N, top_k=K, seed=seed)
    x = W.prefill_inputs(w, with_do=True)
    p = sas.Params(batch=1, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=128, seq_len=N, top_k=K, gate_mode=gate)
    out = sas.empty_prefill_outputs(p, backward=True)
    sas.prefill_step(p, bf16_dev(x["q"]), bf16_dev(x["k"]), bf16_dev(x["v"]), f32_dev(x["s"]), bf16_dev(x["do"]),
                     out, backward=True)
    torch.cuda.synchronize()
    assert sas.sas_get_device_error() == 0
    ref_idx, _ = O.prefill_select(x["s"].astype(np.float64), K)
    assert_idx_equal(out["idx"].cpu().numpy(), ref_idx)
    got = {n: host(out[n]) for n in ("o", "lse_o", "dq", "dk", "dv", "ds")}
    for n in ("o", "dq", "dk", "dv"):
        assert np.isfinite(got[n]).all(), n
    return x, ref_idx, got


def test_full_scope_whole_backward():
    K = NB
    x, idx, got = _run(K, O.GATE_LOG_SOFTMAX, 2, 1, seed=77)
    # every history block selected, ascending, then -1
    for t in (0, 1, 255, 256, 257, NB - 1):
        assert idx[0, 0, t, :t].tolist() == list(range(t)) and (idx[0, 0, t, t:] == -1).all()
    dq, dk, dv, ds, _ = O.backward(x["q"], x["k"], x["v"], x["s"], idx, x["do"])
    errs = {n: rel_fro(got[n], ref) for n, ref in (("dq", dq), ("dk", dk), ("dv", dv), ("ds", ds))}
    assert all(e < TOL_REL for e in errs.values()), errs
    iu = np.triu_indices(NB)
    assert np.all(got["ds"][..., iu[0], iu[1]] == 0)


@pytest.mark.parametrize("K,gate", [(NB, O.GATE_NONE), (300, O.GATE_LOG_SOFTMAX)])
def test_large_k_sampled_blocks(K, gate):
    x, idx, got = _run(K, gate, 4, 1, seed=78 + K)
    ts = [0, 1, 200, 258, 301, NB - 1]
    o, L = O.forward(x["q"], x["k"], x["v"], x["s"], idx, gate_mode=gate, t_list=ts)
    dq, _, _, ds, _ = O.backward(x["q"], x["k"], x["v"], x["s"], idx, x["do"], gate_mode=gate, t_list=ts)
    rows = np.concatenate([np.arange(64 * t, 64 * t + 64) for t in ts])
    assert max_abs(got["o"][:, :, rows], o[:, :, rows]) < TOL_O
    assert max_abs(got["lse_o"][:, :, rows], L[:, :, rows]) < TOL_L
    assert rel_fro(got["dq"][:, :, rows], dq[:, :, rows]) < TOL_REL
    if gate == O.GATE_NONE:
        assert np.all(got["ds"] == 0)
    else:
        for t in ts[1:]:
            assert rel_fro(got["ds"][0, 0, t, :t], ds[0, 0, t, :t]) < TOL_REL, t
