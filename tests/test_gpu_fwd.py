"""GPU parity: gated block-sparse forward (o and the row LSE) against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle.sas_oracle as O
from synth import workloads as W
from tests.parity_util import TOL_L, TOL_O, assert_idx_equal, bf16_dev, f32_dev, host, max_abs

pytestmark = pytest.mark.gpu


def _sas():
    import learned_block_sparse_warp_b200 as sas
    return sas


def run_prefill(w: W.Workload, gate: int, backward: bool = False, idx_override=None, ws_min: bool = False):
    """Runs select + fwd (+ bwd) on the GPU for a small workload; returns host arrays.

    ws_min: give the backward only its smallest workspace, so that its dQ pass
    recomputes S and dP instead of reading stored dZ tiles."""
    sas = _sas()
    x = W.prefill_inputs(w, with_do=backward)
    p = sas.Params(batch=w.batch, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, head_dim=w.head_dim,
                   seq_len=w.seq_len, top_k=w.top_k, gate_mode=gate)
    q, k, v = bf16_dev(x["q"]), bf16_dev(x["k"]), bf16_dev(x["v"])
    s = f32_dev(x["s"])
    out = sas.empty_prefill_outputs(p, backward=backward)
    if backward and ws_min:
        out["ws"] = torch.empty((sas.sas_bwd_workspace_size_min(p),), dtype=torch.uint8, device="cuda")
    sas.sas_topk_select(p, s, out["idx"], out["lse_s"])
    if idx_override is not None:
        out["idx"].copy_(torch.from_numpy(idx_override).cuda())
    sas.sas_fwd(p, q, k, v, s, out["idx"], out["lse_s"], out["o"], out["lse_o"])
    if backward:
        dO = bf16_dev(x["do"])
        sas.sas_bwd(p, q, k, v, out["o"], dO, s, out["idx"], out["lse_s"], out["lse_o"], out["dq"], out["dk"],
                    out["dv"], out["ds"], out["ws"])
    torch.cuda.synchronize()
    err = sas.sas_get_device_error()
    res = {kk: (vv.cpu().numpy() if vv.dtype == torch.int32 else host(vv)) for kk, vv in out.items() if kk != "ws"}
    return x, res, err


CASES = [
    # name, batch, Hq, Hkv, d, N, K
    ("tiny", 1, 2, 2, 64, 1024, 4),
    ("gqa4_d128", 1, 8, 2, 128, 1024, 4),
    ("gqa5_d128", 1, 10, 2, 128, 768, 3),
    ("dense_k", 1, 2, 1, 64, 512, 16),       # K >= every history: dense causal
    ("one_block", 2, 2, 2, 128, 64, 4),      # t = 0 only
    ("k1", 1, 4, 4, 64, 640, 1),
    ("batch3_d64_gqa2", 3, 4, 2, 64, 256, 2),
    # tcgen05 paths (d = 128): one head per head pair, batch 2, eight heads with every block
    # selected, and an odd group with K = 1
    ("g1_d128", 1, 3, 3, 128, 512, 4),
    ("g2_d128_b2", 2, 4, 2, 128, 512, 5),
    ("g8_d128_dense", 1, 8, 1, 128, 512, 16),
    ("g3_d128_k1", 1, 6, 2, 128, 640, 1),
]


@pytest.mark.parametrize("gate", [O.GATE_LOG_SOFTMAX, O.GATE_NONE])
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_fwd_parity(case, gate):
    name, B, Hq, Hkv, d, N, K = case
    w = W.custom(name, batch=B, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, seq_len=N, top_k=K, seed=100 + len(name))
    x, r, err = run_prefill(w, gate)
    assert err == 0
    ref_idx, _ = O.prefill_select(x["s"].astype(np.float64), K)
    assert_idx_equal(r["idx"], ref_idx)
    o, L = O.forward(x["q"], x["k"], x["v"], x["s"], ref_idx, gate_mode=gate)
    assert max_abs(r["o"], o) < TOL_O, max_abs(r["o"], o)
    assert max_abs(r["lse_o"], L) < TOL_L, max_abs(r["lse_o"], L)


def test_fwd_tiny_workload_exact_config():
    w = W.WORKLOADS["tiny"]
    x, r, err = run_prefill(w, O.GATE_LOG_SOFTMAX)
    assert err == 0
    ref_idx, _ = O.prefill_select(x["s"].astype(np.float64), w.top_k)
    o, L = O.forward(x["q"], x["k"], x["v"], x["s"], ref_idx)
    assert max_abs(r["o"], o) < TOL_O
    assert max_abs(r["lse_o"], L) < TOL_L


def test_fwd_out_of_range_index_is_skipped_and_reported():
    """An index at or beyond the query block is skipped by the kernel's own
    check (no out-of-bounds access) and raises SAS_ERR_DEVICE_INDEX."""
    w = W.custom("badidx", batch=1, n_q_heads=2, n_kv_heads=2, head_dim=64, seq_len=512, top_k=2, seed=3)
    x = W.prefill_inputs(w, with_do=False)
    ref_idx, _ = O.prefill_select(x["s"].astype(np.float64), 2)
    bad = ref_idx.copy()
    bad[0, 0, 5, 1] = 6  # t = 5 may not see block 6
    _sas().sas_get_device_error()
    _, r, err = run_prefill(w, O.GATE_NONE, idx_override=bad)
    assert err == 6
    # every other query block is untouched by the bad entry
    keep = bad.copy()
    keep[0, 0, 5, 1] = -1
    o, _ = O.forward(x["q"], x["k"], x["v"], x["s"], keep, gate_mode=O.GATE_NONE)
    assert max_abs(r["o"], o) < TOL_O
