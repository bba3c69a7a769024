"""GPU parity: backward dq/dk/dv and the score gradient ds against the fp64 oracle."""
import numpy as np
import pytest

import oracle.sas_oracle as O
from synth import workloads as W
from tests.parity_util import TOL_L, TOL_O, TOL_REL, assert_idx_equal, max_abs, rel_fro
from tests.test_gpu_fwd import run_prefill

pytestmark = pytest.mark.gpu

CASES = [
    ("tiny", 1, 2, 2, 64, 1024, 4),
    ("gqa4_d128", 1, 8, 2, 128, 1024, 4),
    ("gqa5_d128", 1, 10, 2, 128, 768, 3),
    ("dense_k", 1, 2, 1, 64, 512, 16),
    ("one_block", 2, 2, 2, 128, 64, 4),
    ("k1_batch2", 2, 4, 4, 64, 640, 1),
    # tcgen05 paths (d = 128): one head per head pair, batch 2, eight heads with every block
    # selected, and an odd group with K = 1
    ("g1_d128", 1, 3, 3, 128, 512, 4),
    ("g2_d128_b2", 2, 4, 2, 128, 512, 5),
    ("g8_d128_dense", 1, 8, 1, 128, 512, 16),
    ("g3_d128_k1", 1, 6, 2, 128, 640, 1),
]


ABLATION_CASES = [c for c in CASES if c[0] in ("tiny", "gqa4_d128", "g3_d128_k1", "g2_d128_b2")]


@pytest.mark.parametrize("gate", [O.GATE_LOG_SOFTMAX, O.GATE_NONE])
@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_bwd_parity(case, gate):
    _check_bwd(case, gate)


@pytest.mark.parametrize("gate", [O.GATE_LOG_SIGMOID, O.GATE_LOGIT])
@pytest.mark.parametrize("case", ABLATION_CASES, ids=[c[0] for c in ABLATION_CASES])
def test_bwd_gate_ablations(case, gate):
    """The gate-activation ablations: log σ(s) and the raw logit inside the softmax,
    with their own chain to ds. The forward output is checked on the way."""
    x, r = _check_bwd(case, gate)
    ref_idx, _ = O.prefill_select(x["s"].astype(np.float64), case[6])
    o, L = O.forward(x["q"], x["k"], x["v"], x["s"], ref_idx, gate_mode=gate)
    assert max_abs(r["o"], o) < TOL_O
    assert max_abs(r["lse_o"], L) < TOL_L


SMALL_WS_CASES = [c for c in CASES if c[5] > 64]


@pytest.mark.parametrize("gate", [O.GATE_LOG_SOFTMAX, O.GATE_NONE])
@pytest.mark.parametrize("case", SMALL_WS_CASES, ids=[c[0] for c in SMALL_WS_CASES])
def test_bwd_small_workspace(case, gate):
    """With only the smallest workspace the dQ pass recomputes S and dP instead of
    reading the stored dZ tiles; both forms must match the oracle."""
    _check_bwd(case, gate, ws_min=True)


def test_bwd_workspace_sizes():
    import learned_block_sparse_warp_b200 as sas
    # head_dim 128: the full workspace adds one 16 KB dZ tile per (query block, attended block, head pair)
    p = sas.Params(batch=1, n_q_heads=8, n_kv_heads=2, head_dim=128, seq_len=1024, top_k=4)
    slots = sum(1 + min(4, t) for t in range(16))
    extra = sas.sas_bwd_workspace_size(p) - sas.sas_bwd_workspace_size_min(p)
    assert 2 * slots * 2 * 16384 <= extra < 2 * slots * 2 * 16384 + 256
    # head_dim 64 runs the same passes: the same dZ tiles
    p64 = sas.Params(batch=1, n_q_heads=8, n_kv_heads=2, head_dim=64, seq_len=1024, top_k=4)
    assert sas.sas_bwd_workspace_size(p64) - sas.sas_bwd_workspace_size_min(p64) == extra


def _check_bwd(case, gate, ws_min=False):
    name, B, Hq, Hkv, d, N, K = case
    w = W.custom(name, batch=B, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, seq_len=N, top_k=K, seed=200 + len(name))
    x, r, err = run_prefill(w, gate, backward=True, ws_min=ws_min)
    assert err == 0
    ref_idx, _ = O.prefill_select(x["s"].astype(np.float64), K)
    assert_idx_equal(r["idx"], ref_idx)
    dq, dk, dv, ds, _ = O.backward(x["q"], x["k"], x["v"], x["s"], ref_idx, x["do"], gate_mode=gate)
    errs = {n: rel_fro(r[n], ref) for n, ref in (("dq", dq), ("dk", dk), ("dv", dv))}
    assert all(e < TOL_REL for e in errs.values()), errs
    if gate == O.GATE_NONE:
        assert np.all(r["ds"] == 0)
    elif N > 64:
        e = rel_fro(r["ds"], ds)
        assert e < TOL_REL, e
        # entries at or above the diagonal are exactly zero
        NB = N // 64
        iu = np.triu_indices(NB)
        assert np.all(r["ds"][..., iu[0], iu[1]] == 0)
    else:
        assert np.all(r["ds"] == 0)
    return x, r


def test_bwd_tiny_workload_exact_config():
    w = W.WORKLOADS["tiny"]
    x, r, err = run_prefill(w, O.GATE_LOG_SOFTMAX, backward=True)
    assert err == 0
    ref_idx, _ = O.prefill_select(x["s"].astype(np.float64), w.top_k)
    dq, dk, dv, ds, _ = O.backward(x["q"], x["k"], x["v"], x["s"], ref_idx, x["do"])
    for n, ref in (("dq", dq), ("dk", dk), ("dv", dv), ("ds", ds)):
        assert rel_fro(r[n], ref) < TOL_REL, (n, rel_fro(r[n], ref))
