"""GPU parity for the gate outside the softmax: o = Σ_j g_{m(j)} p_j v_j.

The softmax runs over the plain logits and g = softmax(s) weights each history
block's values; the backward takes dV from g·p, dZ = p·(g·dP − D) and
dl = Σ p·g·dP. Forward, backward (dq, dk, dv, ds) and split-K decode against the
fp64 oracle, on the d = 128 tcgen05 kernels and the d = 64 kernels.
"""
import numpy as np
import pytest
import torch

import oracle.sas_oracle as O
from tests.parity_util import TOL_L, TOL_O, assert_idx_equal, bf16_dev, f32_dev, host, max_abs
from tests.test_gpu_bwd import _check_bwd
from tests.test_gpu_decode import _case

pytestmark = pytest.mark.gpu

OUT = O.GATE_SOFTMAX_OUTSIDE

CASES = [
    # name, batch, Hq, Hkv, d, N, K
    ("tiny_d64", 1, 2, 2, 64, 1024, 4),
    ("gqa4_d128", 1, 8, 2, 128, 1024, 4),
    ("g3_d128_k1", 1, 6, 2, 128, 640, 1),
    ("g2_d128_b2", 2, 4, 2, 128, 512, 5),
    ("dense_d128", 1, 4, 1, 128, 512, 16),  # every history block selected
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_gate_outside_fwd_bwd(case):
    x, r = _check_bwd(case, OUT)  # dq, dk, dv, ds against the oracle
    ref_idx, _ = O.prefill_select(x["s"].astype(np.float64), case[6])
    o, L = O.forward(x["q"], x["k"], x["v"], x["s"], ref_idx, gate_mode=OUT)
    assert max_abs(r["o"], o) < TOL_O
    assert max_abs(r["lse_o"], L) < TOL_L


@pytest.mark.parametrize("d", [64, 128])
def test_gate_outside_decode(d):
    import learned_block_sparse_warp_b200 as sas
    B, Hq, Hkv, Lmax, K, n_split = 3, 16, 4, 2048, 8, 3
    q, kc, vc, s = _case(B, Hq, Hkv, d, Lmax, seed=71 + d)
    cl = np.array([2048, 777, 65], dtype=np.int32)
    p = sas.Params(batch=B, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, seq_len=Lmax, top_k=K, gate_mode=OUT)
    out = sas.empty_decode_outputs(p, n_split)
    sas.decode_step(p, bf16_dev(q), bf16_dev(kc), bf16_dev(vc), torch.from_numpy(cl).cuda(), f32_dev(s), n_split, out)
    torch.cuda.synchronize()
    assert sas.sas_get_device_error() == 0
    ref = O.decode(q, kc, vc, cl, s.astype(np.float64), K, gate_mode=OUT, n_split=n_split)
    assert_idx_equal(out["idx"].cpu().numpy(), ref["idx"])
    assert max_abs(host(out["o_part"]), ref["o_part"]) < TOL_O
    assert max_abs(host(out["o"]), ref["o"]) < TOL_O
    assert max_abs(host(out["lse_o"]), ref["lse"]) < TOL_L
