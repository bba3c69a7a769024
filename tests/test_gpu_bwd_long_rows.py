"""GPU parity of the backward at the edge of the reverse index's two builds.

Rows of up to 4096 blocks build the reverse index (which query blocks selected
each KV block) from a column bitmap of the selection; longer rows test every
(query block, KV block) pair against the row's sorted list. Both builds must
give the same lists, in the same order, so the gradients must match the oracle
on either side of the edge: 4096 blocks (N = 262,144, the bitmap's largest
case, 128 words per row) and 4100 blocks (the pairwise kernels).

The oracle runs on the query blocks that touch a few KV blocks (the first four,
which many query blocks select, two in the middle and the last two): their own
diagonal blocks and every query block that selected one of them. dk and dv of
those KV blocks are then complete sums, and so are dq and the ds rows of those
query blocks.
"""
import numpy as np
import pytest
import torch

import oracle.sas_oracle as O
from synth import workloads as W
from tests.parity_util import TOL_REL, bf16_dev, f32_dev, host, rel_fro

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("nb", [4096, 4100])
def test_bwd_reverse_index_builds_agree(nb):
    import learned_block_sparse_warp_b200 as sas
    N, K, d = 64 * nb, 2, 64
    w = W.custom("long_rows", batch=1, n_q_heads=2, n_kv_heads=1, head_dim=d, seq_len=N, top_k=K, seed=nb)
    x = W.prefill_inputs(w, with_do=True)
    p = sas.Params(batch=1, n_q_heads=2, n_kv_heads=1, head_dim=d, seq_len=N, top_k=K,
                   gate_mode=sas.SAS_GATE_LOG_SOFTMAX)
    out = sas.empty_prefill_outputs(p)
    sas.prefill_step(p, bf16_dev(x["q"]), bf16_dev(x["k"]), bf16_dev(x["v"]), f32_dev(x["s"]), bf16_dev(x["do"]), out)
    torch.cuda.synchronize()
    assert sas.sas_get_device_error() == 0
    idx, _ = O.prefill_select(x["s"].astype(np.float64), K)
    assert np.array_equal(out["idx"].cpu().numpy(), idx)
    js = [0, 1, 2, 3, 1000, 2047, nb - 2, nb - 1]
    ts = sorted(set(js) | {t for t in range(nb) if np.isin(idx[0, 0, t], js).any()})
    assert len(ts) > 3 * len(js)  # the reverse lists are not only the diagonal entries
    dq, dk, dv, ds, _ = O.backward(x["q"], x["k"], x["v"], x["s"], idx, x["do"], t_list=ts)
    qrows = np.concatenate([np.arange(64 * t, 64 * t + 64) for t in ts])
    krows = np.concatenate([np.arange(64 * j, 64 * j + 64) for j in js])
    errs = {"dq": rel_fro(host(out["dq"])[:, :, qrows], dq[:, :, qrows]),
            "dk": rel_fro(host(out["dk"])[:, :, krows], dk[:, :, krows]),
            "dv": rel_fro(host(out["dv"])[:, :, krows], dv[:, :, krows]),
            "ds": rel_fro(host(out["ds"])[:, :, ts], ds[:, :, ts])}
    assert all(e < TOL_REL for e in errs.values()), errs
