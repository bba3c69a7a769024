"""GPU parity: the decode form of sas_topk_select on rows past 2048 blocks.

Those rows run on the cluster radix select. The scores are given in fp32, so
both sides rank the same values and the index lists must match bit for bit.
LSE(s) is an fp32 sum over up to 8191 scores: 1e-4 absolute.
"""
import numpy as np
import pytest
import torch

import oracle.sas_oracle as O
from tests.parity_util import TOL_LSE_S, assert_idx_equal, f32_dev, max_abs

pytestmark = pytest.mark.gpu


def _sas():
    import learned_block_sparse_warp_b200 as sas
    return sas


CASES = [
    # B, Hkv, NB, K, cache lengths, score kind
    (1, 8, 8192, 16, [8192 * 64], "normal"),                        # 512K tokens: 8-CTA clusters
    (2, 4, 3000, 300, [3000 * 64, 64 * 2100 + 9], "normal"),         # K past 256, ragged
    (3, 2, 4096, 64, [4096 * 64, 1, 64 * 2049], "ties"),             # rounded scores: many ties
    (16, 8, 2100, 16, [2100 * 64 - 1] * 16, "normal"),               # 128 rows: one CTA each
]


@pytest.mark.parametrize("B,Hkv,NB,K,lens,kind", CASES)
def test_long_decode_rows_select(B, Hkv, NB, K, lens, kind):
    sas = _sas()
    g = np.random.default_rng(NB + K)
    s = g.standard_normal((B, Hkv, NB)).astype(np.float32) * np.float32(np.sqrt(2))
    if kind == "ties":
        s = np.round(s * 4).astype(np.float32) / 4
    cl = np.array(lens, np.int32)
    p = sas.Params(batch=B, n_q_heads=Hkv, n_kv_heads=Hkv, head_dim=128, seq_len=NB * 64, top_k=K)
    idx = torch.empty((B, Hkv, K), dtype=torch.int32, device="cuda")
    lse = torch.empty((B, Hkv), device="cuda")
    lse_only = torch.empty((B, Hkv), device="cuda")
    clt = torch.from_numpy(cl).cuda()
    sd = f32_dev(s)
    sas.sas_topk_select(p, sd, idx, lse, cache_len=clt)
    sas.sas_gate_lse(p, sd, lse_only, cache_len=clt)
    torch.cuda.synchronize()
    assert sas.sas_get_device_error() == 0
    ref_idx, ref_lse = O.decode_select(s.astype(np.float64), cl, K)
    assert_idx_equal(idx.cpu().numpy(), ref_idx)
    got, got2 = lse.cpu().numpy(), lse_only.cpu().numpy()
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(got), fin) and np.array_equal(got, got2)
    assert max_abs(got[fin], ref_lse[fin]) < TOL_LSE_S * 10
