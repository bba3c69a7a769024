"""GPU parity: Top-K selection (bit-exact index sets) and LSE(s), prefill and decode forms."""
import numpy as np
import pytest
import torch

import oracle.sas_oracle as O
from tests.parity_util import TOL_LSE_S, assert_idx_equal, f32_dev, host

pytestmark = pytest.mark.gpu


def _sas():
    import learned_block_sparse_warp_b200 as sas
    return sas


def _prefill_case(B, Hkv, NB, K, seed, quant=None, scale=np.sqrt(2.0)):
    g = np.random.default_rng(seed)
    s = (g.standard_normal((B, Hkv, NB, NB)) * scale).astype(np.float32)
    if quant is not None:
        s = (np.round(s / quant) * quant).astype(np.float32)
    return s


@pytest.mark.parametrize("B,Hkv,NB,K,quant", [
    (1, 2, 16, 4, None),      # the tiny workload's shape
    (2, 3, 64, 8, 0.5),       # heavy ties
    (1, 2, 40, 1, 1.0),       # K = 1 with ties
    (1, 1, 33, 64, None),     # K larger than every history
    (1, 8, 512, 32, None),    # training workload's row count per head
    (1, 2, 300, 64, 0.25),    # ragged row count, K = 64, ties
    (1, 1, 2048, 64, None),   # 128K-token rows
])
def test_select_prefill_bitexact(B, Hkv, NB, K, quant):
    sas = _sas()
    s = _prefill_case(B, Hkv, NB, K, seed=NB * 7 + K, quant=quant)
    p = sas.Params(batch=B, n_q_heads=Hkv, n_kv_heads=Hkv, head_dim=64, seq_len=NB * 64, top_k=K)
    ds = f32_dev(s)
    idx = torch.full((B, Hkv, NB, K), 12345, dtype=torch.int32, device="cuda")
    lse = torch.empty((B, Hkv, NB), dtype=torch.float32, device="cuda")
    sas.sas_topk_select(p, ds, idx, lse)
    torch.cuda.synchronize()
    ref_idx, ref_lse = O.prefill_select(s.astype(np.float64), K)
    assert_idx_equal(idx.cpu().numpy(), ref_idx)
    got = host(lse)
    assert np.all(np.isneginf(got[:, :, 0]))
    assert np.max(np.abs(got[:, :, 1:] - ref_lse[:, :, 1:])) < TOL_LSE_S
    # LSE alone through its own entry point
    lse2 = torch.empty_like(lse)
    sas.sas_gate_lse(p, ds, lse2)
    torch.cuda.synchronize()
    assert torch.equal(lse2, lse)
    assert sas.sas_get_device_error() == 0


def test_select_extreme_values():
    """Large magnitudes, -0 vs +0, and infinities rank like the fp64 sort."""
    sas = _sas()
    NB, K = 24, 5
    row = np.array([0.0, -0.0, 1e30, -1e30, 3.0, 3.0, -np.inf, 7.5, 1e-38, -1e-38, 2.0, 2.0,
                    -0.0, 0.0, 5.0, 5.0, 5.0, -2.0, 1.0, 1.0, 0.5, 0.5, 9.0, -9.0], dtype=np.float32)
    s = np.tile(row, (NB, 1))[None, None].astype(np.float32)
    p = sas.Params(batch=1, n_q_heads=1, n_kv_heads=1, head_dim=64, seq_len=NB * 64, top_k=K)
    idx = torch.empty((1, 1, NB, K), dtype=torch.int32, device="cuda")
    sas.sas_topk_select(p, f32_dev(s), idx)
    torch.cuda.synchronize()
    ref, _ = O.prefill_select(s.astype(np.float64), K)
    assert_idx_equal(idx.cpu().numpy(), ref)


@pytest.mark.parametrize("gate", [0, 1])
def test_select_decode_bitexact(gate):
    sas = _sas()
    B, Hkv, Lmax, K = 6, 4, 4096, 16
    g = np.random.default_rng(5)
    s = (g.standard_normal((B, Hkv, Lmax // 64)) * np.sqrt(2)).astype(np.float32)
    cl = np.array([1, 64, 65, 1000, 4095, 4096], dtype=np.int32)
    p = sas.Params(batch=B, n_q_heads=Hkv * 2, n_kv_heads=Hkv, head_dim=128, seq_len=Lmax, top_k=K, gate_mode=gate)
    idx = torch.empty((B, Hkv, K), dtype=torch.int32, device="cuda")
    lse = torch.empty((B, Hkv), dtype=torch.float32, device="cuda")
    sas.sas_topk_select(p, f32_dev(s), idx, lse, cache_len=torch.from_numpy(cl).cuda())
    torch.cuda.synchronize()
    ref_idx, ref_lse = O.decode_select(s.astype(np.float64), cl, K)
    assert_idx_equal(idx.cpu().numpy(), ref_idx)
    got = host(lse)
    fin = np.isfinite(ref_lse)
    assert np.all(np.isneginf(got[~fin]))
    assert np.max(np.abs(got[fin] - ref_lse[fin])) < TOL_LSE_S
    assert sas.sas_get_device_error() == 0


def test_select_decode_bad_cache_len_raises_device_error():
    """A cache length outside 1..Lmax is caught by the kernel's own check: no
    access goes out of bounds, the row is treated as empty and the error word
    is set."""
    sas = _sas()
    B, Hkv, Lmax, K = 2, 1, 1024, 4
    s = np.zeros((B, Hkv, Lmax // 64), np.float32)
    cl = np.array([Lmax + 64, 100], dtype=np.int32)
    p = sas.Params(batch=B, n_q_heads=1, n_kv_heads=1, head_dim=64, seq_len=Lmax, top_k=K)
    idx = torch.empty((B, Hkv, K), dtype=torch.int32, device="cuda")
    sas.sas_get_device_error()  # clear
    sas.sas_topk_select(p, f32_dev(s), idx, cache_len=torch.from_numpy(cl).cuda())
    assert sas.sas_get_device_error() == 6
    assert sas.sas_get_device_error() == 0  # cleared by the read
    assert (idx[0].cpu() == -1).all()
