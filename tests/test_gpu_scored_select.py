"""GPU parity: block-mean keys and the fused decode scoring + Top-K.

The scores are fp32 dot products on the GPU and fp64 in the oracle. Near a
Top-K boundary two blocks can be closer than that rounding, so the selection is
checked three ways:
* the scores themselves against the oracle, elementwise;
* the GPU's index list against an exact Top-K of the GPU's own scores, with
  ties to the lower index (the selection must be exact for what was scored);
* against the oracle's selection, every block clearly above the oracle's n-th
  score must be chosen and every block clearly below it must not.
Where the oracle's boundary gap exceeds the rounding (the small pipeline cases)
the index lists must be equal outright.
"""
import math

import numpy as np
import pytest
import torch

import oracle.sas_oracle as O
from synth import workloads as W
from tests.parity_util import TOL_O, assert_idx_equal, bf16_dev, host, max_abs

pytestmark = pytest.mark.gpu

TOL_S = 1e-5  # fp32 vs fp64 dot products of at most 128 bf16 terms, |s| < 10


def _sas():
    import learned_block_sparse_warp_b200 as sas
    return sas


def _bf16(g, shape, std=1.0):
    return W.bf16_round(g.standard_normal(shape).astype(np.float32) * np.float32(std))


def _topk_of(row: np.ndarray, n: int) -> list:
    """Exact Top-n of a float32 row: score descending, then index ascending; returned ascending."""
    order = np.lexsort((np.arange(len(row)), -row.astype(np.float64)))
    return sorted(int(m) for m in order[:n])


def _check_rows(s_gpu, idx_gpu, lse_gpu, s_ref, lse_ref, cache_len, K):
    B, H, _ = s_gpu.shape
    for b in range(B):
        c = (int(cache_len[b]) - 1) // 64
        n = min(K, c)
        for h in range(H):
            got_s = s_gpu[b, h, :c]
            ref_s = s_ref[b, h, :c]
            assert np.all(np.abs(got_s - ref_s) <= TOL_S * (1 + np.abs(ref_s))), (b, h)
            sel = idx_gpu[b, h, :n].tolist()
            assert (idx_gpu[b, h, n:] == -1).all()
            assert sel == _topk_of(got_s.astype(np.float32), n), (b, h)
            if 0 < n < c:
                kth = np.sort(ref_s)[::-1][n - 1]
                band = 4 * TOL_S * (1 + abs(kth))
                chosen = np.zeros(c, bool)
                chosen[sel] = True
                assert chosen[ref_s > kth + band].all() and not chosen[ref_s < kth - band].any(), (b, h)
            if c == 0:
                assert lse_gpu[b, h] == -math.inf
            else:
                assert abs(lse_gpu[b, h] - lse_ref[b, h]) < 1e-4, (b, h)


def _run_scored(B, Hq, Hkv, d, NB, K, cache_len, seed, kmean_np=None):
    sas = _sas()
    g = np.random.default_rng(seed)
    q = _bf16(g, (B, Hq, d))
    km = _bf16(g, (B, Hkv, NB, d), std=1 / 8) if kmean_np is None else kmean_np
    cl = np.asarray(cache_len, np.int32)
    p = sas.Params(batch=B, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, seq_len=NB * 64, top_k=K)
    s = torch.full((B, Hkv, NB), float("nan"), device="cuda")
    idx = torch.empty((B, Hkv, K), dtype=torch.int32, device="cuda")
    lse = torch.empty((B, Hkv), device="cuda")
    sas.sas_decode_select_scored(p, bf16_dev(q), bf16_dev(km), torch.from_numpy(cl).cuda(), s, idx, lse)
    torch.cuda.synchronize()
    err = sas.sas_get_device_error()
    s_ref, idx_ref, lse_ref = O.decode_select_scored(q, km, cl, K)
    return s.cpu().numpy(), idx.cpu().numpy(), lse.cpu().numpy(), s_ref, idx_ref, lse_ref, cl, err


SCORED_CASES = [
    # name, B, Hq, Hkv, d, NB, K, cache_len
    ("b1_512k", 1, 32, 8, 128, 8192, 16, [8192 * 64]),                # 8 rows: clusters of 8 CTAs
    ("b8_64k_ragged", 8, 32, 8, 128, 1024, 16, [65536, 65535, 64 * 700 + 1, 64 * 17, 64, 1, 4000, 65000]),
    ("b16_32k", 16, 32, 8, 128, 512, 16, [32768] * 16),               # 128 rows: one CTA each
    ("d64_k300", 2, 4, 2, 64, 3000, 300, [64 * 3000, 64 * 1000 + 1]),  # K past 256, d = 64
    ("k_ge_history", 3, 8, 2, 128, 40, 32, [1, 64 * 20 + 3, 64 * 40]),  # n = c for two rows
    ("g5", 1, 10, 2, 128, 2048, 64, [64 * 2048 - 7]),
]


@pytest.mark.parametrize("case", SCORED_CASES, ids=[c[0] for c in SCORED_CASES])
def test_scored_select_parity(case):
    name, B, Hq, Hkv, d, NB, K, cl = case
    s, idx, lse, s_ref, idx_ref, lse_ref, cl, err = _run_scored(B, Hq, Hkv, d, NB, K, cl, seed=len(name) * 7 + NB)
    assert err == 0
    _check_rows(s, idx, lse, s_ref, lse_ref, cl, K)


def test_scored_select_ties_across_the_cluster():
    """Zero block means score exactly 0. The positive blocks are taken first; the
    rest of K goes to the lowest-indexed zeros, which sit in the first CTA's
    slice, and blocks with negative scores are never taken."""
    NB, d, K = 4096, 128, 20
    km = np.zeros((1, 1, NB, d), np.float32)
    pos = [3000, 3500, 100, 4000, 2222]
    for j, m in enumerate(pos):
        km[0, 0, m, :] = 0.5 + 0.25 * j
    km[0, 0, 5:12, :] = -1.0  # negative scores among the low indices
    sas = _sas()
    q = np.ones((1, 4, d), np.float32)  # q̄ along +1: the signs above are the scores' signs
    p = sas.Params(batch=1, n_q_heads=4, n_kv_heads=1, head_dim=d, seq_len=NB * 64, top_k=K)
    s = torch.full((1, 1, NB), float("nan"), device="cuda")
    idx = torch.empty((1, 1, K), dtype=torch.int32, device="cuda")
    clt = torch.tensor([NB * 64], dtype=torch.int32, device="cuda")
    sas.sas_decode_select_scored(p, bf16_dev(q), bf16_dev(km), clt, s, idx, None)
    torch.cuda.synchronize()
    assert sas.sas_get_device_error() == 0
    _, idx_ref, _ = O.decode_select_scored(q, km, np.array([NB * 64]), K)
    assert_idx_equal(idx.cpu().numpy(), idx_ref)
    zeros = [m for m in range(NB - 1) if m not in pos and not 5 <= m < 12][:K - len(pos)]
    assert idx.cpu().numpy()[0, 0].tolist() == sorted(pos + zeros)


def test_scored_select_bad_cache_len_raises():
    s, idx, lse, *_, err = _run_scored(2, 4, 2, 128, 64, 4, [64 * 64 + 1, 100], seed=9)
    assert err == 6  # SAS_ERR_DEVICE_INDEX: row 0's cache_len is past Lmax
    assert (idx[0] == -1).all() and np.isneginf(lse[0]).all()
    assert (idx[1, :, 0] == 0).all()  # c = 1: the one history block


@pytest.mark.parametrize("d", [64, 128])
def test_block_mean_keys_full_cache(d):
    sas = _sas()
    g = np.random.default_rng(40 + d)
    B, Hkv, NB = 2, 3, 37
    k = _bf16(g, (B, Hkv, NB * 64, d)) + 0.25  # a nonzero mean
    p = sas.Params(batch=B, n_q_heads=Hkv, n_kv_heads=Hkv, head_dim=d, seq_len=NB * 64, top_k=4)
    km = torch.empty((B, Hkv, NB, d), dtype=torch.bfloat16, device="cuda")
    sas.sas_block_mean_keys(p, bf16_dev(W.bf16_round(k)), km)
    torch.cuda.synchronize()
    assert sas.sas_get_device_error() == 0
    ref = O.block_mean_keys(W.bf16_round(k))
    got = host(km)
    # one rounding to bf16 (half an ulp: 2^-8 relative at most) after an fp32 sum
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-5)


def test_block_mean_keys_decode_update_touches_completed_blocks_only():
    sas = _sas()
    g = np.random.default_rng(41)
    B, Hkv, NB, d = 5, 2, 37, 128
    k = W.bf16_round(_bf16(g, (B, Hkv, NB * 64, d)))
    cl = np.array([64 * 5, 64 * 7 + 3, 64, 1, 64 * 37], np.int32)
    p = sas.Params(batch=B, n_q_heads=2 * Hkv, n_kv_heads=Hkv, head_dim=d, seq_len=NB * 64, top_k=4)
    km = torch.full((B, Hkv, NB, d), 7.0, dtype=torch.bfloat16, device="cuda")
    sas.sas_block_mean_keys(p, bf16_dev(k), km, cache_len=torch.from_numpy(cl).cuda())
    torch.cuda.synchronize()
    assert sas.sas_get_device_error() == 0
    got = host(km)
    ref = O.block_mean_keys(k)
    written = {(0, 4), (2, 0), (4, 36)}
    for b in range(B):
        for m in range(NB):
            if (b, m) in written:
                assert np.all(np.abs(got[b, :, m] - ref[b, :, m]) <= 2.0 ** -8 * np.abs(ref[b, :, m]) + 1e-5)
            else:
                assert np.all(got[b, :, m] == 7.0), (b, m)


@pytest.mark.parametrize("gate", [O.GATE_NONE, O.GATE_LOG_SOFTMAX])
def test_decode_step_scored_pipeline(gate):
    """K cache -> block means -> fused scoring and Top-K -> split-K decode -> merge,
    against the oracle's block means (rounded to bf16 like the side cache),
    scores, selection and decode."""
    sas = _sas()
    w = W.custom("scored_pipe", kind="decode", batch=3, n_q_heads=8, n_kv_heads=2, head_dim=128, seq_len=64 * 50,
                 top_k=8, seed=61, backward=False, heavy_hitters=True)
    cl = np.array([64 * 50, 64 * 20 + 7, 64 * 31], np.int32)
    x = W.decode_inputs(w, cache_len=cl)
    p = sas.Params(batch=3, n_q_heads=8, n_kv_heads=2, head_dim=128, seq_len=64 * 50, top_k=8, gate_mode=gate)
    kc, vc, q = bf16_dev(x["k"]), bf16_dev(x["v"]), bf16_dev(x["q"])
    clt = torch.from_numpy(cl).cuda()
    km = torch.empty((3, 2, 50, 128), dtype=torch.bfloat16, device="cuda")
    sas.sas_block_mean_keys(p, kc, km)  # after the prefill: every block
    s = torch.empty((3, 2, 50), device="cuda")
    n_split = 3
    out = sas.empty_decode_outputs(p, n_split)
    sas.decode_step_scored(p, q, kc, vc, km, clt, s, n_split, out)
    torch.cuda.synchronize()
    assert sas.sas_get_device_error() == 0
    km_ref = W.bf16_round(O.block_mean_keys(x["k"]).astype(np.float32))
    s_ref = O.decode_scores(x["q"], km_ref, cl)
    ref = O.decode(x["q"], x["k"], x["v"], cl, s_ref, 8, gate_mode=gate, n_split=n_split)
    # the oracle's boundary gaps exceed the score rounding, so the lists must be equal
    for b in range(3):
        c = (int(cl[b]) - 1) // 64
        for h in range(2):
            srt = np.sort(s_ref[b, h, :c])[::-1]
            assert srt[7] - srt[8] > 1e-3
    assert_idx_equal(out["idx"].cpu().numpy(), ref["idx"])
    assert max_abs(host(out["o"]), ref["o"]) < TOL_O
    assert max_abs(out["lse_s"].cpu().numpy(), ref["lse_s"]) < 1e-4


def test_decode_graph_scored_replays_eager_step():
    sas = _sas()
    g = np.random.default_rng(62)
    B, Hq, Hkv, d, NB, K = 2, 8, 2, 128, 300, 16
    p = sas.Params(batch=B, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, seq_len=NB * 64, top_k=K,
                   gate_mode=O.GATE_LOG_SOFTMAX)
    kc, vc = bf16_dev(_bf16(g, (B, Hkv, NB * 64, d))), bf16_dev(_bf16(g, (B, Hkv, NB * 64, d)))
    q = bf16_dev(_bf16(g, (B, Hq, d)))
    clt = torch.tensor([NB * 64 - 5, 64 * 123], dtype=torch.int32, device="cuda")
    km = torch.empty((B, Hkv, NB, d), dtype=torch.bfloat16, device="cuda")
    sas.sas_block_mean_keys(p, kc, km)
    s = torch.empty((B, Hkv, NB), device="cuda")
    out = sas.empty_decode_outputs(p, 17)
    sas.decode_step_scored(p, q, kc, vc, km, clt, s, 17, out)
    torch.cuda.synchronize()
    eager = {k: v.clone() for k, v in out.items()}
    graph = sas.DecodeGraph(p, q, kc, vc, clt, s, 17, out, kmean=km)
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    assert sas.sas_get_device_error() == 0
    for k in ("idx", "lse_s", "o", "lse_o"):
        assert torch.equal(out[k], eager[k]), k
