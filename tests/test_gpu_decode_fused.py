"""GPU parity: the one-launch decode step (sas_decode_fused) against the fp64 oracle.

The step selects each row's Top-K blocks inside the kernel, so its picks are
compared bit for bit with the oracle's (lowest block index first among equal
scores), its gate normaliser and its merged output within the parity
tolerances. The shapes cover every cluster size the launcher picks (1, 2, 4
and 8 CTAs per row), d = 64 and 128, G from 1 to 8, every gate mode, ragged
and one-token caches, K at and above the history, and the paged cache.
"""
import numpy as np
import pytest
import torch

import oracle.sas_oracle as O
from tests.parity_util import TOL_L, TOL_O, assert_idx_equal, bf16_dev, f32_dev, host, max_abs
from tests.test_gpu_decode import _case, _paged

pytestmark = pytest.mark.gpu

GATES = [O.GATE_NONE, O.GATE_LOG_SOFTMAX, O.GATE_LOG_SIGMOID, O.GATE_LOGIT, O.GATE_SOFTMAX_OUTSIDE]


def _sas():
    import learned_block_sparse_warp_b200 as sas
    return sas


def _outputs(p):
    B, Hq, Hkv, d, K = p.batch, p.n_q_heads, p.n_kv_heads, p.head_dim, p.top_k
    return dict(o=torch.empty((B, Hq, d), dtype=torch.bfloat16, device="cuda"),
                lse_o=torch.empty((B, Hq), dtype=torch.float32, device="cuda"),
                idx=torch.empty((B, Hkv, K), dtype=torch.int32, device="cuda"),
                lse_s=torch.empty((B, Hkv), dtype=torch.float32, device="cuda"))


def _check(out, ref, gate):
    assert_idx_equal(out["idx"].cpu().numpy(), ref["idx"])
    got = host(out["lse_s"])
    fin = np.isfinite(ref["lse_s"])
    assert np.array_equal(np.isfinite(got), fin) and np.all(got[~fin] == -np.inf)
    assert max_abs(got[fin], ref["lse_s"][fin]) < 1e-4
    o = host(out["o"])
    assert np.isfinite(o).all()
    assert max_abs(o, ref["o"]) < TOL_O, (gate, max_abs(o, ref["o"]))
    assert max_abs(host(out["lse_o"]), ref["lse"]) < TOL_L


# rows = B·Hkv sets the cluster size: 32 rows -> 8 CTAs per row, 128 -> 2, 320 -> 1, 1 row with K = 2 -> 2
SHAPES = [
    (4, 32, 8, 128, 2048, 16, [2048, 1, 1000, 1999]),
    (16, 32, 8, 128, 2048, 16, None),
    (40, 8, 8, 64, 1024, 4, None),
    (3, 8, 8, 64, 1024, 4, [64, 65, 1024]),
    (2, 10, 2, 128, 4096, 8, [4096, 4033]),
    (2, 16, 2, 128, 1024, 32, [1024, 130]),   # K above the history: every block, G = 8
    (1, 4, 1, 64, 512, 2, [300]),
    (2, 6, 2, 128, 8192, 64, [8192, 5000]),   # G = 3, 64 picks over 127 blocks
]


@pytest.mark.parametrize("gate", GATES)
@pytest.mark.parametrize("B,Hq,Hkv,d,Lmax,K,lens", SHAPES)
def test_decode_fused_parity(B, Hq, Hkv, d, Lmax, K, lens, gate):
    sas = _sas()
    q, kc, vc, s = _case(B, Hq, Hkv, d, Lmax, seed=B * 13 + K + gate)
    if lens is None:
        lens = list(np.random.default_rng(B + K).integers(1, Lmax + 1, size=B))
    cl = np.array(lens, dtype=np.int32)
    p = sas.Params(batch=B, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, seq_len=Lmax, top_k=K, gate_mode=gate)
    out = _outputs(p)
    sas.decode_step_fused(p, bf16_dev(q), bf16_dev(kc), bf16_dev(vc), torch.from_numpy(cl).cuda(), f32_dev(s), out)
    torch.cuda.synchronize()
    assert sas.sas_get_device_error() == 0
    ref = O.decode(q, kc, vc, cl, s.astype(np.float64), K, gate_mode=gate, n_split=1)
    _check(out, ref, gate)


def test_decode_fused_ties_take_the_lowest_blocks():
    """Scores drawn from three values: most picks are decided by the block index."""
    sas = _sas()
    B, Hq, Hkv, d, Lmax, K = 4, 16, 4, 128, 4096, 16
    q, kc, vc, _ = _case(B, Hq, Hkv, d, Lmax, seed=3)
    g = np.random.default_rng(4)
    s = g.choice(np.array([-1.0, 0.5, 2.0], np.float32), size=(B, Hkv, Lmax // 64))
    cl = np.array([4096, 4000, 1500, 700], np.int32)
    p = sas.Params(batch=B, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, seq_len=Lmax, top_k=K,
                   gate_mode=O.GATE_LOG_SOFTMAX)
    out = _outputs(p)
    sas.decode_step_fused(p, bf16_dev(q), bf16_dev(kc), bf16_dev(vc), torch.from_numpy(cl).cuda(), f32_dev(s), out)
    torch.cuda.synchronize()
    assert sas.sas_get_device_error() == 0
    ref = O.decode(q, kc, vc, cl, s.astype(np.float64), K, gate_mode=O.GATE_LOG_SOFTMAX, n_split=1)
    _check(out, ref, O.GATE_LOG_SOFTMAX)


def test_decode_fused_equals_the_separate_calls_picks():
    """The in-kernel selection writes exactly the lists of sas_topk_select (decode form)."""
    sas = _sas()
    B, Hq, Hkv, d, Lmax, K = 16, 32, 8, 128, 32768, 16
    q, kc, vc, s = _case(B, Hq, Hkv, d, Lmax, seed=21)
    cl = torch.from_numpy(np.random.default_rng(2).integers(1, Lmax + 1, size=B).astype(np.int32)).cuda()
    p = sas.Params(batch=B, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, seq_len=Lmax, top_k=K,
                   gate_mode=O.GATE_LOG_SOFTMAX)
    sd = f32_dev(s)
    out = _outputs(p)
    sas.decode_step_fused(p, bf16_dev(q), bf16_dev(kc), bf16_dev(vc), cl, sd, out)
    idx = torch.empty_like(out["idx"])
    lse = torch.empty_like(out["lse_s"])
    sas.sas_topk_select(p, sd, idx, lse, cache_len=cl)
    torch.cuda.synchronize()
    assert sas.sas_get_device_error() == 0
    assert torch.equal(out["idx"], idx)
    assert torch.allclose(out["lse_s"], lse, rtol=0, atol=1e-5)


@pytest.mark.parametrize("gate", [O.GATE_NONE, O.GATE_LOG_SOFTMAX])
@pytest.mark.parametrize("B,Hq,Hkv,d,Lmax,K,lens", [
    (4, 32, 8, 128, 2048, 16, [2048, 1, 1000, 1999]),
    (3, 10, 2, 64, 1024, 4, [64, 65, 1024]),
])
def test_decode_fused_paged_parity(B, Hq, Hkv, d, Lmax, K, lens, gate):
    """Through a block table over shuffled pages; NaN in everything the step must not read."""
    sas = _sas()
    q, kc, vc, s = _case(B, Hq, Hkv, d, Lmax, seed=B * 5 + K)
    g = np.random.default_rng(321 + K)
    kp, vp, table = _paged(kc, vc, lens, g)
    cl = np.array(lens, dtype=np.int32)
    p = sas.Params(batch=B, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, seq_len=Lmax, top_k=K, gate_mode=gate)
    out = _outputs(p)
    sas.sas_decode_fused_paged(p, bf16_dev(q), bf16_dev(kp), bf16_dev(vp), torch.from_numpy(table).cuda(),
                               torch.from_numpy(cl).cuda(), f32_dev(s), out["o"], idx=out["idx"],
                               lse_s=out["lse_s"], lse_o=out["lse_o"])
    torch.cuda.synchronize()
    assert sas.sas_get_device_error() == 0
    ref = O.decode_paged(q, kp, vp, table, cl, s.astype(np.float64), K, gate_mode=gate, n_split=1)
    _check(out, ref, gate)


def test_decode_fused_optional_outputs_and_graph():
    """idx, lse_s and lse_o may be omitted; a captured fused step replays fresh inputs."""
    sas = _sas()
    B, Hq, Hkv, d, Lmax, K = 4, 32, 8, 128, 2048, 8
    q, kc, vc, s = _case(B, Hq, Hkv, d, Lmax, seed=91)
    p = sas.Params(batch=B, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, seq_len=Lmax, top_k=K,
                   gate_mode=O.GATE_LOG_SOFTMAX)
    qd, kd, vd, sd = bf16_dev(q), bf16_dev(kc), bf16_dev(vc), f32_dev(s)
    lens = [2048, 700, 65, 1500]
    cld = torch.tensor(lens, dtype=torch.int32, device="cuda")
    o = torch.empty((B, Hq, d), dtype=torch.bfloat16, device="cuda")
    sas.sas_decode_fused(p, qd, kd, vd, cld, sd, o)
    torch.cuda.synchronize()
    assert sas.sas_get_device_error() == 0
    ref = O.decode(q, kc, vc, np.array(lens, np.int32), s.astype(np.float64), K, gate_mode=O.GATE_LOG_SOFTMAX)
    assert max_abs(host(o), ref["o"]) < TOL_O
    out = _outputs(p)
    graph = sas.DecodeGraph(p, qd, kd, vd, cld, sd, 0, out, fused=True)
    for lens, seed in (([1999, 1, 1024, 640], 5), ([64, 2048, 129, 1000], 6)):
        q2, _, _, s2 = _case(B, Hq, Hkv, d, Lmax, seed=seed)
        qd.copy_(bf16_dev(q2))
        sd.copy_(f32_dev(s2))
        cld.copy_(torch.tensor(lens, dtype=torch.int32))
        graph.replay()
        torch.cuda.synchronize()
        assert sas.sas_get_device_error() == 0
        ref = O.decode(q2, kc, vc, np.array(lens, np.int32), s2.astype(np.float64), K,
                       gate_mode=O.GATE_LOG_SOFTMAX)
        _check(out, ref, O.GATE_LOG_SOFTMAX)


def test_decode_fused_limits_and_bad_length():
    """Shapes past the kernel's shared-memory lists are refused before any launch; a cache length
    outside [1, seq_len] raises the device error word and is clamped."""
    sas = _sas()
    B, Hq, Hkv, d, Lmax = 2, 8, 2, 128, 1024
    q, kc, vc, s = _case(B, Hq, Hkv, d, Lmax, seed=8)
    qd, kd, vd, sd = bf16_dev(q), bf16_dev(kc), bf16_dev(vc), f32_dev(s)
    o = torch.empty((B, Hq, d), dtype=torch.bfloat16, device="cuda")
    cl = torch.tensor([1024, 5000], dtype=torch.int32, device="cuda")
    p = sas.Params(batch=B, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, seq_len=Lmax, top_k=256)
    with pytest.raises(sas.SasError) as e:
        sas.sas_decode_fused(p, qd, kd, vd, cl, sd, o)
    assert e.value.code == 2  # SAS_ERR_UNSUPPORTED
    p = sas.Params(batch=B, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, seq_len=Lmax, top_k=4)
    sas.sas_decode_fused(p, qd, kd, vd, cl, sd, o)
    torch.cuda.synchronize()
    assert sas.sas_get_device_error() == 6  # SAS_ERR_DEVICE_INDEX
    assert np.isfinite(host(o)).all()


def test_decode_fused_paged_bad_page_is_reported():
    """A table entry outside the page pool for a block the step reads raises the device error
    word; the kernel reads page 0 in its place and the output stays finite."""
    sas = _sas()
    B, Hq, Hkv, d, Lmax, K = 2, 8, 2, 128, 1024, 4
    q, kc, vc, s = _case(B, Hq, Hkv, d, Lmax, seed=15)
    g = np.random.default_rng(19)
    lens = [700, 1024]
    kp, vp, table = _paged(kc, vc, lens, g, n_extra=0)
    kp = np.nan_to_num(kp)  # every page is read-safe here; only the table entry is wrong
    vp = np.nan_to_num(vp)
    table[1, (lens[1] - 1) // 64] = kp.shape[0] + 3  # the current block of sequence 1
    p = sas.Params(batch=B, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, seq_len=Lmax, top_k=K,
                   gate_mode=O.GATE_NONE)
    o = torch.empty((B, Hq, d), dtype=torch.bfloat16, device="cuda")
    sas.sas_decode_fused_paged(p, bf16_dev(q), bf16_dev(kp), bf16_dev(vp), torch.from_numpy(table).cuda(),
                               torch.tensor(lens, dtype=torch.int32).cuda(), f32_dev(s), o)
    torch.cuda.synchronize()
    assert sas.sas_get_device_error() == 6  # SAS_ERR_DEVICE_INDEX
    assert sas.sas_get_device_error() == 0  # read and cleared
    assert np.isfinite(host(o)).all()
