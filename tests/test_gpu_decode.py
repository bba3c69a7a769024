"""GPU parity: split-K decode partials and their LSE merge against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle.sas_oracle as O
from tests.parity_util import TOL_L, TOL_O, assert_idx_equal, bf16_dev, f32_dev, host, max_abs
from synth.workloads import bf16_round

pytestmark = pytest.mark.gpu


def _sas():
    import learned_block_sparse_warp_b200 as sas
    return sas


def _case(B, Hq, Hkv, d, Lmax, seed):
    g = np.random.default_rng(seed)
    q = bf16_round(g.standard_normal((B, Hq, d)).astype(np.float32))
    kc = bf16_round(g.standard_normal((B, Hkv, Lmax, d)).astype(np.float32))
    vc = bf16_round(g.standard_normal((B, Hkv, Lmax, d)).astype(np.float32))
    s = (g.standard_normal((B, Hkv, Lmax // 64)) * np.sqrt(2)).astype(np.float32)
    return q, kc, vc, s


@pytest.mark.parametrize("gate", [O.GATE_NONE, O.GATE_LOG_SOFTMAX])
@pytest.mark.parametrize("B,Hq,Hkv,d,Lmax,K,n_split,lens", [
    (4, 32, 8, 128, 2048, 16, 17, [2048, 1, 1000, 1999]),
    (3, 8, 8, 64, 1024, 4, 2, [64, 65, 1024]),
    (2, 10, 2, 128, 4096, 8, 3, [4096, 4033]),
    (2, 16, 2, 128, 1024, 32, 33, [1024, 130]),   # K above the history: every block, G = 8
    (1, 4, 1, 64, 512, 2, 1, [300]),
])
def test_decode_parity(B, Hq, Hkv, d, Lmax, K, n_split, lens, gate):
    sas = _sas()
    q, kc, vc, s = _case(B, Hq, Hkv, d, Lmax, seed=B * 31 + K)
    cl = np.array(lens, dtype=np.int32)
    p = sas.Params(batch=B, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, seq_len=Lmax, top_k=K, gate_mode=gate)
    out = sas.empty_decode_outputs(p, n_split)
    sas.decode_step(p, bf16_dev(q), bf16_dev(kc), bf16_dev(vc), torch.from_numpy(cl).cuda(), f32_dev(s), n_split, out)
    torch.cuda.synchronize()
    assert sas.sas_get_device_error() == 0
    ref = O.decode(q, kc, vc, cl, s.astype(np.float64), K, gate_mode=gate, n_split=n_split)
    assert_idx_equal(out["idx"].cpu().numpy(), ref["idx"])
    # split partials: same chunking of the block list on both sides
    lp = host(out["lse_part"])
    fin = np.isfinite(ref["lse_part"])
    assert np.array_equal(np.isfinite(lp), fin)
    assert max_abs(lp[fin], ref["lse_part"][fin]) < TOL_L
    assert max_abs(host(out["o_part"]), ref["o_part"]) < TOL_O
    assert max_abs(host(out["o"]), ref["o"]) < TOL_O
    assert max_abs(host(out["lse_o"]), ref["lse"]) < TOL_L


@pytest.mark.parametrize("d,ns", [(128, 5), (128, 17), (64, 40), (128, 70), (128, 1)])
def test_combine_on_oracle_partials(d, ns):
    """The merge kernel alone, fed partials the oracle computed (including empty splits and rows)."""
    sas = _sas()
    B, Hq = 3, 4
    g = np.random.default_rng(9 + ns)
    o_part = g.standard_normal((B, Hq, ns, d))
    lse_part = g.standard_normal((B, Hq, ns)) * 3
    lse_part[0, 1, min(2, ns - 1)] = -np.inf
    lse_part[2, 3, :] = -np.inf
    lse_part[2, 3, ns - 1] = 0.5
    lse_part[1, 2, :] = -np.inf  # a row with no tokens at all: o = 0, lse = -inf
    o_part[lse_part == -np.inf] = 0.0
    p = sas.Params(batch=B, n_q_heads=Hq, n_kv_heads=Hq, head_dim=d, seq_len=1024, top_k=max(8, ns - 1))
    o = torch.empty((B, Hq, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
    sas.sas_decode_combine(p, ns, f32_dev(o_part), f32_dev(lse_part), o, lse)
    torch.cuda.synchronize()
    ref_o, ref_lse = O.decode_combine(o_part, lse_part)
    assert max_abs(host(o), ref_o) < TOL_O
    got = host(lse)
    fin = np.isfinite(ref_lse)
    assert np.array_equal(np.isfinite(got), fin) and np.all(got[~fin] == -np.inf)
    assert max_abs(got[fin], ref_lse[fin]) < 1e-5


def test_decode_graph_replays_fresh_inputs():
    """A captured decode step, replayed after its inputs change in place, matches the oracle."""
    sas = _sas()
    B, Hq, Hkv, d, Lmax, K, n_split = 4, 32, 8, 128, 2048, 8, 9
    q, kc, vc, s = _case(B, Hq, Hkv, d, Lmax, seed=77)
    p = sas.Params(batch=B, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, seq_len=Lmax, top_k=K,
                   gate_mode=O.GATE_NONE)
    out = sas.empty_decode_outputs(p, n_split)
    qd, kd, vd, sd = bf16_dev(q), bf16_dev(kc), bf16_dev(vc), f32_dev(s)
    cld = torch.tensor([2048, 700, 65, 1500], dtype=torch.int32, device="cuda")
    graph = sas.DecodeGraph(p, qd, kd, vd, cld, sd, n_split, out)
    for lens, seed in (([2048, 700, 65, 1500], None), ([1999, 1, 1024, 640], 5)):
        if seed is not None:  # a new step: new query, new scores, new lengths, same buffers
            q2, _, _, s2 = _case(B, Hq, Hkv, d, Lmax, seed=seed)
            qd.copy_(bf16_dev(q2))
            sd.copy_(f32_dev(s2))
            cld.copy_(torch.tensor(lens, dtype=torch.int32))
            q, s = q2, s2
        graph.replay()
        torch.cuda.synchronize()
        assert sas.sas_get_device_error() == 0
        ref = O.decode(q, kc, vc, np.array(lens, np.int32), s.astype(np.float64), K, gate_mode=O.GATE_NONE,
                       n_split=n_split)
        assert_idx_equal(out["idx"].cpu().numpy(), ref["idx"])
        assert max_abs(host(out["o"]), ref["o"]) < TOL_O
        assert max_abs(host(out["lse_o"]), ref["lse"]) < TOL_L


def _paged(kc, vc, lens, g, n_extra=5):
    """Pages [n_pages, Hkv, 64, d] holding each sequence's blocks 0..c at shuffled
    slots, and the block table. Everything the step must not read is NaN (unused
    pages, tokens past the cache length) or garbage (table entries past c)."""
    B, Hkv, Lmax, d = kc.shape
    NB = Lmax // 64
    used = [(b, m) for b in range(B) for m in range((lens[b] - 1) // 64 + 1)]
    n_pages = len(used) + n_extra
    slots = g.permutation(n_pages)[: len(used)]
    kp = np.full((n_pages, Hkv, 64, d), np.nan, np.float32)
    vp = np.full((n_pages, Hkv, 64, d), np.nan, np.float32)
    table = g.integers(-7, 3 * n_pages, size=(B, NB)).astype(np.int32)
    for (b, m), pg in zip(used, slots):
        n = min(64, lens[b] - 64 * m)
        kp[pg, :, :n] = kc[b, :, 64 * m:64 * m + n]
        vp[pg, :, :n] = vc[b, :, 64 * m:64 * m + n]
        table[b, m] = pg
    return kp, vp, table


@pytest.mark.parametrize("gate", [O.GATE_NONE, O.GATE_LOG_SOFTMAX])
@pytest.mark.parametrize("B,Hq,Hkv,d,Lmax,K,n_split,lens", [
    (4, 32, 8, 128, 2048, 16, 17, [2048, 1, 1000, 1999]),
    (3, 10, 2, 64, 1024, 4, 2, [64, 65, 1024]),
])
def test_decode_paged_parity(B, Hq, Hkv, d, Lmax, K, n_split, lens, gate):
    """Decode through a block table over shuffled pages equals the oracle; NaN in
    every page and token the step must not read never reaches the output."""
    sas = _sas()
    q, kc, vc, s = _case(B, Hq, Hkv, d, Lmax, seed=B * 7 + K)
    g = np.random.default_rng(123 + K)
    kp, vp, table = _paged(kc, vc, lens, g)
    cl = np.array(lens, dtype=np.int32)
    p = sas.Params(batch=B, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, seq_len=Lmax, top_k=K, gate_mode=gate)
    out = sas.empty_decode_outputs(p, n_split)
    sas.decode_step_paged(p, bf16_dev(q), bf16_dev(kp), bf16_dev(vp), torch.from_numpy(table).cuda(),
                          torch.from_numpy(cl).cuda(), f32_dev(s), n_split, out)
    torch.cuda.synchronize()
    assert sas.sas_get_device_error() == 0
    ref = O.decode_paged(q, kp, vp, table, cl, s.astype(np.float64), K, gate_mode=gate, n_split=n_split)
    assert_idx_equal(out["idx"].cpu().numpy(), ref["idx"])
    got = host(out["o"])
    assert np.isfinite(got).all()
    assert max_abs(got, ref["o"]) < TOL_O
    assert max_abs(host(out["lse_o"]), ref["lse"]) < TOL_L


def test_decode_paged_bad_page_is_reported():
    """A table entry outside the page pool for a block the step reads raises the
    device error word; the kernel reads page 0 instead and does not fault."""
    sas = _sas()
    B, Hq, Hkv, d, Lmax, K = 2, 8, 2, 128, 1024, 4
    q, kc, vc, s = _case(B, Hq, Hkv, d, Lmax, seed=5)
    g = np.random.default_rng(9)
    lens = [700, 1024]
    kp, vp, table = _paged(kc, vc, lens, g, n_extra=0)
    table[1, (lens[1] - 1) // 64] = kp.shape[0] + 3  # the current block of sequence 1
    p = sas.Params(batch=B, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, seq_len=Lmax, top_k=K,
                   gate_mode=O.GATE_NONE)
    out = sas.empty_decode_outputs(p, 2)
    sas.decode_step_paged(p, bf16_dev(q), bf16_dev(kp), bf16_dev(vp), torch.from_numpy(table).cuda(),
                          torch.tensor(lens, dtype=torch.int32).cuda(), f32_dev(s), 2, out)
    torch.cuda.synchronize()
    assert sas.sas_get_device_error() == 6  # SAS_ERR_DEVICE_INDEX
    assert sas.sas_get_device_error() == 0  # read and cleared


@pytest.mark.parametrize("gate", [O.GATE_LOG_SIGMOID, O.GATE_LOGIT])
def test_decode_gate_ablations(gate):
    """Decode under the gate-activation ablations (lse_s is not needed and not passed)."""
    sas = _sas()
    B, Hq, Hkv, d, Lmax, K, n_split = 3, 16, 4, 128, 2048, 8, 3
    q, kc, vc, s = _case(B, Hq, Hkv, d, Lmax, seed=61)
    lens = [2048, 777, 65]
    cl = np.array(lens, dtype=np.int32)
    p = sas.Params(batch=B, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, seq_len=Lmax, top_k=K, gate_mode=gate)
    out = sas.empty_decode_outputs(p, n_split)
    qd, kd, vd, sd, cld = bf16_dev(q), bf16_dev(kc), bf16_dev(vc), f32_dev(s), torch.from_numpy(cl).cuda()
    sas.sas_topk_select(p, sd, out["idx"], None, cache_len=cld)
    sas.sas_decode(p, qd, kd, vd, cld, sd, out["idx"], None, n_split, out["o_part"], out["lse_part"])
    sas.sas_decode_combine(p, n_split, out["o_part"], out["lse_part"], out["o"], out["lse_o"])
    torch.cuda.synchronize()
    assert sas.sas_get_device_error() == 0
    ref = O.decode(q, kc, vc, cl, s.astype(np.float64), K, gate_mode=gate, n_split=n_split)
    assert_idx_equal(out["idx"].cpu().numpy(), ref["idx"])
    assert max_abs(host(out["o"]), ref["o"]) < TOL_O
    assert max_abs(host(out["lse_o"]), ref["lse"]) < TOL_L
