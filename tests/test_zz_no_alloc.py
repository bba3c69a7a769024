"""GPU test of sas_decode_noalloc, the decode step that allocates nothing.

Callers that cannot call cudaMalloc use it: a serving loop that may not
synchronise the device per step, a plugin inside a framework whose caching
allocator owns HBM, or a plain C caller without a device allocator. The entry
point keeps its index lists, gate normalisers and split partials in a fixed
16 MiB device array inside the library. This test checks, through the C ABI,
that two calls in a row give the same answers as the regular entry points
(sas_topk_select, sas_decode, sas_decode_combine with caller-owned buffers):
bit for bit, since the same kernels run on the same inputs, and so within the
decode tolerances. It covers d = 128 and d = 64, and a call without lse_o. It also checks that a problem too large for the
fixed scratch is refused before any launch.

The file name sorts last, so a run that stops at the first failure has
already run every other test before this one.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

TOL_O = 2e-2   # decode output, bf16 (same bound as the other decode parity tests)
TOL_L = 1e-2   # output log-sum-exp


def _inputs(B, Hq, Hkv, d, Lmax, seed):
    g = np.random.default_rng(seed)

    def bf(shape):
        return torch.from_numpy(g.standard_normal(shape).astype(np.float32)).to(torch.bfloat16).cuda()

    q, kc, vc = bf((B, Hq, d)), bf((B, Hkv, Lmax, d)), bf((B, Hkv, Lmax, d))
    s = torch.from_numpy((g.standard_normal((B, Hkv, Lmax // 64)) * np.sqrt(2)).astype(np.float32)).cuda()
    return q, kc, vc, s


def _regular(sas, p, q, kc, vc, cl, s):
    out = sas.empty_decode_outputs(p, p.top_k + 1)
    sas.decode_step(p, q, kc, vc, cl, s, p.top_k + 1, out)
    return out["o"], out["lse_o"]


@pytest.mark.parametrize("d", [128, 64])
def test_noalloc_decode_matches_regular_entry_points_twice(d):
    import learned_block_sparse_warp_b200 as sas
    B, Hq, Hkv, Lmax, K = 6, 32, 8, 4096, 16
    calls = [
        (sas.SAS_GATE_NONE, [4096, 1, 1000, 2049, 64, 3333], 11, True),
        (sas.SAS_GATE_LOG_SOFTMAX, [17, 4096, 4095, 128, 129, 700], 12, False),  # lse_o not requested
    ]
    results = []
    for gate, lens, seed, want_lse in calls:
        p = sas.Params(batch=B, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, seq_len=Lmax, top_k=K, gate_mode=gate)
        q, kc, vc, s = _inputs(B, Hq, Hkv, d, Lmax, seed + d)
        cl = torch.tensor(lens, dtype=torch.int32, device="cuda")
        o = torch.empty((B, Hq, d), dtype=torch.bfloat16, device="cuda")
        lse = torch.empty((B, Hq), dtype=torch.float32, device="cuda") if want_lse else None
        sas.sas_decode_noalloc(p, q, kc, vc, cl, s, o, lse)
        o_ref, lse_ref = _regular(sas, p, q, kc, vc, cl, s)
        torch.cuda.synchronize()
        assert sas.sas_get_device_error() == 0
        results.append((o.clone(), None if lse is None else lse.clone(), o_ref, lse_ref))
    for o, lse, o_ref, lse_ref in results:
        assert torch.isfinite(o.float()).all()
        # the same kernels on the same inputs: the scratch layout must not perturb a single value
        assert torch.equal(o, o_ref), (o.float() - o_ref.float()).abs().max().item()
        assert (o.float() - o_ref.float()).abs().max().item() < TOL_O
        if lse is not None:
            assert torch.equal(lse, lse_ref)
            assert (lse - lse_ref).abs().max().item() < TOL_L
    # the two calls really differed, so the second did not just reread the first's scratch
    assert (results[0][0].float() - results[1][0].float()).abs().max().item() > 0.1


def test_noalloc_decode_refuses_sizes_beyond_its_scratch():
    import learned_block_sparse_warp_b200 as sas
    # 64 sequences x 64 query heads x (K + 1 = 65) splits x d 128 fp32 partials = 136 MB > 16 MiB
    p = sas.Params(batch=64, n_q_heads=64, n_kv_heads=8, head_dim=128, seq_len=1024, top_k=64,
                   gate_mode=sas.SAS_GATE_NONE)
    q = torch.zeros((64, 64, 128), dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros((64, 8, 1024, 128), dtype=torch.bfloat16, device="cuda")
    cl = torch.full((64,), 1024, dtype=torch.int32, device="cuda")
    s = torch.zeros((64, 8, 16), dtype=torch.float32, device="cuda")
    o = torch.empty((64, 64, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sas.SasError) as e:
        sas.sas_decode_noalloc(p, q, kc, kc, cl, s, o)
    assert e.value.code == 3  # SAS_ERR_WORKSPACE
