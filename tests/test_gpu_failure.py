"""Failure detection on the GPU without a fault: a bounded wait that runs out.

sas_selftest_wait_timeout runs the tcgen05 kernels' bounded mbarrier wait on a
barrier that nothing completes. The wait must give up by itself after about a
second and report SAS_ERR_TIMEOUT through the device error word. The context
must then still run the library's kernels correctly.
"""
import time

import numpy as np
import pytest
import torch

import oracle.sas_oracle as O
from tests.parity_util import TOL_O, bf16_dev, f32_dev, host, max_abs
from synth.workloads import bf16_round

pytestmark = pytest.mark.gpu

SAS_ERR_TIMEOUT = 5


def test_bounded_wait_times_out_and_the_context_survives():
    import learned_block_sparse_warp_b200 as sas
    sas.sas_get_device_error()  # start from a clear error word
    t0 = time.perf_counter()
    sas.sas_selftest_wait_timeout()
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    assert sas.sas_get_device_error() == SAS_ERR_TIMEOUT
    assert sas.sas_get_device_error() == 0  # read and cleared
    assert 0.2 < waited < 30.0, waited

    # the same context then runs a decode step that matches the oracle
    g = np.random.default_rng(3)
    B, Hq, Hkv, d, Lmax, K = 2, 8, 2, 128, 512, 3
    q = bf16_round(g.standard_normal((B, Hq, d)).astype(np.float32))
    kc = bf16_round(g.standard_normal((B, Hkv, Lmax, d)).astype(np.float32))
    vc = bf16_round(g.standard_normal((B, Hkv, Lmax, d)).astype(np.float32))
    s = g.standard_normal((B, Hkv, Lmax // 64)).astype(np.float32)
    cl = np.array([512, 200], np.int32)
    p = sas.Params(batch=B, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d, seq_len=Lmax, top_k=K,
                   gate_mode=O.GATE_NONE)
    out = sas.empty_decode_outputs(p, K + 1)
    sas.decode_step(p, bf16_dev(q), bf16_dev(kc), bf16_dev(vc), torch.from_numpy(cl).cuda(), f32_dev(s), K + 1, out)
    torch.cuda.synchronize()
    assert sas.sas_get_device_error() == 0
    ref = O.decode(q, kc, vc, cl, s.astype(np.float64), K, gate_mode=O.GATE_NONE, n_split=K + 1)
    assert max_abs(host(out["o"]), ref["o"]) < TOL_O
