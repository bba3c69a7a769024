"""GPU: training steps end to end from host memory (sas_train_steps_host).

Each step's inputs go up, the step runs, its outputs come down, with the copies
of neighbouring steps overlapping the kernels on two device slots. Every kernel
on the path is deterministic (the backward has no atomics), so each step's host
outputs must equal those of the same step run on device buffers; they are also
compared with the fp64 oracle directly.
"""
import numpy as np
import pytest
import torch

from synth import workloads as W

pytestmark = pytest.mark.gpu

OUTS = ("o", "lse_o", "dq", "dk", "dv", "ds")


def _setup(n_sets, gate):
    import learned_block_sparse_warp_b200 as sas
    p = sas.Params(batch=1, n_q_heads=8, n_kv_heads=2, head_dim=128, seq_len=1024, top_k=4, gate_mode=gate)
    sets = []
    for i in range(n_sets):
        w = W.custom("host_steps", batch=1, n_q_heads=8, n_kv_heads=2, head_dim=128, seq_len=1024, top_k=4,
                     seed=500 + i)
        x = W.prefill_inputs(w, with_do=True)
        h = {k: torch.from_numpy(np.ascontiguousarray(x[k])).to(torch.bfloat16 if k != "s" else torch.float32)
             .pin_memory() for k in ("q", "k", "v", "s", "do")}
        sets.append(h)
    return sas, p, sets


def _device_reference(sas, p, h):
    d = {k: v.cuda() for k, v in h.items()}
    out = sas.empty_prefill_outputs(p)
    sas.prefill_step(p, d["q"], d["k"], d["v"], d["s"], d["do"], out)
    torch.cuda.synchronize()
    return {k: out[k].cpu() for k in OUTS}


def _host_outputs(p, gated):
    B, Hq, Hkv, N, d, NB = p.batch, p.n_q_heads, p.n_kv_heads, p.seq_len, p.head_dim, p.n_blocks
    o = dict(o=torch.empty((B, Hq, N, d), dtype=torch.bfloat16).pin_memory(),
             lse_o=torch.empty((B, Hq, N), dtype=torch.float32).pin_memory(),
             dq=torch.empty((B, Hq, N, d), dtype=torch.bfloat16).pin_memory(),
             dk=torch.empty((B, Hkv, N, d), dtype=torch.bfloat16).pin_memory(),
             dv=torch.empty((B, Hkv, N, d), dtype=torch.bfloat16).pin_memory())
    if gated:
        o["ds"] = torch.empty((B, Hkv, NB, NB), dtype=torch.float32).pin_memory()
    return o


@pytest.mark.parametrize("n_steps", [1, 2, 5])
def test_host_steps_equal_device_steps(n_steps):
    import learned_block_sparse_warp_b200 as sas
    sas, p, sets = _setup(3, sas.SAS_GATE_LOG_SOFTMAX)
    refs = [_device_reference(sas, p, h) for h in sets]
    steps, outs = [], []
    for i in range(n_steps):
        ho = _host_outputs(p, True)
        outs.append(ho)
        steps.append({**sets[i % 3], **ho})
    slots = [sas.empty_device_slot(p), sas.empty_device_slot(p)]
    stream = torch.cuda.Stream()
    sas.sas_train_steps_host(p, steps, slots, stream=stream)
    stream.synchronize()
    assert sas.sas_get_device_error() == 0
    for i in range(n_steps):
        for k in OUTS:
            assert torch.equal(outs[i][k], refs[i % 3][k]), (i, k)


def test_host_steps_without_gate_and_shared_buffers():
    """Under SAS_GATE_NONE ds stays on the device; host buffers may be shared by every step."""
    import learned_block_sparse_warp_b200 as sas
    sas, p, sets = _setup(1, sas.SAS_GATE_NONE)
    ref = _device_reference(sas, p, sets[0])
    ho = _host_outputs(p, False)
    steps = [{**sets[0], **ho} for _ in range(4)]
    sas.sas_train_steps_host(p, steps, [sas.empty_device_slot(p), sas.empty_device_slot(p)])
    torch.cuda.synchronize()
    assert sas.sas_get_device_error() == 0
    for k in ("o", "lse_o", "dq", "dk", "dv"):
        assert torch.equal(ho[k], ref[k]), k


@pytest.mark.parametrize("shape", ["tiny", "gqa4_d128"])
def test_host_steps_match_the_oracle(shape):
    """Each step's host outputs against the fp64 oracle directly, at the parity tolerances: the
    tiny configuration (2 heads, d = 64, N = 1024, K = 4) and a GQA-4 d = 128 shape."""
    import learned_block_sparse_warp_b200 as sas
    import oracle.sas_oracle as O
    from tests.parity_util import TOL_L, TOL_O, TOL_REL, max_abs, rel_fro
    if shape == "tiny":
        w = W.WORKLOADS["tiny"]
    else:
        w = W.custom("host_oracle", batch=1, n_q_heads=8, n_kv_heads=2, head_dim=128, seq_len=1024, top_k=4, seed=77)
    p = sas.Params(batch=w.batch, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, head_dim=w.head_dim,
                   seq_len=w.seq_len, top_k=w.top_k, gate_mode=sas.SAS_GATE_LOG_SOFTMAX)
    x = W.prefill_inputs(w, with_do=True)
    h = {k: torch.from_numpy(np.ascontiguousarray(x[k])).to(torch.bfloat16 if k != "s" else torch.float32)
         .pin_memory() for k in ("q", "k", "v", "s", "do")}
    ho = _host_outputs(p, True)
    sas.sas_train_steps_host(p, [{**h, **ho}], [sas.empty_device_slot(p), sas.empty_device_slot(p)])
    torch.cuda.synchronize()
    assert sas.sas_get_device_error() == 0
    f64 = {k: h[k].float().numpy().astype(np.float64) for k in ("q", "k", "v", "s", "do")}
    idx, _ = O.prefill_select(f64["s"], w.top_k)
    o, L = O.forward(f64["q"], f64["k"], f64["v"], f64["s"], idx)
    dq, dk, dv, ds, _ = O.backward(f64["q"], f64["k"], f64["v"], f64["s"], idx, f64["do"])
    got = {k: ho[k].float().numpy().astype(np.float64) for k in OUTS}
    assert max_abs(got["o"], o) < TOL_O
    assert max_abs(got["lse_o"], L) < TOL_L
    for k, ref in (("dq", dq), ("dk", dk), ("dv", dv), ("ds", ds)):
        assert rel_fro(got[k], ref) < TOL_REL, (k, rel_fro(got[k], ref))
