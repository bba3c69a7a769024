"""The work counts behind every TF/s, GB/s and roofline fraction bench.py reports.

fwd_flops follows the selected-tokens rule: per query head and query block t,
4·d·64·(64·n_t + 32) with n_t = min(K, t), the causal current block counted as
half. Here it is checked against a closed form (the sum of min(K, t) in one
expression) and against the per-workload totals the scope table states:
1.081 TFLOP forward for the 32K training workload, 8.725 TFLOP for the 128K
forward, and the sweep's fwd+bwd totals, with bwd = 2.5 fwd. The decode count
is the gathered K and V of the current block and the K selected blocks.
"""
import numpy as np
import pytest

import bench
from synth import workloads as W


def _closed_form(Hq, d, NB, K, B=1):
    # Σ_{t<NB} min(K, t) = K(K−1)/2 + K·(NB − K) when NB ≥ K
    s_min = K * (K - 1) // 2 + K * (NB - K) if NB >= K else NB * (NB - 1) // 2
    return B * Hq * 4.0 * d * 64 * (64 * s_min + 32 * NB)


@pytest.mark.parametrize("name", ["tiny", "qwen3_4b_train_32k", "llama31_8b_fwd_128k"] +
                         [f"qwen3_14b_k{k}_n{n}" for k in (16, 32, 64) for n in (8192, 32768, 65536)])
def test_fwd_flops_closed_form(name):
    w = W.WORKLOADS[name]
    got = bench.fwd_flops(w.n_q_heads, w.head_dim, w.n_blocks, w.top_k, batch=w.batch)
    assert got == pytest.approx(_closed_form(w.n_q_heads, w.head_dim, w.n_blocks, w.top_k, w.batch), rel=1e-12)


def test_fwd_flops_stated_totals():
    w = W.WORKLOADS["qwen3_4b_train_32k"]
    assert bench.fwd_flops(w.n_q_heads, w.head_dim, w.n_blocks, w.top_k) / 1e12 == pytest.approx(1.081, abs=5e-4)
    w = W.WORKLOADS["llama31_8b_fwd_128k"]
    assert bench.fwd_flops(w.n_q_heads, w.head_dim, w.n_blocks, w.top_k) / 1e12 == pytest.approx(8.725, abs=5e-4)
    stated = {16: (0.580, 2.440, 4.921), 32: (1.066, 4.731, 9.616), 64: (1.813, 9.085, 18.78)}
    for k, vals in stated.items():
        for n, v in zip((8192, 32768, 65536), vals):
            w = W.WORKLOADS[f"qwen3_14b_k{k}_n{n}"]
            got = 3.5 * bench.fwd_flops(w.n_q_heads, w.head_dim, w.n_blocks, w.top_k) / 1e12
            assert got == pytest.approx(v, rel=2e-3), (k, n)


def test_fwd_flops_sampled_blocks_add_up():
    w = W.WORKLOADS["qwen3_4b_train_32k"]
    full = bench.fwd_flops(w.n_q_heads, w.head_dim, w.n_blocks, w.top_k)
    halves = [bench.fwd_flops(w.n_q_heads, w.head_dim, w.n_blocks, w.top_k, t_list=ts)
              for ts in (range(0, w.n_blocks, 2), range(1, w.n_blocks, 2))]
    assert sum(halves) == pytest.approx(full, rel=1e-12)


def test_decode_gathered_bytes():
    w = W.WORKLOADS["decode_b16_32k"]
    full = bench.decode_kv_bytes(w, np.full(w.batch, w.seq_len, np.int32))
    assert full == 16 * 8 * (16 * 64 + 64) * 128 * 2 * 2 == 71_303_168
    # a ragged cache: the current block holds L − 64c tokens, and the history gives min(K, c) blocks
    lens = np.array([1, 65, 64 * 10 + 3] + [w.seq_len] * 13, np.int32)
    want = 0
    for L in lens:
        c = (int(L) - 1) // 64
        want += 8 * (min(16, c) * 64 + (int(L) - 64 * c)) * 128 * 2 * 2
    assert bench.decode_kv_bytes(w, lens) == want


def test_bench_sections_name_real_workloads():
    """The sweep and long-context sections look their workloads up by name and shape."""
    for name in bench.SWEEP:
        w = W.WORKLOADS[name]
        assert w.kind == "prefill" and w.seq_len % 64 == 0
    assert W.WORKLOADS["llama31_8b_fwd_128k"].backward is False and W.WORKLOADS["llama31_8b_fwd_128k"].heavy_hitters
    assert all(W.WORKLOADS[n].backward for n in bench.SWEEP[1:])
    for B, L in bench.LONG_DECODE:
        assert B >= 1 and L % 64 == 0 and (L // 64 - 1 + 7) // 8 <= 53248  # fits the scored select's clusters
    assert bench.TRAIN in W.WORKLOADS and bench.DECODE in W.WORKLOADS


def test_sweep_inputs_follow_the_workload_recipe():
    import torch
    w = W.custom("hh", batch=1, n_q_heads=8, n_kv_heads=2, head_dim=128, seq_len=4096, top_k=8, seed=3,
                 backward=False, heavy_hitters=True)
    x = bench.sweep_inputs(w, torch.device("cpu"), torch)
    assert set(x) == {"q", "k", "v", "s"} and x["s"].shape == (1, 2, 64, 64)
    assert x["q"].dtype == torch.bfloat16 and x["s"].dtype == torch.float32
    w2 = W.custom("plain", batch=1, n_q_heads=10, n_kv_heads=2, head_dim=128, seq_len=2048, top_k=8, seed=4)
    x2 = bench.sweep_inputs(w2, torch.device("cpu"), torch)
    assert set(x2) == {"q", "k", "v", "s", "do"}
    assert abs(float(x2["s"].std()) - 2 ** 0.5) < 0.1  # s ~ N(0, 2)
