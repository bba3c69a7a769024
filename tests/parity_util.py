"""Helpers shared by the GPU parity tests: tolerances, comparisons and uploads."""
from __future__ import annotations

import numpy as np
import torch

# Tolerances for bf16 inputs with fp32 accumulation, as stated for this path:
# index sets bit-exact; o max-abs 2e-2; dq/dk/dv/ds relative Frobenius 3e-2.
# The row log-sum-exp L is fp32 over fp32 logits; max-abs 1e-2 leaves room for
# the bf16 rounding of q and k products near large logits. lse_s is a plain
# fp32 log-sum-exp over at most a few thousand N(0, 2) scores: 1e-4 abs.
TOL_O = 2e-2
TOL_REL = 3e-2
TOL_L = 1e-2
TOL_LSE_S = 1e-4


def bf16_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).cuda()


def f32_dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def host(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_fro(got: np.ndarray, ref: np.ndarray) -> float:
    den = float(np.linalg.norm(ref))
    return float(np.linalg.norm(got - ref)) / max(den, 1e-30)


def max_abs(got: np.ndarray, ref: np.ndarray) -> float:
    return float(np.max(np.abs(got - ref))) if got.size else 0.0


def assert_idx_equal(got: np.ndarray, ref: np.ndarray):
    got = np.asarray(got)
    ref = np.asarray(ref)
    bad = np.argwhere(got != ref)
    assert bad.size == 0, f"{len(bad)} index mismatches, first at {bad[0].tolist()}: got {got[tuple(bad[0][:-1])]}, " \
                          f"want {ref[tuple(bad[0][:-1])]}"
