"""Pins for the fp64 oracle: checks against facts the pages and mathematics fix.

None of these checks runs the oracle against a copy of itself. They use:
* hand-derived values (tests/golden),
* a rank-count definition of Top-K (no sorting),
* torch's scaled_dot_product_attention in fp64 (the dense special cases),
* central finite differences (every gradient, including ds),
* the pages' own gate-gradient formula evaluated token by token,
* the invariances the pages state (shift of s, permutation inside a block),
* for the block-mean selector scores: running token sums, and the mean of the
  token-level logits over a block and a head group.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle.sas_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng0 = np.random.default_rng(1234)


def _rand_case(B=1, Hq=2, Hkv=1, N=32, d=8, block=4, seed=0, s_spread=False):
    g = np.random.default_rng(seed)
    q = g.standard_normal((B, Hq, N, d))
    k = g.standard_normal((B, Hkv, N, d))
    v = g.standard_normal((B, Hkv, N, d))
    do = g.standard_normal((B, Hq, N, d))
    nb = N // block
    if s_spread:
        # distinct, well-separated scores so that a small perturbation cannot flip the selection
        s = np.stack([np.stack([g.permutation(nb * nb).reshape(nb, nb) * 0.37 for _ in range(Hkv)])
                      for _ in range(B)]).astype(np.float64)
        s = s - s.mean()
        s *= 0.2
    else:
        s = g.standard_normal((B, Hkv, nb, nb)) * math.sqrt(2.0)
    return q, k, v, do, s


# ---------------------------------------------------------------------------
# Top-K
# ---------------------------------------------------------------------------
def _topk_by_rank(s, K):
    """Block m is in the set iff fewer than K blocks beat it; beat = higher score,
    or equal score and lower index. O(t^2) counting, no sort."""
    t = len(s)
    out = []
    for m in range(t):
        beaten_by = 0
        for m2 in range(t):
            if s[m2] > s[m] or (s[m2] == s[m] and m2 < m):
                beaten_by += 1
        if beaten_by < K:
            out.append(m)
    return out


def test_topk_golden_ties():
    with open(os.path.join(GOLDEN, "topk_ties.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        assert O.topk_blocks(np.array(c["s"], dtype=np.float64), c["K"]) == c["expected"], c


@pytest.mark.parametrize("quant", [None, 0.5, 2.0])
def test_topk_vs_rank_count(quant):
    g = np.random.default_rng(7)
    for _ in range(300):
        t = int(g.integers(0, 40))
        K = int(g.integers(1, 12))
        s = g.standard_normal(t) * 2.0
        if quant is not None:
            s = np.round(s / quant) * quant  # force ties
        assert O.topk_blocks(s, K) == _topk_by_rank(list(s), K)


def test_topk_nan_ranks_last():
    s = np.array([np.nan, 1.0, np.nan, -5.0])
    assert O.topk_blocks(s, 2) == [1, 3]
    assert O.topk_blocks(s, 3) == [0, 1, 3]


def test_prefill_select_shapes_and_padding():
    s = rng0.standard_normal((1, 2, 6, 6))
    idx, lse = O.prefill_select(s, 3)
    assert idx.shape == (1, 2, 6, 3)
    assert (idx[:, :, 0] == -1).all()
    assert list(idx[0, 0, 1]) == [0, -1, -1]
    assert list(idx[0, 0, 2][:2]) == [0, 1] and idx[0, 0, 2, 2] == -1
    assert lse[0, 0, 0] == -math.inf
    for t in range(1, 6):
        row = idx[0, 1, t]
        sel = [m for m in row if m >= 0]
        assert len(sel) == min(3, t) and sel == sorted(sel) and all(m < t for m in sel)


# ---------------------------------------------------------------------------
# LSE and the gate
# ---------------------------------------------------------------------------
def test_lse_closed_forms():
    assert O.logsumexp(np.array([0.0, math.log(2), math.log(3)])) == pytest.approx(math.log(6), abs=1e-15)
    for c in (-40.0, 0.0, 3.5, 1000.0):
        for t in (1, 2, 7, 511):
            assert O.logsumexp(np.full(t, c)) == pytest.approx(c + math.log(t), rel=0, abs=1e-12 * max(1, abs(c)))
    assert O.logsumexp(np.array([])) == -math.inf


def test_lse_vs_fsum():
    g = np.random.default_rng(3)
    for _ in range(100):
        x = g.standard_normal(int(g.integers(1, 50))) * 3
        ref = math.log(math.fsum(math.exp(v) for v in x))
        assert O.logsumexp(x) == pytest.approx(ref, abs=1e-13)


def test_gate_is_softmax_of_scores():
    s = np.array([0.0, math.log(2), math.log(3)])
    lg = O.log_gate(s, [0, 1, 2], O.GATE_LOG_SOFTMAX)
    assert np.allclose(np.exp(lg), [1 / 6, 2 / 6, 3 / 6], atol=1e-15)
    assert np.allclose(O.log_gate(s, [0, 2], O.GATE_NONE), 0.0)


# ---------------------------------------------------------------------------
# Hand example (tests/golden/hand_example.json)
# ---------------------------------------------------------------------------
def test_hand_example():
    with open(os.path.join(GOLDEN, "hand_example.json")) as f:
        ex = json.load(f)
    I, E = ex["inputs"], ex["expected"]
    q = np.array(I["q"]).reshape(1, 1, 3, 1)
    k = np.array(I["k"]).reshape(1, 1, 3, 1)
    v = np.array(I["v"]).reshape(1, 1, 3, 1)
    do = np.array(I["dO"]).reshape(1, 1, 3, 1)
    s = np.array(I["s"]).reshape(1, 1, 3, 3)
    idx, lse_s = O.prefill_select(s, I["top_k"])
    assert idx[0, 0].tolist() == E["idx"]
    assert lse_s[0, 0, 0] == -math.inf
    assert lse_s[0, 0, 1:].tolist() == pytest.approx(E["lse_s"][1:], abs=1e-15)
    o, L = O.forward(q, k, v, s, idx, block=1, softmax_scale=1.0)
    assert o[0, 0, :, 0].tolist() == pytest.approx(E["o_gated"], abs=1e-14)
    assert L[0, 0, 2] == pytest.approx(E["L_gated_row2"], abs=1e-14)
    ou, _ = O.forward(q, k, v, s, idx, block=1, softmax_scale=1.0, gate_mode=O.GATE_NONE)
    assert ou[0, 0, :, 0].tolist() == pytest.approx(E["o_ungated"], abs=1e-14)
    dq, dk, dv, ds, dl = O.backward(q, k, v, s, idx, do, block=1, softmax_scale=1.0)
    assert dl[0, 0, 2, 0] == pytest.approx(E["dl_t2"], abs=1e-14)
    assert ds[0, 0, 2, :2].tolist() == pytest.approx(E["ds_t2"], abs=1e-14)
    assert np.all(ds[0, 0, 1] == 0) and np.all(ds[0, 0, 0] == 0)


# ---------------------------------------------------------------------------
# Dense special cases against torch SDPA (fp64, CPU)
# ---------------------------------------------------------------------------
def _sdpa(q, k, v, G, bias=None, causal=True):
    tq = torch.from_numpy(q)
    tk = torch.from_numpy(k).repeat_interleave(G, dim=1)
    tv = torch.from_numpy(v).repeat_interleave(G, dim=1)
    if bias is None:
        return torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal).numpy()
    return torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=torch.from_numpy(bias)).numpy()


@pytest.mark.parametrize("G", [1, 3])
def test_dense_equality_ungated(G):
    q, k, v, _, s = _rand_case(B=2, Hq=2 * G, Hkv=2, N=48, d=8, block=8, seed=11)
    nb = 48 // 8
    idx, _ = O.prefill_select(s, nb)  # K >= every history
    o, _ = O.forward(q, k, v, s, idx, block=8, gate_mode=O.GATE_NONE)
    ref = _sdpa(q, k, v, G)
    assert np.abs(o - ref).max() < 1e-12


def test_dense_gated_constant_scores_is_biased_attention():
    """Constant s with K = all history gives g_m = 1/t. Every history key of
    query block t then carries a logit shift of -log t; the current block does not."""
    B, Hq, Hkv, N, d, blk = 1, 2, 1, 40, 8, 8
    q, k, v, _, _ = _rand_case(B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, block=blk, seed=5)
    nb = N // blk
    s = np.full((B, Hkv, nb, nb), 0.7)
    idx, _ = O.prefill_select(s, nb)
    o, _ = O.forward(q, k, v, s, idx, block=blk)
    bias = np.full((N, N), -np.inf)
    for i in range(N):
        t = i // blk
        for j in range(i + 1):
            bias[i, j] = 0.0 if j // blk == t else -math.log(t)
    ref = _sdpa(q, k, v, Hq // Hkv, bias=bias[None, None].repeat(Hq, axis=1))
    assert np.abs(o - ref).max() < 1e-12


def test_forward_lse_matches_dense():
    q, k, v, _, s = _rand_case(B=1, Hq=2, Hkv=1, N=32, d=8, block=8, seed=2)
    idx, _ = O.prefill_select(s, 4)
    _, L = O.forward(q, k, v, s, idx, block=8, gate_mode=O.GATE_NONE)
    z = np.einsum("hid,jd->hij", q[0], k[0, 0]) / math.sqrt(8)
    z = np.where(np.tril(np.ones((32, 32), bool))[None], z, -np.inf)
    ref = np.log(np.exp(z).sum(-1))
    assert np.abs(L[0] - ref).max() < 1e-12


# ---------------------------------------------------------------------------
# Invariances the pages state
# ---------------------------------------------------------------------------
def test_shift_invariance_of_scores():
    """g = softmax(s) does not change when a constant is added to s
    ([SAS-summary] §무엇과 다른가); neither does anything downstream."""
    q, k, v, do, s = _rand_case(B=1, Hq=2, Hkv=1, N=48, d=8, block=8, seed=9)
    idx, _ = O.prefill_select(s, 2)
    shift = np.random.default_rng(1).standard_normal((1, 1, 6, 1)) * 5
    s2 = s + shift
    idx2, _ = O.prefill_select(s2, 2)
    assert (idx == idx2).all()
    o1, L1 = O.forward(q, k, v, s, idx, block=8)
    o2, L2 = O.forward(q, k, v, s2, idx2, block=8)
    assert np.abs(o1 - o2).max() < 1e-12 and np.abs(L1 - L2).max() < 1e-12
    g1 = O.backward(q, k, v, s, idx, do, block=8)
    g2 = O.backward(q, k, v, s2, idx2, do, block=8)
    for a, b in zip(g1, g2):
        assert np.abs(a - b).max() < 1e-11


def test_kv_permutation_inside_history_block():
    """Keys and values permuted together inside a block leave every query that
    sees the block as history unchanged (the gate is per block). dk and dv
    permute with them."""
    blk, N = 8, 48
    q, k, v, do, s = _rand_case(B=1, Hq=2, Hkv=1, N=N, d=8, block=blk, seed=21)
    idx, _ = O.prefill_select(s, 3)
    m = 2
    perm = np.arange(N)
    perm[m * blk:(m + 1) * blk] = m * blk + np.random.default_rng(0).permutation(blk)
    kp, vp = k[:, :, perm], v[:, :, perm]
    ts = [t for t in range(N // blk) if t != m]  # block m's own rows see it causally
    o1, _ = O.forward(q, k, v, s, idx, block=blk, t_list=ts)
    o2, _ = O.forward(q, kp, vp, s, idx, block=blk, t_list=ts)
    rows = np.concatenate([np.arange(t * blk, t * blk + blk) for t in ts])
    assert np.abs(o1[:, :, rows] - o2[:, :, rows]).max() < 1e-12
    _, dk1, dv1, ds1, _ = O.backward(q, k, v, s, idx, do, block=blk, t_list=ts)
    _, dk2, dv2, ds2, _ = O.backward(q, kp, vp, s, idx, do, block=blk, t_list=ts)
    assert np.abs(dk1[:, :, perm] - dk2).max() < 1e-12
    assert np.abs(dv1[:, :, perm] - dv2).max() < 1e-12
    assert np.abs(ds1 - ds2).max() < 1e-12


def test_query_head_permutation_in_group():
    q, k, v, do, s = _rand_case(B=1, Hq=3, Hkv=1, N=32, d=8, block=8, seed=4)
    idx, _ = O.prefill_select(s, 2)
    p = [2, 0, 1]
    o1, _ = O.forward(q, k, v, s, idx, block=8)
    o2, _ = O.forward(q[:, p], k, v, s, idx, block=8)
    assert np.abs(o1[:, p] - o2).max() < 1e-12
    dq1, dk1, dv1, ds1, _ = O.backward(q, k, v, s, idx, do, block=8)
    dq2, dk2, dv2, ds2, _ = O.backward(q[:, p], k, v, s, idx, do[:, p], block=8)
    assert np.abs(dq1[:, p] - dq2).max() < 1e-12
    for a, b in ((dk1, dk2), (dv1, dv2), (ds1, ds2)):
        assert np.abs(a - b).max() < 1e-12


def test_gate_reweights_probabilities():
    """exp(z + log g) = g·exp(z) ([SAS-explainer] §仕組み): gated output equals
    the ungated logits' exponentials weighted by g per history block, renormalised."""
    blk, N, d = 4, 16, 8
    q, k, v, _, s = _rand_case(B=1, Hq=1, Hkv=1, N=N, d=d, block=blk, seed=13)
    idx, lse = O.prefill_select(s, 2)
    o, _ = O.forward(q, k, v, s, idx, block=blk)
    t = 3
    sel = [int(m) for m in idx[0, 0, t] if m >= 0]
    g = {m: math.exp(s[0, 0, t, m] - lse[0, 0, t]) for m in sel}
    for r in range(blk):
        i = t * blk + r
        num = np.zeros(d)
        den = 0.0
        for j in range(t * blk, i + 1):
            w = math.exp(q[0, 0, i] @ k[0, 0, j] / math.sqrt(d))
            num += w * v[0, 0, j]
            den += w
        for m in sel:
            for j in range(m * blk, m * blk + blk):
                w = g[m] * math.exp(q[0, 0, i] @ k[0, 0, j] / math.sqrt(d))
                num += w * v[0, 0, j]
                den += w
        assert np.abs(o[0, 0, i] - num / den).max() < 1e-12


# ---------------------------------------------------------------------------
# Gradients: central finite differences and the pages' gate-gradient formula
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("gate_mode", [O.GATE_LOG_SOFTMAX, O.GATE_NONE, O.GATE_LOG_SIGMOID, O.GATE_LOGIT,
                                       O.GATE_SOFTMAX_OUTSIDE])
def test_gradients_finite_differences(gate_mode):
    blk, N, d, K = 4, 16, 4, 2
    q, k, v, do, s = _rand_case(B=1, Hq=2, Hkv=1, N=N, d=d, block=blk, seed=31, s_spread=True)
    idx, _ = O.prefill_select(s, K)

    def f(q_, k_, v_, s_):
        # the selection is held fixed (sparse scope); s only enters through the gate
        o, _ = O.forward(q_, k_, v_, s_, idx, block=blk, gate_mode=gate_mode)
        return float(np.sum(o * do))

    dq, dk, dv, ds, _ = O.backward(q, k, v, s, idx, do, block=blk, gate_mode=gate_mode)
    eps = 1e-6
    for name, x, gx in (("q", q, dq), ("k", k, dk), ("v", v, dv), ("s", s, ds)):
        fd = np.zeros_like(x)
        for ix in np.ndindex(*x.shape):
            if name == "s" and ix[-1] >= ix[-2]:
                continue  # m >= t: not a history score
            xp = x.copy()
            xm = x.copy()
            xp[ix] += eps
            xm[ix] -= eps
            args_p = {"q": q, "k": k, "v": v, "s": s}
            args_m = dict(args_p)
            args_p[name] = xp
            args_m[name] = xm
            fd[ix] = (f(**{a + "_": b for a, b in args_p.items()}) - f(**{a + "_": b for a, b in args_m.items()})) / (2 * eps)
        err = np.abs(fd - gx).max()
        assert err < 1e-7 * max(1.0, np.abs(gx).max()), (name, err)
    if gate_mode == O.GATE_NONE:
        assert np.all(ds == 0)
    else:
        assert np.abs(ds).max() > 1e-3  # the gate really carries gradient


def test_dl_matches_pages_gate_gradient():
    blk, N, d, K = 4, 24, 4, 3
    q, k, v, do, s = _rand_case(B=1, Hq=2, Hkv=1, N=N, d=d, block=blk, seed=17)
    idx, _ = O.prefill_select(s, K)
    _, _, _, _, dl = O.backward(q, k, v, s, idx, do, block=blk)
    for t in range(1, N // blk):
        ref = O.gate_gradient_from_pages(q, k, v, s, idx, do, 0, 0, t, block=blk)
        n = len(ref)
        assert np.abs(dl[0, 0, t, :n] - ref).max() < 1e-12, t


def test_ds_rows_sum_to_zero():
    """Σ_m ds_m = Σ dl − Σ softmax(s)_m Σ dl = 0 for every query block (shift invariance, differentiated)."""
    q, k, v, do, s = _rand_case(B=1, Hq=2, Hkv=2, N=64, d=8, block=8, seed=8)
    idx, _ = O.prefill_select(s, 3)
    _, _, _, ds, _ = O.backward(q, k, v, s, idx, do, block=8)
    assert np.abs(ds.sum(-1)).max() < 1e-12
    nb = 8
    assert np.all(ds[..., np.triu_indices(nb)[0], np.triu_indices(nb)[1]] == 0)


# ---------------------------------------------------------------------------
# Decode
# ---------------------------------------------------------------------------
def _decode_case(B=3, Hq=4, Hkv=2, Lmax=64, d=8, seed=0):
    g = np.random.default_rng(seed)
    q = g.standard_normal((B, Hq, d))
    kc = g.standard_normal((B, Hkv, Lmax, d))
    vc = g.standard_normal((B, Hkv, Lmax, d))
    return q, kc, vc, g


@pytest.mark.parametrize("gate_mode", [O.GATE_NONE, O.GATE_LOG_SOFTMAX, O.GATE_SOFTMAX_OUTSIDE])
def test_decode_equals_last_prefill_row(gate_mode):
    """With L a multiple of the block, the decode query at position L−1 is the
    last row of the prefill forward with the same scores for its block."""
    blk, N, d, K = 8, 48, 8, 2
    q, k, v, _, s = _rand_case(B=1, Hq=4, Hkv=2, N=N, d=d, block=blk, seed=41)
    idx, _ = O.prefill_select(s, K)
    o, L = O.forward(q, k, v, s, idx, block=blk, gate_mode=gate_mode)
    t = N // blk - 1
    dec = O.decode(q[:, :, -1], k, v, np.array([N], np.int32), s[:, :, t], K, block=blk, gate_mode=gate_mode)
    assert np.abs(dec["o"] - o[:, :, -1]).max() < 1e-12
    assert np.abs(dec["lse"] - L[:, :, -1]).max() < 1e-12


def test_decode_dense_ungated_ragged():
    """K covering the whole history and no gate: plain attention of the last
    token over its L−1 predecessors and itself, for L not a multiple of the block."""
    blk, Lmax, d = 8, 64, 8
    q, kc, vc, g = _decode_case(B=4, Hq=4, Hkv=2, Lmax=Lmax, d=d, seed=3)
    cl = np.array([1, 9, 37, 64], np.int32)
    s = g.standard_normal((4, 2, Lmax // blk))
    dec = O.decode(q, kc, vc, cl, s, K=8, block=blk)
    for b in range(4):
        L = cl[b]
        for hq in range(4):
            h = hq // 2
            ref = torch.nn.functional.scaled_dot_product_attention(
                torch.from_numpy(q[b, hq][None, None, None]), torch.from_numpy(kc[b, h, :L][None, None]),
                torch.from_numpy(vc[b, h, :L][None, None])).numpy()[0, 0, 0]
            assert np.abs(dec["o"][b, hq] - ref).max() < 1e-12


@pytest.mark.parametrize("gate_mode", [O.GATE_NONE, O.GATE_LOG_SOFTMAX, O.GATE_SOFTMAX_OUTSIDE])
def test_decode_split_invariance(gate_mode):
    """Merging split partials by their LSE gives the unsplit answer for any split count."""
    blk, Lmax, d = 8, 80, 8
    q, kc, vc, g = _decode_case(B=2, Hq=2, Hkv=1, Lmax=Lmax, d=d, seed=5)
    cl = np.array([80, 43], np.int32)
    s = g.standard_normal((2, 1, Lmax // blk))
    ref = O.decode(q, kc, vc, cl, s, K=3, block=blk, gate_mode=gate_mode, n_split=1)
    for ns in (2, 3, 4, 7):
        out = O.decode(q, kc, vc, cl, s, K=3, block=blk, gate_mode=gate_mode, n_split=ns)
        assert np.abs(out["o"] - ref["o"]).max() < 1e-12
        assert np.abs(out["lse"] - ref["lse"]).max() < 1e-12
        assert (out["idx"] == ref["idx"]).all()


def test_split_ranges_cover():
    for n in range(0, 20):
        for ns in range(1, 9):
            r = O.split_ranges(n, ns)
            assert len(r) == ns
            cov = [i for a, e in r for i in range(a, e)]
            assert cov == list(range(n))


def test_combine_ignores_empty_splits():
    o_part = np.array([[[1.0, 2.0], [0.0, 0.0], [3.0, -1.0]]])
    lse_part = np.array([[0.5, -np.inf, 0.5]])
    o, lse = O.decode_combine(o_part, lse_part)
    assert np.allclose(o, [[2.0, 0.5]]) and lse[0] == pytest.approx(0.5 + math.log(2))


def _page_dense_cache(kc, vc, cl, blk, g, n_extra=3):
    """Pages [n_pages, Hkv, blk, d] holding each sequence's blocks 0..c at shuffled
    positions, and the block table. Unused pages, table entries past c and tokens
    past each cache length are NaN or garbage: the step must never read them."""
    B, Hkv, Lmax, d = kc.shape
    NB = Lmax // blk
    used = [(b, m) for b in range(B) for m in range((int(cl[b]) - 1) // blk + 1)]
    n_pages = len(used) + n_extra
    slots = g.permutation(n_pages)[: len(used)]
    kp = np.full((n_pages, Hkv, blk, d), np.nan)
    vp = np.full((n_pages, Hkv, blk, d), np.nan)
    table = g.integers(-5, 10 * n_pages, size=(B, NB)).astype(np.int32)  # garbage outside 0..c
    for (b, m), pg in zip(used, slots):
        n = min(blk, int(cl[b]) - m * blk)
        kp[pg, :, :n] = kc[b, :, m * blk:m * blk + n]
        vp[pg, :, :n] = vc[b, :, m * blk:m * blk + n]
        table[b, m] = pg
    return kp, vp, table


def test_paged_decode_is_attention_over_the_gathered_pages():
    """Dense ungated K: plain attention of the last token over the tokens the pages
    hold for its sequence, however the pages are laid out; NaN elsewhere is never read."""
    blk, Lmax, d = 8, 64, 8
    q, kc, vc, g = _decode_case(B=3, Hq=4, Hkv=2, Lmax=Lmax, d=d, seed=13)
    cl = np.array([1, 30, 64], np.int32)
    s = g.standard_normal((3, 2, Lmax // blk))
    kp, vp, table = _page_dense_cache(kc, vc, cl, blk, g)
    dec = O.decode_paged(q, kp, vp, table, cl, s, K=8, block=blk)
    assert np.isfinite(dec["o"]).all()
    for b in range(3):
        L = cl[b]
        for hq in range(4):
            h = hq // 2
            ref = torch.nn.functional.scaled_dot_product_attention(
                torch.from_numpy(q[b, hq][None, None, None]), torch.from_numpy(kc[b, h, :L][None, None]),
                torch.from_numpy(vc[b, h, :L][None, None])).numpy()[0, 0, 0]
            assert np.abs(dec["o"][b, hq] - ref).max() < 1e-12


@pytest.mark.parametrize("gate_mode", [O.GATE_NONE, O.GATE_LOG_SOFTMAX, O.GATE_SOFTMAX_OUTSIDE])
def test_paged_decode_equals_dense_decode(gate_mode):
    """Selection and gates too: the paged step gives the dense step's answer."""
    blk, Lmax, d = 8, 96, 8
    q, kc, vc, g = _decode_case(B=2, Hq=4, Hkv=2, Lmax=Lmax, d=d, seed=17)
    cl = np.array([96, 53], np.int32)
    s = g.standard_normal((2, 2, Lmax // blk))
    kp, vp, table = _page_dense_cache(kc, vc, cl, blk, g)
    ref = O.decode(q, kc, vc, cl, s, K=3, block=blk, gate_mode=gate_mode, n_split=2)
    out = O.decode_paged(q, kp, vp, table, cl, s, K=3, block=blk, gate_mode=gate_mode, n_split=2)
    assert (out["idx"] == ref["idx"]).all()
    assert np.abs(out["o"] - ref["o"]).max() < 1e-12
    assert np.abs(out["lse"] - ref["lse"]).max() < 1e-12



def test_gate_ablations_have_their_closed_forms():
    """log σ and the raw logit, as the gate-activation ablations define them, for
    scores far into both tails; the selected set does not matter for either."""
    s_hist = np.array([-40.0, -3.0, 0.0, 2.5, 40.0])
    sel = [0, 1, 2, 3, 4]
    ls = O.log_gate(s_hist, sel, O.GATE_LOG_SIGMOID)
    ref = -np.logaddexp(0.0, -s_hist)  # log σ(x) = −log(1 + e^(−x))
    assert np.abs(ls - ref).max() < 1e-14
    assert O.log_gate(s_hist, sel, O.GATE_LOGIT).tolist() == s_hist.tolist()
    # the softmax-normalised gate is invariant to a global shift of the scores; the ablations are not
    for mode, inv in ((O.GATE_LOG_SOFTMAX, True), (O.GATE_LOG_SIGMOID, False), (O.GATE_LOGIT, False)):
        a = O.log_gate(s_hist[1:4], [0, 2], mode)
        b = O.log_gate(s_hist[1:4] + 1.5, [0, 2], mode)
        assert (np.abs(a - b).max() < 1e-12) == inv


# ---------------------------------------------------------------------------
# Selector scoring from block-mean keys (decode)
# ---------------------------------------------------------------------------
def test_block_mean_keys_by_prefix_sums():
    """Each block mean is a difference of running token sums over 64."""
    g = np.random.default_rng(31)
    k = g.standard_normal((2, 3, 64 * 5 + 17, 8))
    km = O.block_mean_keys(k)
    assert km.shape == (2, 3, 5, 8)
    csum = np.concatenate([np.zeros((2, 3, 1, 8)), np.cumsum(k, axis=2)], axis=2)
    for m in range(5):
        np.testing.assert_allclose(km[:, :, m] * 64, csum[:, :, 64 * (m + 1)] - csum[:, :, 64 * m], rtol=0, atol=1e-11)


def test_block_mean_of_a_constant_block_is_that_key():
    g = np.random.default_rng(32)
    u = np.round(g.standard_normal((4, 16)) * 64) / 64  # short mantissas: every partial sum is exact
    k = np.repeat(u, 64, axis=0)[None, None]  # block m holds 64 copies of u[m]
    assert np.array_equal(O.block_mean_keys(k)[0, 0], u)


@pytest.mark.parametrize("G", [1, 4])
def test_decode_scores_are_mean_token_logits(G):
    """s_m equals the mean over the block's tokens and the group's heads of scale·q_g·k_j."""
    g = np.random.default_rng(33 + G)
    B, Hkv, d, L = 2, 2, 16, 64 * 6
    q = g.standard_normal((B, Hkv * G, d))
    k = g.standard_normal((B, Hkv, L, d))
    cache_len = np.array([L, 64 * 3 + 5])
    s = O.decode_scores(q, O.block_mean_keys(k), cache_len)
    scale = 1 / math.sqrt(d)
    for b in range(B):
        c = (int(cache_len[b]) - 1) // 64
        for h in range(Hkv):
            logits = scale * (q[b, h * G:(h + 1) * G] @ k[b, h].T)  # [G, L]
            want = logits[:, :64 * c].reshape(G, c, 64).mean(axis=(0, 2))
            np.testing.assert_allclose(s[b, h, :c], want, rtol=1e-12, atol=1e-12)
            assert np.isnan(s[b, h, c:]).all()


def test_scored_selection_ranks_aligned_blocks_first():
    """A block whose keys all point along the query ranks first; one pointing against it, last."""
    g = np.random.default_rng(35)
    d, G, L = 32, 4, 64 * 40 + 1
    u = g.standard_normal(d)
    u /= np.linalg.norm(u)
    q = g.standard_normal((1, G, d)) + 4 * u
    k = g.standard_normal((1, 1, L, d))
    k[0, 0, 64 * 7:64 * 8] += 4 * u
    k[0, 0, 64 * 22:64 * 23] -= 4 * u
    s, idx, lse = O.decode_select_scored(q, O.block_mean_keys(k), np.array([L]), K=39)
    row = s[0, 0, :40]
    assert int(np.argmax(row)) == 7 and int(np.argmin(row)) == 22
    # K = 39 of 40 history blocks: every block but the anti-aligned one, ascending
    assert idx[0, 0].tolist() == [m for m in range(40) if m != 22]
    assert lse[0, 0] == pytest.approx(math.log(np.exp(row).sum()), rel=1e-12)


def test_scored_selection_without_history():
    q = np.ones((2, 4, 8))
    k = np.ones((2, 2, 128, 8))
    s, idx, lse = O.decode_select_scored(q, O.block_mean_keys(k), np.array([1, 64]), K=3)
    assert (idx == -1).all() and np.isneginf(lse).all() and np.isnan(s).all()


# ---------------------------------------------------------------------------
# The gate outside the softmax
# ---------------------------------------------------------------------------
def test_outside_gate_is_reweighted_dense_attention():
    """Constant s and K covering the history give g_m = 1/t on every history block.
    The output is then the current block's share of dense attention plus 1/t times
    the history's share. The shares come from torch SDPA over each part and the
    log-sum-exp of each part's logits."""
    blk, N, d = 4, 32, 8
    g = np.random.default_rng(77)
    q = g.standard_normal((1, 2, N, d))
    k = g.standard_normal((1, 1, N, d))
    v = g.standard_normal((1, 1, N, d))
    nb = N // blk
    s = np.zeros((1, 1, nb, nb))
    idx, _ = O.prefill_select(s, nb)
    o, _ = O.forward(q, k, v, s, idx, block=blk, gate_mode=O.GATE_SOFTMAX_OUTSIDE)
    tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
    scale = 1 / math.sqrt(d)
    for t in range(1, nb):
        cur = slice(blk * t, blk * t + blk)
        qb = tq[0, :, cur]  # [2, blk, d]
        kc_, vc_ = tk[0, 0, cur], tv[0, 0, cur]
        kh, vh = tk[0, 0, :blk * t], tv[0, 0, :blk * t]
        causal = torch.ones(blk, blk, dtype=torch.bool).tril()
        o_cur = torch.nn.functional.scaled_dot_product_attention(qb, kc_[None], vc_[None], attn_mask=causal)
        o_hist = torch.nn.functional.scaled_dot_product_attention(qb, kh[None], vh[None])
        z_cur = (qb @ kc_.T * scale).masked_fill(~causal, -math.inf)
        z_hist = qb @ kh.T * scale
        lse_cur = torch.logsumexp(z_cur, -1, keepdim=True)
        lse_all = torch.logsumexp(torch.cat([z_cur, z_hist], -1), -1, keepdim=True)
        w_cur = torch.exp(lse_cur - lse_all)
        ref = w_cur * o_cur + (1 - w_cur) * o_hist / t
        assert np.abs(o[0, :, cur] - ref.numpy()).max() < 1e-12, t


def test_outside_gate_with_one_history_block_is_plain_attention():
    """With one history block, g = softmax of one score = 1, inside or outside."""
    q, k, v, do, s = _rand_case(B=1, Hq=2, Hkv=1, N=16, d=4, block=4, seed=78)
    idx, _ = O.prefill_select(s, 2)
    o4, L4 = O.forward(q, k, v, s, idx, block=4, gate_mode=O.GATE_SOFTMAX_OUTSIDE)
    o1, L1 = O.forward(q, k, v, s, idx, block=4, gate_mode=O.GATE_NONE)
    assert np.abs(o4[:, :, :8] - o1[:, :, :8]).max() < 1e-14
    assert np.abs(L4 - L1).max() < 1e-12  # L is over the plain logits for every query block
    assert np.abs(o4[:, :, 8:] - o1[:, :, 8:]).max() > 1e-3  # two history blocks: g < 1 matters


def test_outside_gate_dl_matches_pages_formula():
    """dl = g·dg, with the page's outside-gate gradient dg_m = Σ p_i dOᵀ v_i over the
    tokens i of block m, summed over the block's rows and the group's heads. p is the
    softmax over the plain logits, from torch."""
    blk, N, d, K = 4, 24, 4, 3
    q, k, v, do, s = _rand_case(B=1, Hq=2, Hkv=1, N=N, d=d, block=blk, seed=79)
    idx, _ = O.prefill_select(s, K)
    _, _, _, _, dl = O.backward(q, k, v, s, idx, do, block=blk, gate_mode=O.GATE_SOFTMAX_OUTSIDE)
    scale = 1 / math.sqrt(d)
    for t in range(1, N // blk):
        sel = [int(m) for m in idx[0, 0, t] if m >= 0]
        tok = np.concatenate([np.arange(blk * t, blk * t + blk)] + [np.arange(blk * m, blk * m + blk) for m in sel])
        hist = s[0, 0, t, :t]
        gate = np.exp(hist - np.log(np.exp(hist).sum()))
        for slot, m in enumerate(sel):
            dg = 0.0
            for hq in range(2):
                for i in range(blk * t, blk * t + blk):
                    z = torch.from_numpy(scale * (k[0, 0, tok] @ q[0, hq, i]))
                    z[:blk][np.arange(blk) > i - blk * t] = -math.inf  # causal inside the current block
                    p = torch.softmax(z, 0).numpy()
                    for jj, j in enumerate(tok):
                        if blk * m <= j < blk * m + blk:
                            dg += p[jj] * float(do[0, hq, i] @ v[0, 0, j])
            assert abs(dl[0, 0, t, slot] - gate[m] * dg) < 1e-12, (t, slot)
