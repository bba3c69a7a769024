"""fp64 CPU oracle for SAS gated block-sparse attention.

TEST INFRASTRUCTURE. This module is the independent checker for the CUDA path.
Only the tests, the smoke check in ``__graft_entry__`` and the benchmark's
CPU-baseline leg may import it. The library itself never does, and this
module imports nothing from the library.

It is plain and slow on purpose. Each query block is processed on its own with
dense NumPy fp64 matrix products over the gathered tokens. There is no tiling,
no online softmax and no fusion. A reader can check each function against the
pages it cites:

* [SAS-explainer]: the ta-paperlens page "論文解説: SAS — 疎注意の「どのブロック
  を読むか」を言語モデル損失で端から端まで学習する". Section 前提 gives block
  sparse attention: C = n/b blocks, the score vector s, the Top-K union S and a
  per-query cost of |S|. Section 仕組み gives the gate g = φ(s) with g0 = 1 for
  the current block B0, Eq. (9), and the inference form with no gate
  (Algorithm 2).
* [SAS-summary]: the onedev.kr page "SAS는 언어모델 손실로 문맥 순위를 직접
  학습하는 사후 어텐션 희소화다." Section 어떻게 동작하나 gives
  o = softmax(qK_Sᵀ + log g_S) V_S. Section 무엇과 다른가 gives the
  softmax-normalised gate log g_m = s_m − LSE(s), the gate gradient with the gate
  inside the softmax, dg_m = Σ_i (p̃_i/g_m) dOᵀ(v_i − o), and "sparse scope"
  training.
* [PBS]: the gist.science page "Sparser Block-Sparse Attention via Token
  Permutation". Section 4 (実装) estimates block importance from mean-pooled
  keys.

Readings where the pages are silent or garbled (page 1's display equations
were lost when the page was extracted):

1. The softmax scale is 1/sqrt(d) unless given. [SAS-explainer] §前提 omits it.
2. LSE(s) runs over all causal history blocks m < t of query block t, not over
   the selected ones only.
3. Query block t covers tokens [b·t, b·t+b). Its history is blocks 0..t−1 and it
   selects n_t = min(K, t) of them. The current block is causally masked.
4. Ties in s go to the lower block index. The index list is written in
   ascending block order and padded with −1.
5. NaN scores rank below every number. Inputs are expected to be finite.
6. Backward uses sparse scope. Content gradients flow only through the selected
   blocks and B0. ds is the exact derivative with the selection held fixed, so
   it is nonzero for unselected history blocks too, through LSE(s).
7. Decode: ``cache_len`` counts the new token. The current block is
   c = (L−1) // b and holds L − b·c tokens with gate 1. History is blocks
   0..c−1.
8. Paged KV cache. [SAS-summary] §전제와 한계 measures decode inside a serving
   engine, which keeps the cache in pages; the pages do not describe a
   layout. A page here holds one block of every KV head, and a block table
   maps logical blocks to pages. Paging changes where tokens are stored, not
   what the step computes: ``decode_paged`` is ``decode`` on the gathered
   dense cache.
9. Selector scoring for decode. The pages' selector is a trained network
   whose weights are not available. The stand-in scores history block m by
   the mean-pooled key: s_m = scale · ⟨q̄, k̄_m⟩, where k̄_m is the mean of the
   block's keys and q̄ the mean of the new token's queries over the KV head's
   group. This is the learned selector with identity projections. It also
   equals the mean over the block's tokens and the group's heads of the
   token-level logits.
10. The gate outside the softmax. [SAS-summary] §무엇과 다른가 contrasts it with
    the gate inside: outside, the attention probabilities are those of the
    plain logits and the gate only re-weights the values, with dg_m = Σ p_i dOᵀv_i
    over block m's tokens. Read with the method's g = softmax(s) and g0 = 1: p is
    the softmax over the plain logits of the whole attended set, and the output
    o = Σ_i g_{m(i)} p_i v_i is not renormalised. dl = g·dg feeds the same chain
    to ds as the gate inside.

All arithmetic is float64. Inputs are taken as given; the generators round
them to bf16 before either side sees them.
"""
from __future__ import annotations

import math
from typing import List, Optional, Sequence, Tuple

import numpy as np

GATE_LOG_SOFTMAX = 0  # training form, Eq. (9)
GATE_NONE = 1  # inference form (Algorithm 2): Top-K only, no gate
# Ablations of the gate activation ([SAS-summary] §무엇과 다른가): a sigmoid gate,
# which saturates to 1, and the raw logit injected unnormalised, which collapses
# to 0. Both stay inside the softmax in log form.
GATE_LOG_SIGMOID = 2  # log g_m = log σ(s_m)
GATE_LOGIT = 3  # log g_m = s_m
# The gate outside the softmax ([SAS-summary] §무엇과 다른가, the first design
# choice): g = softmax(s) multiplies the values of its block after a softmax
# over the plain logits, o = Σ_i g_{m(i)} p_i v_i.
GATE_SOFTMAX_OUTSIDE = 4


def _scale(d: int, softmax_scale: Optional[float]) -> float:
    return 1.0 / math.sqrt(d) if not softmax_scale else float(softmax_scale)


# ---------------------------------------------------------------------------
# Selection: Top-K over the history scores ([SAS-explainer] §前提, the union S;
# ties to the lower block index)
# ---------------------------------------------------------------------------
def topk_blocks(s_hist: np.ndarray, K: int) -> List[int]:
    """The min(K, len(s_hist)) highest-scoring history blocks, ascending.

    The order key is (score descending, block index ascending), with NaN
    below every number. The library sort does the ranking.
    """
    t = len(s_hist)
    n = min(K, t)
    if n <= 0:
        return []
    s = np.asarray(s_hist, dtype=np.float64)
    isnan = np.isnan(s)
    neg = np.where(isnan, 0.0, -s)
    # np.lexsort: the last key is the primary one
    order = np.lexsort((np.arange(t), neg, isnan.astype(np.int8)))
    return sorted(int(m) for m in order[:n])


def logsumexp(x: np.ndarray) -> float:
    """log Σ exp x, with the usual max shift. −inf for an empty row."""
    x = np.asarray(x, dtype=np.float64)
    if x.size == 0:
        return -math.inf
    m = float(np.max(x))
    if m == -math.inf:
        return -math.inf
    return m + math.log(float(np.sum(np.exp(x - m))))


def prefill_select(s: np.ndarray, K: int) -> Tuple[np.ndarray, np.ndarray]:
    """Top-K index sets and gate normaliser for every (batch, KV head, query block).

    s: [B, Hkv, NQB, NKB]. Returns idx int32 [B, Hkv, NQB, K] (ascending, −1 pad)
    and lse_s float64 [B, Hkv, NQB] with lse_s = LSE(s[t, 0:t]), −inf at t = 0.
    """
    B, H, NQB, NKB = s.shape
    idx = np.full((B, H, NQB, K), -1, dtype=np.int32)
    lse = np.full((B, H, NQB), -math.inf)
    for b in range(B):
        for h in range(H):
            for t in range(NQB):
                sel = topk_blocks(s[b, h, t, :t], K)
                idx[b, h, t, : len(sel)] = sel
                lse[b, h, t] = logsumexp(s[b, h, t, :t])
    return idx, lse


def decode_select(s: np.ndarray, cache_len: np.ndarray, K: int, block: int = 64) -> Tuple[np.ndarray, np.ndarray]:
    """Decode form of the selection: s [B, Hkv, NKB]; history of batch b is 0..c_b−1."""
    B, H, _ = s.shape
    idx = np.full((B, H, K), -1, dtype=np.int32)
    lse = np.full((B, H), -math.inf)
    for b in range(B):
        c = (int(cache_len[b]) - 1) // block
        for h in range(H):
            sel = topk_blocks(s[b, h, :c], K)
            idx[b, h, : len(sel)] = sel
            lse[b, h] = logsumexp(s[b, h, :c])
    return idx, lse


# ---------------------------------------------------------------------------
# Gate ([SAS-summary] §무엇과 다른가: g = softmax(s), log g_m = s_m − LSE(s);
# [SAS-explainer] §仕組み: g0 = 1 for B0, one value per block broadcast to its
# tokens)
# ---------------------------------------------------------------------------
def _log_sigmoid(x: float) -> float:
    """log σ(x) = −log(1 + e^(−x)), written so that neither branch overflows."""
    return -math.log1p(math.exp(-x)) if x >= 0 else x - math.log1p(math.exp(x))


def log_gate(s_hist: np.ndarray, selected: Sequence[int], gate_mode: int) -> np.ndarray:
    """log g_m for the selected history blocks (0 for every block under GATE_NONE)."""
    if gate_mode == GATE_NONE:
        return np.zeros(len(selected))
    if gate_mode == GATE_LOG_SIGMOID:
        return np.array([_log_sigmoid(float(s_hist[m])) for m in selected], dtype=np.float64)
    if gate_mode == GATE_LOGIT:
        return np.array([float(s_hist[m]) for m in selected], dtype=np.float64)
    # the softmax-normalised gate, inside (log g in the logits) or outside (g on the values)
    lse = logsumexp(s_hist)
    return np.array([float(s_hist[m]) - lse for m in selected], dtype=np.float64)


def gate_score_gradient(s_hist: np.ndarray, selected: Sequence[int], dl_sel: np.ndarray, gate_mode: int) -> np.ndarray:
    """ds over the history blocks from dl = ∂loss/∂log g of the selected ones.

    log-softmax: ds_m = dl_m·[m ∈ I] − softmax(s)_m Σ dl (every history block
    couples through LSE). log-sigmoid: ds_m = dl_m (1 − σ(s_m)) on the selected
    blocks. logit: ds_m = dl_m on the selected blocks.
    """
    sh = np.asarray(s_hist, np.float64)
    ds_row = np.zeros(len(sh))
    if gate_mode in (GATE_LOG_SOFTMAX, GATE_SOFTMAX_OUTSIDE):
        ds_row = -np.exp(sh - logsumexp(sh)) * float(np.sum(dl_sel))
    for m, x in zip(selected, dl_sel):
        if gate_mode == GATE_LOG_SIGMOID:
            x = x * (1.0 - 1.0 / (1.0 + math.exp(-sh[m])))
        ds_row[m] += x
    return ds_row


def _gathered_tokens(t: int, selected: Sequence[int], block: int, n_cur: int) -> np.ndarray:
    """Token positions of S = B0 ∪ ⋃_{m∈I} B_m: current block first, then history ascending."""
    cur = np.arange(block * t, block * t + n_cur)
    hist = [np.arange(block * m, block * m + block) for m in selected]
    return np.concatenate([cur] + hist) if hist else cur


# ---------------------------------------------------------------------------
# Forward: Eq. (9) of [SAS-explainer] §仕組み, o = softmax(qK_Sᵀ + log g_S) V_S
# ---------------------------------------------------------------------------
def _gate_placement(lam_tok: np.ndarray, gate_mode: int):
    """(logit bias, value weight) per gathered token: (log g, 1) for a gate inside the
    softmax, (0, g) for the gate outside it. The current block has log g = 0 either way."""
    if gate_mode == GATE_SOFTMAX_OUTSIDE:
        return np.zeros_like(lam_tok), np.exp(lam_tok)
    return lam_tok, np.ones_like(lam_tok)


def _block_logits(qb, Kst, lam_tok, scale, causal_n):
    """z = scale·q Kᵀ + log g, with the causal mask inside the current block.

    qb [R, d] are the rows of one head in query block t. Kst [|S|, d] holds the
    gathered keys, current block first. The current block occupies the first
    causal_n columns, and row r may see columns 0..r of it.
    """
    z = scale * (qb @ Kst.T) + lam_tok[None, :]
    R = qb.shape[0]
    rr = np.arange(R)[:, None]
    cc = np.arange(z.shape[1])[None, :]
    z = np.where((cc < causal_n) & (cc > rr), -np.inf, z)
    return z


def forward(q, k, v, s, idx, block: int = 64, gate_mode: int = GATE_LOG_SOFTMAX,
            softmax_scale: Optional[float] = None, t_list: Optional[Sequence[int]] = None):
    """Gated block-sparse attention forward.

    q [B, Hq, N, d], k/v [B, Hkv, N, d], s [B, Hkv, NQB, NKB], idx [B, Hkv, NQB, K]
    (as from ``prefill_select``). Returns o [B, Hq, N, d] and the row
    log-sum-exp L [B, Hq, N] of the gated logits z. With ``t_list`` only those
    query blocks are computed; the other rows stay NaN.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    NQB = N // block
    scale = _scale(d, softmax_scale)
    o = np.full(q.shape, np.nan)
    L = np.full((B, Hq, N), np.nan)
    ts = range(NQB) if t_list is None else t_list
    for b in range(B):
        for h in range(Hkv):
            for t in ts:
                sel = [int(m) for m in idx[b, h, t] if m >= 0]
                lam = log_gate(s[b, h, t, :t], sel, gate_mode)
                tok = _gathered_tokens(t, sel, block, block)
                lam_tok = np.concatenate([np.zeros(block), np.repeat(lam, block)])
                z_bias, g_tok = _gate_placement(lam_tok, gate_mode)
                Kst, Vst = k[b, h, tok], v[b, h, tok]
                rows = slice(block * t, block * t + block)
                for g in range(G):
                    hq = h * G + g
                    z = _block_logits(q[b, hq, rows], Kst, z_bias, scale, block)
                    zmax = z.max(axis=1, keepdims=True)
                    e = np.exp(z - zmax)
                    den = e.sum(axis=1, keepdims=True)
                    P = e / den
                    o[b, hq, rows] = (P * g_tok) @ Vst
                    L[b, hq, rows] = (zmax + np.log(den))[:, 0]
    return o, L


# ---------------------------------------------------------------------------
# Backward: the softmax Jacobian applied to Eq. (9), sparse scope
# ([SAS-summary] §무엇과 다른가, fourth design choice), and the chain through
# g = softmax(s) to the scores
# ---------------------------------------------------------------------------
def backward(q, k, v, s, idx, do, block: int = 64, gate_mode: int = GATE_LOG_SOFTMAX,
             softmax_scale: Optional[float] = None, o=None, t_list: Optional[Sequence[int]] = None):
    """Gradients of ⟨dO, o⟩ with the selection held fixed.

    Returns dq [B, Hq, N, d], dk, dv [B, Hkv, N, d], ds [B, Hkv, NQB, NKB] and
    dl [B, Hkv, NQB, K]. dl[t, slot] is the gradient with respect to log g of the
    block idx[t, slot], summed over the block's tokens, the query block's rows and
    the group's heads. ds follows from log g_m(s) of the gate mode (see
    ``gate_score_gradient``); for the softmax-normalised gate,
    ds_m = dl_m·[m ∈ I] − softmax(s)_m Σ_{m'∈I} dl_m'.

    ``o`` (the forward output) is recomputed when not given. With ``t_list`` only
    those query blocks contribute, so dk/dv are partial sums.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    do = np.asarray(do, np.float64)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    NQB = N // block
    K = idx.shape[-1]
    scale = _scale(d, softmax_scale)
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    ds = np.zeros(s.shape)
    dl = np.zeros((B, Hkv, NQB, K))
    ts = range(NQB) if t_list is None else t_list
    for b in range(B):
        for h in range(Hkv):
            for t in ts:
                sel = [int(m) for m in idx[b, h, t] if m >= 0]
                lam = log_gate(s[b, h, t, :t], sel, gate_mode)
                tok = _gathered_tokens(t, sel, block, block)
                lam_tok = np.concatenate([np.zeros(block), np.repeat(lam, block)])
                z_bias, g_tok = _gate_placement(lam_tok, gate_mode)
                Kst, Vst = k[b, h, tok], v[b, h, tok]
                rows = slice(block * t, block * t + block)
                dlam_tok = np.zeros(len(tok))
                for g in range(G):
                    hq = h * G + g
                    z = _block_logits(q[b, hq, rows], Kst, z_bias, scale, block)
                    zmax = z.max(axis=1, keepdims=True)
                    e = np.exp(z - zmax)
                    P = e / e.sum(axis=1, keepdims=True)
                    ob = (P * g_tok) @ Vst if o is None else np.asarray(o[b, hq, rows], np.float64)
                    dOb = do[b, hq, rows]
                    dP = dOb @ Vst.T  # ∂⟨dO,o⟩/∂(the weight of v_j): g_j p_j is that weight
                    Drow = np.sum(dOb * ob, axis=1, keepdims=True)  # = Σ_j P_ij g_j dP_ij
                    dZ = P * (g_tok * dP - Drow)  # ∂/∂z through the row softmax
                    dq[b, hq, rows] += scale * (dZ @ Kst)
                    # tok holds distinct positions, so fancy-index += sums each row once
                    dk[b, h, tok] += scale * (dZ.T @ q[b, hq, rows])
                    dv[b, h, tok] += (P * g_tok).T @ dOb
                    if gate_mode == GATE_SOFTMAX_OUTSIDE:
                        dlam_tok += (P * g_tok * dP).sum(axis=0)  # g ∂/∂g: ∂g/∂log g = g
                    else:
                        dlam_tok += dZ.sum(axis=0)
                if gate_mode == GATE_NONE or t == 0:
                    continue
                dl_sel = dlam_tok[block:].reshape(len(sel), block).sum(axis=1)
                dl[b, h, t, : len(sel)] = dl_sel
                # chain through log g_m(s_hist) of the gate mode
                ds[b, h, t, :t] = gate_score_gradient(s[b, h, t, :t], sel, dl_sel, gate_mode)
    return dq, dk, dv, ds, dl


def gate_gradient_from_pages(q, k, v, s, idx, do, b, h, t, block: int = 64,
                             softmax_scale: Optional[float] = None) -> np.ndarray:
    """g_m · dg_m for each selected block of query block t, taken straight from
    the formula of [SAS-summary] §무엇과 다른가 (gate inside the softmax):

        dg_m = Σ_{i ∈ B_m} (p̃_i / g_m) · dOᵀ (v_i − o),

    summed over the rows of query block t and the heads of the group. p̃ is the
    gated attention probability. This route goes through v_i − o and never forms
    the softmax Jacobian, so it checks ``backward``'s dl by another path.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    do = np.asarray(do, np.float64)
    _, Hq, _, d = q.shape
    G = Hq // k.shape[1]
    scale = _scale(d, softmax_scale)
    sel = [int(m) for m in idx[b, h, t] if m >= 0]
    sh = np.asarray(s[b, h, t, :t], np.float64)
    g_sel = np.exp(np.array([sh[m] for m in sel]) - logsumexp(sh))
    out = np.zeros(len(sel))
    rows = range(block * t, block * t + block)
    for g in range(G):
        hq = h * G + g
        for i_row in rows:
            # token-level gated softmax of the one query, from Eq. (9) written out
            cur = list(range(block * t, i_row + 1))
            toks = cur + [j for m in sel for j in range(block * m, block * m + block)]
            logit = [scale * float(q[b, hq, i_row] @ k[b, h, j]) for j in cur]
            for mi, m in enumerate(sel):
                for j in range(block * m, block * m + block):
                    logit.append(scale * float(q[b, hq, i_row] @ k[b, h, j]) + math.log(g_sel[mi]))
            logit = np.array(logit)
            p = np.exp(logit - logsumexp(logit))
            o_i = p @ v[b, h, toks]
            base = len(cur)
            for mi in range(len(sel)):
                for jj in range(block):
                    j = toks[base + mi * block + jj]
                    p_t = p[base + mi * block + jj]
                    dg = (p_t / g_sel[mi]) * float(do[b, hq, i_row] @ (v[b, h, j] - o_i))
                    out[mi] += g_sel[mi] * dg
    return out


# ---------------------------------------------------------------------------
# Decode: one new token per sequence, Top-K over the history, the current
# (possibly partial) block always kept ([SAS-explainer] §仕組み, Algorithm 2
# for the ungated inference form)
# ---------------------------------------------------------------------------
def decode_block_list(cache_len: int, idx_row: Sequence[int], block: int = 64) -> List[int]:
    """Blocks read by one decode query: the current block c first, then the selected ones."""
    c = (int(cache_len) - 1) // block
    return [c] + [int(m) for m in idx_row if m >= 0]


def split_ranges(n_items: int, n_split: int) -> List[Tuple[int, int]]:
    """Contiguous chunks of the ordered block list: split j takes [j·per, (j+1)·per)."""
    per = -(-n_items // n_split)
    return [(min(j * per, n_items), min((j + 1) * per, n_items)) for j in range(n_split)]


def _decode_partial(qv, kc, vc, blocks, L, s_hist, sel, gate_mode, scale, block):
    """(o, lse) of one query over the tokens of ``blocks`` (any subset of the block list)."""
    if not blocks:
        return np.zeros(qv.shape[-1]), -math.inf
    c = (L - 1) // block
    lam = dict(zip(sel, log_gate(s_hist, sel, gate_mode)))
    toks, lt = [], []
    for m in blocks:
        if m == c:
            r = np.arange(block * c, L)
            toks.append(r)
            lt.append(np.zeros(len(r)))
        else:
            toks.append(np.arange(block * m, block * m + block))
            lt.append(np.full(block, lam[m]))
    toks = np.concatenate(toks)
    z_bias, g_tok = _gate_placement(np.concatenate(lt), gate_mode)
    z = scale * (kc[toks] @ qv) + z_bias
    lse = logsumexp(z)
    return (np.exp(z - lse) * g_tok) @ vc[toks], lse


def decode(q, kc, vc, cache_len, s, K: int, block: int = 64, gate_mode: int = GATE_NONE,
           softmax_scale: Optional[float] = None, n_split: int = 1):
    """Single-token decode. q [B, Hq, d]; kc/vc [B, Hkv, Lmax, d]; s [B, Hkv, NKB].

    Returns idx [B, Hkv, K], lse_s [B, Hkv], the split partials o_part
    [B, Hq, n_split, d] and lse_part [B, Hq, n_split], and their merge o
    [B, Hq, d] and lse [B, Hq]. With n_split = 1 the partial is the whole answer.
    """
    q = np.asarray(q, np.float64)
    kc = np.asarray(kc, np.float64)
    vc = np.asarray(vc, np.float64)
    B, Hq, d = q.shape
    Hkv = kc.shape[1]
    G = Hq // Hkv
    scale = _scale(d, softmax_scale)
    idx, lse_s = decode_select(s, cache_len, K, block)
    o_part = np.zeros((B, Hq, n_split, d))
    lse_part = np.full((B, Hq, n_split), -math.inf)
    for b in range(B):
        L = int(cache_len[b])
        c = (L - 1) // block
        for h in range(Hkv):
            sel = [int(m) for m in idx[b, h] if m >= 0]
            blist = decode_block_list(L, idx[b, h], block)
            for j, (a, e) in enumerate(split_ranges(len(blist), n_split)):
                for g in range(G):
                    hq = h * G + g
                    o_part[b, hq, j], lse_part[b, hq, j] = _decode_partial(
                        q[b, hq], kc[b, h], vc[b, h], blist[a:e], L, s[b, h, :c], sel, gate_mode, scale, block)
    o, lse = decode_combine(o_part, lse_part)
    return dict(idx=idx, lse_s=lse_s, o_part=o_part, lse_part=lse_part, o=o, lse=lse)


def gather_pages(k_pages, v_pages, block_table, cache_len, block: int = 64):
    """Dense caches [B, Hkv, Lmax, d] from a paged cache.

    A page holds one block of every KV head: k_pages and v_pages are
    [n_pages, Hkv, block, d], and block_table[b, m] is the page of logical block
    m of sequence b. Blocks 0..(L−1)/block of sequence b are copied. Everything
    else stays zero, so a page's tokens past the cache length and the blocks
    past the current one never enter the result.
    """
    k_pages = np.asarray(k_pages)
    v_pages = np.asarray(v_pages)
    B, NB = block_table.shape
    _, Hkv, _, d = k_pages.shape
    kc = np.zeros((B, Hkv, NB * block, d))
    vc = np.zeros((B, Hkv, NB * block, d))
    for b in range(B):
        L = int(cache_len[b])
        for m in range((L - 1) // block + 1):
            n = min(block, L - m * block)  # tokens of block m that exist
            pg = int(block_table[b, m])
            kc[b, :, m * block:m * block + n] = k_pages[pg, :, :n]
            vc[b, :, m * block:m * block + n] = v_pages[pg, :, :n]
    return kc, vc


def decode_paged(q, k_pages, v_pages, block_table, cache_len, s, K: int, block: int = 64,
                 gate_mode: int = GATE_NONE, softmax_scale: Optional[float] = None, n_split: int = 1):
    """Single-token decode over a paged KV cache.

    The paged cache is only a storage layout. The step is the same decode as
    ``decode``, over the dense cache that ``gather_pages`` rebuilds.
    """
    kc, vc = gather_pages(k_pages, v_pages, block_table, cache_len, block)
    return decode(q, kc, vc, cache_len, s, K, block, gate_mode, softmax_scale, n_split)


def decode_combine(o_part: np.ndarray, lse_part: np.ndarray):
    """Merge split partials: LSE = log Σ_j exp lse_j, o = Σ_j exp(lse_j − LSE) o_j."""
    o_part = np.asarray(o_part, np.float64)
    lse_part = np.asarray(lse_part, np.float64)
    shp = lse_part.shape[:-1]
    o = np.zeros(shp + (o_part.shape[-1],))
    lse = np.full(shp, -math.inf)
    for ix in np.ndindex(*shp):
        tot = logsumexp(lse_part[ix])
        lse[ix] = tot
        if tot == -math.inf:
            continue
        w = np.exp(lse_part[ix] - tot)
        o[ix] = w @ o_part[ix]
    return o, lse


# ---------------------------------------------------------------------------
# Selector scoring for decode from mean-pooled keys (reading 9).
# [SAS-summary] §전제와 한계: the decode step's selector scoring and Top-K
# ranking grow with the context, unlike the attention itself. [PBS] §4 実装:
# block importance is estimated from mean-pooled keys.
# ---------------------------------------------------------------------------
def block_mean_keys(k, block: int = 64) -> np.ndarray:
    """k [B, Hkv, L, d] -> k̄ [B, Hkv, L // block, d], the mean of each block's keys."""
    k = np.asarray(k, np.float64)
    B, H, L, d = k.shape
    nb = L // block
    out = np.zeros((B, H, nb, d))
    for m in range(nb):
        out[:, :, m] = k[:, :, m * block:(m + 1) * block].sum(axis=2) / block
    return out


def decode_scores(q, kmean, cache_len, block: int = 64, softmax_scale: Optional[float] = None) -> np.ndarray:
    """Selector scores of a decode step: s [B, Hkv, NKB].

    s[b, h, m] = scale · ⟨q̄, k̄_m⟩ for the history blocks m < c of sequence b,
    with q̄ the mean of the new token's query vectors over the KV head's group.
    Entries m ≥ c are NaN: nothing reads them.
    """
    q = np.asarray(q, np.float64)
    kmean = np.asarray(kmean, np.float64)
    B, Hq, d = q.shape
    Hkv, NKB = kmean.shape[1], kmean.shape[2]
    G = Hq // Hkv
    scale = _scale(d, softmax_scale)
    s = np.full((B, Hkv, NKB), np.nan)
    for b in range(B):
        c = (int(cache_len[b]) - 1) // block
        for h in range(Hkv):
            qbar = q[b, h * G:(h + 1) * G].mean(axis=0)
            s[b, h, :c] = scale * (kmean[b, h, :c] @ qbar)
    return s


def decode_select_scored(q, kmean, cache_len, K: int, block: int = 64, softmax_scale: Optional[float] = None):
    """Scores from block-mean keys, then the decode-form Top-K and LSE(s): (s, idx, lse_s)."""
    s = decode_scores(q, kmean, cache_len, block, softmax_scale)
    idx, lse = decode_select(s, cache_len, K, block)
    return s, idx, lse
