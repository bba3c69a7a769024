/*
 * sas.h — C ABI of the SAS gated block-sparse attention library for NVIDIA
 * B200 (sm_100a).
 *
 * The method: the context is cut into blocks of b = 64 tokens. A selector
 * gives one score s_m per history block. Every query block keeps its own
 * block B0, causally masked and with gate 1. It also keeps the Top-K history
 * blocks by s. For training, the softmax-normalised gate goes inside the
 * attention softmax as log g_m = s_m − LSE(s):
 *
 *     o = softmax(q K_Sᵀ·scale + log g_S) V_S,   S = B0 ∪ ⋃_{m∈I} B_m.
 *
 * Sources:
 *  - SAS explainer (ta-paperlens, "論文解説: SAS — 疎注意の「どのブロックを
 *    読むか」を言語モデル損失で端から端まで学習する"). §前提 covers blocks,
 *    Top-K and the union S. §仕組み covers the gate, Eq. (9) and the ungated
 *    inference form (Algorithm 2).
 *  - SAS summary (onedev.kr, "SAS는 언어모델 손실로 문맥 순위를 직접 학습하는
 *    사후 어텐션 희소화다."). §어떻게 동작하나 gives o_SAS. §무엇과 다른가
 *    gives g = softmax(s), log g_m = s_m − LSE(s), the gate gradient
 *    dg_m = Σ_i (p̃_i/g_m) dOᵀ(v_i − o) and sparse-scope training.
 *
 * Conventions shared by every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller. The library
 *    allocates no device memory. The only host pointers are `p`, the `bytes`
 *    output of sas_bwd_workspace_size and the `code` output of
 *    sas_get_device_error.
 *  - Tensors are dense, row-major, in the stated layouts. The last dimension
 *    is innermost. Every tensor pointer must be 16-byte aligned.
 *  - bf16 tensors hold IEEE bfloat16 bit patterns (sas_bf16 = uint16_t).
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL means the
 *    legacy default stream). Arguments are checked on the host before any
 *    launch. A bad argument returns an error status and launches nothing.
 *    A launch failure returns SAS_ERR_CUDA. Device-side faults that the
 *    kernels detect themselves are raised through sas_get_device_error, for
 *    example an index outside the history or a bounded wait that expired.
 *  - Calls keep no state between them and may be issued from several host
 *    threads, on different streams, with two exceptions. Each device has one
 *    error word, shared by every caller: sas_get_device_error reads and
 *    clears it, so one caller's read also clears what another caller's
 *    kernels raised. And sas_decode_noalloc shares one fixed scratch array
 *    per device (see there). The library looks up the device addresses of
 *    both once per device and keeps them: after cudaDeviceReset on a device,
 *    unload and reload the library before calling it on that device.
 *
 * Shapes (sas_params): B = batch, Hq = n_q_heads, Hkv = n_kv_heads,
 * G = Hq / Hkv (GQA group), d = head_dim, N = seq_len, b = block (64),
 * NQB = NKB = N / b, K = top_k. Query block t covers tokens [b·t, b·t + b).
 * Its history is blocks 0..t−1, and it selects n_t = min(K, t) of them.
 */
#ifndef SAS_H_
#define SAS_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SAS_API __attribute__((visibility("default")))
#else
#define SAS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t sas_bf16;

typedef enum {
  SAS_OK = 0,
  SAS_ERR_INVALID_ARG = 1, /* a pointer, size or layout rule is broken */
  SAS_ERR_UNSUPPORTED = 2, /* valid, but no kernel for it (e.g. head_dim 96) */
  SAS_ERR_WORKSPACE = 3,   /* workspace missing or smaller than required */
  SAS_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed */
  SAS_ERR_TIMEOUT = 5,     /* a device-side bounded wait expired */
  SAS_ERR_DEVICE_INDEX = 6 /* a kernel met a block index outside the history */
} sas_status;

typedef enum {
  /* Training form, Eq. (9): log g_m = s_m − LSE(s) is added to the logits of
   * every token of selected history block m. The current block gets 0. */
  SAS_GATE_LOG_SOFTMAX = 0,
  /* Inference form (Algorithm 2): Top-K selection only, no gate term. */
  SAS_GATE_NONE = 1,
  /* Ablations of the gate activation (SAS summary §무엇과 다른가: a sigmoid
   * gate saturates to 1, unnormalised logits collapse to 0). Both stay inside
   * the softmax in log form, like SAS_GATE_LOG_SOFTMAX, and need s but not
   * lse_s (which may be NULL and is not read).
   * log g_m = log σ(s_m): */
  SAS_GATE_LOG_SIGMOID = 2,
  /* log g_m = s_m: */
  SAS_GATE_LOGIT = 3,
  /* The gate outside the softmax (SAS summary §무엇과 다른가, contrasted with
   * the gate inside): g_m = softmax(s)_m over the history multiplies the
   * values of block m after a softmax over the plain logits,
   * o_i = Σ_j g_{m(j)} p_ij v_j (g = 1 for the current block), with no
   * renormalisation. lse_o is the log-sum-exp of the plain logits. Needs s and
   * lse_s, like SAS_GATE_LOG_SOFTMAX, and its ds chain is the same. */
  SAS_GATE_SOFTMAX_OUTSIDE = 4
} sas_gate_mode;

typedef struct {
  int batch;           /* B >= 1 */
  int n_q_heads;       /* Hq >= 1, a multiple of n_kv_heads */
  int n_kv_heads;      /* Hkv >= 1 */
  int head_dim;        /* d: 64 or 128 */
  int seq_len;         /* prefill: N; decode: KV-cache capacity Lmax; a multiple of block.
                          SAS_ERR_UNSUPPORTED above 2^19 blocks, or when
                          batch * n_kv_heads * blocks exceeds 2^30 */
  int block;           /* b: must be 64 */
  int top_k;           /* K: 1..2048 (K >= t selects every history block: full scope) */
  float softmax_scale; /* 0 selects 1/sqrt(d) */
  int gate_mode;       /* sas_gate_mode */
} sas_params;

/* ---------------------------------------------------------------------------
 * Selection and gate normaliser
 * SAS explainer §前提: Top-K of the history scores. SAS summary §무엇과 다른가:
 * LSE(s) is the normaliser of g = softmax(s).
 * ------------------------------------------------------------------------- */

/* Top-K history blocks of every query block, and optionally LSE(s).
 *
 * Prefill form (cache_len == NULL):
 *   s       fp32  [B, Hkv, NQB, NKB]. Only entries m < t of row t are read.
 *   idx     int32 [B, Hkv, NQB, K]. Output. The n_t = min(K, t) blocks with
 *           the highest s[t, m] for m < t, ties to the lower m, written in
 *           ascending m. Slots n_t..K−1 hold −1.
 *   lse_s   fp32  [B, Hkv, NQB]. Output, may be NULL.
 *           lse_s[t] = log Σ_{m<t} exp s[t, m], and −inf at t = 0.
 * Decode form (cache_len != NULL):
 *   cache_len int32 [B]. Tokens in each sequence's cache, the new token
 *           included, 1 <= L <= seq_len. The current block is c = (L−1)/b.
 *           History is blocks 0..c−1.
 *   s       fp32  [B, Hkv, NKB]. Only m < c is read.
 *   idx     int32 [B, Hkv, K]; lse_s fp32 [B, Hkv] (may be NULL).
 * Scores must be finite. NaN ranks below every number. */
SAS_API sas_status sas_topk_select(const sas_params* p, const float* s, const int32_t* cache_len, int32_t* idx,
                           float* lse_s, void* stream);

/* LSE(s) alone, with the same layouts and forms as sas_topk_select. */
SAS_API sas_status sas_gate_lse(const sas_params* p, const float* s, const int32_t* cache_len, float* lse_s,
                        void* stream);

/* ---------------------------------------------------------------------------
 * Forward, Eq. (9) (SAS explainer §仕組み; SAS summary §어떻게 동작하나)
 * ------------------------------------------------------------------------- */

/* o_i = Σ_{j∈S_t} softmax_j(z_ij) v_j with z_ij = scale·q_i·k_j + λ_j.
 * λ_j = log g_{m(j)} for tokens of the selected history blocks: s[t, m] −
 * lse_s[t] (SAS_GATE_LOG_SOFTMAX), log σ(s[t, m]) (SAS_GATE_LOG_SIGMOID),
 * s[t, m] (SAS_GATE_LOGIT) or 0 (SAS_GATE_NONE). λ is 0 for the current
 * block. In the current block, column j is visible to row i only when j <= i.
 *   q      bf16 [B, Hq, N, d]
 *   k, v   bf16 [B, Hkv, N, d]
 *   s      fp32 [B, Hkv, NQB, NKB]. Read under every gate mode but SAS_GATE_NONE.
 *   idx    int32 [B, Hkv, NQB, K], as written by sas_topk_select.
 *   lse_s  fp32 [B, Hkv, NQB]. Required under SAS_GATE_LOG_SOFTMAX and SAS_GATE_SOFTMAX_OUTSIDE,
 *          ignored (may be NULL) under the other modes.
 *   o      bf16 [B, Hq, N, d]. Output.
 *   lse_o  fp32 [B, Hq, N]. Output, may be NULL. Row log-sum-exp of z,
 *          which the backward needs.
 * An idx entry outside [0, t) is skipped and raises SAS_ERR_DEVICE_INDEX. */
SAS_API sas_status sas_fwd(const sas_params* p, const sas_bf16* q, const sas_bf16* k, const sas_bf16* v, const float* s,
                   const int32_t* idx, const float* lse_s, sas_bf16* o, float* lse_o, void* stream);

/* ---------------------------------------------------------------------------
 * Backward with the gate/score gradient (SAS summary §무엇과 다른가: the gate
 * inside the softmax, chained through g = softmax(s); sparse scope)
 * ------------------------------------------------------------------------- */

/* Bytes of device workspace for the fastest form of sas_bwd. At head_dim 128
 * it includes one bf16 dZ tile per (query block, attended block, pair of
 * query heads): 16 KB × B·Hkv·Σ_t (1 + min(K, t))·ceil(G/2), about 4.3 GB at
 * B 1, 8 KV heads, G 4, N 32768, K 32. The KV-major pass stores dZ there and
 * the dQ pass reads it back instead of recomputing S and dP. */
SAS_API sas_status sas_bwd_workspace_size(const sas_params* p, size_t* bytes);

/* The smallest workspace sas_bwd accepts. With less than
 * sas_bwd_workspace_size bytes (but at least this many) the dQ pass
 * recomputes S and dP itself: the same results, more time, no dZ tiles. */
SAS_API sas_status sas_bwd_workspace_size_min(const sas_params* p, size_t* bytes);

/* Gradients of ⟨dO, o⟩ with the selection idx held fixed.
 *   Inputs: q, k, v, s, idx, lse_s as in sas_fwd. o and lse_o are the
 *   forward's outputs. dO is bf16 [B, Hq, N, d].
 *   dq     bf16 [B, Hq, N, d]. Output.
 *   dk, dv bf16 [B, Hkv, N, d]. Output. Summed over the G query heads.
 *   ds     fp32 [B, Hkv, NQB, NKB]. Output. With dl[t, m] the gradient for
 *          log g_m summed over block m's tokens, the rows of query block t and
 *          the G heads,
 *            ds[t, m] = dl[t, m]·[m ∈ I_t] − softmax(s[t, 0:t])_m · Σ_{m'∈I_t} dl[t, m']
 *          under SAS_GATE_LOG_SOFTMAX and SAS_GATE_SOFTMAX_OUTSIDE (where
 *          dl = g·∂/∂g = Σ p·g·dOᵀv over the block), dl[t, m]·(1 − σ(s[t, m]))·[m ∈ I_t]
 *          under SAS_GATE_LOG_SIGMOID and dl[t, m]·[m ∈ I_t] under
 *          SAS_GATE_LOGIT. Zero for m >= t, and zero everywhere under
 *          SAS_GATE_NONE. May be NULL under SAS_GATE_NONE.
 *   ws     device workspace, 256-byte aligned, of at least
 *          sas_bwd_workspace_size_min bytes (SAS_ERR_WORKSPACE otherwise).
 *          With sas_bwd_workspace_size bytes or more the faster form runs.
 *          Its contents on entry do not matter. The call overwrites it.
 * idx must be in the form sas_topk_select writes: ascending, −1 padded.
 * Other index lists are memory-safe but their gradients are unspecified. */
SAS_API sas_status sas_bwd(const sas_params* p, const sas_bf16* q, const sas_bf16* k, const sas_bf16* v,
                   const sas_bf16* o, const sas_bf16* dO, const float* s, const int32_t* idx, const float* lse_s,
                   const float* lse_o, sas_bf16* dq, sas_bf16* dk, sas_bf16* dv, float* ds, void* ws,
                   size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Split-K single-token decode (SAS explainer §仕組み: at inference Top-K on s,
 * then ordinary sparse attention; SAS summary §전제와 한계: decode is the
 * sparsified stage)
 * ------------------------------------------------------------------------- */

/* One new query token per sequence, at position L−1 with L = cache_len[b].
 * It attends to the current block c = (L−1)/b, whose tokens b·c..L−1 carry
 * gate 1, and to the selected history blocks idx[b, h, 0..n−1], n = min(K, c).
 * Under a gate mode those blocks get λ = log g (see sas_fwd). The ordered
 * block list [c, idx...] is cut into n_split contiguous chunks of
 * ceil((n+1)/n_split) blocks. Split j covers its chunk and writes that
 * chunk's normalised output and log-sum-exp. An empty chunk gives o = 0 and
 * lse = −inf.
 *   q          bf16 [B, Hq, d]
 *   kc, vc     bf16 [B, Hkv, Lmax, d]   (Lmax = seq_len)
 *   cache_len  int32 [B], 1 <= L <= Lmax
 *   s          fp32 [B, Hkv, NKB]. Read under every gate mode but SAS_GATE_NONE.
 *   idx        int32 [B, Hkv, K] from sas_topk_select (decode form)
 *   lse_s      fp32 [B, Hkv]. Required under SAS_GATE_LOG_SOFTMAX and
 *              SAS_GATE_SOFTMAX_OUTSIDE only.
 *   n_split    1..K+1, with ceil((K+1) / n_split) <= 64 (SAS_ERR_UNSUPPORTED
 *              otherwise): a split covers at most 64 blocks.
 *   o_part     fp32 [B, Hq, n_split, d]. Output.
 *   lse_part   fp32 [B, Hq, n_split]. Output. */
SAS_API sas_status sas_decode(const sas_params* p, const sas_bf16* q, const sas_bf16* kc, const sas_bf16* vc,
                      const int32_t* cache_len, const float* s, const int32_t* idx, const float* lse_s, int n_split,
                      float* o_part, float* lse_part, void* stream);

/* The same split-K decode over a paged KV cache (serving layout). A page holds
 * one 64-token block of every KV head, and a block table maps each sequence's
 * logical blocks to pages, so sequences grow without moving their history.
 *   k_pages, v_pages  bf16 [n_pages, Hkv, 64, d]
 *   n_pages           >= 1
 *   block_table       int32 [B, NKB] with NKB = seq_len / 64: the page of
 *                     logical block m of sequence b. Only the entries of the
 *                     blocks the step reads (the current block and the
 *                     selected history blocks) are read. An entry outside
 *                     [0, n_pages) raises SAS_ERR_DEVICE_INDEX, and page 0 is
 *                     read in its place.
 *   seq_len           bounds cache_len, as Lmax does for sas_decode.
 * Tokens of the current block's page past cache_len are never read. Every other
 * argument and output is as in sas_decode. */
SAS_API sas_status sas_decode_paged(const sas_params* p, const sas_bf16* q, const sas_bf16* k_pages,
                                    const sas_bf16* v_pages, int n_pages, const int32_t* block_table,
                                    const int32_t* cache_len, const float* s, const int32_t* idx, const float* lse_s,
                                    int n_split, float* o_part, float* lse_part, void* stream);

/* Merge of the split partials:
 *   LSE = log Σ_j exp lse_part[j],   o = Σ_j exp(lse_part[j] − LSE) · o_part[j].
 *   o      bf16 [B, Hq, d]. Output.
 *   lse_o  fp32 [B, Hq]. Output, may be NULL. */
SAS_API sas_status sas_decode_combine(const sas_params* p, int n_split, const float* o_part, const float* lse_part,
                              sas_bf16* o, float* lse_o, void* stream);

/* The whole decode step in one launch: the Top-K select of sas_topk_select
 * (decode form) on s, the attention of sas_decode over the current block and
 * the picks, and the merge of sas_decode_combine. SAS explainer §仕組み,
 * Algorithm 2: scores pick the Top-K history blocks, attention runs over them
 * and the current block; the gate modes apply as in sas_decode.
 *
 * One cluster of up to 8 CTAs serves each (sequence, KV head) row. Each CTA
 * selects the row's blocks itself, attends to its share of the ordered list
 * and keeps its partial in shared memory; the cluster merges the partials over
 * distributed shared memory. No partial goes to HBM and no workspace is taken.
 *
 *   q, kc, vc, cache_len  as in sas_decode.
 *   s      fp32 [B, Hkv, NKB], always read (it drives the selection).
 *   idx    int32 [B, Hkv, K]. Output, may be NULL: the picks, ascending, −1
 *          padded, bit for bit those of sas_topk_select.
 *   lse_s  fp32 [B, Hkv]. Output, may be NULL: LSE of the history scores.
 *   o      bf16 [B, Hq, d]. Output.
 *   lse_o  fp32 [B, Hq]. Output, may be NULL.
 * Limits: G <= 8, K <= 255 and NKB <= 2048 (the row's keys and picks live in
 * shared memory); other shapes return SAS_ERR_UNSUPPORTED before any launch
 * and are served by the separate calls. A cache_len outside [1, seq_len]
 * raises SAS_ERR_DEVICE_INDEX and is clamped. */
SAS_API sas_status sas_decode_fused(const sas_params* p, const sas_bf16* q, const sas_bf16* kc, const sas_bf16* vc,
                                    const int32_t* cache_len, const float* s, int32_t* idx, float* lse_s, sas_bf16* o,
                                    float* lse_o, void* stream);

/* sas_decode_fused over the paged cache of sas_decode_paged (k_pages, v_pages,
 * n_pages, block_table as there). Only the table entries of the blocks the
 * step reads are read. */
SAS_API sas_status sas_decode_fused_paged(const sas_params* p, const sas_bf16* q, const sas_bf16* k_pages,
                                          const sas_bf16* v_pages, int n_pages, const int32_t* block_table,
                                          const int32_t* cache_len, const float* s, int32_t* idx, float* lse_s,
                                          sas_bf16* o, float* lse_o, void* stream);

/* ---------------------------------------------------------------------------
 * Selector scoring fused with Top-K for long decode caches (SAS summary
 * §전제와 한계: in decode, the selector's scoring and the Top-K ranking grow
 * with the context while the attention does not. PBS §4: block importance
 * from mean-pooled keys.)
 * ------------------------------------------------------------------------- */

/* Block-mean keys: kmean[b, h, m, :] = (1/64) Σ_{j<64} k[b, h, 64m + j, :],
 * summed in fp32 and rounded once to bf16.
 *   k          bf16 [B, Hkv, Lmax, d] (Lmax = seq_len), the K cache.
 *   cache_len  NULL: every block m < Lmax/64 of every sequence is written.
 *              int32 [B]: the decode update. For each sequence whose
 *              cache_len[b] is a multiple of 64, only block cache_len[b]/64 − 1
 *              (the block the newest token completed) is written; nothing is
 *              written for the other sequences. A cache_len outside
 *              [1, Lmax] raises SAS_ERR_DEVICE_INDEX.
 *   kmean      bf16 [B, Hkv, Lmax/64, d]. Output, caller-owned.
 * Blocks must be complete when summarised: a block with tokens past the
 * sequence's cache_len is summarised over whatever the cache holds there. */
SAS_API sas_status sas_block_mean_keys(const sas_params* p, const sas_bf16* k, const int32_t* cache_len,
                                       sas_bf16* kmean, void* stream);

/* Selector scores of one decode step and their Top-K, in one launch.
 *   s[b, h, m] = scale · ⟨q̄, kmean[b, h, m]⟩ for the history blocks m < c,
 *   c = (cache_len[b] − 1)/64, with q̄ = (1/G) Σ_g q[b, h·G + g] and scale
 *   p->softmax_scale (0 selects 1/sqrt(d)). Then, as the decode form of
 *   sas_topk_select on these scores: idx = the n = min(K, c) highest-scoring
 *   history blocks, ties to the lower m, ascending, padded with −1; lse_s =
 *   log Σ_{m<c} exp s[b, h, m], −inf when c = 0.
 *   q          bf16 [B, Hq, d]
 *   kmean      bf16 [B, Hkv, NKB, d] from sas_block_mean_keys
 *   cache_len  int32 [B], 1 <= L <= seq_len (otherwise SAS_ERR_DEVICE_INDEX,
 *              and the row is treated as having no history)
 *   s          fp32 [B, Hkv, NKB]. Output: entries m < c are written, the
 *              rest are left as they were. sas_decode reads it for the gate.
 *   idx        int32 [B, Hkv, K]. Output.
 *   lse_s      fp32 [B, Hkv]. Output, may be NULL.
 * The selection is exact for the scores written to s (a full sort of s would
 * pick the same blocks). Each row is split over a cluster of up to 8 CTAs,
 * each holding at most 53,248 scores in shared memory: SAS_ERR_UNSUPPORTED
 * beyond 8 × 53,248 history blocks (about 27M tokens). */
SAS_API sas_status sas_decode_select_scored(const sas_params* p, const sas_bf16* q, const sas_bf16* kmean,
                                            const int32_t* cache_len, float* s, int32_t* idx, float* lse_s,
                                            void* stream);

/* ---------------------------------------------------------------------------
 * Decode step that allocates nothing. The paper has no counterpart to this
 * entry point; it exists for callers of this library that cannot allocate.
 * ------------------------------------------------------------------------- */

/* Size of the library's fixed decode scratch, on every GPU that loads it. */
#define SAS_NOALLOC_SCRATCH_BYTES (16 * 1024 * 1024)

/* The whole decode step in one call: the decode form of sas_topk_select, then
 * sas_decode with n_split = K + 1 (one block per split), then
 * sas_decode_combine. The caller passes the inputs and the outputs only. The
 * index lists, gate normalisers and split partials between the kernels live in
 * a fixed device array inside the library, so the call allocates nothing.
 *
 * Who needs it: callers that cannot call cudaMalloc. cudaMalloc synchronises
 * the device, which a serving loop with a per-step latency budget cannot
 * afford. A plugin inside a host framework whose caching allocator already
 * holds most of HBM would see cudaMalloc fail or fragment memory behind the
 * framework's back. A plain C caller may have no device allocator at all.
 *
 * Arguments: q, kc, vc, cache_len and s as in sas_decode (s is always
 * required, it drives the selection). o bf16 [B, Hq, d] and lse_o fp32
 * [B, Hq] (may be NULL) as in sas_decode_combine.
 *
 * Limits and behaviour:
 *  - The scratch holds B·Hkv·K int32 indices, B·Hkv fp32 normalisers and
 *    B·Hq·(K+1)·(d+1) fp32 partials, each region rounded up to 256 bytes.
 *    Sizes beyond SAS_NOALLOC_SCRATCH_BYTES return SAS_ERR_WORKSPACE before
 *    any launch. For example, 16 sequences × 32 query heads × K = 16 × d = 128
 *    need about 4.5 MB.
 *  - The array is a file-scope device variable: every GPU that loads the
 *    library holds these 16 MiB until the process exits.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress, with that device current). Make that first call
 *    before any stream capture on that device. The address is kept for the
 *    life of the library: after cudaDeviceReset, reload the library.
 *  - Every call shares the one array per device. Calls that overlap on the
 *    GPU (other streams, other host threads) race on it; the caller must
 *    order them. Each call writes all the scratch it reads, so nothing needs
 *    clearing between calls.
 *  - No cudaMalloc, cudaFree or allocating library routine is called. */
SAS_API sas_status sas_decode_noalloc(const sas_params* p, const sas_bf16* q, const sas_bf16* kc, const sas_bf16* vc,
                                      const int32_t* cache_len, const float* s, sas_bf16* o, float* lse_o,
                                      void* stream);

/* ---------------------------------------------------------------------------
 * Training steps end to end from host memory. The pages have no counterpart:
 * this is the library's I/O path for callers whose batches live on the host.
 * ------------------------------------------------------------------------- */

/* One step's host buffers (pinned memory, for the copies to overlap; pageable
 * memory works but serialises them). Inputs as in sas_fwd / sas_bwd; outputs
 * as those calls write them. lse_o may be NULL (not copied back). ds must be
 * NULL under SAS_GATE_NONE and may be NULL otherwise (not copied back). */
typedef struct {
  const sas_bf16* q;   /* [B, Hq, N, d] */
  const sas_bf16* k;   /* [B, Hkv, N, d] */
  const sas_bf16* v;   /* [B, Hkv, N, d] */
  const float* s;      /* [B, Hkv, NQB, NKB] */
  const sas_bf16* dO;  /* [B, Hq, N, d] */
  sas_bf16* o;         /* [B, Hq, N, d] */
  float* lse_o;        /* [B, Hq, N] or NULL */
  sas_bf16* dq;        /* [B, Hq, N, d] */
  sas_bf16* dk;        /* [B, Hkv, N, d] */
  sas_bf16* dv;        /* [B, Hkv, N, d] */
  float* ds;           /* [B, Hkv, NQB, NKB] or NULL */
} sas_host_step;

/* One set of caller-owned device buffers for a step, with the layouts of the
 * host buffers, plus idx int32 [B, Hkv, NQB, K], lse_s fp32 [B, Hkv, NQB], and
 * the backward workspace (at least sas_bwd_workspace_size_min bytes, 256-byte
 * aligned; sas_bwd_workspace_size bytes select the faster backward). ds
 * is required under every gate mode but SAS_GATE_NONE. */
typedef struct {
  sas_bf16 *q, *k, *v, *dO, *o, *dq, *dk, *dv;
  float *s, *lse_s, *lse_o, *ds;
  int32_t* idx;
  void* ws;
  size_t ws_bytes;
} sas_device_slot;

/* Runs n_steps training steps (select + LSE, forward, backward with ds), step
 * i on device slot i % 2 (slots[0..1]; one slot is enough when n_steps = 1).
 * Step i's inputs are copied from steps[i] to the slot, its kernels run on
 * `stream`, and its outputs are copied back to steps[i]. The upload of step
 * i + 1 and the download of step i − 1 run on two internal copy streams while
 * step i's kernels run. The call is asynchronous: when `stream` has completed,
 * every step's outputs are in host memory. Host buffers may be shared between
 * steps (the copies of one direction run in step order), but a step's host
 * outputs must not be read before `stream` completes.
 * Errors: the argument checks of sas_fwd and sas_bwd for every slot and step,
 * before anything is enqueued (SAS_ERR_INVALID_ARG, SAS_ERR_WORKSPACE);
 * SAS_ERR_CUDA if a copy or launch cannot be enqueued. After such an error
 * the caller's stream still waits for every copy already enqueued, so buffers
 * may be released once it completes. */
SAS_API sas_status sas_train_steps_host(const sas_params* p, int n_steps, const sas_host_step* steps,
                                        const sas_device_slot* slots, void* stream);

/* ---------------------------------------------------------------------------
 * Diagnostics
 * ------------------------------------------------------------------------- */

/* Launches one thread that waits, through the same bounded wait as the
 * tcgen05 kernels, on an mbarrier that nothing completes. After about one
 * second of GPU clock cycles the wait gives up and raises SAS_ERR_TIMEOUT in
 * the device error word (read it with sas_get_device_error). It lets a caller
 * check the timeout path and that the context stays usable afterwards; nothing
 * faults or hangs. Asynchronous on `stream`. */
SAS_API sas_status sas_selftest_wait_timeout(void* stream);

/* Synchronises `stream`, then reads and clears the device error word of the
 * current device. *code is SAS_OK when no kernel raised an error since the
 * last read, else the first sas_status a kernel raised (SAS_ERR_TIMEOUT or
 * SAS_ERR_DEVICE_INDEX). The word is one per device and shared by every
 * caller of the library in the process: a kernel of any caller may have
 * raised it, and this read clears it for all of them. */
SAS_API sas_status sas_get_device_error(void* stream, int* code);

/* Static, human-readable name of a status code. */
SAS_API const char* sas_status_string(sas_status status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
SAS_API int sas_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SAS_H_ */
