// Top-K history-block selection and gate normaliser LSE(s).
//
// SAS explainer (ta-paperlens), section 前提: the selector's score vector s
// picks the K highest-scoring history blocks; their union with the current
// block is the attended set S. SAS summary (onedev.kr), section 무엇과 다른가:
// the gate is g = softmax(s), so log g_m = s_m − LSE(s).
//
// One warp owns one row of scores (one query block of one KV head, or one
// decode sequence of one KV head). It finds the n-th largest score key by a
// 32-step bitwise search on an order-preserving integer key, then takes ties
// at the threshold from the lowest block index, then writes the chosen blocks
// in ascending order with ballots. The row stays in L1 across the passes.
// Every selected set is exact, so the result matches a full sort bit for bit.
#include "common.cuh"

namespace sas {

// Counts keys >= thr in row[0..n). The result is the same on every lane.
__device__ __forceinline__ int count_ge(const float* __restrict__ row, int n, uint32_t thr) {
  int c = 0;
  for (int m = threadIdx.x & 31; m < n; m += 32) c += (score_key(__ldg(row + m)) >= thr) ? 1 : 0;
  return warp_isum(c);
}

// One warp: selection (idx != nullptr) and/or LSE (lse != nullptr) of row[0..t).
__device__ void select_row(const float* __restrict__ row, int t, int K, int32_t* __restrict__ idx,
                           float* __restrict__ lse) {
  const int lane = threadIdx.x & 31;
  if (lse != nullptr) {
    float mx = -INFINITY;
    for (int m = lane; m < t; m += 32) mx = fmaxf(mx, __ldg(row + m));
    mx = warp_max(mx);
    float sum = 0.f;
    if (mx != -INFINITY) {
      for (int m = lane; m < t; m += 32) sum += expf(__ldg(row + m) - mx);
    }
    sum = warp_sum(sum);
    if (lane == 0) *lse = (t == 0 || mx == -INFINITY) ? -INFINITY : mx + logf(sum);
  }
  if (idx == nullptr) return;
  const int n = min(K, t);
  uint32_t thr = 0;  // every key >= 0: take all when n == t
  int need_eq = 0x7fffffff;
  if (n < t) {
    // largest thr with count(key >= thr) >= n is the n-th largest key
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = thr | (1u << bit);
      if (count_ge(row, t, cand) >= n) thr = cand;
    }
    const int gt = (thr == 0xffffffffu) ? 0 : count_ge(row, t, thr + 1);
    need_eq = n - gt;  // ties at the threshold, lowest block index first
  }
  int written = 0, eq_seen = 0;
  for (int base = 0; base < t; base += 32) {
    const int m = base + lane;
    const uint32_t key = (m < t) ? score_key(__ldg(row + m)) : 0u;
    const bool valid = m < t;
    const bool eq = valid && key == thr && n < t;
    const unsigned eq_mask = __ballot_sync(0xffffffffu, eq);
    const int eq_rank = eq_seen + __popc(eq_mask & ((1u << lane) - 1u));
    const bool take = valid && ((n == t) || key > thr || (eq && eq_rank < need_eq));
    const unsigned take_mask = __ballot_sync(0xffffffffu, take);
    if (take) idx[written + __popc(take_mask & ((1u << lane) - 1u))] = m;
    written += __popc(take_mask);
    eq_seen += __popc(eq_mask);
  }
  for (int k = written + lane; k < K; k += 32) idx[k] = -1;
}

// Prefill: rows are (b, h, t) with t < NQB; row t reads s[b, h, t, 0..t).
__global__ void __launch_bounds__(256) select_prefill_kernel(const float* __restrict__ s, int rows, int NB, int K,
                                                             int32_t* __restrict__ idx, float* __restrict__ lse) {
  const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= rows) return;
  const int t = r % NB;
  select_row(s + size_t(r) * NB, t, K, idx ? idx + size_t(r) * K : nullptr, lse ? lse + r : nullptr);
}

// Decode: rows are (b, h); the history of sequence b is blocks 0..c-1 with
// c = (cache_len[b] - 1) / 64.
__global__ void __launch_bounds__(256) select_decode_kernel(const float* __restrict__ s,
                                                            const int32_t* __restrict__ cache_len, int B, int Hkv,
                                                            int NB, int K, int32_t* __restrict__ idx,
                                                            float* __restrict__ lse, int* err) {
  const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= B * Hkv) return;
  const int b = r / Hkv;
  const int L = cache_len[b];
  int c = (L - 1) / kBlock;
  if (L < 1 || L > NB * kBlock) {
    if ((threadIdx.x & 31) == 0) raise_error(err, SAS_ERR_DEVICE_INDEX);
    c = 0;
  }
  select_row(s + size_t(r) * NB, c, K, idx ? idx + size_t(r) * K : nullptr, lse ? lse + r : nullptr);
}

cudaError_t launch_select(const Shape& sh, const float* s, const int32_t* cache_len, int32_t* idx, float* lse,
                          int* err, cudaStream_t st) {
  const int warps = 8;
  if (cache_len == nullptr) {
    const int rows = sh.B * sh.Hkv * sh.NB;
    select_prefill_kernel<<<(rows + warps - 1) / warps, warps * 32, 0, st>>>(s, rows, sh.NB, sh.K, idx, lse);
  } else {
    const int rows = sh.B * sh.Hkv;
    select_decode_kernel<<<(rows + warps - 1) / warps, warps * 32, 0, st>>>(s, cache_len, sh.B, sh.Hkv, sh.NB, sh.K,
                                                                            idx, lse, err);
  }
  return cudaGetLastError();
}

}  // namespace sas
