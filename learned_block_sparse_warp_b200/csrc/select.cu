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
// Decode rows of up to 2048 blocks take one CTA each; longer decode rows go to
// the cluster radix select of score.cu.
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

// Register-resident variant for rows of at most 32·R scores: lane j holds
// blocks j, j + 32, ... as order keys shifted up by one, so an empty slot (key
// 0) never counts against a threshold. The search stops as soon as a
// threshold isolates exactly n blocks.
template <int R>
__device__ void select_row_reg(const float* __restrict__ row, int t, int K, int32_t* __restrict__ idx,
                               float* __restrict__ lse) {
  const int lane = threadIdx.x & 31;
  uint32_t key[R];
  float mx = -INFINITY;
#pragma unroll
  for (int j = 0; j < R; ++j) {
    const int m = lane + 32 * j;
    const float f = (m < t) ? __ldg(row + m) : -INFINITY;
    key[j] = (m < t) ? score_key(f) + 1u : 0u;
    mx = fmaxf(mx, f);
  }
  if (lse != nullptr) {
    mx = warp_max(mx);
    float sum = 0.f;
    if (mx != -INFINITY) {
#pragma unroll
      for (int j = 0; j < R; ++j) {
        const int m = lane + 32 * j;
        if (m < t) sum += expf(__ldg(row + m) - mx);
      }
    }
    sum = warp_sum(sum);
    if (lane == 0) *lse = (t == 0 || mx == -INFINITY) ? -INFINITY : mx + logf(sum);
  }
  if (idx == nullptr) return;
  const int n = min(K, t);
  uint32_t thr = 1u;  // every filled slot has key >= 1
  bool exact = (n == t);
  int need_eq = 0;
  if (!exact) {
    uint32_t acc = 0u;
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = acc | (1u << bit);
      int c = 0;
#pragma unroll
      for (int j = 0; j < R; ++j) c += (key[j] >= cand) ? 1 : 0;
      c = warp_isum(c);
      if (c >= n) acc = cand;
      if (c == n) {  // exactly n keys at or above cand: take them all
        exact = true;
        break;
      }
    }
    thr = acc;
    if (!exact) {
      int gt = 0;
#pragma unroll
      for (int j = 0; j < R; ++j) gt += (key[j] > thr) ? 1 : 0;
      need_eq = n - warp_isum(gt);
    }
  }
  int written = 0, eq_seen = 0;
#pragma unroll
  for (int j = 0; j < R; ++j) {
    if (32 * j >= t) break;
    const uint32_t k = key[j];
    const bool eq = !exact && k == thr;
    const unsigned eq_mask = __ballot_sync(0xffffffffu, eq);
    const int eq_rank = eq_seen + __popc(eq_mask & ((1u << lane) - 1u));
    const bool take = exact ? (k >= thr) : (k > thr || (eq && eq_rank < need_eq));
    const unsigned take_mask = __ballot_sync(0xffffffffu, take);
    if (take) idx[written + __popc(take_mask & ((1u << lane) - 1u))] = lane + 32 * j;
    written += __popc(take_mask);
    eq_seen += __popc(eq_mask);
  }
  for (int k = written + lane; k < K; k += 32) idx[k] = -1;
}

template <int R>
__device__ __forceinline__ void select_any(const float* row, int t, int K, int32_t* idx, float* lse) {
  if (R > 0) select_row_reg<(R > 0 ? R : 1)>(row, t, K, idx, lse);
  else select_row(row, t, K, idx, lse);
}

// Prefill: rows are (b, h, t) with t < NQB; row t reads s[b, h, t, 0..t).
template <int R>
__global__ void __launch_bounds__(256) select_prefill_kernel(const float* __restrict__ s, int rows, int NB, int K,
                                                             int32_t* __restrict__ idx, float* __restrict__ lse) {
  const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= rows) return;
  const int t = r % NB;
  select_any<R>(s + size_t(r) * NB, t, K, idx ? idx + size_t(r) * K : nullptr, lse ? lse + r : nullptr);
}

// Decode: rows are (b, h); the history of sequence b is blocks 0..c-1 with
// c = (cache_len[b] - 1) / 64.
template <int R>
__global__ void __launch_bounds__(256) select_decode_kernel(const float* __restrict__ s,
                                                            const int32_t* __restrict__ cache_len, int B, int Hkv,
                                                            int NB, int K, int32_t* __restrict__ idx,
                                                            float* __restrict__ lse, int* err) {
  griddep_wait();  // s and cache_len may come from the work just before this launch
  griddep_launch_dependents();
  const int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (r >= B * Hkv) return;
  const int b = r / Hkv;
  const int L = cache_len[b];
  int c = (L - 1) / kBlock;
  if (L < 1 || L > NB * kBlock) {
    if ((threadIdx.x & 31) == 0) raise_error(err, SAS_ERR_DEVICE_INDEX);
    c = 0;
  }
  select_any<R>(s + size_t(r) * NB, c, K, idx ? idx + size_t(r) * K : nullptr, lse ? lse + r : nullptr);
}

// One CTA of 256 threads per row, for few long rows (decode). Thread i holds
// blocks i, i + 256, ... as shifted order keys in registers. Each threshold
// candidate costs one __syncthreads_count per register slot, and the chosen
// blocks are written in ascending order with block-wide ballot scans.
constexpr int kRowThreads = 256;
constexpr int kRowSlots = 8;  // rows of up to 2048 history blocks

__device__ __forceinline__ int block_excl_scan(bool flag, int* warp_tot, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned m = __ballot_sync(0xffffffffu, flag);
  if (lane == 0) warp_tot[warp] = __popc(m);
  __syncthreads();
  int before = 0;
  total = 0;
#pragma unroll
  for (int w = 0; w < kRowThreads / 32; ++w) {
    const int c = warp_tot[w];
    before += (w < warp) ? c : 0;
    total += c;
  }
  __syncthreads();
  return before + __popc(m & ((1u << lane) - 1u));
}

__global__ void __launch_bounds__(kRowThreads) select_decode_cta_kernel(const float* __restrict__ s,
                                                                       const int32_t* __restrict__ cache_len,
                                                                       int B, int Hkv, int NB, int K,
                                                                       int32_t* __restrict__ idx,
                                                                       float* __restrict__ lse, int* err) {
  __shared__ int warp_tot[kRowThreads / 32];
  __shared__ float red[kRowThreads / 32];
  griddep_wait();  // s and cache_len may come from the work just before this launch
  griddep_launch_dependents();
  const int r = blockIdx.x;
  const int b = r / Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* row = s + size_t(r) * NB;
  // the whole row is read while cache_len is still in flight, then masked to the history
  float f[kRowSlots];
#pragma unroll
  for (int v = 0; v < kRowSlots; ++v) {
    const int m = tid + kRowThreads * v;
    f[v] = (m < NB) ? __ldg(row + m) : -INFINITY;
  }
  const int L = cache_len[b];
  int t = (L - 1) / kBlock;
  if (L < 1 || L > NB * kBlock) {
    if (tid == 0) raise_error(err, SAS_ERR_DEVICE_INDEX);
    t = 0;
  }
  uint32_t key[kRowSlots];
  float mx = -INFINITY;
#pragma unroll
  for (int v = 0; v < kRowSlots; ++v) {
    const int m = tid + kRowThreads * v;
    if (m >= t) f[v] = -INFINITY;
    key[v] = (m < t) ? score_key(f[v]) + 1u : 0u;
    mx = fmaxf(mx, f[v]);
  }
  if (lse != nullptr) {
    mx = warp_max(mx);
    if (lane == 0) red[warp] = mx;
    __syncthreads();
    mx = red[0];
#pragma unroll
    for (int w = 1; w < kRowThreads / 32; ++w) mx = fmaxf(mx, red[w]);
    __syncthreads();
    float sum = 0.f;
    if (mx != -INFINITY) {
#pragma unroll
      for (int v = 0; v < kRowSlots; ++v)
        if (tid + kRowThreads * v < t) sum += expf(f[v] - mx);
    }
    sum = warp_sum(sum);
    if (lane == 0) red[warp] = sum;
    __syncthreads();
    if (tid == 0) {
      float tot = 0.f;
      for (int w = 0; w < kRowThreads / 32; ++w) tot += red[w];
      lse[r] = (t == 0 || mx == -INFINITY) ? -INFINITY : mx + logf(tot);
    }
  }
  if (idx == nullptr) return;
  int32_t* out = idx + size_t(r) * K;
  const int n = min(K, t);
  const int slots = (t + kRowThreads - 1) / kRowThreads;  // uniform
  uint32_t thr = 1u;
  bool exact = (n == t);
  int need_eq = 0;
  if (!exact) {
    uint32_t acc = 0u;
    for (int bit = 31; bit >= 0; --bit) {
      const uint32_t cand = acc | (1u << bit);
      int c = 0;
#pragma unroll
      for (int v = 0; v < kRowSlots; ++v)
        if (v < slots) c += __syncthreads_count(key[v] >= cand);  // slots is uniform over the block
      if (c >= n) acc = cand;
      if (c == n) {
        exact = true;
        break;
      }
    }
    thr = acc;
    if (!exact) {
      int gt = 0;
#pragma unroll
      for (int v = 0; v < kRowSlots; ++v)
        if (v < slots) gt += __syncthreads_count(key[v] > thr);
      need_eq = n - gt;
    }
  }
  // ascending order: slot-major, then thread
  int written = 0, eq_seen = 0;
#pragma unroll
  for (int v = 0; v < kRowSlots; ++v) {
    if (v >= slots) break;
    const uint32_t k = key[v];
    const bool eq = !exact && k == thr;
    int eq_tot = 0;
    const int eq_rank = eq_seen + block_excl_scan(eq, warp_tot, eq_tot);
    const bool take = exact ? (k >= thr) : (k > thr || (eq && eq_rank < need_eq));
    int take_tot = 0;
    const int pos = written + block_excl_scan(take, warp_tot, take_tot);
    if (take) out[pos] = tid + kRowThreads * v;
    written += take_tot;
    eq_seen += eq_tot;
  }
  for (int k = written + tid; k < K; k += kRowThreads) out[k] = -1;
}

template <int R>
static void launch_select_r(const Shape& sh, const float* s, const int32_t* cache_len, int32_t* idx, float* lse,
                            int* err, cudaStream_t st) {
  const int warps = 8;
  if (cache_len == nullptr) {
    const int rows = sh.B * sh.Hkv * sh.NB;
    select_prefill_kernel<R><<<(rows + warps - 1) / warps, warps * 32, 0, st>>>(s, rows, sh.NB, sh.K, idx, lse);
  } else if (sh.NB <= kRowThreads * kRowSlots) {  // decode: one CTA per (sequence, KV head)
    launch_pdl(select_decode_cta_kernel, dim3(sh.B * sh.Hkv), dim3(kRowThreads), 0, st, s, cache_len, sh.B, sh.Hkv,
               sh.NB, sh.K, idx, lse, err);
  } else {
    const int rows = sh.B * sh.Hkv;
    launch_pdl(select_decode_kernel<R>, dim3((rows + warps - 1) / warps), dim3(warps * 32), 0, st, s, cache_len, sh.B,
               sh.Hkv, sh.NB, sh.K, idx, lse, err);
  }
}

bool scored_rows_fit(int NB);
cudaError_t launch_select_cluster(const Shape& sh, const float* s, const int32_t* cache_len, int32_t* idx,
                                  float* lse, int* err, cudaStream_t st);

cudaError_t launch_select(const Shape& sh, const float* s, const int32_t* cache_len, int32_t* idx, float* lse,
                          int* err, cudaStream_t st) {
  // decode rows past 2048 blocks: a radix select over a cluster of CTAs per row
  if (cache_len != nullptr && sh.NB > kRowThreads * kRowSlots && scored_rows_fit(sh.NB))
    return launch_select_cluster(sh, s, cache_len, idx, lse, err, st);
  // rows hold at most NB - 1 history scores
  if (sh.NB <= 4 * 32) launch_select_r<4>(sh, s, cache_len, idx, lse, err, st);
  else if (sh.NB <= 16 * 32) launch_select_r<16>(sh, s, cache_len, idx, lse, err, st);
  else if (sh.NB <= 64 * 32) launch_select_r<64>(sh, s, cache_len, idx, lse, err, st);
  else launch_select_r<0>(sh, s, cache_len, idx, lse, err, st);
  return cudaGetLastError();
}

}  // namespace sas
