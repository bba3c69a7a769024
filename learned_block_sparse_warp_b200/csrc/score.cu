// Selector scoring fused with Top-K for long decode caches.
//
// SAS summary (onedev.kr), section 전제와 한계: in decode the attention over the
// selected blocks costs the same at any context length, while the selector's
// scoring and the Top-K ranking grow with it; at 512K tokens the selection is
// most of the step. PBS (gist.science, "Sparser Block-Sparse Attention via
// Token Permutation"), section 4: block importance from mean-pooled keys.
//
// The selector score of history block m for a new token is
//   s_m = scale · ⟨q̄, k̄_m⟩,
// with k̄_m the mean of block m's 64 keys and q̄ the mean of the token's query
// vectors over the KV head's group (the learned selector with identity
// projections; it equals the mean of the token-level logits over the block
// and the group).
//
// block_mean_keys_kernel keeps k̄ as a bf16 side cache, 1/64 the size of the K
// cache. One warp sums one block's keys in fp32 and rounds the mean to bf16
// once. The whole cache is summarised at once after a prefill. During decode
// only the block that the newest token completed is.
//
// select_scored_kernel does one (sequence, KV head) row per thread-block
// cluster of C CTAs. CTA r streams a contiguous slice of the row's k̄ from HBM
// once with 16-byte loads and keeps its scores in shared memory (they also go
// to s, which the decode kernel reads for the gate). The cluster then finds
// LSE(s), and the n-th largest score key by an 8-bit radix select over all
// slices. Each pass's 256-bin histograms are summed through distributed shared
// memory. Ties at the threshold go to the lower block index, which is the
// lower-ranked CTA's slice first, and the chosen blocks are written in
// ascending order. The selected set is exact: it is the one a full sort of the
// kernel's scores picks.
//
// The same kernel with D = 0 reads the scores from s instead of computing
// them. The decode form of sas_topk_select uses it for rows past 2048 blocks,
// where one CTA or warp per row would walk the row 32 times.
#include <cooperative_groups.h>

#include <atomic>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace sas {

namespace ssc {
constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 256;            // 8-bit digits: four passes over a 32-bit key
constexpr int kMaxCluster = 8;        // portable cluster size
constexpr int kUnroll = 8;            // 16-byte loads in flight per lane
constexpr int kMinSlice = 64;         // blocks per CTA below which a row is not split further
constexpr int kMaxSlice = 53248;      // fp32 scores per CTA: 208 KB of shared memory
static_assert(kThreads >= kBins, "one thread per histogram bin");
}  // namespace ssc

struct ScoredSelectArgs {
  const uint16_t* q;      // [B, Hq, d] bf16
  const uint16_t* kmean;  // [B, Hkv, NB, d] bf16
  const int32_t* cache_len;
  float* s;               // [B, Hkv, NB]: entries m < c written (D > 0) or read (D = 0)
  int32_t* idx;           // [B, Hkv, K], or null for LSE(s) alone
  float* lse;             // [B, Hkv] or null
  int* err;
  int Hq, Hkv, G, NB, K;
  float qscale;           // softmax scale / G
};

// Values each CTA publishes to the rest of its cluster.
struct ClusterXch {
  float mx, sum;
  int gt, eq;
};

// Dot product of 8 bf16 (one 16-byte load) with 8 fp32.
__device__ __forceinline__ float dot8(const uint4& v, const float* w) {
  const uint32_t x[4] = {v.x, v.y, v.z, v.w};
  float acc = 0.f;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    acc = fmaf(__uint_as_float(x[j] << 16), w[2 * j], acc);
    acc = fmaf(__uint_as_float(x[j] & 0xffff0000u), w[2 * j + 1], acc);
  }
  return acc;
}

__device__ __forceinline__ float cta_max(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_max(v);
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int w = 1; w < ssc::kWarps; ++w) r = fmaxf(r, red[w]);
  __syncthreads();
  return r;
}

__device__ __forceinline__ float cta_sum(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_sum(v);
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = 0.f;
#pragma unroll
  for (int w = 0; w < ssc::kWarps; ++w) r += red[w];
  __syncthreads();
  return r;
}

__device__ __forceinline__ int cta_isum(int v, int* wtot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = warp_isum(v);
  if (lane == 0) wtot[warp] = v;
  __syncthreads();
  int r = 0;
#pragma unroll
  for (int w = 0; w < ssc::kWarps; ++w) r += wtot[w];
  __syncthreads();
  return r;
}

// Exclusive prefix count of `flag` over the CTA's threads in thread order;
// `total` receives the CTA-wide count.
__device__ __forceinline__ int cta_excl_scan(bool flag, int* wtot, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned m = __ballot_sync(0xffffffffu, flag);
  if (lane == 0) wtot[warp] = __popc(m);
  __syncthreads();
  int before = 0;
  total = 0;
#pragma unroll
  for (int w = 0; w < ssc::kWarps; ++w) {
    const int c = wtot[w];
    before += (w < warp) ? c : 0;
    total += c;
  }
  __syncthreads();
  return before + __popc(m & ((1u << lane) - 1u));
}

// Inclusive prefix sum of v over threads 0..kBins-1 (eight warps). Threads
// past kBins take part in the barriers and get 0.
__device__ __forceinline__ uint32_t bins_incl_scan(uint32_t v, uint32_t* wsum) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += u;
  }
  if (lane == 31 && warp < ssc::kBins / 32) wsum[warp] = v;
  __syncthreads();
  uint32_t before = 0;
  for (int w = 0; w < warp && w < ssc::kBins / 32; ++w) before += wsum[w];
  __syncthreads();
  return threadIdx.x < ssc::kBins ? v + before : 0u;
}

// D = 64 or 128: scores from q and k̄; D = 0: scores read from s.
template <int D>
__global__ void __launch_bounds__(ssc::kThreads) select_scored_kernel(ScoredSelectArgs a) {
  extern __shared__ float sc[];  // this CTA's slice of the row's scores
  __shared__ float qbar[D > 0 ? D : 1];
  __shared__ uint32_t hist[2][ssc::kBins];
  __shared__ float red[ssc::kWarps];
  __shared__ int wtot[ssc::kWarps];
  __shared__ uint32_t wsum[ssc::kBins / 32];
  __shared__ uint32_t pick[3];  // digit, keys above it, keys at it
  __shared__ ClusterXch xch;

  cg::cluster_group cluster = cg::this_cluster();
  const int C = int(cluster.num_blocks());
  const int rank = int(cluster.block_rank());
  const int row = blockIdx.x / C;  // (b, h)
  const int b = row / a.Hkv, h = row - b * a.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  griddep_wait();  // q, k̄ (or s) and cache_len may come from the work just before this launch
  griddep_launch_dependents();
  const int L = a.cache_len[b];
  int c = (L - 1) / kBlock;
  if (L < 1 || L > a.NB * kBlock) {
    if (tid == 0 && rank == 0) raise_error(a.err, SAS_ERR_DEVICE_INDEX);
    c = 0;
  }
  const int per = (c + C - 1) / C;
  const int m0 = min(c, rank * per), m1 = min(c, m0 + per), n_loc = m1 - m0;

  if constexpr (D == 0) {  // the given scores of blocks m0..m1-1
    const float* srow = a.s + size_t(row) * a.NB + m0;
    for (int i = tid; i < n_loc; i += ssc::kThreads) sc[i] = __ldg(srow + i);
  } else {
  for (int i = tid; i < D; i += ssc::kThreads) {
    const uint16_t* qp = a.q + (size_t(b) * a.Hq + size_t(h) * a.G) * D + i;
    float acc = 0.f;
    for (int g = 0; g < a.G; ++g) acc += bf16_to_f32(qp[size_t(g) * D]);
    qbar[i] = acc * a.qscale;
  }
  __syncthreads();

  // ---- scores of blocks m0..m1-1: LPB lanes per block, 8 dims per lane ----
  {
    constexpr int LPB = D / 8, BPW = 32 / LPB, kStep = ssc::kWarps * BPW;
    const int sub = lane % LPB, grp = lane / LPB;
    float w[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) w[j] = qbar[sub * 8 + j];
    const uint16_t* kb = a.kmean + size_t(row) * a.NB * D + sub * 8;
    float* srow = a.s + size_t(row) * a.NB;
    for (int wb = m0 + warp * BPW; wb < m1; wb += kStep * ssc::kUnroll) {  // warp-uniform bounds
      uint4 v[ssc::kUnroll];
#pragma unroll
      for (int u = 0; u < ssc::kUnroll; ++u) {
        const int m = wb + grp + u * kStep;
        v[u] = m < m1 ? __ldg(reinterpret_cast<const uint4*>(kb + size_t(m) * D)) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < ssc::kUnroll; ++u) {
        const int m = wb + grp + u * kStep;
        float d = dot8(v[u], w);
#pragma unroll
        for (int o = LPB / 2; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
        if (sub == 0 && m < m1) {
          sc[m - m0] = d;
          srow[m] = d;
        }
      }
    }
  }
  }  // scores computed
  __syncthreads();

  // ---- LSE(s) over the whole row ----
  if (a.lse != nullptr) {
    float mx = -INFINITY;
    for (int i = tid; i < n_loc; i += ssc::kThreads) mx = fmaxf(mx, sc[i]);
    mx = cta_max(mx, red);
    if (tid == 0) xch.mx = mx;
    cluster.sync();
    float gmx = -INFINITY;
    for (int r = 0; r < C; ++r) gmx = fmaxf(gmx, cluster.map_shared_rank(&xch, r)->mx);
    float sum = 0.f;
    if (gmx != -INFINITY)
      for (int i = tid; i < n_loc; i += ssc::kThreads) sum += expf(sc[i] - gmx);
    sum = cta_sum(sum, red);
    if (tid == 0) xch.sum = sum;
    cluster.sync();
    if (rank == 0 && tid == 0) {
      float tot = 0.f;
      for (int r = 0; r < C; ++r) tot += cluster.map_shared_rank(&xch, r)->sum;
      a.lse[row] = (c == 0 || gmx == -INFINITY) ? -INFINITY : gmx + logf(tot);
    }
  }

  // ---- Top-K: n = min(K, c) blocks, ascending ----
  const int n = min(a.K, c);
  int32_t* irow = a.idx + size_t(row) * a.K;
  if (a.idx == nullptr) {
    // LSE(s) alone
  } else if (n == c) {
    for (int m = m0 + tid; m < m1; m += ssc::kThreads) irow[m] = m;
  } else {
    // Radix select of the n-th largest key, 8 bits a pass from the top. After
    // a pass, `prefix` holds the chosen digits and `need` how many keys under
    // that prefix are still to be taken. When the keys under the prefix are
    // exactly `need`, every key >= prefix is taken and the search stops.
    uint32_t prefix = 0u, need = uint32_t(n);
    bool exact = false;
    int shift = 24;
    for (int pass = 0; pass < 4; ++pass, shift -= 8) {
      uint32_t* hs = hist[pass & 1];
      if (tid < ssc::kBins) hs[tid] = 0u;
      __syncthreads();
      const uint32_t hi = pass == 0 ? 0u : (0xffffffffu << (shift + 8));
      for (int i = tid; i < n_loc; i += ssc::kThreads) {
        const uint32_t key = score_key(sc[i]);
        if ((key & hi) == prefix) atomicAdd(&hs[(key >> shift) & 0xffu], 1u);
      }
      cluster.sync();  // every slice's histogram of this pass is complete
      // thread t holds bin 255 - t: the scan runs from the largest digit down
      const int bin = ssc::kBins - 1 - tid;
      uint32_t v = 0u;
      if (tid < ssc::kBins)
        for (int r = 0; r < C; ++r) v += cluster.map_shared_rank(hs, r)[bin];
      const uint32_t incl = bins_incl_scan(v, wsum);
      if (tid < ssc::kBins && incl >= need && incl - v < need) {
        pick[0] = uint32_t(bin);
        pick[1] = incl - v;
        pick[2] = v;
      }
      __syncthreads();
      prefix |= pick[0] << shift;
      need -= pick[1];
      const uint32_t at = pick[2];
      // pick is next written after the next pass's cluster barrier, so no
      // thread can still be reading it then
      if (at == need) {
        exact = true;
        break;
      }
    }
    // exact: take every key >= prefix. Otherwise prefix is the threshold key:
    // take keys above it, and the first `need` keys equal to it.
    const uint32_t thr = prefix;
    int my_gt = 0, my_eq = 0;
    for (int i = tid; i < n_loc; i += ssc::kThreads) {
      const uint32_t key = score_key(sc[i]);
      my_gt += (exact ? key >= thr : key > thr) ? 1 : 0;
      my_eq += (!exact && key == thr) ? 1 : 0;
    }
    my_gt = cta_isum(my_gt, wtot);
    my_eq = cta_isum(my_eq, wtot);
    if (tid == 0) {
      xch.gt = my_gt;
      xch.eq = my_eq;
    }
    cluster.sync();
    int out_before = 0, eq_before = 0;
    for (int r = 0; r < rank; ++r) {
      const ClusterXch* x = cluster.map_shared_rank(&xch, r);
      out_before += x->gt + min(x->eq, max(0, int(need) - eq_before));
      eq_before += x->eq;
    }
    int written = 0, eq_seen = 0;
    for (int base = 0; base < n_loc; base += ssc::kThreads) {
      const int i = base + tid;
      const bool valid = i < n_loc;
      const uint32_t key = valid ? score_key(sc[i]) : 0u;
      const bool e = valid && !exact && key == thr;
      const bool g = valid && (exact ? key >= thr : key > thr);
      int e_tot = 0;
      const int e_rank = eq_before + eq_seen + cta_excl_scan(e, wtot, e_tot);
      const bool take = g || (e && e_rank < int(need));
      int t_tot = 0;
      const int pos = cta_excl_scan(take, wtot, t_tot);
      if (take) irow[out_before + written + pos] = m0 + i;
      written += t_tot;
      eq_seen += e_tot;
    }
  }
  if (rank == 0 && a.idx != nullptr)
    for (int k = n + tid; k < a.K; k += ssc::kThreads) irow[k] = -1;
  cluster.sync();  // no CTA leaves while another may still read its shared memory
}

// One warp per (row, block): the fp32 sum of the block's 64 keys, times 1/64,
// rounded to bf16. With cache_len, item (b, h) covers only the block that the
// newest token completed (cache_len[b] a multiple of 64), if any.
template <int D>
__global__ void __launch_bounds__(256) block_mean_keys_kernel(const uint16_t* __restrict__ k,
                                                              const int32_t* __restrict__ cache_len, int Hkv,
                                                              int NB, int n_items, uint16_t* __restrict__ kmean,
                                                              int* err) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int item = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (item >= n_items) return;
  int bh, m;
  if (cache_len == nullptr) {
    bh = item / NB;
    m = item - bh * NB;
  } else {
    bh = item;
    const int L = cache_len[bh / Hkv];
    if (L < 1 || L > NB * kBlock) {
      if (lane == 0) raise_error(err, SAS_ERR_DEVICE_INDEX);
      return;
    }
    if (L % kBlock != 0) return;
    m = L / kBlock - 1;
  }
  constexpr int LPR = D / 8, RPI = 32 / LPR, kIter = kBlock / RPI;  // lanes per row, rows per step
  const int sub = lane % LPR, r0 = lane / LPR;
  const uint16_t* src = k + (size_t(bh) * NB * kBlock + size_t(m) * kBlock + r0) * D + sub * 8;
  float acc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = 0.f;
#pragma unroll
  for (int it0 = 0; it0 < kIter; it0 += 8) {
    uint4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = __ldg(reinterpret_cast<const uint4*>(src + size_t(it0 + u) * RPI * D));
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const uint32_t x[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        acc[2 * j] += __uint_as_float(x[j] << 16);
        acc[2 * j + 1] += __uint_as_float(x[j] & 0xffff0000u);
      }
    }
  }
#pragma unroll
  for (int o = LPR; o < 32; o <<= 1)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], o);
  if (r0 == 0) {
    constexpr float kInv = 1.0f / kBlock;
    uint4 out;
    out.x = pack_bf16x2(acc[0] * kInv, acc[1] * kInv);
    out.y = pack_bf16x2(acc[2] * kInv, acc[3] * kInv);
    out.z = pack_bf16x2(acc[4] * kInv, acc[5] * kInv);
    out.w = pack_bf16x2(acc[6] * kInv, acc[7] * kInv);
    *reinterpret_cast<uint4*>(kmean + (size_t(bh) * NB + m) * D + sub * 8) = out;
  }
}

cudaError_t launch_block_mean_keys(const Shape& sh, const uint16_t* k, const int32_t* cache_len, uint16_t* kmean,
                                   int* err, cudaStream_t st) {
  const int n_items = cache_len == nullptr ? sh.B * sh.Hkv * sh.NB : sh.B * sh.Hkv;
  const dim3 grid((n_items + 7) / 8);
  if (sh.d == 128)
    return launch_pdl(block_mean_keys_kernel<128>, grid, dim3(256), 0, st, k, cache_len, sh.Hkv, sh.NB, n_items,
                      kmean, err);
  return launch_pdl(block_mean_keys_kernel<64>, grid, dim3(256), 0, st, k, cache_len, sh.Hkv, sh.NB, n_items, kmean,
                    err);
}

// Whether rows of NB blocks (at most NB - 1 history blocks) fit the largest
// cluster's shared memory.
bool scored_rows_fit(int NB) { return (NB - 1 + ssc::kMaxCluster - 1) / ssc::kMaxCluster <= ssc::kMaxSlice; }

// Cluster size for rows of NB blocks: doubled while the grid stays within one
// CTA per SM and each CTA keeps at least kMinSlice blocks, and further while a
// slice does not fit shared memory. 0 when no size fits.
int scored_cluster_size(int rows, int NB, int sms) {
  const int hist = NB - 1;
  int C = 1;
  while (C < ssc::kMaxCluster && rows * 2 * C <= sms && hist / (2 * C) >= ssc::kMinSlice) C *= 2;
  while (C < ssc::kMaxCluster && (hist + C - 1) / C > ssc::kMaxSlice) C *= 2;
  return (hist + C - 1) / C > ssc::kMaxSlice ? 0 : C;
}

// SM count of the current device, fetched once per device. Threads that race
// on the first fetch all store the same value.
static cudaError_t device_sm_count(int* out) {
  static std::atomic<int> sm_count[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  int n = sm_count[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if ((e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    sm_count[dev].store(n, std::memory_order_relaxed);
  }
  *out = n;
  return cudaSuccess;
}

template <int D>
static cudaError_t launch_scored_d(const ScoredSelectArgs& a, int rows, int C, cudaStream_t st) {
  const int slice = (a.NB - 1 + C - 1) / C;
  const size_t smem = size_t(slice > 0 ? slice : 1) * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(select_scored_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(rows * C);
  cfg.blockDim = dim3(ssc::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, select_scored_kernel<D>, a);
}

cudaError_t launch_select_scored(const Shape& sh, const uint16_t* q, const uint16_t* kmean,
                                 const int32_t* cache_len, float* s, int32_t* idx, float* lse, int* err,
                                 cudaStream_t st) {
  int sms = 0;
  cudaError_t e = device_sm_count(&sms);
  if (e != cudaSuccess) return e;
  const int rows = sh.B * sh.Hkv;
  const int C = scored_cluster_size(rows, sh.NB, sms);
  if (C == 0) return cudaErrorInvalidValue;  // the host entry rules this out first
  ScoredSelectArgs a{q, kmean, cache_len, s, idx, lse, err, sh.Hq, sh.Hkv, sh.G, sh.NB, sh.K,
                     sh.scale / float(sh.G)};
  if (sh.d == 128) return launch_scored_d<128>(a, rows, C, st);
  return launch_scored_d<64>(a, rows, C, st);
}

// The decode form of sas_topk_select on given scores, one cluster per row.
cudaError_t launch_select_cluster(const Shape& sh, const float* s, const int32_t* cache_len, int32_t* idx,
                                  float* lse, int* err, cudaStream_t st) {
  int sms = 0;
  cudaError_t e = device_sm_count(&sms);
  if (e != cudaSuccess) return e;
  const int rows = sh.B * sh.Hkv;
  const int C = scored_cluster_size(rows, sh.NB, sms);
  if (C == 0) return cudaErrorInvalidValue;
  ScoredSelectArgs a{nullptr, nullptr, cache_len, const_cast<float*>(s), idx, lse, err, sh.Hq, sh.Hkv, sh.G,
                     sh.NB, sh.K, 0.f};
  return launch_scored_d<0>(a, rows, C, st);
}

}  // namespace sas

// ---------------------------------------------------------------------------
// C ABI
// ---------------------------------------------------------------------------
namespace sas {
sas_status check_params(const sas_params* p, Shape* sh);
int* error_word();
}  // namespace sas

namespace {
bool ok16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool opt16(const void* p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
}  // namespace

extern "C" {

sas_status sas_block_mean_keys(const sas_params* p, const sas_bf16* k, const int32_t* cache_len, sas_bf16* kmean,
                               void* stream) {
  sas::Shape sh;
  sas_status r = sas::check_params(p, &sh);
  if (r != SAS_OK) return r;
  if (!ok16(k) || !ok16(kmean) || !opt16(cache_len)) return SAS_ERR_INVALID_ARG;
  int* err = sas::error_word();
  if (err == nullptr) return SAS_ERR_CUDA;
  return sas::launch_block_mean_keys(sh, k, cache_len, kmean, err, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SAS_OK
             : SAS_ERR_CUDA;
}

sas_status sas_decode_select_scored(const sas_params* p, const sas_bf16* q, const sas_bf16* kmean,
                                    const int32_t* cache_len, float* s, int32_t* idx, float* lse_s, void* stream) {
  sas::Shape sh;
  sas_status r = sas::check_params(p, &sh);
  if (r != SAS_OK) return r;
  if (!ok16(q) || !ok16(kmean) || !ok16(cache_len) || !ok16(s) || !ok16(idx) || !opt16(lse_s))
    return SAS_ERR_INVALID_ARG;
  if (!sas::scored_rows_fit(sh.NB)) return SAS_ERR_UNSUPPORTED;
  int* err = sas::error_word();
  if (err == nullptr) return SAS_ERR_CUDA;
  return sas::launch_select_scored(sh, q, kmean, cache_len, s, idx, lse_s, err,
                                   static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SAS_OK
             : SAS_ERR_CUDA;
}

}  // extern "C"
