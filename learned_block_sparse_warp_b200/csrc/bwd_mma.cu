// Backward of gated block-sparse attention: the small kernels around the
// tcgen05 passes, the workspace layout, and the launcher.
//
// SAS summary (onedev.kr), section 무엇과 다른가: with the gate inside the
// softmax the gate gradient is dg_m = Σ_i (p̃_i/g_m) dOᵀ(v_i − o), and
// g = softmax(s) chains it to the scores. Training uses "sparse scope":
// content gradients reach only the selected blocks. Per query row i and
// attended token j:
//   P_ij = exp(z_ij − L_i),  dP_ij = dO_i·v_j,  D_i = dO_i·o_i,
//   dZ_ij = P_ij (dP_ij − D_i),
//   dV_j += P_ij dO_i,  dK_j += scale·dZ_ij q_i,  dQ_i += scale·dZ_ij k_j,
//   dl[t, m] = Σ_{i∈t, heads} Σ_{j∈B_m} dZ_ij   (= g_m·dg_m),
//   ds[t, m] = dl[t, m]·[m∈I_t] − softmax(s_t)_m Σ_{m'∈I_t} dl[t, m'].
//
// Kernels, in launch order:
//   bwd_prep         D_i = rowsum(dO ∘ o)
//   revidx_count/scan/fill
//                    for every KV block j, the query blocks t > j that
//                    selected it, ascending in t, with j's slot in idx[t]
//                    and the block's log2 gate for t
//   the tcgen05 passes (bwd_sm100.cu): dK, dV, dl (and the dZ tiles), then dQ
//   bwd_ds_chain     ds from dl through the gate's activation
#include <algorithm>

#include "common.cuh"

namespace sas {

struct BwdWs {
  float* drow;     // [B, Hq, N]
  float* dl;       // [B, Hkv, NB, K]
  int* rev_cnt;    // [B, Hkv, NB]
  uint32_t* col_bits;  // [B, Hkv, NB, W]: bit t of block j's row is set when idx[t] holds j (NB <= kBitmapMaxNB)
  int* col_pre;        // [B, Hkv, NB, W]: set bits of block j's row in the words before w
  int* rev_off;    // [B, Hkv, NB + 1]
  int* rev_list;   // [B, Hkv, NB * K]: (t << kSlotBits) | slot
  float* rev_lam;  // [B, Hkv, NB * K]: log2-domain gate of each reverse-index entry
  uint16_t* dz;    // with spill: [B, Hkv, Σ_t (1 + min(K, t)), ceil(G/2)] tiles of 128 x 64 bf16
};

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Up to this many blocks the reverse index is built from a bitmap of which
// query blocks selected each block (two words of workspace per 32 blocks and
// block); longer rows test every (t, j) pair against the row's sorted list.
constexpr int kBitmapMaxNB = 4096;
static int bitmap_words(const Shape& sh) { return sh.NB <= kBitmapMaxNB ? (sh.NB + 31) / 32 : 0; }

long long bwd_dz_tiles(const Shape& sh);

// The stored-dZ backward needs one 16 KB tile per (query block, attended block,
// head pair); its tile index must fit a TMA coordinate.
bool bwd_can_spill(const Shape& sh) { return bwd_dz_tiles(sh) < (1LL << 31); }

size_t bwd_ws_layout(const Shape& sh, bool spill, void* base, BwdWs* ws) {
  const size_t bhq = size_t(sh.B) * sh.Hq, bhk = size_t(sh.B) * sh.Hkv;
  size_t off = 0;
  size_t o_dr = off;
  off = align256(off + bhq * sh.N * sizeof(float));
  size_t o_dl = off;
  off = align256(off + bhk * sh.NB * sh.K * sizeof(float));
  size_t o_cnt = off;
  off = align256(off + bhk * sh.NB * sizeof(int));
  size_t o_off = off;
  off = align256(off + bhk * (sh.NB + 1) * sizeof(int));
  size_t o_list = off;
  off = align256(off + bhk * sh.NB * sh.K * sizeof(int));
  size_t o_lam = off;
  off = align256(off + bhk * sh.NB * sh.K * sizeof(float));
  const size_t n_bits = bhk * sh.NB * size_t(bitmap_words(sh));
  size_t o_bits = off;
  off = align256(off + n_bits * sizeof(uint32_t));
  size_t o_pre = off;
  off = align256(off + n_bits * sizeof(int));
  size_t o_dz = off;
  if (spill) off = align256(off + size_t(bwd_dz_tiles(sh)) * 128 * 64 * sizeof(uint16_t));
  if (ws != nullptr) {
    char* p = static_cast<char*>(base);
    ws->drow = reinterpret_cast<float*>(p + o_dr);
    ws->dl = reinterpret_cast<float*>(p + o_dl);
    ws->rev_cnt = reinterpret_cast<int*>(p + o_cnt);
    ws->rev_off = reinterpret_cast<int*>(p + o_off);
    ws->rev_list = reinterpret_cast<int*>(p + o_list);
    ws->rev_lam = reinterpret_cast<float*>(p + o_lam);
    ws->col_bits = n_bits ? reinterpret_cast<uint32_t*>(p + o_bits) : nullptr;
    ws->col_pre = n_bits ? reinterpret_cast<int*>(p + o_pre) : nullptr;
    ws->dz = spill ? reinterpret_cast<uint16_t*>(p + o_dz) : nullptr;
  }
  return off;
}

// ---------------------------------------------------------------------------
// D_i = dO_i · o_i. HBM-bound: each thread reads 16-byte chunks of o and dO,
// a row is 256 (d = 128) or 128 bytes, so 16 or 8 lanes share a row and reduce
// with shuffles. Each thread keeps four rows' loads in flight.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const uint16_t* __restrict__ o, const uint16_t* __restrict__ dO,
                                                       size_t rows, float* __restrict__ drow) {
  constexpr int CPR = D / 8;     // 16-byte chunks per row
  constexpr int RPW = 32 / CPR;  // rows per warp and unroll step
  constexpr int U = 4;
  const int lane = threadIdx.x & 31;
  const int c = lane % CPR, sub = lane / CPR;
  const size_t warp_g = (size_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const size_t n_warps = (size_t(gridDim.x) * blockDim.x) >> 5;
  const uint4* o4 = reinterpret_cast<const uint4*>(o);
  const uint4* d4 = reinterpret_cast<const uint4*>(dO);
  for (size_t r0 = warp_g * RPW * U; r0 < rows; r0 += n_warps * RPW * U) {
    uint4 x[U], y[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const size_t r = r0 + u * RPW + sub;
      x[u] = r < rows ? __ldg(o4 + r * CPR + c) : make_uint4(0, 0, 0, 0);
      y[u] = r < rows ? __ldg(d4 + r * CPR + c) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint32_t xa[4] = {x[u].x, x[u].y, x[u].z, x[u].w}, ya[4] = {y[u].x, y[u].y, y[u].z, y[u].w};
      float acc = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        acc = fmaf(__uint_as_float(xa[k] << 16), __uint_as_float(ya[k] << 16), acc);
        acc = fmaf(__uint_as_float(xa[k] & 0xffff0000u), __uint_as_float(ya[k] & 0xffff0000u), acc);
      }
#pragma unroll
      for (int off = CPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      const size_t r = r0 + u * RPW + sub;
      if (c == 0 && r < rows) drow[r] = acc;
    }
  }
}

// ---------------------------------------------------------------------------
// Reverse index: which query blocks selected KV block j (ascending t)
// ---------------------------------------------------------------------------
// Slot of block j in the ascending list idx_row[0..n), or -1.
__device__ __forceinline__ int find_slot(const int32_t* __restrict__ idx_row, int n, int j) {
  int lo = 0, hi = n;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    const int m = idx_row[mid];
    if (m < j && m >= 0) lo = mid + 1;
    else hi = mid;
  }
  return (lo < n && idx_row[lo] == j) ? lo : -1;
}

__global__ void __launch_bounds__(256) revidx_count_kernel(const int32_t* __restrict__ idx, int nbh, int NB, int K,
                                                           int* __restrict__ cnt) {
  const int w = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (w >= nbh * NB) return;
  const int lane = threadIdx.x & 31;
  const int bh = w / NB, j = w % NB;
  int c = 0;
  for (int t = j + 1 + lane; t < NB; t += 32) {
    const int32_t* row = idx + (size_t(bh) * NB + t) * K;
    c += (find_slot(row, min(K, t), j) >= 0) ? 1 : 0;
  }
  c = warp_isum(c);
  if (lane == 0) cnt[w] = c;
}

__global__ void revidx_scan_kernel(const int* __restrict__ cnt, int NB, int* __restrict__ off) {
  const int bh = blockIdx.x;
  const int lane = threadIdx.x;
  const int* c = cnt + size_t(bh) * NB;
  int* o = off + size_t(bh) * (NB + 1);
  int run = 0;
  for (int base = 0; base < NB; base += 32) {
    const int j = base + lane;
    int v = (j < NB) ? c[j] : 0;
    int inc = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, inc, d);
      if (lane >= d) inc += u;
    }
    if (j < NB) o[j] = run + inc - v;
    run += __shfl_sync(0xffffffffu, inc, 31);
  }
  if (lane == 0) o[NB] = run;
}

__global__ void __launch_bounds__(256) revidx_fill_kernel(const int32_t* __restrict__ idx, int nbh, int NB, int K,
                                                          const int* __restrict__ off, int* __restrict__ list,
                                                          const float* __restrict__ s, const float* __restrict__ lse_s,
                                                          int gate, float* __restrict__ lam) {
  const int w = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (w >= nbh * NB) return;
  const int lane = threadIdx.x & 31;
  const int bh = w / NB, j = w % NB;
  int pos = off[size_t(bh) * (NB + 1) + j];
  int* out = list + size_t(bh) * NB * K;
  for (int base = j + 1; base < NB; base += 32) {
    const int t = base + lane;
    int slot = -1;
    if (t < NB) slot = find_slot(idx + (size_t(bh) * NB + t) * K, min(K, t), j);
    const unsigned mask = __ballot_sync(0xffffffffu, slot >= 0);
    if (slot >= 0) {
      const int at = pos + __popc(mask & ((1u << lane) - 1u));
      out[at] = (t << kSlotBits) | slot;
      if (lam != nullptr) {  // the gate of block j for query block t, log2 domain
        const size_t row = size_t(bh) * NB + t;
        lam[size_t(bh) * NB * K + at] =
            gate != SAS_GATE_NONE ? gate_lam2(gate, s[row * NB + j], lse_s != nullptr ? lse_s[row] : 0.f) : 0.f;
      }
    }
    pos += __popc(mask);
  }
}

// The same reverse index from a bitmap, with every step parallel over the
// selection's entries or the blocks:
//   mark     one thread per entry (b, h, t, s): j = idx[t][s] sets bit t of
//            block j's row (a zeroed [NB, W] bitmap per (b, h));
//   colscan  one warp per (b, h, j): the row's count of set bits, and per
//            word the set bits before it;
//   fill     one thread per entry: its place in j's list is j's offset plus
//            the set bits of j's row below t, and the entry is (t, s).
// The lists come out ascending in t, as from the pairwise kernels above.
__global__ void __launch_bounds__(256) revidx_mark_kernel(const int32_t* __restrict__ idx, int nbh, int NB, int K,
                                                         int W, uint32_t* __restrict__ bits) {
  const size_t e = size_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= size_t(nbh) * NB * K) return;
  const int s = int(e % K);
  const size_t row = e / K;  // (b, h, t)
  const int t = int(row % NB);
  if (s >= min(K, t)) return;
  const int j = idx[e];
  if (j < 0 || j >= t) return;
  const size_t bh = row / NB;
  atomicOr(bits + (bh * NB + j) * W + (t >> 5), 1u << (t & 31));
}

__global__ void __launch_bounds__(256) revidx_colscan_kernel(const uint32_t* __restrict__ bits, int rows, int W,
                                                            int* __restrict__ pre, int* __restrict__ cnt) {
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (r >= rows) return;
  const int lane = threadIdx.x & 31;
  int run = 0;
  for (int w0 = 0; w0 < W; w0 += 32) {
    const int w = w0 + lane;
    const int c = w < W ? __popc(bits[size_t(r) * W + w]) : 0;
    int incl = c;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += u;
    }
    if (w < W) pre[size_t(r) * W + w] = run + incl - c;
    run += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) cnt[r] = run;
}

__global__ void __launch_bounds__(256) revidx_fill_cols_kernel(const int32_t* __restrict__ idx, int nbh, int NB, int K,
                                                              int W, const uint32_t* __restrict__ bits,
                                                              const int* __restrict__ pre, const int* __restrict__ off,
                                                              int* __restrict__ list, const float* __restrict__ s,
                                                              const float* __restrict__ lse_s, int gate,
                                                              float* __restrict__ lam) {
  const size_t e = size_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (e >= size_t(nbh) * NB * K) return;
  const int slot = int(e % K);
  const size_t row = e / K;
  const int t = int(row % NB);
  if (slot >= min(K, t)) return;
  const int j = idx[e];
  if (j < 0 || j >= t) return;
  const size_t bh = row / NB;
  const size_t wi = (bh * NB + j) * W + (t >> 5);
  const int pos = off[bh * (NB + 1) + j] + pre[wi] + __popc(bits[wi] & ((1u << (t & 31)) - 1u));
  list[bh * NB * K + pos] = (t << kSlotBits) | slot;
  if (lam != nullptr)
    lam[bh * NB * K + pos] =
        gate != SAS_GATE_NONE ? gate_lam2(gate, s[row * NB + j], lse_s != nullptr ? lse_s[row] : 0.f) : 0.f;
}

// One warp per (b, h, t): ds[t, m] = dl[t, m]·[m∈I] − softmax(s_t)_m Σ dl.
__global__ void __launch_bounds__(256) bwd_ds_chain_kernel(const float* __restrict__ s, const float* __restrict__ lse_s,
                                                           const int32_t* __restrict__ idx,
                                                           const float* __restrict__ dl, int rows, int NB, int K,
                                                           int gate, float* __restrict__ ds) {
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (r >= rows) return;
  const int lane = threadIdx.x & 31;
  const int t = r % NB;
  float* dsr = ds + size_t(r) * NB;
  if (gate == SAS_GATE_NONE || t == 0) {
    for (int m = lane; m < NB; m += 32) dsr[m] = 0.f;
    return;
  }
  const int n = min(K, t);
  const int32_t* ir = idx + size_t(r) * K;
  const float* dlr = dl + size_t(r) * K;
  const float* sr = s + size_t(r) * NB;
  if (gate == SAS_GATE_LOG_SOFTMAX || gate == SAS_GATE_SOFTMAX_OUTSIDE) {  // every history block couples through LSE(s)
    float sum = 0.f;
    for (int kk = lane; kk < n; kk += 32) {
      const int m = ir[kk];
      if (m >= 0 && m < t) sum += dlr[kk];
    }
    sum = warp_sum(sum);
    const float lse = lse_s[r];
    for (int m = lane; m < NB; m += 32) dsr[m] = (m < t) ? -expf(sr[m] - lse) * sum : 0.f;
  } else {  // log σ(s) and the raw logit act on each selected block alone
    for (int m = lane; m < NB; m += 32) dsr[m] = 0.f;
  }
  __syncwarp();
  for (int kk = lane; kk < n; kk += 32) {
    const int m = ir[kk];
    if (m < 0 || m >= t) continue;
    float x = dlr[kk];
    if (gate == SAS_GATE_LOG_SIGMOID) x *= 1.f / (1.f + expf(sr[m]));  // d log σ(s) / ds = 1 − σ(s) = σ(−s)
    dsr[m] += x;
  }
}

// ---------------------------------------------------------------------------
// Host launcher
// ---------------------------------------------------------------------------
cudaError_t launch_bwd_passes_sm100(const Shape& sh, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                   const uint16_t* dO, const float* s, const int32_t* idx, const float* lse_s,
                                   const float* lse_o, const float* drow, const int* rev_off, const int* rev_list,
                                   const float* rev_lam, float* dl, uint16_t* dz, uint16_t* dq, uint16_t* dk,
                                   uint16_t* dv, int* err, cudaStream_t st);

template <int D>
static cudaError_t launch_bwd_d(const Shape& sh, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                const uint16_t* o, const uint16_t* dO, const float* s, const int32_t* idx,
                                const float* lse_s, const float* lse_o, uint16_t* dq, uint16_t* dk, uint16_t* dv,
                                float* ds, void* ws_base, bool spill, int* err, cudaStream_t st) {
  BwdWs ws;
  bwd_ws_layout(sh, spill, ws_base, &ws);
  const size_t rows_q = size_t(sh.B) * sh.Hq * sh.N;
  const int nbh = sh.B * sh.Hkv;
  cudaError_t e;
  if ((e = cudaMemsetAsync(ws.dl, 0, size_t(nbh) * sh.NB * sh.K * sizeof(float), st)) != cudaSuccess) return e;
  {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const size_t rows_per_cta = size_t(8) * (32 / (D / 8)) * 4;  // warps x rows per warp step x unroll
    const unsigned grid = unsigned(std::min<size_t>((rows_q + rows_per_cta - 1) / rows_per_cta, size_t(sms) * 8));
    bwd_prep_kernel<D><<<std::max(1u, grid), 256, 0, st>>>(o, dO, rows_q, ws.drow);
  }
  const int nw = nbh * sh.NB;
  const int W = bitmap_words(sh);
  if (W > 0) {
    const size_t n_ent = size_t(nw) * sh.K;
    const unsigned ent_blocks = unsigned((n_ent + 255) / 256);
    if ((e = cudaMemsetAsync(ws.col_bits, 0, size_t(nw) * W * sizeof(uint32_t), st)) != cudaSuccess) return e;
    revidx_mark_kernel<<<ent_blocks, 256, 0, st>>>(idx, nbh, sh.NB, sh.K, W, ws.col_bits);
    revidx_colscan_kernel<<<(nw + 7) / 8, 256, 0, st>>>(ws.col_bits, nw, W, ws.col_pre, ws.rev_cnt);
    revidx_scan_kernel<<<nbh, 32, 0, st>>>(ws.rev_cnt, sh.NB, ws.rev_off);
    revidx_fill_cols_kernel<<<ent_blocks, 256, 0, st>>>(idx, nbh, sh.NB, sh.K, W, ws.col_bits, ws.col_pre,
                                                        ws.rev_off, ws.rev_list, s, lse_s, sh.gate, ws.rev_lam);
  } else {
    revidx_count_kernel<<<(nw + 7) / 8, 256, 0, st>>>(idx, nbh, sh.NB, sh.K, ws.rev_cnt);
    revidx_scan_kernel<<<nbh, 32, 0, st>>>(ws.rev_cnt, sh.NB, ws.rev_off);
    revidx_fill_kernel<<<(nw + 7) / 8, 256, 0, st>>>(idx, nbh, sh.NB, sh.K, ws.rev_off, ws.rev_list, s, lse_s,
                                                      sh.gate, ws.rev_lam);
  }
  // tcgen05 passes: dK/dV/dl (and the dZ tiles) KV-major, then dQ query-major
  if ((e = launch_bwd_passes_sm100(sh, q, k, v, dO, s, idx, lse_s, lse_o, ws.drow, ws.rev_off, ws.rev_list,
                                   ws.rev_lam, ws.dl, ws.dz, dq, dk, dv, err, st)) != cudaSuccess)
    return e;
  if (ds != nullptr) {
    const int rows = nbh * sh.NB;
    bwd_ds_chain_kernel<<<(rows + 7) / 8, 256, 0, st>>>(s, lse_s, idx, ws.dl, rows, sh.NB, sh.K, sh.gate, ds);
  }
  return cudaGetLastError();
}

cudaError_t launch_bwd_mma(const Shape& sh, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                           const uint16_t* o, const uint16_t* dO, const float* s, const int32_t* idx,
                           const float* lse_s, const float* lse_o, uint16_t* dq, uint16_t* dk, uint16_t* dv, float* ds,
                           void* ws, bool spill, int* err, cudaStream_t st) {
  if (sh.d == 128)
    return launch_bwd_d<128>(sh, q, k, v, o, dO, s, idx, lse_s, lse_o, dq, dk, dv, ds, ws, spill, err, st);
  return launch_bwd_d<64>(sh, q, k, v, o, dO, s, idx, lse_s, lse_o, dq, dk, dv, ds, ws, spill, err, st);
}

}  // namespace sas
