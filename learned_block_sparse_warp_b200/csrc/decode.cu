// Split-K single-token decode over the selected blocks, and the LSE merge.
//
// SAS explainer (ta-paperlens), section 仕組み: at inference the scores pick
// the Top-K history blocks, and attention runs over them and the current
// block. Algorithm 2 adds no gate; SAS_GATE_LOG_SOFTMAX keeps the
// training-time gate. SAS summary (onedev.kr), section 전제와 한계: decode is
// the sparsified stage, and its attention cost stays flat as the context grows.
//
// The work is HBM-bound: every selected 64-token block is read once. The split
// kernel is persistent. Each CTA owns a strided set of items (sequence, KV
// head, split) and expands them into tasks, one per 64-token block. It streams
// the tasks' K, V and q rows through a multi-stage cp.async ring in shared
// memory. Every CTA therefore keeps several 32 KB blocks in flight while it
// computes on another, and there is no per-block launch or index-lookup
// latency. The task list (block index, token count, gate) is built in shared
// memory before the ring starts, so no global load sits between two copies.
// The ring uses only cp.async groups, with no spin-waits.
//
// The K/V arrays are either the dense cache [B, Hkv, Lmax, d] or a paged cache
// [n_pages, Hkv, 64, d] with a block table: each task resolves its block to a
// 64-row slice of the array when the task list is built, so the ring is the
// same for both.
//
// The arithmetic runs on mma.sync, so that the instruction count stays below
// the memory time. The G <= 8 query heads of a KV head are padded to one
// 16-row A fragment that serves every K/V load (GQA grouping). Each warp
// scores 16 of the block's 64 tokens. Row maxima and sums are exchanged
// through shared memory. P goes through a swizzled 16 x 64 bf16 tile, and
// each warp then accumulates PV for a quarter of the head dimension.
#include <cooperative_groups.h>

#include <type_traits>

#include "common.cuh"

namespace sas {

namespace cg = cooperative_groups;

namespace dec {
constexpr int kThreads = 128;
constexpr int kMaxTasks = kMaxDecodeBlocksPerSplit;  // task slots per chunk of items (2 CTAs per SM at d = 128)
constexpr int kFusedMaxK = 255;     // the fused step keeps the whole selected list in shared memory
constexpr int kFusedMaxNB = 2048;   // and the row's keys (4 bytes each) in one ring stage
constexpr int kMaxCluster = 8;      // portable cluster size
}  // namespace dec

struct DecodeArgs {
  const uint16_t* q;
  const uint16_t* kc;
  const uint16_t* vc;
  const int32_t* cache_len;
  const float* s;
  const int32_t* idx;
  const float* lse_s;
  const int32_t* table;  // paged cache: page of logical block m of sequence b at table[b * NB + m]; null if dense
  int n_pages;
  float* o_part;
  float* lse_part;
  int* err;
  int B, Hkv, Lmax, K, gate, gated, outside, n_split, per_max, items_per_chunk;
  float scale;
};

struct DecodeFusedArgs {
  const uint16_t* q;
  const uint16_t* kc;
  const uint16_t* vc;
  const int32_t* cache_len;
  const float* s;
  const int32_t* table;  // paged cache block table, or null for the dense cache
  int n_pages;
  int32_t* idx;    // [B, Hkv, K] picks, may be null
  float* lse_s;    // [B, Hkv], may be null
  uint16_t* o;     // [B, Hq, d]
  float* lse_o;    // [B, Hq], may be null
  int* err;
  int B, Hkv, Lmax, K, gate, gated, outside, need_lse;
  float scale;
};

// The running state of one item's online softmax in one thread: the O fragments
// of this warp's d columns (rows are heads; rows >= G are padding), the row max
// and sum of head g_row (log2 domain, the same in every warp), and the A
// fragments of the padded query rows.
template <int D>
struct DecAcc {
  float o[D / 32][4];
  float m, l;
  uint32_t qa[D / 16][4];
};

// One 64-token block of an item, run by all 128 threads: S = q Kᵀ on mma.sync
// (each warp scores 16 tokens), the block's softmax update with the maxima and
// sums exchanged through shared memory, P through the swizzled tile at sP, and
// O += P V over each warp's quarter of d. `st` is the ring stage that holds the
// block's K and V tiles (and, for the item's first block, its query rows).
// Tokens past ntok are masked. lam2 biases the logits (log2 domain); gw
// weights P·V. Contains two __syncthreads.
template <int D, int G>
__device__ __forceinline__ void dec_block(DecAcc<D>& A, uint32_t st, uint32_t sP, int ntok, float lam2, float gw,
                                          bool first, float sc2, float (*red_max)[8], float (*red_sum)[8]) {
  constexpr int CH = D / 8;             // 16-byte chunks per row
  constexpr int TILEB = kBlock * D * 2;  // one 64-token tile
  constexpr int DW = D / 4;             // d columns per warp in PV
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g_row = lane >> 2;  // the head this thread's C-fragment row 0 belongs to
  if (first) {
#pragma unroll
    for (int j = 0; j < DW / 8; ++j) A.o[j][0] = A.o[j][1] = A.o[j][2] = A.o[j][3] = 0.f;
    A.m = -INFINITY;
    A.l = 0.f;
    // this stage holds the item's query rows; keep their A fragments in registers
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk)
      ldsm_x4(st + 2 * TILEB + swz<CH>(lane & 15, 2 * kk + (lane >> 4)), A.qa[kk][0], A.qa[kk][1], A.qa[kk][2], A.qa[kk][3]);
  }
  // S = q Kᵀ for this warp's 16 tokens (two n8 tiles); rows are heads
  float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    uint32_t b0, b1, b2, b3;
    ldsm_x4(st + swz<CH>(16 * warp + (lane & 7) + ((lane >> 4) << 3), 2 * kk + ((lane >> 3) & 1)), b0, b1, b2, b3);
    mma_bf16_16816(sacc[0], A.qa[kk], b0, b1);
    mma_bf16_16816(sacc[1], A.qa[kk], b2, b3);
  }
  // gated logits (log2 domain) of head g_row; tokens past ntok are masked
  float z[4];
  float mx = -INFINITY;
#pragma unroll
  for (int n = 0; n < 2; ++n)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int tok = 16 * warp + 8 * n + 2 * (lane & 3) + e;
      const float v = tok < ntok ? fmaf(sacc[n][e], sc2, lam2) : -INFINITY;
      z[2 * n + e] = v;
      mx = fmaxf(mx, v);
    }
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
  mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
  if ((lane & 3) == 0 && g_row < 8) red_max[warp][g_row] = mx;
  __syncthreads();
  const float m_blk = fmaxf(fmaxf(red_max[0][g_row], red_max[1][g_row]), fmaxf(red_max[2][g_row], red_max[3][g_row]));
  const float m_new = fmaxf(A.m, m_blk);
  const float alpha = (A.m == -INFINITY) ? 0.f : exp2f(A.m - m_new);
  float ps = 0.f;
  float pv[4];
#pragma unroll
  for (int x = 0; x < 4; ++x) {
    pv[x] = (z[x] == -INFINITY) ? 0.f : exp2f(z[x] - m_new);
    ps += pv[x];
  }
  ps += __shfl_xor_sync(0xffffffffu, ps, 1);
  ps += __shfl_xor_sync(0xffffffffu, ps, 2);
  if ((lane & 3) == 0 && g_row < 8) red_sum[warp][g_row] = ps;
  // P (bf16) of head g_row at tokens 16 warp + 8 n + 2 (lane & 3) + {0, 1}
#pragma unroll
  for (int n = 0; n < 2; ++n) {
    const int tok = 16 * warp + 8 * n + 2 * (lane & 3);
    const uint32_t addr = sP + swz<8>(g_row, tok >> 3) + (tok & 7) * 2;
    asm volatile("st.shared.b32 [%0], %1;\n" ::"r"(addr), "r"(pack_bf16x2(pv[2 * n] * gw, pv[2 * n + 1] * gw)));
  }
#pragma unroll
  for (int j = 0; j < DW / 8; ++j) {
    A.o[j][0] *= alpha;
    A.o[j][1] *= alpha;
  }
  __syncthreads();
  A.l = A.l * alpha + ((red_sum[0][g_row] + red_sum[1][g_row]) + (red_sum[2][g_row] + red_sum[3][g_row]));
  A.m = m_new;
  // O += P V over this warp's d columns [DW warp, DW warp + DW)
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    uint32_t pa[4];
    ldsm_x4(sP + swz<8>(lane & 15, 2 * kk + (lane >> 4)), pa[0], pa[1], pa[2], pa[3]);
#pragma unroll
    for (int dp = 0; dp < DW / 16; ++dp) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(st + TILEB + swz<CH>(16 * kk + (lane & 7) + (((lane >> 3) & 1) << 3), (DW / 8) * warp + 2 * dp + (lane >> 4)),
                b0, b1, b2, b3);
      mma_bf16_16816(A.o[2 * dp], pa, b0, b1);
      mma_bf16_16816(A.o[2 * dp + 1], pa, b2, b3);
    }
  }
}

template <int D, int G, int STAGES>
__global__ void __launch_bounds__(dec::kThreads) decode_split_kernel(DecodeArgs a) {
  constexpr int CH = D / 8;             // 16-byte chunks per row
  constexpr int ROWB = D * 2;           // bytes per K/V row
  constexpr int TILEB = kBlock * ROWB;  // one 64-token tile, XOR-swizzled
  constexpr int QB = 16 * ROWB;         // the group's query rows, padded to 16
  constexpr int STAGEB = 2 * TILEB + QB;
  constexpr int DW = D / 4;             // d columns per warp in PV
  extern __shared__ __align__(128) uint8_t smem[];
  // per task: item, 64-row block of the K/V arrays (row b · 64), token count, first/last flags, gate
  __shared__ int t_item[dec::kMaxTasks], t_blk[dec::kMaxTasks], t_ntok[dec::kMaxTasks], t_flags[dec::kMaxTasks];
  __shared__ float t_lam[dec::kMaxTasks];
  __shared__ int wsum_s[dec::kThreads / 32];
  __shared__ float red_max[4][8], red_sum[4][8];
  __shared__ __align__(128) uint16_t p_s[16 * kBlock];  // P tile: 16 rows x 64 tokens, bf16, swizzled

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int NB = a.Lmax / kBlock;
  const int n_items = a.B * a.Hkv * a.n_split;
  const float sc2 = a.scale * kLog2e;
  const uint32_t ring = smem_u32(smem);
  const uint32_t sP = smem_u32(p_s);

  griddep_launch_dependents();  // the merge kernel may begin its launch; it waits for this grid's writes
  // The padding rows G..15 of each stage's query tile and of the P tile are
  // never loaded; they only feed output rows that are discarded, but are kept
  // at zero so that every product stays finite. K/V rows past a block's token
  // count are zero-filled by the copies themselves.
  for (int i = tid; i < STAGES * (16 - G) * CH; i += dec::kThreads) {
    const int stg = i / ((16 - G) * CH), rem = i % ((16 - G) * CH);
    asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};\n" ::"r"(ring + stg * STAGEB + 2 * TILEB +
                                                                  swz<CH>(G + rem / CH, rem % CH)),
                 "r"(0));
  }
  for (int i = tid; i < 16 * kBlock / 8; i += dec::kThreads)
    asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};\n" ::"r"(sP + i * 16), "r"(0));
  __syncthreads();
  griddep_wait();  // idx and lse_s come from the select kernel that precedes this one

  const int my_items = (n_items > int(blockIdx.x)) ? (n_items - 1 - int(blockIdx.x)) / int(gridDim.x) + 1 : 0;
  const int g_row = lane >> 2;  // the head this thread's C-fragment row 0 belongs to


  for (int chunk0 = 0; chunk0 < my_items; chunk0 += a.items_per_chunk) {
    const int n_chunk = min(a.items_per_chunk, my_items - chunk0);
    // ---- task list of this chunk: thread i expands item i ----
    int pos0 = 0, cnt = 0, item = -1, c = 0, L = 1;
    if (tid < n_chunk) {
      item = int(blockIdx.x) + (chunk0 + tid) * int(gridDim.x);
      const int split = item % a.n_split;
      const int bh = item / a.n_split;
      const int b = bh / a.Hkv;
      L = a.cache_len[b];
      if (L < 1 || L > a.Lmax) {
        raise_error(a.err, SAS_ERR_DEVICE_INDEX);
        L = max(1, min(L, a.Lmax));
      }
      c = (L - 1) / kBlock;
      const int nl = 1 + min(a.K, c);
      const int per = (nl + a.n_split - 1) / a.n_split;
      pos0 = min(split * per, nl);
      cnt = min(pos0 + per, nl) - pos0;
      if (cnt == 0) {  // an empty chunk: o = 0, lse = -inf
        for (int g = 0; g < G; ++g) {
          const size_t row = (size_t(bh) * G + g) * a.n_split + split;
          for (int e = 0; e < D; ++e) a.o_part[row * D + e] = 0.f;
          a.lse_part[row] = -INFINITY;
        }
      }
    }
    // exclusive scan of the per-item task counts: shuffles within a warp, then the warp totals
    int incl = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    if (lane == 31) wsum_s[warp] = incl;
    __syncthreads();
    int base = incl - cnt, nt = 0;
#pragma unroll
    for (int w = 0; w < dec::kThreads / 32; ++w) {
      const int v = wsum_s[w];
      base += (w < warp) ? v : 0;
      nt += v;
    }
    if (tid < n_chunk) {
      const int bh = item / a.n_split;
      const float lse_bh = (a.gated && a.lse_s != nullptr) ? a.lse_s[bh] : 0.f;
      for (int j = 0; j < cnt; ++j) {
        const int pos = pos0 + j;
        int m = c, ntok = L - c * kBlock;
        float lam = 0.f;
        if (pos > 0) {
          m = a.idx[size_t(bh) * a.K + pos - 1];
          ntok = kBlock;
          if (m < 0 || m >= c) {
            if (m >= c) raise_error(a.err, SAS_ERR_DEVICE_INDEX);
            m = 0;
            ntok = 0;  // an empty block
          } else if (a.gated) {
            lam = gate_lam2(a.gate, a.s[size_t(bh) * NB + m], lse_bh);
          }
        }
        int blk = bh * NB + m;  // dense cache [B, Hkv, Lmax, d]
        if (a.table != nullptr) {  // paged cache [n_pages, Hkv, 64, d]
          int pg = 0;
          if (ntok > 0) {
            const int b = bh / a.Hkv;
            pg = a.table[size_t(b) * NB + m];
            if (pg < 0 || pg >= a.n_pages) {
              raise_error(a.err, SAS_ERR_DEVICE_INDEX);
              pg = 0;
            }
          }
          blk = pg * a.Hkv + bh % a.Hkv;
        }
        t_item[base + j] = item;
        t_blk[base + j] = blk;
        t_ntok[base + j] = ntok;
        t_lam[base + j] = lam;
        t_flags[base + j] = (j == 0 ? 1 : 0) | (j == cnt - 1 ? 2 : 0);
      }
    }
    __syncthreads();

    auto issue = [&](int task) {
      const uint32_t st = ring + (task % STAGES) * STAGEB;
      const int it = t_item[task];
      const int bh = it / a.n_split;
      const int ntok = t_ntok[task];
      const size_t row0 = size_t(t_blk[task]) * kBlock;
      const uint16_t* kb = a.kc + row0 * D;
      const uint16_t* vb = a.vc + row0 * D;
      // rows past ntok are zero-filled (no bytes read), so masked tokens multiply finite zeros
#pragma unroll 4
      for (int i = tid; i < kBlock * CH; i += dec::kThreads) {
        const int r = i / CH, ch = i % CH;
        const int nb = r < ntok ? 16 : 0;
        const size_t off = r < ntok ? size_t(r) * D + ch * 8 : 0;
        cp_async16_zfill(st + swz<CH>(r, ch), kb + off, nb);
        cp_async16_zfill(st + TILEB + swz<CH>(r, ch), vb + off, nb);
      }
      if (t_flags[task] & 1) {  // the item's first block brings its G query rows
        const uint16_t* qb = a.q + size_t(bh) * G * D;
        for (int i = tid; i < G * CH; i += dec::kThreads)
          cp_async16(st + 2 * TILEB + swz<CH>(i / CH, i % CH), qb + (i / CH) * D + (i % CH) * 8);
      }
    };

#pragma unroll
    for (int s = 0; s < STAGES - 1; ++s) {
      if (s < nt) issue(s);
      cp_async_commit();
    }
    DecAcc<D> acc;  // the running O fragments, max and sum of the item in flight
    for (int task = 0; task < nt; ++task) {
      if (task + STAGES - 1 < nt) issue(task + STAGES - 1);
      cp_async_commit();
      cp_async_wait<STAGES - 1>();
      __syncthreads();
      const uint32_t st = ring + (task % STAGES) * STAGEB;
      // the gate inside the softmax biases the logits by log2 g; outside, it weights P·V by g
      const float lam2 = a.outside ? 0.f : t_lam[task];
      const float gw = a.outside ? exp2f(t_lam[task]) : 1.f;
      const int flags = t_flags[task];
      dec_block<D, G>(acc, st, sP, t_ntok[task], lam2, gw, (flags & 1) != 0, sc2, red_max, red_sum);
      if (flags & 2) {  // the item's last block: write its normalised partial for the G heads
        const int it = t_item[task];
        const int split = it % a.n_split, bh = it / a.n_split;
        if (g_row < G) {
          const size_t row = (size_t(bh) * G + g_row) * a.n_split + split;
          const float inv = acc.l > 0.f ? 1.f / acc.l : 0.f;
#pragma unroll
          for (int j = 0; j < DW / 8; ++j) {
            const int col = DW * warp + 8 * j + 2 * (lane & 3);
            *reinterpret_cast<float2*>(a.o_part + row * D + col) = make_float2(acc.o[j][0] * inv, acc.o[j][1] * inv);
          }
          if (warp == 0 && (lane & 3) == 0)
            a.lse_part[row] = acc.l > 0.f ? (acc.m + log2f(acc.l)) * kLn2 : -INFINITY;
        }
      }
      __syncthreads();
    }
    cp_async_wait<0>();
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// The whole decode step in one launch (sas_decode_fused): one cluster of CS
// CTAs per (sequence, KV head) row. Every CTA of the cluster selects the row's
// Top-K blocks itself (the row is 2 KB at 32K, so the redundant work is cheaper
// than a hand-over) while the first CTA's load of the current block is in
// flight. Each CTA then streams its share of the ordered list [current block,
// picks...] through the same cp.async ring and block step as the split kernel,
// and leaves its unnormalised partial (O fragments, row max, row sum) in its own
// shared memory. After a cluster barrier every CTA merges a slice of the G x d
// outputs from all partials over distributed shared memory, so no partial
// touches HBM and no second kernel runs.

// Exclusive sum over the 128 threads of the CTA (tot gets the total). Contains
// two __syncthreads; wtot holds 4 ints of shared memory.
__device__ __forceinline__ int cta_excl_sum(int v, int* wtot, int& tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += u;
  }
  if (lane == 31) wtot[warp] = incl;
  __syncthreads();
  int before = incl - v;
  tot = 0;
#pragma unroll
  for (int w = 0; w < dec::kThreads / 32; ++w) {
    before += (w < warp) ? wtot[w] : 0;
    tot += wtot[w];
  }
  __syncthreads();
  return before;
}

// One 8-bit radix pass over the keys of key[0, c) whose bits above `shift + 8`
// equal prefix's: fixes the digit at which the count from the top bin reaches
// need. xch gets the digit, the number still needed within its bin, and the
// bin's count. (Plain shared atomics: aggregating equal digits within a warp
// first, by match.any, measured slower on sm_100a.)
__device__ void cta_radix_pass(const uint32_t* key, int c, int pass, uint32_t prefix, int need, int* hist, int* xch) {
  const int tid = threadIdx.x, lane = tid & 31;
  const int shift = 24 - 8 * pass;
  for (int i = tid; i < 256; i += dec::kThreads) hist[i] = 0;
  __syncthreads();
  for (int m = tid; m < c; m += dec::kThreads) {
    const uint32_t k = key[m];
    if (pass == 0 || ((k ^ prefix) >> (shift + 8)) == 0u) atomicAdd(&hist[(k >> shift) & 255u], 1);
  }
  __syncthreads();
  if (tid < 32) {  // lane owns bins [8 lane, 8 lane + 8); counts run from the top bin down
    int cnt[8], own = 0;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      cnt[u] = hist[8 * lane + u];
      own += cnt[u];
    }
    int incl = own;  // own plus every lane above
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int u = __shfl_down_sync(0xffffffffu, incl, off);
      if (lane + off < 32) incl += u;
    }
    int acc = incl - own;  // keys in bins above this lane's
    if (acc < need && need <= incl) {
#pragma unroll
      for (int u = 7; u >= 0; --u) {
        if (acc + cnt[u] >= need) {
          xch[0] = 8 * lane + u;
          xch[1] = need - acc;
          xch[2] = cnt[u];
          break;
        }
        acc += cnt[u];
      }
    }
  }
  __syncthreads();
}

// The n largest of key[0, c) in shared memory (0 < n < c), ties to the lowest
// index. The first 8-bit radix pass fixes the leading byte of the n-th largest
// key. When at most 128 keys share that byte (the usual case: scores spread
// over several exponents), those candidates are ranked against each other
// directly, one per thread, and the picks (every key with a larger leading
// byte, and the candidates ranked below the number still needed) are appended
// to app in any order. Otherwise three more passes find the exact threshold;
// the picks are appended likewise unless a tie is cut at it, in which case
// the function returns true with the threshold and the number of its equals
// to take, and the caller places the picks in index order.
__device__ bool cta_select(const uint32_t* key, int c, int n, int* hist, int* xch, int* app, int* napp,
                           uint32_t* cand_k, int* cand_m, int* ncand, uint32_t& thr, int& need_eq) {
  const int tid = threadIdx.x;
  if (tid == 0) *ncand = 0;
  cta_radix_pass(key, c, 0, 0u, n, hist, xch);
  const uint32_t d0 = uint32_t(xch[0]);
  const int need1 = xch[1], cnt0 = xch[2];
  if (cnt0 <= dec::kThreads) {
    for (int m = tid; m < c; m += dec::kThreads) {
      const uint32_t k = key[m], top = k >> 24;
      if (top > d0) {
        app[atomicAdd(napp, 1)] = m;
      } else if (top == d0) {
        const int s = atomicAdd(ncand, 1);
        cand_k[s] = k;
        cand_m[s] = m;
      }
    }
    __syncthreads();
    if (tid < cnt0) {
      const uint32_t k = cand_k[tid];
      const int mi = cand_m[tid];
      int r = 0;  // candidates ahead of this one: larger keys, and equal keys at lower indexes
#pragma unroll 8
      for (int j = 0; j < cnt0; ++j) {
        const uint32_t kj = cand_k[j];
        r += (kj > k || (kj == k && cand_m[j] < mi)) ? 1 : 0;
      }
      if (r < need1) app[atomicAdd(napp, 1)] = mi;
    }
    return false;
  }
  uint32_t prefix = d0 << 24;
  int need = need1;
#pragma unroll 1
  for (int pass = 1; pass < 4; ++pass) {
    cta_radix_pass(key, c, pass, prefix, need, hist, xch);
    prefix |= uint32_t(xch[0]) << (24 - 8 * pass);
    need = xch[1];
  }
  thr = prefix;
  need_eq = need;
  if (need_eq != xch[2]) return true;  // a tie is cut at the threshold
  for (int m = tid; m < c; m += dec::kThreads)
    if (key[m] >= thr) app[atomicAdd(napp, 1)] = m;
  return false;
}

template <int D, int G, int STAGES>
__global__ void __launch_bounds__(dec::kThreads) decode_fused_kernel(DecodeFusedArgs a) {
  constexpr int CH = D / 8;
  constexpr int ROWB = D * 2;
  constexpr int TILEB = kBlock * ROWB;
  constexpr int QB = 16 * ROWB;
  constexpr int STAGEB = 2 * TILEB + QB;
  constexpr int DW = D / 4;
  static_assert(dec::kFusedMaxNB * 4 + 768 * 4 <= STAGEB, "keys, histogram, picks and candidates fit one ring stage");
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int sel_s[dec::kFusedMaxK];         // the row's picks, ascending
  __shared__ float lam_s[dec::kFusedMaxK + 1];   // log2 gate of each of this CTA's tasks
  __shared__ int xch_s[4], wtot_s[dec::kThreads / 32], napp_s;
  __shared__ float redf_s[dec::kThreads / 32];
  __shared__ float red_max[4][8], red_sum[4][8];
  __shared__ __align__(128) uint16_t p_s[16 * kBlock];

  cg::cluster_group cluster = cg::this_cluster();
  const int CS = int(cluster.num_blocks()), rank = int(cluster.block_rank());
  const int bh = int(blockIdx.x) / CS;
  const int b = bh / a.Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g_row = lane >> 2;
  const int NB = a.Lmax / kBlock;
  const float sc2 = a.scale * kLog2e;
  const uint32_t ring = smem_u32(smem);
  const uint32_t sP = smem_u32(p_s);

  griddep_launch_dependents();
  if (tid == 0) napp_s = 0;
  for (int i = tid; i < STAGES * (16 - G) * CH; i += dec::kThreads) {  // padding rows, as in the split kernel
    const int stg = i / ((16 - G) * CH), rem = i % ((16 - G) * CH);
    asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};\n" ::"r"(ring + stg * STAGEB + 2 * TILEB +
                                                                  swz<CH>(G + rem / CH, rem % CH)),
                 "r"(0));
  }
  for (int i = tid; i < 16 * kBlock / 8; i += dec::kThreads)
    asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};\n" ::"r"(sP + i * 16), "r"(0));
  griddep_wait();  // q, the caches, the scores and cache_len may come from the work just before

  // the row's scores are read while the cache length is still in flight
  const float* srow = a.s + size_t(bh) * NB;
  uint32_t* key_s = reinterpret_cast<uint32_t*>(smem + (STAGES - 1) * STAGEB);
  int* hist_s = reinterpret_cast<int*>(key_s + dec::kFusedMaxNB);
  for (int m = tid; m < NB - 1; m += dec::kThreads) key_s[m] = __float_as_uint(__ldg(srow + m));
  int L = a.cache_len[b];
  if (L < 1 || L > a.Lmax) {
    if (tid == 0) raise_error(a.err, SAS_ERR_DEVICE_INDEX);
    L = max(1, min(L, a.Lmax));
  }
  const int c = (L - 1) / kBlock;  // the current block; history blocks are [0, c)
  const int n = min(a.K, c);

  // ---- this CTA's share of the ordered list [c, picks...]
  const int nl = 1 + n;
  const int share = (nl + CS - 1) / CS;
  const int p0 = min(rank * share, nl);
  const int nt = min(p0 + share, nl) - p0;
  auto issue = [&](int j) {
    const uint32_t st = ring + (j % STAGES) * STAGEB;
    const int pos = p0 + j;
    const int m = pos == 0 ? c : sel_s[pos - 1];
    const int ntok = pos == 0 ? L - c * kBlock : kBlock;
    int blk = bh * NB + m;  // dense cache [B, Hkv, Lmax, d]
    if (a.table != nullptr) {  // paged cache [n_pages, Hkv, 64, d]
      int pg = a.table[size_t(b) * NB + m];
      if (pg < 0 || pg >= a.n_pages) {
        raise_error(a.err, SAS_ERR_DEVICE_INDEX);
        pg = 0;
      }
      blk = pg * a.Hkv + bh % a.Hkv;
    }
    const size_t row0 = size_t(blk) * kBlock;
    const uint16_t* kb = a.kc + row0 * D;
    const uint16_t* vb = a.vc + row0 * D;
#pragma unroll 4
    for (int i = tid; i < kBlock * CH; i += dec::kThreads) {
      const int r = i / CH, ch = i % CH;
      const int nb = r < ntok ? 16 : 0;
      const size_t off = r < ntok ? size_t(r) * D + ch * 8 : 0;
      cp_async16_zfill(st + swz<CH>(r, ch), kb + off, nb);
      cp_async16_zfill(st + TILEB + swz<CH>(r, ch), vb + off, nb);
    }
    if (j == 0) {  // the first block of the CTA brings the G query rows
      const uint16_t* qb = a.q + size_t(bh) * G * D;
      for (int i = tid; i < G * CH; i += dec::kThreads)
        cp_async16(st + 2 * TILEB + swz<CH>(i / CH, i % CH), qb + (i / CH) * D + (i % CH) * 8);
    }
  };

  // the first CTA of the cluster starts on the current block, which needs no selection
  if (p0 == 0) {
    if (nt > 0) issue(0);
    cp_async_commit();
  }
  // ---- selection: keys of the history scores in the last ring stage (not loaded before the loop)
  float mx = -INFINITY;
  for (int m = tid; m < c; m += dec::kThreads) {  // each thread converts the scores it read
    const float v = __uint_as_float(key_s[m]);
    key_s[m] = score_key(v) + 1u;  // >= 1, so the threshold 1 takes every block
    mx = fmaxf(mx, v);
  }
  float lse = 0.f;
  if (a.need_lse) {  // LSE of the history scores, as the select kernels take it
    mx = warp_max(mx);
    if (lane == 0) redf_s[warp] = mx;
    __syncthreads();
    mx = fmaxf(fmaxf(redf_s[0], redf_s[1]), fmaxf(redf_s[2], redf_s[3]));
    __syncthreads();
    float sum = 0.f;
    if (mx != -INFINITY)
      for (int m = tid; m < c; m += dec::kThreads) sum += expf(__ldg(srow + m) - mx);
    sum = warp_sum(sum);
    if (lane == 0) redf_s[warp] = sum;
    __syncthreads();
    const float tot = (redf_s[0] + redf_s[1]) + (redf_s[2] + redf_s[3]);
    lse = (c == 0 || mx == -INFINITY) ? -INFINITY : mx + logf(tot);
  }
  __syncthreads();  // every key is in place
  const bool all = (n == c), none = (n == 0);
  int need_eq = 0;
  uint32_t thr = 1u;
  int32_t* idx_row = (rank == 0 && a.idx != nullptr) ? a.idx + size_t(bh) * a.K : nullptr;
  int* app_s = hist_s + 256;
  uint32_t* cand_k = reinterpret_cast<uint32_t*>(app_s + 256);
  int* cand_m = app_s + 384;
  bool tie = false;
  if (all) {
    for (int m = tid; m < c; m += dec::kThreads) app_s[m] = m;
  } else if (!none) {
    tie = cta_select(key_s, c, n, hist_s, xch_s, app_s, &napp_s, cand_k, cand_m, &xch_s[3], thr, need_eq);
  }
  const bool fast = !none && !tie;
  if (fast) {
    __syncthreads();
    for (int i = tid; i < n; i += dec::kThreads) {
      const int v = app_s[i];
      int r = 0;
      for (int j = 0; j < n; ++j) r += app_s[j] < v ? 1 : 0;
      sel_s[r] = v;
      if (idx_row != nullptr) idx_row[r] = v;
      const int jt = r + 1 - p0;  // this CTA's task at list position r + 1
      if (jt >= 0 && jt < nt) lam_s[jt] = a.gated ? gate_lam2(a.gate, __ldg(srow + v), lse) : 0.f;
    }
  } else if (!none) {
    // ties cut at the threshold, taken from the lowest block index: each thread
    // owns a contiguous run of blocks, and two block-wide scans place the picks
    const int per = (c + dec::kThreads - 1) / dec::kThreads;
    const int lo = min(c, tid * per), hi = min(c, lo + per);
    int eq = 0;
    for (int m = lo; m < hi; ++m) eq += key_s[m] == thr ? 1 : 0;
    int tot = 0;
    const int eq0 = cta_excl_sum(eq, wtot_s, tot);
    int take = 0;
    for (int m = lo, e = eq0; m < hi; ++m) {
      const uint32_t k = key_s[m];
      const bool is_eq = k == thr;
      take += (k > thr || (is_eq && e < need_eq)) ? 1 : 0;
      e += is_eq ? 1 : 0;
    }
    int pos = cta_excl_sum(take, wtot_s, tot);
    for (int m = lo, e = eq0; m < hi; ++m) {
      const uint32_t k = key_s[m];
      const bool is_eq = k == thr;
      if (k > thr || (is_eq && e < need_eq)) sel_s[pos++] = m;
      e += is_eq ? 1 : 0;
    }
  }
  if (idx_row != nullptr)
    for (int i = n + tid; i < a.K; i += dec::kThreads) idx_row[i] = -1;
  if (rank == 0 && a.lse_s != nullptr && tid == 0) a.lse_s[bh] = lse;
  if (p0 == 0 && nt > 0 && tid == 0) lam_s[0] = 0.f;  // the current block takes no gate
  __syncthreads();  // the picks are placed, and the keys' stage is free for the ring
  if (!fast && !none) {  // the tie path placed the picks by block scans: write them out and take their gates
    if (idx_row != nullptr)
      for (int i = tid; i < n; i += dec::kThreads) idx_row[i] = sel_s[i];
    for (int j = tid; j < nt; j += dec::kThreads)
      if (p0 + j > 0) lam_s[j] = a.gated ? gate_lam2(a.gate, __ldg(srow + sel_s[p0 + j - 1]), lse) : 0.f;
  }

  DecAcc<D> acc;
#pragma unroll
  for (int j = 0; j < DW / 8; ++j) acc.o[j][0] = acc.o[j][1] = acc.o[j][2] = acc.o[j][3] = 0.f;
  acc.m = -INFINITY;
  acc.l = 0.f;
  if (p0 != 0) {  // the other CTAs' first block is a pick
    if (nt > 0) issue(0);
    cp_async_commit();
  }
#pragma unroll
  for (int s = 1; s < STAGES - 1; ++s) {
    if (s < nt) issue(s);
    cp_async_commit();
  }
  for (int j = 0; j < nt; ++j) {
    if (j + STAGES - 1 < nt) issue(j + STAGES - 1);
    cp_async_commit();
    cp_async_wait<STAGES - 1>();
    __syncthreads();
    const float lam2 = a.outside ? 0.f : lam_s[j];
    const float gw = a.outside ? exp2f(lam_s[j]) : 1.f;
    dec_block<D, G>(acc, ring + (j % STAGES) * STAGEB, sP, (p0 + j) == 0 ? L - c * kBlock : kBlock, lam2, gw, j == 0,
                    sc2, red_max, red_sum);
    __syncthreads();
  }
  cp_async_wait<0>();
  __syncthreads();

  // ---- the partial of this CTA, unnormalised, in its first ring stage: m[G], l[G], o[G][D]
  float* part = reinterpret_cast<float*>(smem);
  if (g_row < G) {
#pragma unroll
    for (int j = 0; j < DW / 8; ++j) {
      const int col = DW * warp + 8 * j + 2 * (lane & 3);
      *reinterpret_cast<float2*>(part + 16 + g_row * D + col) = make_float2(acc.o[j][0], acc.o[j][1]);
    }
    if (warp == 0 && (lane & 3) == 0) {
      part[g_row] = acc.m;
      part[8 + g_row] = acc.l;
    }
  }
  cluster.sync();  // every partial of the cluster is in place
  // ---- merge: CTA `rank` writes pairs of d columns rank·128 + tid, + CS·128, ...
  for (int e = rank * dec::kThreads + tid; e < G * D / 2; e += CS * dec::kThreads) {
    const int g = (2 * e) / D, col = (2 * e) % D;
    float M = -INFINITY;
    for (int r = 0; r < CS; ++r) M = fmaxf(M, cluster.map_shared_rank(part, r)[g]);
    float den = 0.f, n0 = 0.f, n1 = 0.f;
    for (int r = 0; r < CS; ++r) {
      const float* pr = cluster.map_shared_rank(part, r);
      const float mr = pr[g];
      const float w = (mr == -INFINITY) ? 0.f : exp2f(mr - M);
      const float2 ov = *reinterpret_cast<const float2*>(pr + 16 + g * D + col);
      den = fmaf(w, pr[8 + g], den);
      n0 = fmaf(w, ov.x, n0);
      n1 = fmaf(w, ov.y, n1);
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    const size_t row = size_t(bh) * G + g;
    *reinterpret_cast<uint32_t*>(a.o + row * D + col) = pack_bf16x2(n0 * inv, n1 * inv);
    if (col == 0 && a.lse_o != nullptr) a.lse_o[row] = den > 0.f ? (M + log2f(den)) * kLn2 : -INFINITY;
  }
  cluster.sync();  // no CTA leaves while another may still read its partial
}

// One warp per (sequence, query head). The lanes read the split LSEs in
// parallel and reduce them with shuffles. The partials are then streamed in
// batches of 16 float4 (d = 128) or float2 (d = 64) loads per lane, all
// issued before the first is used, so a batch costs one L2 round trip. The
// weight is applied by a select, with no branch around the loads.
template <int D>
__global__ void __launch_bounds__(256) decode_combine_kernel(const float* __restrict__ o_part,
                                                             const float* __restrict__ lse_part, int n_split,
                                                             int rows, uint16_t* __restrict__ o,
                                                             float* __restrict__ lse_o) {
  constexpr int PER = D / 32;  // d values per lane: 4 or 2
  constexpr int BATCH = 16;
  using VecT = typename std::conditional<PER == 4, float4, float2>::type;
  griddep_wait();  // the partials come from the split kernel that precedes this one
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int lane = threadIdx.x & 31;
  const float* lp = lse_part + size_t(row) * n_split;
  const float l0 = lane < n_split ? lp[lane] : -INFINITY;
  float mx = l0;
  for (int j = lane + 32; j < n_split; j += 32) mx = fmaxf(mx, lp[j]);
  mx = warp_max(mx);
  const float mref = (mx == -INFINITY) ? 0.f : mx;  // all splits empty: every weight is 0
  const float* op = o_part + size_t(row) * n_split * D + lane * PER;
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  float den = 0.f;
  for (int j0 = 0; j0 < n_split; j0 += 32) {
    const int jl = j0 + lane;
    const float l = j0 == 0 ? l0 : (jl < n_split ? lp[jl] : -INFINITY);
    const float wl = exp2f((l - mref) * kLog2e);  // 0 for an empty split (lse = -inf)
    den += wl;
    const int nj = min(32, n_split - j0);
    for (int u0 = 0; u0 < nj; u0 += BATCH) {
      VecT x[BATCH];
#pragma unroll
      for (int u = 0; u < BATCH; ++u) {
        const int j = j0 + min(u0 + u, nj - 1);  // a valid split; surplus slots get weight 0
        x[u] = *reinterpret_cast<const VecT*>(op + size_t(j) * D);
      }
#pragma unroll
      for (int u = 0; u < BATCH; ++u) {
        const float w0 = __shfl_sync(0xffffffffu, wl, (u0 + u) & 31);
        const float w = (u0 + u < nj && w0 > 0.f) ? w0 : 0.f;
        const float* xv = reinterpret_cast<const float*>(&x[u]);
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[e] = w > 0.f ? fmaf(w, xv[e], acc[e]) : acc[e];
      }
    }
  }
  den = warp_sum(den);
  const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] *= inv;
  uint16_t* dst = o + size_t(row) * D + lane * PER;
  if (PER == 4) {
    *reinterpret_cast<uint2*>(dst) =
        make_uint2(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[PER > 2 ? 2 : 0], acc[PER > 3 ? 3 : 0]));
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(acc[0], acc[1]);
  }
  if (lse_o != nullptr && lane == 0) lse_o[row] = (mx == -INFINITY) ? -INFINITY : mx + logf(den);
}

template <int D, int G>
static cudaError_t launch_decode_dg(const Shape& sh, const DecodeArgs& a, cudaStream_t st) {
  constexpr int STAGES = 3;
  constexpr int smem = STAGES * (2 * kBlock * D * 2 + 16 * D * 2);
  auto kern = decode_split_kernel<D, G, STAGES>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0, per_sm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, dec::kThreads, smem)) != cudaSuccess)
    return e;
  const int n_items = a.B * a.Hkv * a.n_split;
  const int grid = max(1, min(n_items, sms * max(1, per_sm)));
  e = launch_pdl(kern, dim3(grid), dim3(dec::kThreads), smem, st, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_decode_d(const Shape& sh, const uint16_t* q, const uint16_t* kc, const uint16_t* vc,
                                   const int32_t* table, int n_pages, const int32_t* cl, const float* s,
                                   const int32_t* idx, const float* lse_s, int n_split, float* o_part,
                                   float* lse_part, int* err, cudaStream_t st) {
  DecodeArgs a;
  a.table = table;
  a.n_pages = n_pages;
  a.q = q;
  a.kc = kc;
  a.vc = vc;
  a.cache_len = cl;
  a.s = s;
  a.idx = idx;
  a.lse_s = lse_s;
  a.o_part = o_part;
  a.lse_part = lse_part;
  a.err = err;
  a.B = sh.B;
  a.Hkv = sh.Hkv;
  a.Lmax = sh.N;
  a.K = sh.K;
  a.gate = sh.gate;
  a.gated = sh.gated;
  a.outside = sh.outside;
  a.n_split = n_split;
  a.per_max = (sh.K + 1 + n_split - 1) / n_split;
  a.items_per_chunk = max(1, min(dec::kThreads, dec::kMaxTasks / a.per_max));
  a.scale = sh.scale;
  switch (sh.G) {
    case 1: return launch_decode_dg<D, 1>(sh, a, st);
    case 2: return launch_decode_dg<D, 2>(sh, a, st);
    case 3: return launch_decode_dg<D, 3>(sh, a, st);
    case 4: return launch_decode_dg<D, 4>(sh, a, st);
    case 5: return launch_decode_dg<D, 5>(sh, a, st);
    case 6: return launch_decode_dg<D, 6>(sh, a, st);
    case 7: return launch_decode_dg<D, 7>(sh, a, st);
    case 8: return launch_decode_dg<D, 8>(sh, a, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_decode(const Shape& sh, const uint16_t* q, const uint16_t* kc, const uint16_t* vc,
                          const int32_t* cl, const float* s, const int32_t* idx, const float* lse_s, int n_split,
                          float* o_part, float* lse_part, int* err, cudaStream_t st) {
  if (sh.d == 128)
    return launch_decode_d<128>(sh, q, kc, vc, nullptr, 0, cl, s, idx, lse_s, n_split, o_part, lse_part, err, st);
  return launch_decode_d<64>(sh, q, kc, vc, nullptr, 0, cl, s, idx, lse_s, n_split, o_part, lse_part, err, st);
}

cudaError_t launch_decode_paged(const Shape& sh, const uint16_t* q, const uint16_t* kp, const uint16_t* vp,
                                int n_pages, const int32_t* table, const int32_t* cl, const float* s,
                                const int32_t* idx, const float* lse_s, int n_split, float* o_part, float* lse_part,
                                int* err, cudaStream_t st) {
  if (sh.d == 128)
    return launch_decode_d<128>(sh, q, kp, vp, table, n_pages, cl, s, idx, lse_s, n_split, o_part, lse_part, err, st);
  return launch_decode_d<64>(sh, q, kp, vp, table, n_pages, cl, s, idx, lse_s, n_split, o_part, lse_part, err, st);
}

// The cluster size: the largest power of two of CTAs per row that keeps the
// whole grid in one wave of resident CTAs (2 per SM at d = 128), at most 8
// and at most one per block of the list.
template <int D, int G>
static cudaError_t launch_decode_fused_dg(const Shape& sh, const DecodeFusedArgs& a, cudaStream_t st) {
  constexpr int STAGES = 3;
  constexpr int smem = STAGES * (2 * kBlock * D * 2 + 16 * D * 2);
  auto kern = decode_fused_kernel<D, G, STAGES>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0, per_sm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, dec::kThreads, smem)) != cudaSuccess)
    return e;
  const int rows = a.B * a.Hkv;
  const int want = max(1, min(min(dec::kMaxCluster, a.K + 1), (sms * max(1, per_sm)) / rows));
  int cs = 1;
  while (cs * 2 <= want) cs *= 2;  // a power of two
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(rows * cs);
  cfg.blockDim = dim3(dec::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if ((e = cudaLaunchKernelEx(&cfg, kern, a)) != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_decode_fused_d(const Shape& sh, const DecodeFusedArgs& a, cudaStream_t st) {
  switch (sh.G) {
    case 1: return launch_decode_fused_dg<D, 1>(sh, a, st);
    case 2: return launch_decode_fused_dg<D, 2>(sh, a, st);
    case 3: return launch_decode_fused_dg<D, 3>(sh, a, st);
    case 4: return launch_decode_fused_dg<D, 4>(sh, a, st);
    case 5: return launch_decode_fused_dg<D, 5>(sh, a, st);
    case 6: return launch_decode_fused_dg<D, 6>(sh, a, st);
    case 7: return launch_decode_fused_dg<D, 7>(sh, a, st);
    case 8: return launch_decode_fused_dg<D, 8>(sh, a, st);
    default: return cudaErrorInvalidValue;
  }
}

bool decode_fused_fits(const Shape& sh) {
  return sh.G <= 8 && sh.K <= dec::kFusedMaxK && sh.NB <= dec::kFusedMaxNB;
}

cudaError_t launch_decode_fused(const Shape& sh, const uint16_t* q, const uint16_t* kc, const uint16_t* vc,
                                const int32_t* table, int n_pages, const int32_t* cl, const float* s, int32_t* idx,
                                float* lse_s, uint16_t* o, float* lse_o, int* err, cudaStream_t st) {
  DecodeFusedArgs a;
  a.q = q;
  a.kc = kc;
  a.vc = vc;
  a.cache_len = cl;
  a.s = s;
  a.table = table;
  a.n_pages = n_pages;
  a.idx = idx;
  a.lse_s = lse_s;
  a.o = o;
  a.lse_o = lse_o;
  a.err = err;
  a.B = sh.B;
  a.Hkv = sh.Hkv;
  a.Lmax = sh.N;
  a.K = sh.K;
  a.gate = sh.gate;
  a.gated = sh.gated;
  a.outside = sh.outside;
  a.need_lse = (lse_s != nullptr || sh.gate == SAS_GATE_LOG_SOFTMAX || sh.gate == SAS_GATE_SOFTMAX_OUTSIDE) ? 1 : 0;
  a.scale = sh.scale;
  return sh.d == 128 ? launch_decode_fused_d<128>(sh, a, st) : launch_decode_fused_d<64>(sh, a, st);
}

cudaError_t launch_decode_combine(const Shape& sh, int n_split, const float* o_part, const float* lse_part,
                                  uint16_t* o, float* lse_o, cudaStream_t st) {
  const int rows = sh.B * sh.Hq;
  const dim3 grid((rows + 7) / 8), block(256);
  const cudaError_t e =
      sh.d == 128 ? launch_pdl(decode_combine_kernel<128>, grid, block, 0, st, o_part, lse_part, n_split, rows, o, lse_o)
                  : launch_pdl(decode_combine_kernel<64>, grid, block, 0, st, o_part, lse_part, n_split, rows, o, lse_o);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace sas
