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
#include <type_traits>

#include "common.cuh"

namespace sas {

namespace dec {
constexpr int kThreads = 128;
constexpr int kMaxTasks = kMaxDecodeBlocksPerSplit;  // task slots per chunk of items (2 CTAs per SM at d = 128)
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

  float oacc[DW / 8][4];
  float m_run = -INFINITY, l_run = 0.f;  // for head g_row (log2 domain), same in every warp

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
    uint32_t qa[D / 16][4];  // A fragments of the padded query rows (rows >= G are zero)
    for (int task = 0; task < nt; ++task) {
      if (task + STAGES - 1 < nt) issue(task + STAGES - 1);
      cp_async_commit();
      cp_async_wait<STAGES - 1>();
      __syncthreads();
      const uint32_t st = ring + (task % STAGES) * STAGEB;
      const int ntok = t_ntok[task];
      // the gate inside the softmax biases the logits by log2 g; outside, it weights P·V by g
      const float lam2 = a.outside ? 0.f : t_lam[task];
      const float gw = a.outside ? exp2f(t_lam[task]) : 1.f;
      const int flags = t_flags[task];
      if (flags & 1) {
#pragma unroll
        for (int j = 0; j < DW / 8; ++j) oacc[j][0] = oacc[j][1] = oacc[j][2] = oacc[j][3] = 0.f;
        m_run = -INFINITY;
        l_run = 0.f;
        // this stage holds the item's query rows; keep their A fragments in registers
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          ldsm_x4(st + 2 * TILEB + swz<CH>(lane & 15, 2 * kk + (lane >> 4)), qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3]);
      }
      // S = q Kᵀ for this warp's 16 tokens (two n8 tiles); rows are heads
      float sacc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(st + swz<CH>(16 * warp + (lane & 7) + ((lane >> 4) << 3), 2 * kk + ((lane >> 3) & 1)), b0, b1, b2, b3);
        mma_bf16_16816(sacc[0], qa[kk], b0, b1);
        mma_bf16_16816(sacc[1], qa[kk], b2, b3);
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
      const float m_new = fmaxf(m_run, m_blk);
      const float alpha = (m_run == -INFINITY) ? 0.f : exp2f(m_run - m_new);
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
        oacc[j][0] *= alpha;
        oacc[j][1] *= alpha;
      }
      __syncthreads();
      l_run = l_run * alpha + ((red_sum[0][g_row] + red_sum[1][g_row]) + (red_sum[2][g_row] + red_sum[3][g_row]));
      m_run = m_new;
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
          mma_bf16_16816(oacc[2 * dp], pa, b0, b1);
          mma_bf16_16816(oacc[2 * dp + 1], pa, b2, b3);
        }
      }
      if (flags & 2) {  // the item's last block: write its normalised partial for the G heads
        const int it = t_item[task];
        const int split = it % a.n_split, bh = it / a.n_split;
        if (g_row < G) {
          const size_t row = (size_t(bh) * G + g_row) * a.n_split + split;
          const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll
          for (int j = 0; j < DW / 8; ++j) {
            const int col = DW * warp + 8 * j + 2 * (lane & 3);
            *reinterpret_cast<float2*>(a.o_part + row * D + col) = make_float2(oacc[j][0] * inv, oacc[j][1] * inv);
          }
          if (warp == 0 && (lane & 3) == 0)
            a.lse_part[row] = l_run > 0.f ? (m_run + log2f(l_run)) * kLn2 : -INFINITY;
        }
      }
      __syncthreads();
    }
    cp_async_wait<0>();
    __syncthreads();
  }
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
