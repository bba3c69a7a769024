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
// latency. The G query heads of a KV head share every K/V load (GQA grouping).
// The task list (block index, token count, gate) is built in shared memory
// before the ring starts, so no global load sits between two copies. The ring
// uses only cp.async groups, with no spin-waits.
#include "common.cuh"

namespace sas {

namespace dec {
constexpr int kThreads = 128;
constexpr int kMaxTasks = 128;  // task slots per chunk of items
}  // namespace dec

__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(addr));
  return r;
}

struct DecodeArgs {
  const uint16_t* q;
  const uint16_t* kc;
  const uint16_t* vc;
  const int32_t* cache_len;
  const float* s;
  const int32_t* idx;
  const float* lse_s;
  float* o_part;
  float* lse_part;
  int* err;
  int B, Hkv, Lmax, K, gated, n_split, per_max, items_per_chunk;
  float scale;
};

template <int D, int G, int STAGES>
__global__ void __launch_bounds__(dec::kThreads) decode_split_kernel(DecodeArgs a) {
  constexpr int CH = D / 8;            // 16-byte chunks per row
  constexpr int ROWB = D * 2;          // bytes per K/V row
  constexpr int TILEB = kBlock * ROWB;  // one 64-token tile
  constexpr int QB = G * ROWB;          // the group's query rows
  constexpr int STAGEB = 2 * TILEB + QB;
  constexpr int LPR = CH;               // lanes per row: one 16-byte chunk each
  constexpr int RPW = 32 / LPR;         // rows per warp per step
  constexpr int RG = dec::kThreads / LPR;  // row groups in the PV product
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int t_item[dec::kMaxTasks], t_m[dec::kMaxTasks], t_ntok[dec::kMaxTasks], t_flags[dec::kMaxTasks];
  __shared__ float t_lam[dec::kMaxTasks];
  __shared__ int n_tasks_s;
  __shared__ int cnt_s[dec::kThreads];
  __shared__ float sc_s[G][kBlock];
  __shared__ float m_s[G], l_s[G], a_s[G];
  __shared__ float red_s[4][G][D];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int NB = a.Lmax / kBlock;
  const int n_items = a.B * a.Hkv * a.n_split;
  const float sc2 = a.scale * kLog2e;
  const uint32_t ring = smem_u32(smem);

  // this CTA's items: blockIdx.x + k * gridDim.x
  const int my_items = (n_items > int(blockIdx.x)) ? (n_items - 1 - int(blockIdx.x)) / int(gridDim.x) + 1 : 0;

  float acc[G][8];

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
    cnt_s[tid] = cnt;
    __syncthreads();
    if (tid == 0) {  // exclusive scan of at most 128 counts
      int run = 0;
      for (int i = 0; i < dec::kThreads; ++i) {
        const int v = cnt_s[i];
        cnt_s[i] = run;
        run += v;
      }
      n_tasks_s = run;
    }
    __syncthreads();
    if (tid < n_chunk) {
      const int bh = item / a.n_split;
      const float lse_bh = (a.gated && a.lse_s != nullptr) ? a.lse_s[bh] : 0.f;
      const int base = cnt_s[tid];
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
            lam = (a.s[size_t(bh) * NB + m] - lse_bh) * kLog2e;
          }
        }
        t_item[base + j] = item;
        t_m[base + j] = m;
        t_ntok[base + j] = ntok;
        t_lam[base + j] = lam;
        t_flags[base + j] = (j == 0 ? 1 : 0) | (j == cnt - 1 ? 2 : 0);
      }
    }
    __syncthreads();
    const int nt = n_tasks_s;

    auto issue = [&](int task) {
      const uint32_t st = ring + (task % STAGES) * STAGEB;
      const int it = t_item[task];
      const int bh = it / a.n_split;
      const int ntok = t_ntok[task];
      const size_t row0 = size_t(bh) * a.Lmax + size_t(t_m[task]) * kBlock;
      const uint16_t* kb = a.kc + row0 * D;
      const uint16_t* vb = a.vc + row0 * D;
      for (int i = tid; i < ntok * CH; i += dec::kThreads) {
        const int r = i / CH, ch = i % CH;
        cp_async16(st + r * ROWB + ch * 16, kb + size_t(r) * D + ch * 8);
        cp_async16(st + TILEB + r * ROWB + ch * 16, vb + size_t(r) * D + ch * 8);
      }
      const uint16_t* qb = a.q + size_t(bh) * G * D;
      for (int i = tid; i < G * CH; i += dec::kThreads) cp_async16(st + 2 * TILEB + i * 16, qb + i * 8);
    };

#pragma unroll
    for (int s = 0; s < STAGES - 1; ++s) {
      if (s < nt) issue(s);
      cp_async_commit();
    }
    for (int task = 0; task < nt; ++task) {
      if (task + STAGES - 1 < nt) issue(task + STAGES - 1);
      cp_async_commit();
      cp_async_wait<STAGES - 1>();
      __syncthreads();
      const uint32_t st = ring + (task % STAGES) * STAGEB;
      const int ntok = t_ntok[task];
      const float lam2 = t_lam[task];
      const int flags = t_flags[task];
      if (flags & 1) {
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[g][e] = 0.f;
      }
      // scores: half-warps own rows, 16 lanes per row, one 16-byte chunk each
      {
        const int hh = lane / LPR, cl = lane % LPR;
#pragma unroll 2
        for (int i = 0; i < 16 / RPW; ++i) {
          const int r = 16 * warp + RPW * i + hh;
          float kf[8];
          if (r < ntok) {
            unpack8(lds128(st + r * ROWB + cl * 16), kf);
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) kf[e] = 0.f;
          }
#pragma unroll
          for (int g = 0; g < G; ++g) {
            float qf[8];
            unpack8(lds128(st + 2 * TILEB + g * ROWB + cl * 16), qf);
            float dot = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) dot = fmaf(qf[e], kf[e], dot);
#pragma unroll
            for (int o = LPR / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
            if (cl == 0) sc_s[g][r] = (r < ntok) ? fmaf(dot, sc2, lam2) : -INFINITY;
          }
        }
      }
      __syncthreads();
      // online softmax per head (one warp per head)
      for (int g = warp; g < G; g += 4) {
        const float z0 = sc_s[g][lane], z1 = sc_s[g][lane + 32];
        const float m_old = (flags & 1) ? -INFINITY : m_s[g];
        const float m_new = fmaxf(m_old, warp_max(fmaxf(z0, z1)));
        const float p0 = (z0 == -INFINITY) ? 0.f : exp2f(z0 - m_new);
        const float p1 = (z1 == -INFINITY) ? 0.f : exp2f(z1 - m_new);
        const float bs = warp_sum(p0 + p1);
        sc_s[g][lane] = p0;
        sc_s[g][lane + 32] = p1;
        if (lane == 0) {
          const float alpha = (m_old == -INFINITY) ? 0.f : exp2f(m_old - m_new);
          a_s[g] = alpha;
          l_s[g] = ((flags & 1) ? 0.f : l_s[g]) * alpha + bs;
          m_s[g] = m_new;
        }
      }
      __syncthreads();
      // PV: 8 row groups of 16 lanes, one 16-byte chunk of d per lane
      {
        const int rg = tid / LPR, cl = tid % LPR;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float al = a_s[g];
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[g][e] *= al;
        }
        for (int r = rg; r < ntok; r += RG) {
          float vf[8];
          unpack8(lds128(st + TILEB + r * ROWB + cl * 16), vf);
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float pw = sc_s[g][r];
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[g][e] = fmaf(pw, vf[e], acc[g][e]);
          }
        }
      }
      if (flags & 2) {  // last block of the item: reduce the row groups and write the partial
        const int cl = tid % LPR;
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            float v = acc[g][e];
#pragma unroll
            for (int o = LPR; o < 32; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
            acc[g][e] = v;
          }
        if (lane < LPR) {
#pragma unroll
          for (int g = 0; g < G; ++g)
#pragma unroll
            for (int e = 0; e < 8; ++e) red_s[warp][g][cl * 8 + e] = acc[g][e];
        }
        __syncthreads();
        const int it = t_item[task];
        const int split = it % a.n_split, bh = it / a.n_split;
        for (int i = tid; i < G * D; i += dec::kThreads) {
          const int g = i / D, e = i % D;
          const float v = red_s[0][g][e] + red_s[1][g][e] + red_s[2][g][e] + red_s[3][g][e];
          const float l = l_s[g];
          a.o_part[((size_t(bh) * G + g) * a.n_split + split) * D + e] = (l > 0.f) ? v / l : 0.f;
        }
        if (tid < G) {
          const float l = l_s[tid];
          a.lse_part[(size_t(bh) * G + tid) * a.n_split + split] = (l > 0.f) ? (m_s[tid] + log2f(l)) * kLn2 : -INFINITY;
        }
      }
      __syncthreads();
    }
    cp_async_wait<0>();
    __syncthreads();
  }
}

template <int D>
__global__ void decode_combine_kernel(const float* __restrict__ o_part, const float* __restrict__ lse_part,
                                      int n_split, uint16_t* __restrict__ o, float* __restrict__ lse_o) {
  const size_t row = blockIdx.x;
  const float* lp = lse_part + row * n_split;
  float mx = -INFINITY;
  for (int j = 0; j < n_split; ++j) mx = fmaxf(mx, lp[j]);
  float den = 0.f;
  if (mx != -INFINITY)
    for (int j = 0; j < n_split; ++j) den += exp2f((lp[j] - mx) * kLog2e);
  const int e = threadIdx.x;
  float acc = 0.f;
  if (mx != -INFINITY) {
    for (int j = 0; j < n_split; ++j) {
      const float w = exp2f((lp[j] - mx) * kLog2e);
      if (w > 0.f) acc = fmaf(w, o_part[(row * n_split + j) * D + e], acc);
    }
    acc /= den;
  }
  const __nv_bfloat16 r = __float2bfloat16_rn(acc);
  o[row * D + e] = *reinterpret_cast<const uint16_t*>(&r);
  if (lse_o != nullptr && e == 0) lse_o[row] = (mx == -INFINITY) ? -INFINITY : mx + logf(den);
}

template <int D, int G>
static cudaError_t launch_decode_dg(const Shape& sh, const DecodeArgs& a, cudaStream_t st) {
  constexpr int STAGES = 3;
  constexpr int smem = STAGES * (2 * kBlock * D * 2 + G * D * 2);
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
  kern<<<grid, dec::kThreads, smem, st>>>(a);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_decode_d(const Shape& sh, const uint16_t* q, const uint16_t* kc, const uint16_t* vc,
                                   const int32_t* cl, const float* s, const int32_t* idx, const float* lse_s,
                                   int n_split, float* o_part, float* lse_part, int* err, cudaStream_t st) {
  DecodeArgs a;
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
  a.gated = sh.gated;
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
  if (sh.d == 128) return launch_decode_d<128>(sh, q, kc, vc, cl, s, idx, lse_s, n_split, o_part, lse_part, err, st);
  return launch_decode_d<64>(sh, q, kc, vc, cl, s, idx, lse_s, n_split, o_part, lse_part, err, st);
}

cudaError_t launch_decode_combine(const Shape& sh, int n_split, const float* o_part, const float* lse_part,
                                  uint16_t* o, float* lse_o, cudaStream_t st) {
  const int rows = sh.B * sh.Hq;
  if (sh.d == 128)
    decode_combine_kernel<128><<<rows, 128, 0, st>>>(o_part, lse_part, n_split, o, lse_o);
  else
    decode_combine_kernel<64><<<rows, 64, 0, st>>>(o_part, lse_part, n_split, o, lse_o);
  return cudaGetLastError();
}

}  // namespace sas
