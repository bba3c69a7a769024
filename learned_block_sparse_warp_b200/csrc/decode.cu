// Split-K single-token decode over the selected blocks, and the LSE merge.
//
// SAS explainer (ta-paperlens), section 仕組み: at inference the scores pick
// the Top-K history blocks and attention runs over them and the current block.
// Algorithm 2 adds no gate; SAS_GATE_LOG_SOFTMAX keeps the training-time gate.
// SAS summary (onedev.kr), section 전제와 한계: decode is the sparsified stage,
// and its attention cost stays flat as the context grows.
//
// The work is HBM-bound: every selected 64-token block is read once. One CTA
// covers one split of one (sequence, KV head). Its G query heads share every
// K/V load (GQA grouping). Each thread issues all of its 128-bit loads for a
// block before using any of them, so a CTA keeps 32 KB (d = 128) in flight.
#include "common.cuh"

namespace sas {

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

template <int D, int G>
__global__ void __launch_bounds__(256) decode_split_kernel(
    const uint16_t* __restrict__ q, const uint16_t* __restrict__ kc, const uint16_t* __restrict__ vc,
    const int32_t* __restrict__ cache_len, const float* __restrict__ s, const int32_t* __restrict__ idx,
    const float* __restrict__ lse_s, int Hkv, int Lmax, int K, float scale, int gated, int n_split,
    float* __restrict__ o_part, float* __restrict__ lse_part, int* err) {
  constexpr int CH = D / 8;         // 16-byte chunks per row
  constexpr int RP = 256 / CH;      // rows per pass
  constexpr int PASSES = kBlock / RP;
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int ch = tid % CH, rg = tid / CH;
  const int NB = Lmax / kBlock;

  __shared__ float q_s[G][D];
  __shared__ float p_s[G][kBlock];
  __shared__ float m_s[G], l_s[G], a_s[G];
  __shared__ int list_s[kMaxTopK + 1];
  __shared__ int nlist_s;
  __shared__ float red_s[RP][D];

  int L = cache_len[b];
  if (L < 1 || L > Lmax) {
    if (tid == 0) raise_error(err, SAS_ERR_DEVICE_INDEX);
    L = max(1, min(L, Lmax));
  }
  const int c = (L - 1) / kBlock;
  const size_t bh = size_t(b) * Hkv + h;

  // ordered block list: the current block, then the valid selected blocks
  if (warp == 0) {
    const int n = min(K, c);
    int cnt = 0;
    bool stop = false;
    for (int base = 0; base < n && !stop; base += 32) {
      const int k = base + lane;
      const int m = (k < n) ? idx[bh * K + k] : -1;
      const bool end = (k < n) && m < 0;
      const bool bad = (k < n) && m >= c;
      if (bad) raise_error(err, SAS_ERR_DEVICE_INDEX);
      const unsigned end_mask = __ballot_sync(0xffffffffu, end);
      const int first_end = end_mask ? __ffs(end_mask) - 1 : 32;
      const bool ok = (k < n) && !bad && m >= 0 && lane < first_end;
      const unsigned ok_mask = __ballot_sync(0xffffffffu, ok);
      if (ok) list_s[1 + cnt + __popc(ok_mask & ((1u << lane) - 1u))] = m;
      cnt += __popc(ok_mask);
      stop = end_mask != 0;
    }
    if (lane == 0) {
      list_s[0] = c;
      nlist_s = 1 + cnt;
    }
  }
  for (int i = tid; i < G * D; i += 256) {
    const int g = i / D, e = i % D;
    q_s[g][e] = bf16_to_f32(q[(bh * G + g) * D + e]);
  }
  if (tid < G) {
    m_s[tid] = -INFINITY;
    l_s[tid] = 0.f;
  }
  __syncthreads();

  const int nl = nlist_s;
  const int per = (nl + n_split - 1) / n_split;
  const int pos0 = min(split * per, nl), pos1 = min(pos0 + per, nl);
  const float lse_bh = (gated && lse_s != nullptr) ? lse_s[bh] : 0.f;
  const float sc2 = scale * kLog2e;

  float acc[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[g][e] = 0.f;

  for (int pos = pos0; pos < pos1; ++pos) {
    const int m = list_s[pos];
    const int ntok = (m == c) ? (L - c * kBlock) : kBlock;
    const float lam2 = (m != c && gated) ? (s[bh * NB + m] - lse_bh) * kLog2e : 0.f;
    const uint16_t* kb = kc + (bh * Lmax + size_t(m) * kBlock) * D;
    const uint16_t* vb = vc + (bh * Lmax + size_t(m) * kBlock) * D;
    uint4 kr[PASSES], vr[PASSES];
#pragma unroll
    for (int p = 0; p < PASSES; ++p) {
      const int row = p * RP + rg;
      if (row < ntok) {
        kr[p] = ld_stream_v4(kb + size_t(row) * D + ch * 8);
        vr[p] = ld_stream_v4(vb + size_t(row) * D + ch * 8);
      } else {
        kr[p] = make_uint4(0, 0, 0, 0);
        vr[p] = make_uint4(0, 0, 0, 0);
      }
    }
    // scores of the G heads for this block's tokens (log2 domain)
#pragma unroll
    for (int p = 0; p < PASSES; ++p) {
      const int row = p * RP + rg;
      float kf[8];
      unpack8(kr[p], kf);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float dot = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) dot = fmaf(q_s[g][ch * 8 + e], kf[e], dot);
#pragma unroll
        for (int o = CH / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
        if (ch == 0) p_s[g][row] = (row < ntok) ? fmaf(dot, sc2, lam2) : -INFINITY;
      }
    }
    __syncthreads();
    // online softmax update, one warp per head
    for (int g = warp; g < G; g += 8) {
      const float z0 = p_s[g][lane], z1 = p_s[g][lane + 32];
      const float bm = warp_max(fmaxf(z0, z1));
      const float m_old = m_s[g];
      const float m_new = fmaxf(m_old, bm);
      const float p0 = exp2f(z0 - m_new), p1 = exp2f(z1 - m_new);
      const float bs = warp_sum(p0 + p1);
      p_s[g][lane] = p0;
      p_s[g][lane + 32] = p1;
      __syncwarp();
      if (lane == 0) {
        const float alpha = exp2f(m_old - m_new);
        a_s[g] = alpha;
        l_s[g] = l_s[g] * alpha + bs;
        m_s[g] = m_new;
      }
    }
    __syncthreads();
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float alpha = a_s[g];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[g][e] *= alpha;
    }
#pragma unroll
    for (int p = 0; p < PASSES; ++p) {
      const int row = p * RP + rg;
      float vf[8];
      unpack8(vr[p], vf);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float pw = p_s[g][row];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[g][e] = fmaf(pw, vf[e], acc[g][e]);
      }
    }
    __syncthreads();
  }

  // reduce the RP row groups and write the split's normalised partial
  for (int g = 0; g < G; ++g) {
#pragma unroll
    for (int e = 0; e < 8; ++e) red_s[rg][ch * 8 + e] = acc[g][e];
    __syncthreads();
    const size_t row = (bh * G + g) * size_t(n_split) + split;
    const float l = l_s[g];
    for (int e = tid; e < D; e += 256) {
      float v = 0.f;
#pragma unroll 4
      for (int r = 0; r < RP; ++r) v += red_s[r][e];
      o_part[row * D + e] = (l > 0.f) ? v / l : 0.f;
    }
    if (tid == 0) lse_part[row] = (l > 0.f) ? (m_s[g] + log2f(l)) * kLn2 : -INFINITY;
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

template <int D>
static cudaError_t launch_decode_d(const Shape& sh, const uint16_t* q, const uint16_t* kc, const uint16_t* vc,
                                   const int32_t* cl, const float* s, const int32_t* idx, const float* lse_s,
                                   int n_split, float* o_part, float* lse_part, int* err, cudaStream_t st) {
  dim3 grid(n_split, sh.Hkv, sh.B);
#define SAS_DEC(GG)                                                                                          \
  case GG:                                                                                                   \
    decode_split_kernel<D, GG><<<grid, 256, 0, st>>>(q, kc, vc, cl, s, idx, lse_s, sh.Hkv, sh.N, sh.K,       \
                                                     sh.scale, sh.gated, n_split, o_part, lse_part, err);    \
    break;
  switch (sh.G) {
    SAS_DEC(1)
    SAS_DEC(2)
    SAS_DEC(3)
    SAS_DEC(4)
    SAS_DEC(5)
    SAS_DEC(6)
    SAS_DEC(7)
    SAS_DEC(8)
    default:
      return cudaErrorInvalidValue;
  }
#undef SAS_DEC
  return cudaGetLastError();
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
