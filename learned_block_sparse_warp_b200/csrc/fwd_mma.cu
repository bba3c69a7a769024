// Gated block-sparse attention forward, warp-level tensor-core version.
//
// SAS explainer (ta-paperlens), section 仕組み, Eq. (9):
//   o = softmax(q K_Sᵀ + log g_S) V_S,  S = B0 ∪ ⋃_{m∈I} B_m,
// with the gate log g_m = s_m − LSE(s) (SAS summary, onedev.kr, section
// 무엇과 다른가) added to every logit of block m and 0 on the current block.
//
// One CTA of four warps owns one (batch, query head, query block): 64 query
// rows, 16 per warp. The block list [t, I_t...] is walked once. Each selected
// block's K and V rows are gathered by index with cp.async into a
// double-buffered, XOR-swizzled shared tile. QKᵀ and PV run on mma.sync
// m16n8k16 (bf16 in, fp32 accumulate). The per-block gate is one scalar add
// in the online-softmax update. The probabilities stay in registers and feed
// PV directly as the A operand.
#include "common.cuh"

namespace sas {

template <int D>
__device__ __forceinline__ void load_tile_async(uint32_t s_base, const uint16_t* __restrict__ g, int tid,
                                                int nthreads) {
  constexpr int CH = D / 8;
  for (int i = tid; i < kBlock * CH; i += nthreads) {
    const int r = i / CH, c = i % CH;
    cp_async16(s_base + swz<CH>(r, c), g + size_t(r) * D + c * 8);
  }
}

template <int D>
__global__ void __launch_bounds__(128) fwd_mma_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                                                      const uint16_t* __restrict__ v, const float* __restrict__ s,
                                                      const int32_t* __restrict__ idx,
                                                      const float* __restrict__ lse_s, uint16_t* __restrict__ o,
                                                      float* __restrict__ lse_o, Shape sh, int* err) {
  constexpr int CH = D / 8;
  constexpr int TILE = kBlock * D * 2;  // bytes of one 64 x D bf16 tile
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int list_s[kMaxTopK + 1];
  __shared__ float lam_s[kMaxTopK + 1];
  __shared__ int nlist_s;

  const int t = sh.NB - 1 - int(blockIdx.x);  // heavy query blocks first
  const int hq = blockIdx.y, b = blockIdx.z;
  const int h = hq / sh.G;
  const size_t bh = size_t(b) * sh.Hkv + h;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sK = sQ + TILE;
  const uint32_t sV = sK + 2 * TILE;

  if (warp == 0) {
    const size_t row = bh * sh.NB + t;
    build_block_list(idx + row * sh.K, sh.K, t, sh.gated ? s + row * sh.NB : nullptr,
                     lse_s != nullptr ? lse_s[row] : 0.f, sh.gate, list_s, lam_s, &nlist_s, err);
  }
  const uint16_t* qg = q + ((size_t(b) * sh.Hq + hq) * sh.N + size_t(t) * kBlock) * D;
  const uint16_t* kg = k + bh * size_t(sh.N) * D;
  const uint16_t* vg = v + bh * size_t(sh.N) * D;
  load_tile_async<D>(sQ, qg, tid, 128);
  __syncthreads();
  const int nl = nlist_s;
  load_tile_async<D>(sK, kg + size_t(list_s[0]) * kBlock * D, tid, 128);
  load_tile_async<D>(sV, vg + size_t(list_s[0]) * kBlock * D, tid, 128);
  cp_async_commit();

  float oacc[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  const float sc2 = sh.scale * kLog2e;
  const int ra = 16 * warp + (lane >> 2);  // this thread's rows: ra and ra + 8

  for (int i = 0; i < nl; ++i) {
    if (i + 1 < nl) {
      const int st = (i + 1) & 1;
      const size_t off = size_t(list_s[i + 1]) * kBlock * D;
      load_tile_async<D>(sK + st * TILE, kg + off, tid, 128);
      load_tile_async<D>(sV + st * TILE, vg + off, tid, 128);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const uint32_t cK = sK + (i & 1) * TILE, cV = sV + (i & 1) * TILE;

    // S = Q Kᵀ for this warp's 16 rows x 64 keys
    float sacc[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) sacc[j][0] = sacc[j][1] = sacc[j][2] = sacc[j][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t a[4];
      ldsm_x4(sQ + swz<CH>(16 * warp + (lane & 15), 2 * kk + (lane >> 4)), a[0], a[1], a[2], a[3]);
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(cK + swz<CH>(16 * np + (lane & 7) + ((lane >> 4) << 3), 2 * kk + ((lane >> 3) & 1)), b0, b1, b2, b3);
        mma_bf16_16816(sacc[2 * np], a, b0, b1);
        mma_bf16_16816(sacc[2 * np + 1], a, b2, b3);
      }
    }
    // gated logits in the log2 domain; causal mask on the current block. The gate
    // outside the softmax leaves the logits plain and weights P·V by g instead.
    const float lam2 = sh.outside ? 0.f : lam_s[i];
    const float gw = sh.outside ? exp2f(lam_s[i]) : 1.f;
    const bool diag = (i == 0);
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int col = 8 * j + 2 * (lane & 3) + (e & 1);
        const int row = ra + ((e >> 1) << 3);
        float z = fmaf(sacc[j][e], sc2, lam2);
        if (diag && col > row) z = -INFINITY;
        sacc[j][e] = z;
        mx[e >> 1] = fmaxf(mx[e >> 1], z);
      }
    }
    float alpha[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
      const float m_new = fmaxf(m_run[r], mx[r]);
      alpha[r] = exp2f(m_run[r] - m_new);
      m_run[r] = m_new;
    }
    float rs[2] = {0.f, 0.f};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float p = exp2f(sacc[j][e] - m_run[e >> 1]);
        sacc[j][e] = p;
        rs[e >> 1] += p;
      }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) l_run[r] = l_run[r] * alpha[r] + rs[r];
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
      oacc[j][0] *= alpha[0];
      oacc[j][1] *= alpha[0];
      oacc[j][2] *= alpha[1];
      oacc[j][3] *= alpha[1];
    }
    // O += P V
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t a[4];
      a[0] = pack_bf16x2(sacc[2 * kk][0] * gw, sacc[2 * kk][1] * gw);
      a[1] = pack_bf16x2(sacc[2 * kk][2] * gw, sacc[2 * kk][3] * gw);
      a[2] = pack_bf16x2(sacc[2 * kk + 1][0] * gw, sacc[2 * kk + 1][1] * gw);
      a[3] = pack_bf16x2(sacc[2 * kk + 1][2] * gw, sacc[2 * kk + 1][3] * gw);
#pragma unroll
      for (int dp = 0; dp < D / 16; ++dp) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(cV + swz<CH>(16 * kk + (lane & 7) + (((lane >> 3) & 1) << 3), 2 * dp + (lane >> 4)), b0, b1, b2,
                  b3);
        mma_bf16_16816(oacc[2 * dp], a, b0, b1);
        mma_bf16_16816(oacc[2 * dp + 1], a, b2, b3);
      }
    }
    __syncthreads();
  }

  // epilogue: normalise, stage the bf16 tile in shared memory, store coalesced
  float inv[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    float l = l_run[r];
    l += __shfl_xor_sync(0xffffffffu, l, 1);
    l += __shfl_xor_sync(0xffffffffu, l, 2);
    inv[r] = 1.f / l;
    if (lse_o != nullptr && (lane & 3) == 0)
      lse_o[(size_t(b) * sh.Hq + hq) * sh.N + size_t(t) * kBlock + ra + 8 * r] = (m_run[r] + log2f(l)) * kLn2;
  }
#pragma unroll
  for (int j = 0; j < D / 8; ++j) {
    const int col = 8 * j + 2 * (lane & 3);
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int row = ra + 8 * r;
      const uint32_t val = pack_bf16x2(oacc[j][2 * r] * inv[r], oacc[j][2 * r + 1] * inv[r]);
      const uint32_t addr = sQ + swz<CH>(row, col >> 3) + (col & 7) * 2;
      asm volatile("st.shared.b32 [%0], %1;\n" ::"r"(addr), "r"(val));
    }
  }
  __syncthreads();
  uint16_t* og = o + ((size_t(b) * sh.Hq + hq) * sh.N + size_t(t) * kBlock) * D;
  for (int i = tid; i < kBlock * CH; i += 128) {
    const int r = i / CH, c = i % CH;
    uint4 val;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(val.x), "=r"(val.y), "=r"(val.z), "=r"(val.w)
                 : "r"(sQ + swz<CH>(r, c)));
    *reinterpret_cast<uint4*>(og + size_t(r) * D + c * 8) = val;
  }
}

template <int D>
static cudaError_t launch_fwd_d(const Shape& sh, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                const float* s, const int32_t* idx, const float* lse_s, uint16_t* o, float* lse_o,
                                int* err, cudaStream_t st) {
  const int smem = 5 * kBlock * D * 2;
  cudaError_t e = cudaFuncSetAttribute(fwd_mma_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(sh.NB, sh.Hq, sh.B);
  fwd_mma_kernel<D><<<grid, 128, smem, st>>>(q, k, v, s, idx, lse_s, o, lse_o, sh, err);
  return cudaGetLastError();
}

cudaError_t launch_fwd_mma(const Shape& sh, const uint16_t* q, const uint16_t* k, const uint16_t* v, const float* s,
                           const int32_t* idx, const float* lse_s, uint16_t* o, float* lse_o, int* err,
                           cudaStream_t st) {
  if (sh.d == 128) return launch_fwd_d<128>(sh, q, k, v, s, idx, lse_s, o, lse_o, err, st);
  return launch_fwd_d<64>(sh, q, k, v, s, idx, lse_s, o, lse_o, err, st);
}

}  // namespace sas
