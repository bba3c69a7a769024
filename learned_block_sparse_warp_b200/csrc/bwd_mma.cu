// Backward of gated block-sparse attention, with the gate/score gradient.
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
//   bwd_main         one CTA per (batch, KV head, KV block j), eight warps.
//                    It walks its diagonal query block and then every query
//                    block that selected j, for each of the G heads, and
//                    recomputes P from the saved row LSE. dK_j and dV_j stay
//                    in registers for the whole walk. dQ is added to an fp32
//                    workspace with red.global. dl[t, slot] has exactly one
//                    writer, the CTA that owns j, so the score path uses no
//                    atomics.
//   bwd_dq_convert   fp32 dQ -> bf16
//   bwd_ds_chain     ds from dl through the softmax over s
#include <algorithm>

#include "common.cuh"

namespace sas {

struct BwdWs {
  float* dq_acc;   // [B, Hq, N, d] fp32 (d = 64 path only)
  float* drow;     // [B, Hq, N]
  float* dl;       // [B, Hkv, NB, K]
  int* rev_cnt;    // [B, Hkv, NB]
  int* rev_off;    // [B, Hkv, NB + 1]
  int* rev_list;   // [B, Hkv, NB * K]: (t << kSlotBits) | slot
  float* rev_lam;  // [B, Hkv, NB * K]: log2-domain gate of each reverse-index entry
  uint16_t* dz;    // d = 128 with spill: [B, Hkv, Σ_t (1 + min(K, t)), ceil(G/2)] tiles of 128 x 64 bf16
};

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

long long bwd_dz_tiles(const Shape& sh);

// The stored-dZ backward needs one 16 KB tile per (query block, attended block,
// head pair); its tile index must fit a TMA coordinate.
bool bwd_can_spill(const Shape& sh) { return sh.d == 128 && bwd_dz_tiles(sh) < (1LL << 31); }

size_t bwd_ws_layout(const Shape& sh, bool spill, void* base, BwdWs* ws) {
  const size_t bhq = size_t(sh.B) * sh.Hq, bhk = size_t(sh.B) * sh.Hkv;
  size_t off = 0;
  size_t o_dq = off;
  if (sh.d != 128) off = align256(off + bhq * sh.N * sh.d * sizeof(float));
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
  size_t o_dz = off;
  if (spill) off = align256(off + size_t(bwd_dz_tiles(sh)) * 128 * 64 * sizeof(uint16_t));
  if (ws != nullptr) {
    char* p = static_cast<char*>(base);
    ws->dq_acc = sh.d != 128 ? reinterpret_cast<float*>(p + o_dq) : nullptr;
    ws->drow = reinterpret_cast<float*>(p + o_dr);
    ws->dl = reinterpret_cast<float*>(p + o_dl);
    ws->rev_cnt = reinterpret_cast<int*>(p + o_cnt);
    ws->rev_off = reinterpret_cast<int*>(p + o_off);
    ws->rev_list = reinterpret_cast<int*>(p + o_list);
    ws->rev_lam = reinterpret_cast<float*>(p + o_lam);
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

// ---------------------------------------------------------------------------
// Main backward kernel
// ---------------------------------------------------------------------------
template <int D>
__device__ __forceinline__ void bwd_load_tile(uint32_t s_base, const uint16_t* __restrict__ g, int tid) {
  constexpr int CH = D / 8;
  for (int i = tid; i < kBlock * CH; i += 256) {
    const int r = i / CH, c = i % CH;
    cp_async16(s_base + swz<CH>(r, c), g + size_t(r) * D + c * 8);
  }
}

__device__ __forceinline__ void st_shared_b32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.b32 [%0], %1;\n" ::"r"(addr), "r"(v));
}

__device__ __forceinline__ void red_add_f32x2(float* p, float a, float b) {
  asm volatile("red.global.add.v2.f32 [%0], {%1, %2};\n" ::"l"(p), "f"(a), "f"(b) : "memory");
}

template <int D>
__global__ void __launch_bounds__(256, 1) bwd_main_kernel(
    const uint16_t* __restrict__ q, const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
    const uint16_t* __restrict__ dO, const float* __restrict__ s, const float* __restrict__ lse_s,
    const float* __restrict__ lse_o, const float* __restrict__ drow, const int* __restrict__ rev_off,
    const int* __restrict__ rev_list, float* __restrict__ dq_acc, float* __restrict__ dl, uint16_t* __restrict__ dk,
    uint16_t* __restrict__ dv, Shape sh) {
  constexpr int CH = D / 8;
  constexpr int TILE = kBlock * D * 2;
  constexpr int PT = kBlock * kBlock * 2;  // 64 x 64 bf16
  constexpr int NT = D / 16;               // 8-wide d tiles per warp (half of D)
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(16) float sL[2][kBlock];
  __shared__ __align__(16) float sD[2][kBlock];
  __shared__ float sdl[8];

  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const size_t bh = size_t(b) * sh.Hkv + h;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wm = warp & 3, wn = warp >> 2;
  const uint32_t sK = smem_u32(smem);
  const uint32_t sV = sK + TILE;
  const uint32_t sQ = sV + TILE;       // 2 stages
  const uint32_t sdO = sQ + 2 * TILE;  // 2 stages
  const uint32_t sP = sdO + 2 * TILE;
  const uint32_t sZ = sP + PT;
  const int G = sh.G;

  const int off0 = rev_off[bh * (sh.NB + 1) + j];
  const int n_sel = rev_off[bh * (sh.NB + 1) + j + 1] - off0;
  const int* lst = rev_list + bh * size_t(sh.NB) * sh.K + off0;
  const int n_steps = (1 + n_sel) * G;

  auto step_t = [&](int e) -> int { return e == 0 ? j : (lst[e - 1] >> kSlotBits); };
  auto issue_step = [&](int st, int stage) {
    const int e = st / G, g = st % G;
    const int t = step_t(e);
    const int hq = h * G + g;
    const size_t rowbase = (size_t(b) * sh.Hq + hq) * sh.N + size_t(t) * kBlock;
    bwd_load_tile<D>(sQ + stage * TILE, q + rowbase * D, tid);
    bwd_load_tile<D>(sdO + stage * TILE, dO + rowbase * D, tid);
    if (tid < 16) cp_async16(smem_u32(&sL[stage][tid * 4]), lse_o + rowbase + tid * 4);
    else if (tid < 32) cp_async16(smem_u32(&sD[stage][(tid - 16) * 4]), drow + rowbase + (tid - 16) * 4);
  };

  const uint16_t* kg = k + (bh * sh.N + size_t(j) * kBlock) * D;
  const uint16_t* vg = v + (bh * sh.N + size_t(j) * kBlock) * D;
  bwd_load_tile<D>(sK, kg, tid);
  bwd_load_tile<D>(sV, vg, tid);
  issue_step(0, 0);
  cp_async_commit();

  float dk_acc[NT][4], dv_acc[NT][4];
#pragma unroll
  for (int i = 0; i < NT; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk_acc[i][e] = dv_acc[i][e] = 0.f;
  float dl_part = 0.f;
  const float sc2 = sh.scale * kLog2e;
  const int ra = 16 * wm + (lane >> 2);  // this thread's S rows: ra, ra + 8
  const int ca = 32 * wn;                // this warp's S columns: ca .. ca + 31

  for (int st = 0; st < n_steps; ++st) {
    const int stage = st & 1;
    if (st + 1 < n_steps) {
      issue_step(st + 1, stage ^ 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const int e = st / G, g = st % G;
    const int t = step_t(e);
    const int slot = e == 0 ? -1 : (lst[e - 1] & ((1 << kSlotBits) - 1));
    const bool diag = (e == 0);
    float lam2 = 0.f;
    if (!diag && sh.gated) {
      const size_t row = bh * sh.NB + t;
      lam2 = gate_lam2(sh.gate, s[row * sh.NB + j], lse_s != nullptr ? lse_s[row] : 0.f);
    }
    const uint32_t cQ = sQ + stage * TILE, cdO = sdO + stage * TILE;
    // Gate inside the softmax: log2 g biases the logits. Outside: the logits are
    // plain, v carries the weight g·p, so dV takes g·p, dZ = p·(g·dP − D), and
    // dl = Σ p·g·dP (= g ∂/∂g).
    const float zb = sh.outside ? 0.f : lam2;
    const float gw = sh.outside ? exp2f(lam2) : 1.f;

    // S = Q Kᵀ and dP = dO Vᵀ for rows 16wm.., columns 32wn..
    float sacc[4][4], pacc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int c = 0; c < 4; ++c) sacc[i][c] = pacc[i][c] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t a[4], ad[4];
      ldsm_x4(cQ + swz<CH>(16 * wm + (lane & 15), 2 * kk + (lane >> 4)), a[0], a[1], a[2], a[3]);
      ldsm_x4(cdO + swz<CH>(16 * wm + (lane & 15), 2 * kk + (lane >> 4)), ad[0], ad[1], ad[2], ad[3]);
#pragma unroll
      for (int np = 0; np < 2; ++np) {
        const int brow = ca + 16 * np + (lane & 7) + ((lane >> 4) << 3);
        const int bch = 2 * kk + ((lane >> 3) & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(sK + swz<CH>(brow, bch), b0, b1, b2, b3);
        mma_bf16_16816(sacc[2 * np], a, b0, b1);
        mma_bf16_16816(sacc[2 * np + 1], a, b2, b3);
        ldsm_x4(sV + swz<CH>(brow, bch), b0, b1, b2, b3);
        mma_bf16_16816(pacc[2 * np], ad, b0, b1);
        mma_bf16_16816(pacc[2 * np + 1], ad, b2, b3);
      }
    }
    // P and dZ, stored to shared memory as bf16; dl partial sum in fp32
    {
      const float L0 = sL[stage][ra] * kLog2e, L1 = sL[stage][ra + 8] * kLog2e;
      const float D0 = sD[stage][ra], D1 = sD[stage][ra + 8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int col = ca + 8 * i + 2 * (lane & 3);
        float p[4], z[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int row = ra + ((c >> 1) << 3);
          const int cc = col + (c & 1);
          const float Lr = (c >> 1) ? L1 : L0;
          const float Dr = (c >> 1) ? D1 : D0;
          float pv = exp2f(fmaf(sacc[i][c], sc2, zb) - Lr);
          if (diag && cc > row) pv = 0.f;
          const float gdp = gw * pacc[i][c];
          p[c] = pv * gw;
          z[c] = pv * (gdp - Dr);
          dl_part += sh.outside ? pv * gdp : z[c];
        }
        st_shared_b32(sP + swz<8>(ra, col >> 3) + (col & 7) * 2, pack_bf16x2(p[0], p[1]));
        st_shared_b32(sP + swz<8>(ra + 8, col >> 3) + (col & 7) * 2, pack_bf16x2(p[2], p[3]));
        st_shared_b32(sZ + swz<8>(ra, col >> 3) + (col & 7) * 2, pack_bf16x2(z[0], z[1]));
        st_shared_b32(sZ + swz<8>(ra + 8, col >> 3) + (col & 7) * 2, pack_bf16x2(z[2], z[3]));
      }
    }
    const bool last_head = (g == G - 1);
    if (last_head && !diag) {
      const float w = warp_sum(dl_part);
      if (lane == 0) sdl[warp] = w;
    }
    __syncthreads();

    // dV += Pᵀ dO and dK += dZᵀ Q: rows = KV tokens 16wm.., cols = d (D/2)wn..
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t ap[4], az[4];
      const int arow = 16 * kk + (lane & 7) + ((lane >> 4) << 3);
      const int ach = 2 * wm + ((lane >> 3) & 1);
      ldsm_x4_t(sP + swz<8>(arow, ach), ap[0], ap[1], ap[2], ap[3]);
      ldsm_x4_t(sZ + swz<8>(arow, ach), az[0], az[1], az[2], az[3]);
#pragma unroll
      for (int dp = 0; dp < NT / 2; ++dp) {
        const int brow = 16 * kk + (lane & 7) + (((lane >> 3) & 1) << 3);
        const int bch = (D / 16) * wn + 2 * dp + (lane >> 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(cdO + swz<CH>(brow, bch), b0, b1, b2, b3);
        mma_bf16_16816(dv_acc[2 * dp], ap, b0, b1);
        mma_bf16_16816(dv_acc[2 * dp + 1], ap, b2, b3);
        ldsm_x4_t(cQ + swz<CH>(brow, bch), b0, b1, b2, b3);
        mma_bf16_16816(dk_acc[2 * dp], az, b0, b1);
        mma_bf16_16816(dk_acc[2 * dp + 1], az, b2, b3);
      }
    }
    // dQ = scale · dZ K: rows = queries 16wm.., cols = d (D/2)wn..
    {
      float qacc[NT][4];
#pragma unroll
      for (int i = 0; i < NT; ++i) qacc[i][0] = qacc[i][1] = qacc[i][2] = qacc[i][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        uint32_t a[4];
        ldsm_x4(sZ + swz<8>(16 * wm + (lane & 15), 2 * kk + (lane >> 4)), a[0], a[1], a[2], a[3]);
#pragma unroll
        for (int dp = 0; dp < NT / 2; ++dp) {
          const int brow = 16 * kk + (lane & 7) + (((lane >> 3) & 1) << 3);
          const int bch = (D / 16) * wn + 2 * dp + (lane >> 4);
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(sK + swz<CH>(brow, bch), b0, b1, b2, b3);
          mma_bf16_16816(qacc[2 * dp], a, b0, b1);
          mma_bf16_16816(qacc[2 * dp + 1], a, b2, b3);
        }
      }
      const int hq = h * G + g;
      float* dqb = dq_acc + ((size_t(b) * sh.Hq + hq) * sh.N + size_t(t) * kBlock) * D;
#pragma unroll
      for (int i = 0; i < NT; ++i) {
        const int col = (D / 2) * wn + 8 * i + 2 * (lane & 3);
        red_add_f32x2(dqb + size_t(ra) * D + col, qacc[i][0] * sh.scale, qacc[i][1] * sh.scale);
        red_add_f32x2(dqb + size_t(ra + 8) * D + col, qacc[i][2] * sh.scale, qacc[i][3] * sh.scale);
      }
    }
    __syncthreads();
    if (last_head) {
      if (!diag && sh.gated && tid == 0) {
        float w = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) w += sdl[i];
        dl[(bh * sh.NB + t) * sh.K + slot] = w;
      }
      dl_part = 0.f;
    }
  }

  // dK (scaled) and dV of block j, summed over the G heads
  uint16_t* dkg = dk + (bh * sh.N + size_t(j) * kBlock) * D;
  uint16_t* dvg = dv + (bh * sh.N + size_t(j) * kBlock) * D;
#pragma unroll
  for (int i = 0; i < NT; ++i) {
    const int col = (D / 2) * wn + 8 * i + 2 * (lane & 3);
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int row = ra + 8 * r;
      *reinterpret_cast<uint32_t*>(dkg + size_t(row) * D + col) =
          pack_bf16x2(dk_acc[i][2 * r] * sh.scale, dk_acc[i][2 * r + 1] * sh.scale);
      *reinterpret_cast<uint32_t*>(dvg + size_t(row) * D + col) = pack_bf16x2(dv_acc[i][2 * r], dv_acc[i][2 * r + 1]);
    }
  }
}

// ---------------------------------------------------------------------------
// Epilogues
// ---------------------------------------------------------------------------
__global__ void bwd_dq_convert_kernel(const float4* __restrict__ acc, size_t n4, uint2* __restrict__ out) {
  for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += size_t(gridDim.x) * blockDim.x) {
    const float4 a = acc[i];
    out[i] = make_uint2(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w));
  }
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
  revidx_count_kernel<<<(nw + 7) / 8, 256, 0, st>>>(idx, nbh, sh.NB, sh.K, ws.rev_cnt);
  revidx_scan_kernel<<<nbh, 32, 0, st>>>(ws.rev_cnt, sh.NB, ws.rev_off);
  revidx_fill_kernel<<<(nw + 7) / 8, 256, 0, st>>>(idx, nbh, sh.NB, sh.K, ws.rev_off, ws.rev_list, s, lse_s,
                                                    sh.gate, D == 128 ? ws.rev_lam : nullptr);
  if (D == 128) {  // tcgen05 passes: dK/dV/dl (and the dZ tiles) KV-major, then dQ query-major
    if ((e = launch_bwd_passes_sm100(sh, q, k, v, dO, s, idx, lse_s, lse_o, ws.drow, ws.rev_off, ws.rev_list,
                                     ws.rev_lam, ws.dl, ws.dz, dq, dk, dv, err, st)) != cudaSuccess)
      return e;
    if (ds != nullptr) {
      const int rows = nbh * sh.NB;
      bwd_ds_chain_kernel<<<(rows + 7) / 8, 256, 0, st>>>(s, lse_s, idx, ws.dl, rows, sh.NB, sh.K, sh.gate, ds);
    }
    return cudaGetLastError();
  }
  if ((e = cudaMemsetAsync(ws.dq_acc, 0, rows_q * D * sizeof(float), st)) != cudaSuccess) return e;
  const int smem = 6 * kBlock * D * 2 + 2 * kBlock * kBlock * 2;
  if ((e = cudaFuncSetAttribute(bwd_main_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=
      cudaSuccess)
    return e;
  bwd_main_kernel<D><<<dim3(sh.NB, sh.Hkv, sh.B), 256, smem, st>>>(q, k, v, dO, s, lse_s, lse_o, ws.drow, ws.rev_off,
                                                                   ws.rev_list, ws.dq_acc, ws.dl, dk, dv, sh);
  const size_t n4 = rows_q * D / 4;
  bwd_dq_convert_kernel<<<148 * 8, 256, 0, st>>>(reinterpret_cast<const float4*>(ws.dq_acc), n4,
                                                  reinterpret_cast<uint2*>(dq));
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
  return launch_bwd_d<64>(sh, q, k, v, o, dO, s, idx, lse_s, lse_o, dq, dk, dv, ds, ws, false, err, st);
}

}  // namespace sas
