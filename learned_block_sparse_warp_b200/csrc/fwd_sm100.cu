// Gated block-sparse attention forward on the Blackwell tensor cores.
//
// SAS explainer (ta-paperlens), section 仕組み, Eq. (9):
//   o = softmax(q K_Sᵀ + log g_S) V_S,  S = B0 ∪ ⋃_{m∈I} B_m,
// with log g_m = s_m − LSE(s) (SAS summary, onedev.kr, section 무엇과 다른가)
// on every logit of history block m and 0 on the causally masked current
// block B0.
//
// One CTA owns one (batch, KV head, query block) and up to four query heads
// of the group. That is 256 rows, packed as two M = 128 tiles of two heads
// each, so every gathered K/V block serves four heads (GQA packing). Roles:
//   warp 0       builds the block list [t, I_t...], then issues TMA loads:
//                the Q rows once, then the selected K/V blocks two at a time
//                (N = 128) into a 2-stage shared-memory ring. Blocks are
//                gathered by index with no copy in HBM.
//   warp 1       allocates 512 TMEM columns and issues every tcgen05.mma:
//                S_r = Q_r Kᵀ (SS, fp32 in TMEM), then O_r += P_r V (TS:
//                P_r read from TMEM).
//   warps 4-7    softmax of tile 0; warps 8-11 softmax of tile 1. Each thread
//                owns one row: it reads S from TMEM, adds the block's
//                log-gate (one scalar per 64 columns), masks the current
//                block causally, updates the row max and sum, and writes
//                bf16 P back over the consumed S columns. O is rescaled in
//                TMEM only when the row max grows by more than 2^8, so the
//                result is exact and rescales are rare.
// TMEM: S0 [0,128), S1 [128,256), O0 [256,384), O1 [384,512).
// Every mbarrier wait is bounded and raises SAS_ERR_TIMEOUT instead of hanging.
#include <mutex>

#include "sm100.cuh"

namespace sas {

namespace fsm {
constexpr int kThreads = 384;                    // 0 TMA, 1 and 3 MMA (one per tile), 4-11 softmax
constexpr int kStages = 2;
constexpr int kHalf = 128 * 128;                 // one d-half of a 128-row tile: 128 rows x 128 B
constexpr int kQBytes = 4 * kHalf;               // 2 tiles x 2 d-halves
constexpr int kStageBytes = 4 * kHalf;           // K and V, 2 d-halves each, 128 token rows
constexpr int kSmemBytes = kQBytes + kStages * kStageBytes + 1024;  // + room to align to 1 KB
constexpr float kRescale = 8.0f;                 // log2 headroom before O is rescaled
}  // namespace fsm

struct FwdSm100Args {
  const int32_t* idx;
  const float* s;
  const float* lse_s;
  uint16_t* o;
  float* lse_o;
  int* err;
  int B, Hq, Hkv, G, N, NB, K, gate, gated, n_tp;
  float scale;
};

// kOut: the gate weights the values after a softmax over the plain logits
// (SAS_GATE_SOFTMAX_OUTSIDE) instead of entering the logits as log g.
template <bool kOut>
__global__ void __launch_bounds__(fsm::kThreads, 1)
    fwd_sm100_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, FwdSm100Args a) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  __shared__ int list_s[kMaxTopK + 1];
  __shared__ float lam_s[kMaxTopK + 1];
  __shared__ int nlist_s;
  // bar_turn[r]: tile r's softmax may run its exponentials. The two tiles take
  // turns, so one tile's exponentials overlap the other tile's MMAs instead of
  // both contending for the SM's exponential units at once.
  // bar_p[r] / bar_pb[r]: tile r's P of the pair's first / second 64-column block is in TMEM,
  // so the PV of the first block starts while the second block's exponentials run.
  __shared__ __align__(8) uint64_t bar_q, bar_full[fsm::kStages], bar_empty[fsm::kStages], bar_s[2], bar_p[2],
      bar_pb[2], bar_o[2], bar_fin, bar_turn[2];
  __shared__ uint32_t tmem_s;
  __shared__ int abort_s;

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sQ = base, sKV = base + fsm::kQBytes;
  const int t = a.NB - 1 - int(blockIdx.x);
  const int h = int(blockIdx.y) / a.n_tp, tp = int(blockIdx.y) % a.n_tp;
  const int b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g_first = 4 * tp;
  const int n_heads = min(4, a.G - g_first);
  const int n_tiles = (n_heads + 1) / 2;
  const size_t bh = size_t(b) * a.Hkv + h;
  volatile int* abort_flag = &abort_s;

  if (threadIdx.x == 0) abort_s = 0;
  if (warp == 0) {
    const size_t row = bh * a.NB + t;
    build_block_list(a.idx + row * a.K, a.K, t, a.gated ? a.s + row * a.NB : nullptr,
                     a.lse_s != nullptr ? a.lse_s[row] : 0.f, a.gate, list_s, lam_s, &nlist_s, a.err);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_s), 512);
    if (lane == 0) {
      mbar_init(smem_u32(&bar_q), 1);
      for (int s = 0; s < fsm::kStages; ++s) {
        mbar_init(smem_u32(&bar_full[s]), 1);
        mbar_init(smem_u32(&bar_empty[s]), n_tiles);  // one commit per tile's MMA thread
      }
      for (int r = 0; r < 2; ++r) {
        mbar_init(smem_u32(&bar_s[r]), 1);
        mbar_init(smem_u32(&bar_p[r]), 128);
        mbar_init(smem_u32(&bar_pb[r]), 128);
        mbar_init(smem_u32(&bar_o[r]), 1);
      }
      mbar_init(smem_u32(&bar_fin), n_tiles);
      mbar_init(smem_u32(&bar_turn[0]), 4);  // one arrival per softmax warp of the other tile
      mbar_init(smem_u32(&bar_turn[1]), 4);
      fence_barrier_init();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_s;
  const int nl = nlist_s;
  const int n_pairs = (nl + 1) / 2;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(smem_u32(&bar_q), uint32_t(n_heads) * 2u * 8192u);
      for (int hh = 0; hh < n_heads; ++hh) {
        const int r = hh >> 1, half = hh & 1;
        const int row = int((size_t(b) * a.Hq + size_t(h) * a.G + g_first + hh) * a.N + size_t(t) * kBlock);
        for (int c = 0; c < 2; ++c)
          tma_load_2d(sQ + (r * 2 + c) * fsm::kHalf + half * 8192, &tmQ, c * 64, row, smem_u32(&bar_q));
      }
      int issued = 0;
      for (int p = 0; p < n_pairs; ++p) {
        const int st = p % fsm::kStages, use = p / fsm::kStages;
        if (!mbar_wait(smem_u32(&bar_empty[st]), (use & 1) ^ 1, abort_flag, a.err)) break;
        const int nb = min(2, nl - 2 * p);
        mbar_arrive_expect_tx(smem_u32(&bar_full[st]), uint32_t(nb) * 4u * 8192u);
        const uint32_t sk = sKV + st * fsm::kStageBytes, sv = sk + 2 * fsm::kHalf;
        for (int bb = 0; bb < nb; ++bb) {
          const int row = int(bh * a.N + size_t(list_s[2 * p + bb]) * kBlock);
          for (int c = 0; c < 2; ++c) {
            tma_load_2d(sk + c * fsm::kHalf + bb * 8192, &tmK, c * 64, row, smem_u32(&bar_full[st]));
            tma_load_2d(sv + c * fsm::kHalf + bb * 8192, &tmV, c * 64, row, smem_u32(&bar_full[st]));
          }
        }
        ++issued;
      }
      if (*abort_flag) {  // let the loads already in flight land before the CTA exits
        for (int p = max(0, issued - fsm::kStages); p < issued; ++p) {
          const long long t0 = clock64();
          while (!mbar_try_wait(smem_u32(&bar_full[p % fsm::kStages]), (p / fsm::kStages) & 1) &&
                 clock64() - t0 < kWaitCycles) {
          }
        }
      }
    }
  } else if ((warp == 1 || warp == 3) && (warp >> 1) < n_tiles) {
    // ------------------------------------------------------------ MMA issuers, one thread per tile
    // (each tile's chain S → softmax → PV is latency-bound; two threads let the
    // two tiles' MMAs overlap)
    if (lane == 0) {
      const int r = warp >> 1;
      const uint32_t idS2 = idesc_bf16_f32(128, 128, 0, 0), idS1 = idesc_bf16_f32(128, 64, 0, 0);
      const uint32_t idPV = idesc_bf16_f32(128, 128, 0, 1);
      const uint64_t dQ0 = smem_desc_sw128(sQ + r * 2 * fsm::kHalf, 16, 1024);
      const uint64_t dK0 = smem_desc_sw128(sKV, 16, 1024);
      const uint64_t dV0 = smem_desc_sw128(sKV + 2 * fsm::kHalf, fsm::kHalf, 1024);
      const uint32_t tS = tmem + r * 128, tO = tmem + 256 + r * 128;
      bool ok = mbar_wait(smem_u32(&bar_q), 0, abort_flag, a.err);
      tc_fence_after();
      for (int p = 0; ok && p < n_pairs; ++p) {
        const int st = p % fsm::kStages, use = p / fsm::kStages;
        if (!(ok = mbar_wait(smem_u32(&bar_full[st]), use & 1, abort_flag, a.err))) break;
        if (p > 0) {  // PV(p-1) reads P from the columns that S(p) overwrites
          if (!(ok = mbar_wait(smem_u32(&bar_o[r]), (p - 1) & 1, abort_flag, a.err))) break;
        }
        tc_fence_after();
        const int nb = min(2, nl - 2 * p);
        const uint32_t so = st * fsm::kStageBytes;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t oc = (k >> 2) * fsm::kHalf + (k & 3) * 32;
          mma_ss(tS, desc_advance(dQ0, oc), desc_advance(dK0, so + oc), nb == 2 ? idS2 : idS1, k > 0 ? 1u : 0u);
        }
        mma_commit(smem_u32(&bar_s[r]));
        if (!(ok = mbar_wait(smem_u32(&bar_p[r]), p & 1, abort_flag, a.err))) break;
        tc_fence_after();
        for (int jj = 0; jj < 4; ++jj)  // the first block's 64 tokens
          mma_ts(tO, tS + jj * 8, desc_advance(dV0, so + jj * 2048), idPV, (p > 0 || jj > 0) ? 1u : 0u);
        if (nb > 1) {  // the second block's, once its P is in (every pair but an odd last one)
          if (!(ok = mbar_wait(smem_u32(&bar_pb[r]), p & 1, abort_flag, a.err))) break;
          tc_fence_after();
          for (int jj = 4; jj < 8; ++jj)
            mma_ts(tO, tS + jj * 8, desc_advance(dV0, so + jj * 2048), idPV, 1u);
        }
        mma_commit(smem_u32(&bar_o[r]));
        mma_commit(smem_u32(&bar_empty[st]));
      }
      mma_commit(smem_u32(&bar_fin));
    }
  } else if (warp >= 4 && (warp - 4) / 4 < n_tiles) {
    // ------------------------------------------------------------ softmax, one row per thread
    const int r = (warp - 4) / 4;
    const int quarter = warp & 3;
    const int row = 32 * quarter + lane;
    const uint32_t lane_addr = uint32_t(32 * quarter) << 16;
    const uint32_t tS = tmem + lane_addr + r * 128, tO = tmem + lane_addr + 256 + r * 128;
    const int qpos = row & 63;
    const float sc2 = a.scale * kLog2e;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int p = 0; p < n_pairs; ++p) {
      ok = mbar_wait(smem_u32(&bar_s[r]), p & 1, abort_flag, a.err);
      if (!__all_sync(0xffffffffu, ok)) {  // TMEM loads below are warp-collective
        ok = false;
        break;
      }
      tc_fence_after();
      const int nb = min(2, nl - 2 * p);
      // log2 g of the pair's two blocks, as a logit bias (the gate outside the softmax adds none)
      const float lamA = kOut ? 0.f : lam_s[2 * p], lamB = (kOut || nb < 2) ? 0.f : lam_s[2 * p + 1];
      const bool diag = (p == 0);  // block A of pair 0 is the causal current block
      // The pair's S row (up to 128 columns) comes out of TMEM in four loads and
      // one wait, and stays in registers. Raw row max per 64-column block; the
      // scale and gate are applied to the max. The current block is causal.
      uint32_t v[128];
      tmem_ld32(tS, v);
      tmem_ld32(tS + 32, v + 32);
      if (nb > 1) {
        tmem_ld32(tS + 64, v + 64);
        tmem_ld32(tS + 96, v + 96);
      }
      tmem_wait_ld();
      if (diag) {
#pragma unroll
        for (int e = 0; e < 64; ++e) v[e] = e <= qpos ? v[e] : __float_as_uint(-INFINITY);
      }
      float rmA = -INFINITY, rmB = -INFINITY;
      {
        float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
        for (int e = 0; e < 64; e += 2) {
          m0 = fmaxf(m0, __uint_as_float(v[e]));
          m1 = fmaxf(m1, __uint_as_float(v[e + 1]));
        }
        rmA = fmaxf(m0, m1);
      }
      if (nb > 1) {
        float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
        for (int e = 64; e < 128; e += 2) {
          m0 = fmaxf(m0, __uint_as_float(v[e]));
          m1 = fmaxf(m1, __uint_as_float(v[e + 1]));
        }
        rmB = fmaxf(m0, m1);
      }
      float mx = rmA == -INFINITY ? -INFINITY : fmaf(rmA, sc2, lamA);
      if (nb > 1) mx = fmaxf(mx, fmaf(rmB, sc2, lamB));
      // The stabiliser moves only when the row max grows by more than 2^8. The
      // decision is per row, but the TMEM round trip that rescales O is a
      // warp-collective instruction, so a warp runs it whenever any of its rows
      // moved, with alpha = 1 for the rows that did not.
      float alpha = 1.f;
      const bool grow = mx > m_used + fsm::kRescale;
      if (grow) {
        alpha = (m_used == -INFINITY) ? 0.f : exp2f(m_used - mx);
        l *= alpha;
        m_used = mx;
      }
      // Turn order: tile 0 pair 0, tile 1 pair 0, tile 0 pair 1, ... Tile 0 waits for
      // tile 1's turn of pair p - 1, tile 1 for tile 0's turn of pair p. Neither
      // barrier can run a phase ahead: its next phase needs the waiter's own turn.
      if (n_tiles == 2 && (r == 1 || p > 0)) {
        const bool got = mbar_wait(smem_u32(&bar_turn[r]), (r == 0 ? p - 1 : p) & 1, abort_flag, a.err);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
      }
      // probabilities, row sum, bf16 P over the S columns (all read above), one 64-column
      // block at a time: block ch2's P goes to TMEM columns [32 ch2, 32 ch2 + 32)
      auto block_p = [&](const int ch2) {
        const float off = (ch2 == 0 ? lamA : lamB) - m_used;  // p = 2^(S·sc2 + λ − m)
        uint32_t pk[32];
        float s0 = 0.f, s1 = 0.f;
        // gate outside: the row sum takes p, the values take g·p
        __nv_bfloat162 gw2;
        if constexpr (kOut) gw2 = __float2bfloat162_rn(fast_exp2(lam_s[2 * p + ch2]));
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float p0 = fast_exp2(fmaf(__uint_as_float(v[64 * ch2 + 2 * e]), sc2, off));
          const float p1 = fast_exp2(fmaf(__uint_as_float(v[64 * ch2 + 2 * e + 1]), sc2, off));
          s0 += p0;
          s1 += p1;
          pk[e] = pack_bf16x2(p0, p1);
          if constexpr (kOut) {  // g·p in bf16: p and g rounded once each, then their product
            __nv_bfloat162 pg = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&pk[e]), gw2);
            pk[e] = *reinterpret_cast<uint32_t*>(&pg);
          }
        }
        l += s0 + s1;
        tmem_st32(tS + ch2 * 32, pk);
      };
      // the turn guards the exponentials only: it passes as soon as the last block's are done
      auto pass_turn = [&]() {
        if (n_tiles == 2) {
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&bar_turn[r ^ 1]));
        }
      };
      block_p(0);
      if (nb == 1) pass_turn();
      if (p > 0 && __any_sync(0xffffffffu, grow)) {
        // O holds PV of earlier pairs, complete because S_r(p) completed after it. It is
        // rescaled before the first block's PV of this pair is released, 16 columns at a time.
        for (int ch = 0; ch < 8; ++ch) {
          uint32_t w[16];
          tmem_ld16(tO + ch * 16, w);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) w[e] = __float_as_uint(__uint_as_float(w[e]) * alpha);
          tmem_st16(tO + ch * 16, w);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&bar_p[r]));
      if (nb > 1) {
        block_p(1);
        pass_turn();
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(smem_u32(&bar_pb[r]));
      }
    }
    if (ok) ok = mbar_wait(smem_u32(&bar_o[r]), (n_pairs - 1) & 1, abort_flag, a.err);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
      const int hh = row >> 6;
      if (2 * r + hh < n_heads) {
        const int hq = h * a.G + g_first + 2 * r + hh;
        const size_t orow = (size_t(b) * a.Hq + hq) * a.N + size_t(t) * kBlock + qpos;
        const float inv = 1.f / l;
        uint4* og = reinterpret_cast<uint4*>(a.o + orow * 128);
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t v[32];
          tmem_ld32(tO + ch * 32, v);
          tmem_wait_ld();
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(v[8 * q4 + 0]) * inv, __uint_as_float(v[8 * q4 + 1]) * inv);
            w.y = pack_bf16x2(__uint_as_float(v[8 * q4 + 2]) * inv, __uint_as_float(v[8 * q4 + 3]) * inv);
            w.z = pack_bf16x2(__uint_as_float(v[8 * q4 + 4]) * inv, __uint_as_float(v[8 * q4 + 5]) * inv);
            w.w = pack_bf16x2(__uint_as_float(v[8 * q4 + 6]) * inv, __uint_as_float(v[8 * q4 + 7]) * inv);
            og[ch * 4 + q4] = w;
          }
        }
        if (a.lse_o != nullptr) a.lse_o[orow] = (m_used + log2f(l)) * kLn2;
      }
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (lane == 0) {  // every MMA this CTA issued has completed
      const long long t0 = clock64();
      while (!mbar_try_wait(smem_u32(&bar_fin), 0) && clock64() - t0 < kWaitCycles) {
      }
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// Host side: tensor maps and launch
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Row-major bf16 matrix [rows, cols] read in 64 x 64 boxes with the 128-byte swizzle.
bool make_tmap_bf16_2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols) {
  EncodeTiledFn fn = encode_tiled();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {64, 64};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 [heads, N, 128] read in boxes of 2 heads x 64 tokens x 64 d (128-byte swizzle), so one
// load brings both heads of a head pair for one d-half: 128 rows of 128 B.
bool make_tmap_bf16_3d_heads(CUtensorMap* m, const void* base, uint64_t heads, uint64_t N) {
  EncodeTiledFn fn = encode_tiled();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {128, N, heads};
  const cuuint64_t strides[2] = {128 * 2, N * 128 * 2};
  const cuuint32_t box[3] = {64, 64, 2};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 [rows, N] read in boxes of 2 rows x 64 values (no swizzle).
bool make_tmap_f32_rows(CUtensorMap* m, const void* base, uint64_t rows, uint64_t N) {
  EncodeTiledFn fn = encode_tiled();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {N, rows};
  const cuuint64_t strides[1] = {N * 4};
  const cuuint32_t box[2] = {64, 2};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 [tiles, 128, 64] in boxes of one whole tile (128-byte swizzle): the backward's dZ tiles.
bool make_tmap_bf16_tiles(CUtensorMap* m, const void* base, uint64_t tiles) {
  EncodeTiledFn fn = encode_tiled();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {64, 128, tiles};
  const cuuint64_t strides[2] = {64 * 2, 128 * 64 * 2};
  const cuuint32_t box[3] = {64, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_fwd_sm100(const Shape& sh, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                             const float* s, const int32_t* idx, const float* lse_s, uint16_t* o, float* lse_o,
                             int* err, cudaStream_t st) {
  CUtensorMap tq, tk, tv;
  const uint64_t rq = uint64_t(sh.B) * sh.Hq * sh.N, rkv = uint64_t(sh.B) * sh.Hkv * sh.N;
  if (!make_tmap_bf16_2d(&tq, q, rq, 128) || !make_tmap_bf16_2d(&tk, k, rkv, 128) ||
      !make_tmap_bf16_2d(&tv, v, rkv, 128))
    return cudaErrorInvalidValue;
  auto kern = sh.outside ? fwd_sm100_kernel<true> : fwd_sm100_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, fsm::kSmemBytes);
  if (e != cudaSuccess) return e;
  FwdSm100Args a;
  a.idx = idx;
  a.s = s;
  a.lse_s = lse_s;
  a.o = o;
  a.lse_o = lse_o;
  a.err = err;
  a.B = sh.B;
  a.Hq = sh.Hq;
  a.Hkv = sh.Hkv;
  a.G = sh.G;
  a.N = sh.N;
  a.NB = sh.NB;
  a.K = sh.K;
  a.gate = sh.gate;
  a.gated = sh.gated;
  a.n_tp = (sh.G + 3) / 4;
  a.scale = sh.scale;
  dim3 grid(sh.NB, sh.Hkv * a.n_tp, sh.B);
  kern<<<grid, fsm::kThreads, fsm::kSmemBytes, st>>>(tq, tk, tv, a);
  return cudaGetLastError();
}

}  // namespace sas
