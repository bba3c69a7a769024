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
// each, so every gathered K/V block serves four heads (GQA packing). A step
// is one gathered 64-token block. Roles:
//   warp 0       builds the block list [t, I_t...], then issues TMA loads:
//                the Q rows once, then each selected K/V block into a
//                4-stage shared-memory ring. Blocks are gathered by index
//                with no copy in HBM.
//   warps 1, 3   one MMA-issuing warp per tile (warp 1 also allocates the
//                512 TMEM columns): S_r(b) = Q_r K_bᵀ (SS, fp32 in TMEM), then
//                O_r += P_r(b) V_b (TS: P read from TMEM). The whole warp
//                walks the loop and waits; elect.sync picks the lane that
//                issues, so the operands stay warp-uniform.
//   warps 4-7    softmax of tile 0; warps 8-11 softmax of tile 1. Each thread
//                owns one row: it reads the block's 64 logits from TMEM,
//                masks the current block causally, adds the block's log-gate,
//                updates the row max and sum, and writes bf16 P back over the
//                consumed S columns. O is rescaled in TMEM only when the row
//                max grows by more than 2^8, so the result is exact and
//                rescales are rare.
//                With two tiles, their exponential sections take turns
//                (tile 0 on block b, then tile 1 on block b, then tile 0 on
//                b + 1), handed over by an mbarrier, so the two groups do
//                not contend for the same issue slots at the same moment.
// Each tile has two 64-column S buffers: S of block b + 1 is computed while
// the softmax works on block b and PV of block b − 1 runs, so no tile waits
// for its own PV before its next S.
// TMEM, tile r at column 256 r: S buffers [0, 64) and [64, 128), O [128, 256).
// Every mbarrier wait is bounded and raises SAS_ERR_TIMEOUT instead of hanging.
#include <mutex>

#include "sm100.cuh"

namespace sas {

namespace fsm {
constexpr int kThreads = 384;            // 0 TMA, 1 and 3 MMA (one warp per tile), 4-11 softmax
constexpr int kStages = 4;               // one gathered K/V block per stage
constexpr int kHalf = 128 * 128;         // one d-half of a 128-row Q tile: 128 rows x 128 B
constexpr int kQBytes = 4 * kHalf;       // 2 tiles x 2 d-halves
constexpr int kHalfKV = 64 * 128;        // one d-half of a 64-row K or V block
constexpr int kStageBytes = 4 * kHalfKV;  // K and V of one block, two d-halves each
constexpr int kSmemBytes = kQBytes + kStages * kStageBytes + 1024;  // + room to align to 1 KB
constexpr float kRescale = 8.0f;         // log2 headroom before O is rescaled
}  // namespace fsm

struct FwdSm100Args {
  const int32_t* idx;
  const float* s;
  const float* lse_s;
  uint16_t* o;
  float* lse_o;
  int* err;
  int B, Hq, Hkv, G, N, NB, K, gate, gated, n_tp;
  int d;  // head dim, 64 or 128; at 64 the tensor maps zero-fill the second 64-column half of every box
  float scale;
};

// kOut: the gate weights the values after a softmax over the plain logits
// (SAS_GATE_SOFTMAX_OUTSIDE) instead of entering the logits as log g.
//
// Barriers, for tile r and block b (c = b & 1 selects the S buffer):
//   producer   waits empty[st] (block b − 4), loads K_b, V_b        -> full[st]
//   MMA r      waits full of b + 1 and pv[c'] (PV of b − 1, the buffer S(b + 1)
//              reuses), issues S(b + 1)                               -> s[c']
//              waits p[c] (P of b in TMEM), issues PV(b)             -> pv[c], empty[st]
//   softmax r  waits s[c], writes P(b)                                -> p[c]
//              (waits pv of b − 1 before a rare rescale of O)
// No waiter can fall two phases behind: every barrier's next phase needs the
// waiter's own next action first.
template <bool kOut>
__global__ void __launch_bounds__(fsm::kThreads, 1)
    fwd_sm100_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, FwdSm100Args a) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  __shared__ int list_s[kMaxTopK + 1];
  __shared__ float lam_s[kMaxTopK + 1];
  __shared__ int nlist_s;
  __shared__ __align__(8) uint64_t bar_q, bar_full[fsm::kStages], bar_empty[fsm::kStages], bar_s[2][2], bar_p[2][2],
      bar_pv[2][2], bar_fin, bar_turn[2];
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
      for (int r = 0; r < 2; ++r)
        for (int c = 0; c < 2; ++c) {
          mbar_init(smem_u32(&bar_s[r][c]), 1);
          mbar_init(smem_u32(&bar_p[r][c]), 128);
          mbar_init(smem_u32(&bar_pv[r][c]), 1);
        }
      mbar_init(smem_u32(&bar_fin), n_tiles);
      mbar_init(smem_u32(&bar_turn[0]), 4);
      mbar_init(smem_u32(&bar_turn[1]), 4);
      fence_barrier_init();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_s;
  const int nl = nlist_s;

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
      for (int i = 0; i < nl; ++i) {
        const int st = i % fsm::kStages, use = i / fsm::kStages;
        if (!mbar_wait(smem_u32(&bar_empty[st]), (use & 1) ^ 1, abort_flag, a.err)) break;
        mbar_arrive_expect_tx(smem_u32(&bar_full[st]), 4u * 8192u);
        const uint32_t sk = sKV + st * fsm::kStageBytes, sv = sk + 2 * fsm::kHalfKV;
        const int row = int(bh * a.N + size_t(list_s[i]) * kBlock);
        for (int c = 0; c < 2; ++c) {
          tma_load_2d(sk + c * fsm::kHalfKV, &tmK, c * 64, row, smem_u32(&bar_full[st]));
          tma_load_2d(sv + c * fsm::kHalfKV, &tmV, c * 64, row, smem_u32(&bar_full[st]));
        }
        ++issued;
      }
      if (*abort_flag) {  // let the loads already in flight land before the CTA exits
        for (int i = max(0, issued - fsm::kStages); i < issued; ++i) {
          const long long t0 = clock64();
          while (!mbar_try_wait(smem_u32(&bar_full[i % fsm::kStages]), (i / fsm::kStages) & 1) &&
                 clock64() - t0 < kWaitCycles) {
          }
        }
      }
    }
  } else if ((warp == 1 || warp == 3) && (warp >> 1) < n_tiles) {
    // ------------------------------------------------------------ MMA issuers, one warp per tile
    // The whole warp walks the loop and waits; one elected lane issues each MMA.
    {
      const int r = warp >> 1;
      const uint32_t idS = idesc_bf16_f32(128, 64, 0, 0);   // q rows x kv, K = d
      const uint32_t idPV = idesc_bf16_f32(128, 128, 0, 1);  // q rows x d, K = kv; V MN-major
      // descriptors are built once; a stage or K step only moves the start address
      const uint64_t dQ0 = smem_desc_sw128(sQ + r * 2 * fsm::kHalf, 16, 1024);
      const uint64_t dK0 = smem_desc_sw128(sKV, 16, 1024);
      const uint64_t dV0 = smem_desc_sw128(sKV + 2 * fsm::kHalfKV, fsm::kHalfKV, 1024);
      const uint32_t tT = tmem + r * 256, tO = tT + 128;
      auto issue_s = [&](const int i) {  // S of block i into buffer i & 1
        const uint32_t so = (i % fsm::kStages) * fsm::kStageBytes;
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mma_ss_e(tT + (i & 1) * 64, desc_advance(dQ0, (k >> 2) * fsm::kHalf + (k & 3) * 32),
                   desc_advance(dK0, so + (k >> 2) * fsm::kHalfKV + (k & 3) * 32), idS, k > 0 ? 1u : 0u);
        mma_commit_e(smem_u32(&bar_s[r][i & 1]));
      };
      bool ok = mbar_wait(smem_u32(&bar_q), 0, abort_flag, a.err);
      ok = ok && mbar_wait(smem_u32(&bar_full[0]), 0, abort_flag, a.err);
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
      if (ok) issue_s(0);
      for (int i = 0; ok && i < nl; ++i) {
        if (i + 1 < nl) {
          const int n = i + 1;
          ok = mbar_wait(smem_u32(&bar_full[n % fsm::kStages]), (n / fsm::kStages) & 1, abort_flag, a.err);
          // PV of block n − 2 read its P from the buffer that S(n) overwrites
          if (ok && n >= 2) ok = mbar_wait(smem_u32(&bar_pv[r][n & 1]), ((n - 2) >> 1) & 1, abort_flag, a.err);
          if (!(ok = __all_sync(0xffffffffu, ok))) break;
          tc_fence_after();
          issue_s(n);
        }
        ok = mbar_wait(smem_u32(&bar_p[r][i & 1]), (i >> 1) & 1, abort_flag, a.err);
        if (!(ok = __all_sync(0xffffffffu, ok))) break;
        tc_fence_after();
        const uint32_t sv = (i % fsm::kStages) * fsm::kStageBytes;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj)  // P(i) packed over the first 32 columns of its S buffer
          mma_ts_e(tO, tT + (i & 1) * 64 + jj * 8, desc_advance(dV0, sv + jj * 2048), idPV, (i > 0 || jj > 0) ? 1u : 0u);
        mma_commit_e(smem_u32(&bar_pv[r][i & 1]));
        mma_commit_e(smem_u32(&bar_empty[i % fsm::kStages]));
      }
      mma_commit_e(smem_u32(&bar_fin));
    }
  } else if (warp >= 4 && (warp - 4) / 4 < n_tiles) {
    // ------------------------------------------------------------ softmax, one row per thread
    const int r = (warp - 4) / 4;
    const int quarter = warp & 3;
    const int row = 32 * quarter + lane;
    const uint32_t lane_addr = uint32_t(32 * quarter) << 16;
    const uint32_t tT = tmem + lane_addr + r * 256, tO = tT + 128;
    const int qpos = row & 63;
    const float sc2 = a.scale * kLog2e;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int i = 0; i < nl; ++i) {
      const uint32_t tS = tT + (i & 1) * 64;
      ok = mbar_wait(smem_u32(&bar_s[r][i & 1]), (i >> 1) & 1, abort_flag, a.err);
      if (!__all_sync(0xffffffffu, ok)) {  // TMEM loads below are warp-collective
        ok = false;
        break;
      }
      tc_fence_after();
      // log2 g of the block as a logit bias (the gate outside the softmax adds none)
      const float lam = kOut ? 0.f : lam_s[i];
      uint32_t v[64];
      tmem_ld32(tS, v);
      tmem_ld32(tS + 32, v + 32);
      tmem_wait_ld();
      if (i == 0) {  // the current block is causal
#pragma unroll
        for (int e = 0; e < 64; ++e) v[e] = e <= qpos ? v[e] : __float_as_uint(-INFINITY);
      }
      float mm[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) mm[c] = fmaxf(__uint_as_float(v[c]), __uint_as_float(v[c + 8]));
#pragma unroll
      for (int e = 16; e < 64; e += 8)
#pragma unroll
        for (int c = 0; c < 8; ++c) mm[c] = fmaxf(mm[c], __uint_as_float(v[e + c]));
      const float rm = fmaxf(fmaxf(fmaxf(mm[0], mm[1]), fmaxf(mm[2], mm[3])), fmaxf(fmaxf(mm[4], mm[5]), fmaxf(mm[6], mm[7])));
      const float mx = rm == -INFINITY ? -INFINITY : fmaf(rm, sc2, lam);
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
      if (n_tiles == 2 && (r == 1 || i > 0)) {
        const bool got = mbar_wait(smem_u32(&bar_turn[r]), (r == 0 ? i - 1 : i) & 1, abort_flag, a.err);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
      }
      // probabilities, row sum, bf16 P over the S columns just read
      {
        const float off = lam - m_used;  // p = 2^(S·sc2 + λ − m)
        uint32_t pk[32];
        float s0 = 0.f, s1 = 0.f;
        // gate outside: the row sum takes p, the values take g·p
        __nv_bfloat162 gw2;
        if constexpr (kOut) gw2 = __float2bfloat162_rn(fast_exp2(lam_s[i]));
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float p0 = fast_exp2(fmaf(__uint_as_float(v[2 * e]), sc2, off));
          const float p1 = fast_exp2(fmaf(__uint_as_float(v[2 * e + 1]), sc2, off));
          s0 += p0;
          s1 += p1;
          pk[e] = pack_bf16x2(p0, p1);
          if constexpr (kOut) {  // g·p in bf16: p and g rounded once each, then their product
            __nv_bfloat162 pg = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&pk[e]), gw2);
            pk[e] = *reinterpret_cast<uint32_t*>(&pg);
          }
        }
        l += s0 + s1;
        if (n_tiles == 2) {
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&bar_turn[r ^ 1]));
        }
        tmem_st32(tS, pk);
      }
      if (i > 0 && __any_sync(0xffffffffu, grow)) {
        // O holds PV of the earlier blocks once PV(i − 1) has completed
        ok = mbar_wait(smem_u32(&bar_pv[r][(i - 1) & 1]), ((i - 1) >> 1) & 1, abort_flag, a.err);
        if (!__all_sync(0xffffffffu, ok)) {
          ok = false;
          break;
        }
        tc_fence_after();
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
      mbar_arrive(smem_u32(&bar_p[r][i & 1]));
    }
    if (ok) ok = mbar_wait(smem_u32(&bar_pv[r][(nl - 1) & 1]), ((nl - 1) >> 1) & 1, abort_flag, a.err);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
      const int hh = row >> 6;
      if (2 * r + hh < n_heads) {
        const int hq = h * a.G + g_first + 2 * r + hh;
        const size_t orow = (size_t(b) * a.Hq + hq) * a.N + size_t(t) * kBlock + qpos;
        const float inv = 1.f / l;
        uint4* og = reinterpret_cast<uint4*>(a.o + orow * a.d);
        for (int ch = 0; ch < a.d / 32; ++ch) {
          uint32_t w[32];
          tmem_ld32(tO + ch * 32, w);
          tmem_wait_ld();
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint4 x;
            x.x = pack_bf16x2(__uint_as_float(w[8 * q4 + 0]) * inv, __uint_as_float(w[8 * q4 + 1]) * inv);
            x.y = pack_bf16x2(__uint_as_float(w[8 * q4 + 2]) * inv, __uint_as_float(w[8 * q4 + 3]) * inv);
            x.z = pack_bf16x2(__uint_as_float(w[8 * q4 + 4]) * inv, __uint_as_float(w[8 * q4 + 5]) * inv);
            x.w = pack_bf16x2(__uint_as_float(w[8 * q4 + 6]) * inv, __uint_as_float(w[8 * q4 + 7]) * inv);
            og[ch * 4 + q4] = x;
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

// bf16 [heads, N, d] read in boxes of 2 heads x 64 tokens x 64 d (128-byte swizzle), so one
// load brings both heads of a head pair for one d-half: 128 rows of 128 B. At d = 64 the
// second d-half is past the extent and arrives as zeros.
bool make_tmap_bf16_3d_heads(CUtensorMap* m, const void* base, uint64_t heads, uint64_t N, uint64_t d) {
  EncodeTiledFn fn = encode_tiled();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {d, N, heads};
  const cuuint64_t strides[2] = {d * 2, N * d * 2};
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
  // [rows, d] with d = 64 or 128: the kernel always loads two 64-column boxes per row; at d = 64 the
  // second lies past the extent, so TMA fills it with zeros and it adds nothing to S or to PV
  if (!make_tmap_bf16_2d(&tq, q, rq, sh.d) || !make_tmap_bf16_2d(&tk, k, rkv, sh.d) ||
      !make_tmap_bf16_2d(&tv, v, rkv, sh.d))
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
  a.d = sh.d;
  a.scale = sh.scale;
  dim3 grid(sh.NB, sh.Hkv * a.n_tp, sh.B);
  kern<<<grid, fsm::kThreads, fsm::kSmemBytes, st>>>(tq, tk, tv, a);
  return cudaGetLastError();
}

}  // namespace sas
