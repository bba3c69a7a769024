// Backward of gated block-sparse attention on the Blackwell tensor cores.
//
// SAS summary (onedev.kr), section 무엇과 다른가: the gate sits inside the
// softmax, and its gradient dg_m = Σ_i (p̃_i/g_m) dOᵀ(v_i − o) chains through
// g = softmax(s). Training uses sparse scope: content gradients reach only
// the selected blocks. Per query row i and attended token j:
//   P_ij = exp(z_ij − L_i),  dP_ij = dO_i·v_j,  dZ_ij = P_ij (dP_ij − D_i),
//   dV_j = Σ_i P_ij dO_i,  dK_j = scale Σ_i dZ_ij q_i,  dQ_i = scale Σ_j dZ_ij k_j,
//   dl[t, m] = Σ_{rows of t, heads, tokens of m} dZ   (= g_m·dg_m).
//
// Two passes with no atomics and no reduction traffic:
//   bwd_kv_sm100_kernel  one CTA per (batch, KV head, KV block j). It walks the
//       query blocks that attend j (its own diagonal block first, then the
//       reverse index), two query heads (128 rows) per step. S = Q Kᵀ and
//       dP = dO Vᵀ land in double-buffered TMEM. The softmax-gradient warps
//       write P and dZ as bf16 rows, 128-byte swizzled, into shared memory.
//       dVᵀ += dOᵀ P and dKᵀ += Qᵀ dZ then accumulate in TMEM as M = 128
//       (d-major) MMAs with MN-major operands, so dK_j and dV_j stay on chip
//       for the whole walk. The CTA is also the only writer of dl[t, slot(j)].
//   bwd_q_sm100_kernel   one CTA per (batch, KV head, query block, up to four
//       heads), structured like the forward: two M = 128 tiles, S and dP per
//       selected block in TMEM, dZ written back as bf16 over S, and
//       dQ += dZ K as a TS MMA with K MN-major. dQ is written once, in bf16.
// The first pass recomputes S and dP a second time (7 GEMM-shaped products
// instead of 5), but no partial sum is ever sent to L2.
#include "sm100.cuh"

namespace sas {

struct BwdSm100Args {
  const int* rev_off;
  const int* rev_list;
  const float* s;
  const float* lse_s;
  const float* lse_o;
  const float* drow;
  float* dl;
  uint16_t* dq;
  uint16_t* dk;
  uint16_t* dv;
  const int32_t* idx;
  int* err;
  int B, Hq, Hkv, G, N, NB, K, gated, n_hp, n_tp;
  float scale;
};

// ===========================================================================
// Pass 1: dK, dV and dl, KV-major
// ===========================================================================
namespace bkv {
constexpr int kThreads = 384;                 // 0 TMA, 1 MMA, 2-3 spare, 4-7 and 8-11 softmax gradient
constexpr int kHalf64 = 64 * 128;             // one d-half of a 64-row tile
constexpr int kKV = 4 * kHalf64;              // K_j and V_j
constexpr int kHalf128 = 128 * 128;           // one d-half of a 128-row tile
constexpr int kTile = 2 * kHalf128;           // 128 rows x d 128
constexpr int kStage = 2 * kTile + 1024;      // Q tile, dO tile, L and D rows (128 floats each)
constexpr int kStages = 2;
constexpr int kPZ = 128 * 128;                // P or dZ: 128 q rows x 64 kv bf16
constexpr int kSmem = kKV + kStages * kStage + 2 * kPZ + 1024;
struct Meta {
  int t, slot, nv;
  float lam2;
};
}  // namespace bkv

__global__ void __launch_bounds__(bkv::kThreads, 1)
    bwd_kv_sm100_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                        BwdSm100Args a) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_kv, bar_full[bkv::kStages], bar_empty[bkv::kStages], bar_s[2], bar_p, bar_pz,
      bar_fin;
  __shared__ bkv::Meta meta[bkv::kStages];
  __shared__ float red_s[2][8];
  __shared__ uint32_t tmem_s;
  __shared__ int abort_s;

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sK = base, sV = base + 2 * bkv::kHalf64;
  const uint32_t sStage = base + bkv::kKV;
  const uint32_t sP = sStage + bkv::kStages * bkv::kStage, sZ = sP + bkv::kPZ;
  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t bh = size_t(b) * a.Hkv + h;
  const int off0 = a.rev_off[bh * (a.NB + 1) + j];
  const int n_sel = a.rev_off[bh * (a.NB + 1) + j + 1] - off0;
  const int* lst = a.rev_list + bh * size_t(a.NB) * a.K + off0;
  const int n_steps = (1 + n_sel) * a.n_hp;
  volatile int* abort_flag = &abort_s;

  if (threadIdx.x == 0) abort_s = 0;
  if (a.G & 1) {  // a half head pair leaves rows 64..127 unloaded: keep them finite (zero)
    for (int i = threadIdx.x; i < bkv::kStages * 2 * bkv::kTile / 16; i += bkv::kThreads) {
      const int st = i / (2 * bkv::kTile / 16), rem = i % (2 * bkv::kTile / 16);
      asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};\n" ::"r"(sStage + st * bkv::kStage + rem * 16), "r"(0));
    }
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_s), 512);
    if (lane == 0) {
      mbar_init(smem_u32(&bar_kv), 1);
      for (int s = 0; s < bkv::kStages; ++s) {
        mbar_init(smem_u32(&bar_full[s]), 1);
        mbar_init(smem_u32(&bar_empty[s]), 1);
      }
      mbar_init(smem_u32(&bar_s[0]), 1);
      mbar_init(smem_u32(&bar_s[1]), 1);
      mbar_init(smem_u32(&bar_p), 256);
      mbar_init(smem_u32(&bar_pz), 1);
      mbar_init(smem_u32(&bar_fin), 1);
      fence_barrier_init();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_s;
  // TMEM columns: S buffers 0 / 64, dP buffers 128 / 192, dVᵀ 256, dKᵀ 320
  constexpr uint32_t kColDV = 256, kColDK = 320;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
      const int krow = int(bh * a.N + size_t(j) * kBlock);
      mbar_arrive_expect_tx(smem_u32(&bar_kv), 4u * 8192u);
      for (int c = 0; c < 2; ++c) {
        tma_load_2d(sK + c * bkv::kHalf64, &tmK, c * 64, krow, smem_u32(&bar_kv));
        tma_load_2d(sV + c * bkv::kHalf64, &tmV, c * 64, krow, smem_u32(&bar_kv));
      }
      int issued = 0;
      for (int i = 0; i < n_steps; ++i) {
        const int st = i % bkv::kStages, use = i / bkv::kStages;
        if (!mbar_wait(smem_u32(&bar_empty[st]), (use & 1) ^ 1, abort_flag, a.err)) break;
        const int e = i / a.n_hp, hp = i % a.n_hp;
        int t = j, slot = -1;
        if (e > 0) {
          const int w = lst[e - 1];
          t = w >> 8;
          slot = w & 255;
        }
        float lam2 = 0.f;
        if (e > 0 && a.gated) {
          const size_t row = bh * a.NB + t;
          lam2 = (a.s[row * a.NB + j] - a.lse_s[row]) * kLog2e;
        }
        const int nv = min(2, a.G - 2 * hp);
        meta[st] = bkv::Meta{t, slot, nv, lam2};
        const uint32_t bar = smem_u32(&bar_full[st]);
        mbar_arrive_expect_tx(bar, uint32_t(nv) * (4u * 8192u + 512u));
        const uint32_t sq = sStage + st * bkv::kStage, sdo = sq + bkv::kTile, sl = sdo + bkv::kTile;
        for (int hh = 0; hh < nv; ++hh) {
          const size_t qrow = (size_t(b) * a.Hq + size_t(h) * a.G + 2 * hp + hh) * a.N + size_t(t) * kBlock;
          for (int c = 0; c < 2; ++c) {
            tma_load_2d(sq + c * bkv::kHalf128 + hh * 8192, &tmQ, c * 64, int(qrow), bar);
            tma_load_2d(sdo + c * bkv::kHalf128 + hh * 8192, &tmDO, c * 64, int(qrow), bar);
          }
          bulk_load(sl + hh * 256, a.lse_o + qrow, 256, bar);
          bulk_load(sl + 512 + hh * 256, a.drow + qrow, 256, bar);
        }
        ++issued;
      }
      if (*abort_flag) {
        for (int i = max(0, issued - bkv::kStages); i < issued; ++i) {
          const long long t0 = clock64();
          while (!mbar_try_wait(smem_u32(&bar_full[i % bkv::kStages]), (i / bkv::kStages) & 1) &&
                 clock64() - t0 < kWaitCycles) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idS = idesc_bf16_f32(128, 64, 0, 0);     // S, dP: q rows x kv, K = d
      const uint32_t idG = idesc_bf16_f32(128, 64, 1, 1);     // dVᵀ, dKᵀ: d x kv, K = q rows
      bool ok = mbar_wait(smem_u32(&bar_kv), 0, abort_flag, a.err);
      tc_fence_after();
      auto grads = [&](int i) {  // dVᵀ += dOᵀ P, dKᵀ += Qᵀ dZ for step i
        const int st = i % bkv::kStages;
        const uint32_t sq = sStage + st * bkv::kStage, sdo = sq + bkv::kTile;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t acc = (i > 0 || k > 0) ? 1u : 0u;
          mma_ss(tmem + kColDV, smem_desc_sw128(sdo + k * 2048, bkv::kHalf128, 1024),
                 smem_desc_sw128(sP + k * 2048, bkv::kHalf128, 1024), idG, acc);
          mma_ss(tmem + kColDK, smem_desc_sw128(sq + k * 2048, bkv::kHalf128, 1024),
                 smem_desc_sw128(sZ + k * 2048, bkv::kHalf128, 1024), idG, acc);
        }
        mma_commit(smem_u32(&bar_pz));
        mma_commit(smem_u32(&bar_empty[st]));
      };
      for (int i = 0; ok && i < n_steps; ++i) {
        const int st = i % bkv::kStages, use = i / bkv::kStages, sb = i & 1;
        if (!(ok = mbar_wait(smem_u32(&bar_full[st]), use & 1, abort_flag, a.err))) break;
        tc_fence_after();
        const uint32_t sq = sStage + st * bkv::kStage, sdo = sq + bkv::kTile;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int c = k >> 2, kk = k & 3;
          mma_ss(tmem + sb * 64, smem_desc_sw128(sq + c * bkv::kHalf128 + kk * 32, 16, 1024),
                 smem_desc_sw128(sK + c * bkv::kHalf64 + kk * 32, 16, 1024), idS, k > 0 ? 1u : 0u);
          mma_ss(tmem + 128 + sb * 64, smem_desc_sw128(sdo + c * bkv::kHalf128 + kk * 32, 16, 1024),
                 smem_desc_sw128(sV + c * bkv::kHalf64 + kk * 32, 16, 1024), idS, k > 0 ? 1u : 0u);
        }
        mma_commit(smem_u32(&bar_s[sb]));
        if (i > 0) {
          if (!(ok = mbar_wait(smem_u32(&bar_p), (i - 1) & 1, abort_flag, a.err))) break;
          tc_fence_after();
          grads(i - 1);
        }
      }
      if (ok && n_steps > 0 && mbar_wait(smem_u32(&bar_p), (n_steps - 1) & 1, abort_flag, a.err)) {
        tc_fence_after();
        grads(n_steps - 1);
      }
      mma_commit(smem_u32(&bar_fin));
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax gradient
    // Thread (wg, row): q row `row`, kv columns [32 wg, 32 wg + 32).
    const int wg = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int row = 32 * quarter + lane;
    const uint32_t lane_addr = uint32_t(32 * quarter) << 16;
    const int hh = row >> 6, qpos = row & 63;
    const float sc2 = a.scale * kLog2e;
    float dl_part = 0.f;
    bool ok = true;
    for (int i = 0; i < n_steps; ++i) {
      const int st = i % bkv::kStages, use = i / bkv::kStages, sb = i & 1;
      ok = mbar_wait(smem_u32(&bar_full[st]), use & 1, abort_flag, a.err);
      ok = ok && mbar_wait(smem_u32(&bar_s[sb]), use & 1, abort_flag, a.err);
      if (i > 0) ok = ok && mbar_wait(smem_u32(&bar_pz), (i - 1) & 1, abort_flag, a.err);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const bkv::Meta m = meta[st];
      const int e = i / a.n_hp, hp = i % a.n_hp;
      const bool diag = (e == 0), valid = hh < m.nv;
      const uint32_t sl = sStage + st * bkv::kStage + 2 * bkv::kTile;
      float L2 = 0.f, Dr = 0.f;
      asm volatile("ld.shared.f32 %0, [%1];\n" : "=f"(L2) : "r"(sl + row * 4));
      asm volatile("ld.shared.f32 %0, [%1];\n" : "=f"(Dr) : "r"(sl + 512 + row * 4));
      L2 = L2 * kLog2e - m.lam2;  // P = exp2(S·sc2 − (L·log2e − λ))
      uint32_t vs[32], vp[32];
      tmem_ld32(tmem + lane_addr + sb * 64 + wg * 32, vs);
      tmem_ld32(tmem + lane_addr + 128 + sb * 64 + wg * 32, vp);
      tmem_wait_ld();
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {  // 16-byte chunk: 8 kv columns
        uint32_t wp[4], wz[4];
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2) {
          float pp[2], zz[2];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int x = c4 * 8 + e2 * 2 + u;
            const int col = wg * 32 + x;
            float p = exp2f(fmaf(__uint_as_float(vs[x]), sc2, -L2));
            if (!valid || (diag && col > qpos)) p = 0.f;
            const float z = valid ? p * (__uint_as_float(vp[x]) - Dr) : 0.f;  // L, D of a missing head are unset
            dl_part += z;
            pp[u] = p;
            zz[u] = z;
          }
          wp[e2] = pack_bf16x2(pp[0], pp[1]);
          wz[e2] = pack_bf16x2(zz[0], zz[1]);
        }
        const int chunk = wg * 4 + c4;
        const uint32_t off = uint32_t(row * 128 + ((chunk ^ (row & 7)) << 4));
        asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(sP + off), "r"(wp[0]), "r"(wp[1]), "r"(wp[2]),
                     "r"(wp[3]));
        asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(sZ + off), "r"(wz[0]), "r"(wz[1]), "r"(wz[2]),
                     "r"(wz[3]));
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(smem_u32(&bar_p));
      if (hp == a.n_hp - 1) {  // the entry's last head pair: dl[t, slot] has this CTA as its only writer
        if (!diag) {
          const float w = warp_sum(dl_part);
          if (lane == 0) red_s[e & 1][warp - 4] = w;
          named_bar_sync(1, 256);
          if (warp == 4 && lane == 0 && a.gated) {
            float tot = 0.f;
#pragma unroll
            for (int k = 0; k < 8; ++k) tot += red_s[e & 1][k];
            a.dl[(bh * a.NB + m.t) * a.K + m.slot] = tot;
          }
        }
        dl_part = 0.f;
      }
    }
    // epilogue: warpgroup 0 writes dV, warpgroup 1 writes dK. TMEM lanes are d
    // rows, so each row is transposed through shared memory into [kv][d].
    ok = ok && mbar_wait(smem_u32(&bar_fin), 0, abort_flag, a.err);
    ok = __all_sync(0xffffffffu, ok);
    const uint32_t stage_buf = wg == 0 ? sP : sZ;  // [64 kv][128 d] bf16, plain row-major
    if (ok) {
      tc_fence_after();
      const int d = row;
      const float mul = wg == 0 ? 1.f : a.scale;
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_addr + (wg == 0 ? kColDV : kColDK) + ch * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          const __nv_bfloat16 bv = __float2bfloat16_rn(__uint_as_float(v[x]) * mul);
          const uint16_t bits = *reinterpret_cast<const uint16_t*>(&bv);
          asm volatile("st.shared.u16 [%0], %1;\n" ::"r"(stage_buf + (ch * 32 + x) * 256 + d * 2), "h"(bits));
        }
      }
    }
    named_bar_sync(2 + wg, 128);
    if (ok) {
      uint16_t* dst = (wg == 0 ? a.dv : a.dk) + (bh * a.N + size_t(j) * kBlock) * 128;
      uint4* g = reinterpret_cast<uint4*>(dst);
      for (int i = row; i < 64 * 16; i += 128) {
        uint4 x;
        asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n" : "=r"(x.x), "=r"(x.y), "=r"(x.z), "=r"(x.w)
                     : "r"(stage_buf + i * 16));
        g[i] = x;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (lane == 0) {
      const long long t0 = clock64();
      while (!mbar_try_wait(smem_u32(&bar_fin), 0) && clock64() - t0 < kWaitCycles) {
      }
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ===========================================================================
// Pass 2: dQ, query-major
// ===========================================================================
namespace bq {
constexpr int kThreads = 640;                 // 0 TMA, 1 MMA, 2-3 spare, 4-19 softmax gradient (tile, half)
constexpr int kHalf = 128 * 128;              // one d-half of a 128-row tile
constexpr int kQ = 4 * kHalf;                 // 2 tiles x 2 d-halves
constexpr int kHalfKV = 64 * 128;             // one d-half of a 64-row block
constexpr int kStage = 4 * kHalfKV;           // K and V of one block
constexpr int kStages = 2;
constexpr int kSmem = 2 * kQ + kStages * kStage + 1024;
}  // namespace bq

__global__ void __launch_bounds__(bq::kThreads, 1)
    bwd_q_sm100_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                       BwdSm100Args a) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  __shared__ int list_s[kMaxTopK + 1];
  __shared__ float lam_s[kMaxTopK + 1];
  __shared__ int nlist_s;
  __shared__ __align__(8) uint64_t bar_q, bar_full[bq::kStages], bar_empty[bq::kStages], bar_s[2], bar_p[2], bar_o[2],
      bar_fin;
  __shared__ uint32_t tmem_s;
  __shared__ int abort_s;

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sQ = base, sDO = base + bq::kQ, sKV = base + 2 * bq::kQ;
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
                     a.gated ? a.lse_s[row] : 0.f, a.gated, list_s, lam_s, &nlist_s, a.err);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_s), 512);
    if (lane == 0) {
      mbar_init(smem_u32(&bar_q), 1);
      for (int s = 0; s < bq::kStages; ++s) {
        mbar_init(smem_u32(&bar_full[s]), 1);
        mbar_init(smem_u32(&bar_empty[s]), 1);
      }
      for (int r = 0; r < 2; ++r) {
        mbar_init(smem_u32(&bar_s[r]), 1);
        mbar_init(smem_u32(&bar_p[r]), 256);
        mbar_init(smem_u32(&bar_o[r]), 1);
      }
      mbar_init(smem_u32(&bar_fin), 1);
      fence_barrier_init();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_s;
  const int nl = nlist_s;
  // TMEM columns: S_r at 64 r, dP_r at 128 + 64 r, dQ_r at 256 + 128 r. The two
  // warpgroups of a tile split its 64 kv columns; each writes its packed dZ over
  // the first 16 of its own 32 S columns, so tokens 0-31 sit at S_r columns
  // 0-15 and tokens 32-63 at columns 32-47.

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
      mbar_arrive_expect_tx(smem_u32(&bar_q), uint32_t(n_heads) * 4u * 8192u);
      for (int hh = 0; hh < n_heads; ++hh) {
        const int r = hh >> 1, half = hh & 1;
        const int row = int((size_t(b) * a.Hq + size_t(h) * a.G + g_first + hh) * a.N + size_t(t) * kBlock);
        for (int c = 0; c < 2; ++c) {
          tma_load_2d(sQ + (r * 2 + c) * bq::kHalf + half * 8192, &tmQ, c * 64, row, smem_u32(&bar_q));
          tma_load_2d(sDO + (r * 2 + c) * bq::kHalf + half * 8192, &tmDO, c * 64, row, smem_u32(&bar_q));
        }
      }
      int issued = 0;
      for (int i = 0; i < nl; ++i) {
        const int st = i % bq::kStages, use = i / bq::kStages;
        if (!mbar_wait(smem_u32(&bar_empty[st]), (use & 1) ^ 1, abort_flag, a.err)) break;
        mbar_arrive_expect_tx(smem_u32(&bar_full[st]), 4u * 8192u);
        const uint32_t sk = sKV + st * bq::kStage, sv = sk + 2 * bq::kHalfKV;
        const int row = int(bh * a.N + size_t(list_s[i]) * kBlock);
        for (int c = 0; c < 2; ++c) {
          tma_load_2d(sk + c * bq::kHalfKV, &tmK, c * 64, row, smem_u32(&bar_full[st]));
          tma_load_2d(sv + c * bq::kHalfKV, &tmV, c * 64, row, smem_u32(&bar_full[st]));
        }
        ++issued;
      }
      if (*abort_flag) {
        for (int i = max(0, issued - bq::kStages); i < issued; ++i) {
          const long long t0 = clock64();
          while (!mbar_try_wait(smem_u32(&bar_full[i % bq::kStages]), (i / bq::kStages) & 1) &&
                 clock64() - t0 < kWaitCycles) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idS = idesc_bf16_f32(128, 64, 0, 0);
      const uint32_t idQ = idesc_bf16_f32(128, 128, 0, 1);  // dQ: q rows x d, K = kv tokens (K MN-major)
      bool ok = mbar_wait(smem_u32(&bar_q), 0, abort_flag, a.err);
      tc_fence_after();
      for (int i = 0; ok && i < nl; ++i) {
        const int st = i % bq::kStages, use = i / bq::kStages;
        if (!(ok = mbar_wait(smem_u32(&bar_full[st]), use & 1, abort_flag, a.err))) break;
        tc_fence_after();
        const uint32_t sk = sKV + st * bq::kStage, sv = sk + 2 * bq::kHalfKV;
        for (int r = 0; r < n_tiles; ++r) {
          if (i > 0) {  // dQ_r(i-1) reads dZ_r from the columns S_r(i) overwrites
            if (!(ok = mbar_wait(smem_u32(&bar_o[r]), (i - 1) & 1, abort_flag, a.err))) break;
            tc_fence_after();
          }
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int c = k >> 2, kk = k & 3;
            mma_ss(tmem + r * 64, smem_desc_sw128(sQ + (r * 2 + c) * bq::kHalf + kk * 32, 16, 1024),
                   smem_desc_sw128(sk + c * bq::kHalfKV + kk * 32, 16, 1024), idS, k > 0 ? 1u : 0u);
            mma_ss(tmem + 128 + r * 64, smem_desc_sw128(sDO + (r * 2 + c) * bq::kHalf + kk * 32, 16, 1024),
                   smem_desc_sw128(sv + c * bq::kHalfKV + kk * 32, 16, 1024), idS, k > 0 ? 1u : 0u);
          }
          mma_commit(smem_u32(&bar_s[r]));
        }
        if (!ok) break;
        for (int r = 0; r < n_tiles; ++r) {
          if (!(ok = mbar_wait(smem_u32(&bar_p[r]), i & 1, abort_flag, a.err))) break;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_ts(tmem + 256 + r * 128, tmem + r * 64 + (k >> 1) * 32 + (k & 1) * 8,
                   smem_desc_sw128(sk + k * 2048, bq::kHalfKV, 1024), idQ, (i > 0 || k > 0) ? 1u : 0u);
          mma_commit(smem_u32(&bar_o[r]));
        }
        if (!ok) break;
        mma_commit(smem_u32(&bar_empty[st]));
      }
      mma_commit(smem_u32(&bar_fin));
    }
  } else if (warp >= 4 && (warp - 4) / 8 < n_tiles) {
    // ------------------------------------------------------------ softmax gradient
    // Thread (r, w, row): row `row` of tile r, kv columns [32 w, 32 w + 32).
    const int r = (warp - 4) / 8, w = ((warp - 4) >> 2) & 1;
    const int quarter = warp & 3;
    const int row = 32 * quarter + lane;
    const uint32_t lane_addr = uint32_t(32 * quarter) << 16;
    const uint32_t tS = tmem + lane_addr + r * 64 + w * 32, tP = tmem + lane_addr + 128 + r * 64 + w * 32;
    const uint32_t tQ = tmem + lane_addr + 256 + r * 128 + w * 64;
    const int hh = row >> 6, qpos = row & 63;
    const bool valid = 2 * r + hh < n_heads;
    const int hq = h * a.G + g_first + 2 * r + hh;
    const size_t grow = (size_t(b) * a.Hq + (valid ? hq : h * a.G)) * a.N + size_t(t) * kBlock + qpos;
    const float L2 = valid ? a.lse_o[grow] * kLog2e : 0.f;
    const float Dr = valid ? a.drow[grow] : 0.f;
    const float sc2 = a.scale * kLog2e;
    bool ok = true;
    for (int i = 0; i < nl; ++i) {
      ok = mbar_wait(smem_u32(&bar_s[r]), i & 1, abort_flag, a.err);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float off2 = L2 - lam_s[i];
      const bool diag = (i == 0);
      uint32_t vs[32], vp[32], dz[16];
      tmem_ld32(tS, vs);
      tmem_ld32(tP, vp);
      tmem_wait_ld();
#pragma unroll
      for (int x = 0; x < 16; ++x) {
        float zz[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int col = w * 32 + 2 * x + u;
          float p = exp2f(fmaf(__uint_as_float(vs[2 * x + u]), sc2, -off2));
          if (!valid || (diag && col > qpos)) p = 0.f;
          zz[u] = valid ? p * (__uint_as_float(vp[2 * x + u]) - Dr) : 0.f;
        }
        dz[x] = pack_bf16x2(zz[0], zz[1]);
      }
      tmem_st16(tS, dz);  // packed dZ over this warpgroup's own, already read S columns
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&bar_p[r]));
    }
    if (ok) ok = mbar_wait(smem_u32(&bar_o[r]), (nl - 1) & 1, abort_flag, a.err);
    ok = __all_sync(0xffffffffu, ok);
    if (ok && valid) {  // rows 64..127 of a one-head tile form whole warps
      tc_fence_after();
      uint4* og = reinterpret_cast<uint4*>(a.dq + grow * 128) + w * 8;  // d columns [64 w, 64 w + 64)
      for (int ch = 0; ch < 2; ++ch) {
        uint32_t v[32];
        tmem_ld32(tQ + ch * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint4 o4;
          o4.x = pack_bf16x2(__uint_as_float(v[8 * q4 + 0]) * a.scale, __uint_as_float(v[8 * q4 + 1]) * a.scale);
          o4.y = pack_bf16x2(__uint_as_float(v[8 * q4 + 2]) * a.scale, __uint_as_float(v[8 * q4 + 3]) * a.scale);
          o4.z = pack_bf16x2(__uint_as_float(v[8 * q4 + 4]) * a.scale, __uint_as_float(v[8 * q4 + 5]) * a.scale);
          o4.w = pack_bf16x2(__uint_as_float(v[8 * q4 + 6]) * a.scale, __uint_as_float(v[8 * q4 + 7]) * a.scale);
          og[ch * 4 + q4] = o4;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (lane == 0) {
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
// Host side
// ---------------------------------------------------------------------------
cudaError_t launch_bwd_passes_sm100(const Shape& sh, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                   const uint16_t* dO, const float* s, const int32_t* idx, const float* lse_s,
                                   const float* lse_o, const float* drow, const int* rev_off, const int* rev_list,
                                   float* dl, uint16_t* dq, uint16_t* dk, uint16_t* dv, int* err, cudaStream_t st) {
  CUtensorMap tq, tk, tv, tdo;
  const uint64_t rq = uint64_t(sh.B) * sh.Hq * sh.N, rkv = uint64_t(sh.B) * sh.Hkv * sh.N;
  if (!make_tmap_bf16_2d(&tq, q, rq, 128) || !make_tmap_bf16_2d(&tdo, dO, rq, 128) ||
      !make_tmap_bf16_2d(&tk, k, rkv, 128) || !make_tmap_bf16_2d(&tv, v, rkv, 128))
    return cudaErrorInvalidValue;
  BwdSm100Args a;
  a.rev_off = rev_off;
  a.rev_list = rev_list;
  a.s = s;
  a.lse_s = lse_s;
  a.lse_o = lse_o;
  a.drow = drow;
  a.dl = dl;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.idx = idx;
  a.err = err;
  a.B = sh.B;
  a.Hq = sh.Hq;
  a.Hkv = sh.Hkv;
  a.G = sh.G;
  a.N = sh.N;
  a.NB = sh.NB;
  a.K = sh.K;
  a.gated = sh.gated;
  a.n_hp = (sh.G + 1) / 2;
  a.n_tp = (sh.G + 3) / 4;
  a.scale = sh.scale;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(bwd_kv_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bkv::kSmem)) !=
      cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(bwd_q_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bq::kSmem)) !=
      cudaSuccess)
    return e;
  bwd_kv_sm100_kernel<<<dim3(sh.NB, sh.Hkv, sh.B), bkv::kThreads, bkv::kSmem, st>>>(tq, tk, tv, tdo, a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  bwd_q_sm100_kernel<<<dim3(sh.NB, sh.Hkv * a.n_tp, sh.B), bq::kThreads, bq::kSmem, st>>>(tq, tk, tv, tdo, a);
  return cudaGetLastError();
}

}  // namespace sas
