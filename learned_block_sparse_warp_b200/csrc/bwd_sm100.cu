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
  const float* rev_lam;
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
constexpr int kThreads = 384;                 // 0 TMA, 1 and 3 MMA, 2 spare, 4-7 and 8-11 softmax gradient
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

// tmQ3 / tmDO3 load both heads of a head pair per box; tmL / tmD load their
// saved row LSE and D. Two threads issue the MMAs, one for S and dVᵀ and one
// for dP and dKᵀ, because a single thread needs about 70 cycles per MMA issue,
// more than an N = 64 MMA takes to run.
__global__ void __launch_bounds__(bkv::kThreads, 1)
    bwd_kv_sm100_kernel(const __grid_constant__ CUtensorMap tmQ3, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO3,
                        const __grid_constant__ CUtensorMap tmL, const __grid_constant__ CUtensorMap tmD,
                        BwdSm100Args a) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t bar_kv, bar_full[bkv::kStages], bar_empty[bkv::kStages], bar_s[2], bar_p, bar_pz,
      bar_fin;
  __shared__ bkv::Meta meta[bkv::kStages];
  __shared__ int ring_w[64];
  __shared__ float ring_l[64];
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
  const float* lam_lst = a.rev_lam + bh * size_t(a.NB) * a.K + off0;
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
        mbar_init(smem_u32(&bar_empty[s]), 2);
      }
      mbar_init(smem_u32(&bar_s[0]), 2);
      mbar_init(smem_u32(&bar_s[1]), 2);
      mbar_init(smem_u32(&bar_p), 256);
      mbar_init(smem_u32(&bar_pz), 2);
      mbar_init(smem_u32(&bar_fin), 2);
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
    // Lane 0 issues the loads. The whole warp keeps a 64-entry ring of
    // reverse-index entries (t, slot) and their gates, filled 32 entries at a
    // time with cp.async one batch ahead, so no global load sits between two
    // TMA issues.
    const int n_ent = 1 + n_sel;
    auto fetch = [&](int batch) {
      const int e = 32 * batch + lane;
      if (e >= 1 && e < n_ent) {
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(smem_u32(&ring_w[e & 63])), "l"(lst + e - 1));
        asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(smem_u32(&ring_l[e & 63])),
                     "l"(lam_lst + e - 1));
      }
      cp_async_commit();
    };
    fetch(0);
    fetch(1);
    if (lane == 0) {
      tma_prefetch_desc(&tmQ3);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO3);
      tma_prefetch_desc(&tmL);
      tma_prefetch_desc(&tmD);
      const int krow = int(bh * a.N + size_t(j) * kBlock);
      mbar_arrive_expect_tx(smem_u32(&bar_kv), 4u * 8192u);
      for (int c = 0; c < 2; ++c) {
        tma_load_2d(sK + c * bkv::kHalf64, &tmK, c * 64, krow, smem_u32(&bar_kv));
        tma_load_2d(sV + c * bkv::kHalf64, &tmV, c * 64, krow, smem_u32(&bar_kv));
      }
    }
    int issued = 0;
    bool live = true;
    for (int i = 0; i < n_steps; ++i) {
      const int e = i / a.n_hp, hp = i % a.n_hp;
      if (hp == 0 && (e & 31) == 0) {  // entering batch e / 32
        __syncwarp();
        if (e >= 32) fetch(e / 32 + 1);  // into the half that batch e / 32 - 1 used
        cp_async_wait<1>();
        __syncwarp();
      }
      if (lane == 0 && live) {
        const int st = i % bkv::kStages, use = i / bkv::kStages;
        if (!mbar_wait(smem_u32(&bar_empty[st]), (use & 1) ^ 1, abort_flag, a.err)) {
          live = false;
          continue;
        }
        int t = j, slot = -1;
        float lam2 = 0.f;
        if (e > 0) {
          const int w = ring_w[e & 63];
          t = w >> 8;
          slot = w & 255;
          lam2 = ring_l[e & 63];
        }
        const int nv = min(2, a.G - 2 * hp);
        meta[st] = bkv::Meta{t, slot, nv, lam2};
        const uint32_t bar = smem_u32(&bar_full[st]);
        // a box always holds two heads; for a one-head pair the second head's rows
        // are another head's (or zero-filled past the tensor) and are masked to zero
        mbar_arrive_expect_tx(bar, 4u * 16384u + 2u * 512u);
        const uint32_t sq = sStage + st * bkv::kStage, sdo = sq + bkv::kTile, sl = sdo + bkv::kTile;
        const int hq0 = int(size_t(b) * a.Hq + size_t(h) * a.G + 2 * hp);
        for (int c = 0; c < 2; ++c) {
          tma_load_3d(sq + c * bkv::kHalf128, &tmQ3, c * 64, t * kBlock, hq0, bar);
          tma_load_3d(sdo + c * bkv::kHalf128, &tmDO3, c * 64, t * kBlock, hq0, bar);
        }
        tma_load_2d(sl, &tmL, t * kBlock, hq0, bar);
        tma_load_2d(sl + 512, &tmD, t * kBlock, hq0, bar);
        ++issued;
      }
    }
    cp_async_wait<0>();
    if (lane == 0 && *abort_flag) {
      for (int i = max(0, issued - bkv::kStages); i < issued; ++i) {
        const long long t0 = clock64();
        while (!mbar_try_wait(smem_u32(&bar_full[i % bkv::kStages]), (i / bkv::kStages) & 1) &&
               clock64() - t0 < kWaitCycles) {
        }
      }
    }
  } else if (warp == 1 || warp == 3) {
    // ------------------------------------------------------------ MMA issuers
    // warp 1: S = Q Kᵀ and dVᵀ += dOᵀ P; warp 3: dP = dO Vᵀ and dKᵀ += Qᵀ dZ
    if (lane == 0) {
      const bool first = (warp == 1);
      const uint32_t idS = idesc_bf16_f32(128, 64, 0, 0);     // S, dP: q rows x kv, K = d
      const uint32_t idG = idesc_bf16_f32(128, 64, 1, 1);     // dVᵀ, dKᵀ: d x kv, K = q rows
      // Descriptors are built once; a stage or K step only moves the start address.
      const uint32_t sA = sStage + (first ? 0u : uint32_t(bkv::kTile));      // Q or dO tile of stage 0
      const uint32_t sG = sStage + (first ? uint32_t(bkv::kTile) : 0u);      // dO or Q tile of stage 0
      const uint64_t dA = smem_desc_sw128(sA, 16, 1024);
      const uint64_t dB = smem_desc_sw128(first ? sK : sV, 16, 1024);
      const uint64_t dGa = smem_desc_sw128(sG, bkv::kHalf128, 1024);
      const uint64_t dGb = smem_desc_sw128(first ? sP : sZ, bkv::kHalf128, 1024);
      const uint32_t tD = tmem + (first ? 0u : 128u), tG = tmem + (first ? kColDV : kColDK);
      auto grads = [&](int i) {
        const uint32_t so = (i % bkv::kStages) * bkv::kStage;
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mma_ss(tG, desc_advance(dGa, so + k * 2048), desc_advance(dGb, k * 2048), idG, (i > 0 || k > 0) ? 1u : 0u);
        mma_commit(smem_u32(&bar_pz));
        mma_commit(smem_u32(&bar_empty[i % bkv::kStages]));
      };
      bool ok = mbar_wait(smem_u32(&bar_kv), 0, abort_flag, a.err);
      tc_fence_after();
      for (int i = 0; ok && i < n_steps; ++i) {
        const int st = i % bkv::kStages, use = i / bkv::kStages, sb = i & 1;
        if (!(ok = mbar_wait(smem_u32(&bar_full[st]), use & 1, abort_flag, a.err))) break;
        tc_fence_after();
        const uint32_t so = st * bkv::kStage;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t oa = (k >> 2) * bkv::kHalf128 + (k & 3) * 32, ob = (k >> 2) * bkv::kHalf64 + (k & 3) * 32;
          mma_ss(tD + sb * 64, desc_advance(dA, so + oa), desc_advance(dB, ob), idS, k > 0 ? 1u : 0u);
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
      // Columns this row may use: all 32, none for a missing head, and the causal
      // prefix on the diagonal block. L and D of a missing head are never read.
      int n_ok = valid ? 32 : 0;
      if (valid && diag) n_ok = min(32, max(0, qpos + 1 - wg * 32));
      if (!valid) L2 = 0.f, Dr = 0.f;
      uint32_t vs[32], vp[32];
      tmem_ld32(tmem + lane_addr + sb * 64 + wg * 32, vs);
      tmem_ld32(tmem + lane_addr + 128 + sb * 64 + wg * 32, vp);
      tmem_wait_ld();
      float pr[32];
#pragma unroll
      for (int x = 0; x < 32; ++x) pr[x] = fast_exp2(fmaf(__uint_as_float(vs[x]), sc2, -L2));
#pragma unroll
      for (int x = 0; x < 32; ++x) pr[x] = x < n_ok ? pr[x] : 0.f;
      float zr[32];
#pragma unroll
      for (int x = 0; x < 32; ++x) zr[x] = x < n_ok ? pr[x] * (__uint_as_float(vp[x]) - Dr) : 0.f;
      float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
#pragma unroll
      for (int x = 0; x < 32; x += 4) {
        s0 += zr[x];
        s1 += zr[x + 1];
        s2 += zr[x + 2];
        s3 += zr[x + 3];
      }
      dl_part += (s0 + s1) + (s2 + s3);
#pragma unroll
      for (int c4 = 0; c4 < 4; ++c4) {  // 16-byte chunk: 8 kv columns
        const uint32_t off = uint32_t(row * 128 + (((wg * 4 + c4) ^ (row & 7)) << 4));
        asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(sP + off),
                     "r"(pack_bf16x2(pr[8 * c4], pr[8 * c4 + 1])), "r"(pack_bf16x2(pr[8 * c4 + 2], pr[8 * c4 + 3])),
                     "r"(pack_bf16x2(pr[8 * c4 + 4], pr[8 * c4 + 5])), "r"(pack_bf16x2(pr[8 * c4 + 6], pr[8 * c4 + 7])));
        asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(sZ + off),
                     "r"(pack_bf16x2(zr[8 * c4], zr[8 * c4 + 1])), "r"(pack_bf16x2(zr[8 * c4 + 2], zr[8 * c4 + 3])),
                     "r"(pack_bf16x2(zr[8 * c4 + 4], zr[8 * c4 + 5])), "r"(pack_bf16x2(zr[8 * c4 + 6], zr[8 * c4 + 7])));
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
constexpr int kThreads = 384;                 // 0 TMA, 1 and 3 MMA, 2 spare, 4-7 and 8-11 softmax gradient
constexpr int kHalf = 128 * 128;              // one d-half of a 128-row tile
constexpr int kTile = 2 * kHalf;              // 128 rows x d 128
constexpr int kHalfKV = 64 * 128;             // one d-half of a 64-row block
constexpr int kStage = 4 * kHalfKV;           // K and V of one block
constexpr int kStages = 3;
constexpr int kSmem = 2 * kTile + kStages * kStage + 1024;
}  // namespace bq

// One CTA per (batch, KV head, query block, head pair): 128 rows. S and dP of
// consecutive blocks alternate between two TMEM buffers, so the tensor cores
// compute block i+1 while the softmax-gradient warps work on block i.
__global__ void __launch_bounds__(bq::kThreads, 1)
    bwd_q_sm100_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                       BwdSm100Args a) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  __shared__ int list_s[kMaxTopK + 1];
  __shared__ float lam_s[kMaxTopK + 1];
  __shared__ int nlist_s;
  // bar_p is per S/dP buffer: with one barrier the softmax warps could complete
  // two phases before the MMA thread observed the first, and its parity wait
  // would then never return.
  __shared__ __align__(8) uint64_t bar_q, bar_full[bq::kStages], bar_empty[bq::kStages], bar_s[2], bar_p[2],
      bar_o[2], bar_fin;
  __shared__ uint32_t tmem_s;
  __shared__ int abort_s;

  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const uint32_t sQ = base, sDO = base + bq::kTile, sKV = base + 2 * bq::kTile;
  const int t = a.NB - 1 - int(blockIdx.x);
  const int h = int(blockIdx.y) / a.n_hp, hp = int(blockIdx.y) % a.n_hp;
  const int b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nv = min(2, a.G - 2 * hp);  // heads in this tile
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
        mbar_init(smem_u32(&bar_empty[s]), 2);
      }
      for (int r = 0; r < 2; ++r) {
        mbar_init(smem_u32(&bar_s[r]), 2);
        mbar_init(smem_u32(&bar_o[r]), 1);
        mbar_init(smem_u32(&bar_p[r]), 256);
      }
      mbar_init(smem_u32(&bar_fin), 2);
      fence_barrier_init();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_s;
  const int nl = nlist_s;
  // TMEM columns: S buffers at 0 / 64, dP buffers at 128 / 192, dQ at 256. The
  // two warpgroups split the 64 kv columns; each writes its packed dZ over the
  // first 16 of its own 32 S columns, so tokens 0-31 sit at buffer columns
  // 0-15 and tokens 32-63 at columns 32-47.

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
      mbar_arrive_expect_tx(smem_u32(&bar_q), uint32_t(nv) * 4u * 8192u);
      for (int hh = 0; hh < nv; ++hh) {
        const int row = int((size_t(b) * a.Hq + size_t(h) * a.G + 2 * hp + hh) * a.N + size_t(t) * kBlock);
        for (int c = 0; c < 2; ++c) {
          tma_load_2d(sQ + c * bq::kHalf + hh * 8192, &tmQ, c * 64, row, smem_u32(&bar_q));
          tma_load_2d(sDO + c * bq::kHalf + hh * 8192, &tmDO, c * 64, row, smem_u32(&bar_q));
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
    // ------------------------------------------------------------ MMA issuer: S and dQ
    if (lane == 0) {
      const uint32_t idS = idesc_bf16_f32(128, 64, 0, 0);
      const uint32_t idQ = idesc_bf16_f32(128, 128, 0, 1);  // dQ: q rows x d, K = kv tokens (K MN-major)
      // Descriptors are built once; a stage or K step only moves the start address.
      const uint64_t dKmn0 = smem_desc_sw128(sKV, bq::kHalfKV, 1024);
      const uint64_t dQk0 = smem_desc_sw128(sQ, 16, 1024), dKk0 = smem_desc_sw128(sKV, 16, 1024);
      auto dq_mma = [&](int i) {  // dQ += dZ(i) K(i)
        const uint32_t so = (i % bq::kStages) * bq::kStage;
        const uint32_t zb = tmem + (i & 1) * 64;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_ts(tmem + 256, zb + (k >> 1) * 32 + (k & 1) * 8, desc_advance(dKmn0, so + k * 2048), idQ,
                 (i > 0 || k > 0) ? 1u : 0u);
        mma_commit(smem_u32(&bar_o[i & 1]));
        mma_commit(smem_u32(&bar_empty[i % bq::kStages]));
      };
      bool ok = mbar_wait(smem_u32(&bar_q), 0, abort_flag, a.err);
      tc_fence_after();
      for (int i = 0; ok && i < nl; ++i) {
        const int st = i % bq::kStages, use = i / bq::kStages, sb = i & 1;
        if (!(ok = mbar_wait(smem_u32(&bar_full[st]), use & 1, abort_flag, a.err))) break;
        // dQ(i - 2) read dZ from the S buffer that S(i) overwrites
        if (i >= 2 && !(ok = mbar_wait(smem_u32(&bar_o[sb]), ((i - 2) >> 1) & 1, abort_flag, a.err))) break;
        tc_fence_after();
        const uint32_t so = st * bq::kStage;
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mma_ss(tmem + sb * 64, desc_advance(dQk0, (k >> 2) * bq::kHalf + (k & 3) * 32),
                 desc_advance(dKk0, so + (k >> 2) * bq::kHalfKV + (k & 3) * 32), idS, k > 0 ? 1u : 0u);
        mma_commit(smem_u32(&bar_s[sb]));
        if (i > 0) {
          if (!(ok = mbar_wait(smem_u32(&bar_p[(i - 1) & 1]), ((i - 1) >> 1) & 1, abort_flag, a.err))) break;
          tc_fence_after();
          dq_mma(i - 1);
        }
      }
      if (ok && nl > 0 && mbar_wait(smem_u32(&bar_p[(nl - 1) & 1]), ((nl - 1) >> 1) & 1, abort_flag, a.err)) {
        tc_fence_after();
        dq_mma(nl - 1);
      }
      mma_commit(smem_u32(&bar_fin));
    }
  } else if (warp == 3) {
    // ------------------------------------------------------------ MMA issuer: dP
    if (lane == 0) {
      const uint32_t idS = idesc_bf16_f32(128, 64, 0, 0);
      const uint64_t dOk0 = smem_desc_sw128(sDO, 16, 1024);
      const uint64_t dVk0 = smem_desc_sw128(sKV + 2 * bq::kHalfKV, 16, 1024);
      bool ok = mbar_wait(smem_u32(&bar_q), 0, abort_flag, a.err);
      tc_fence_after();
      for (int i = 0; ok && i < nl; ++i) {
        const int st = i % bq::kStages, use = i / bq::kStages, sb = i & 1;
        if (!(ok = mbar_wait(smem_u32(&bar_full[st]), use & 1, abort_flag, a.err))) break;
        // the softmax warps finished reading dP(i - 2) from this buffer
        if (i >= 2 && !(ok = mbar_wait(smem_u32(&bar_p[sb]), ((i - 2) >> 1) & 1, abort_flag, a.err))) break;
        tc_fence_after();
        const uint32_t so = st * bq::kStage;
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mma_ss(tmem + 128 + sb * 64, desc_advance(dOk0, (k >> 2) * bq::kHalf + (k & 3) * 32),
                 desc_advance(dVk0, so + (k >> 2) * bq::kHalfKV + (k & 3) * 32), idS, k > 0 ? 1u : 0u);
        mma_commit(smem_u32(&bar_s[sb]));
        mma_commit(smem_u32(&bar_empty[st]));
      }
      mma_commit(smem_u32(&bar_fin));
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax gradient
    // Thread (w, row): row `row` of the tile, kv columns [32 w, 32 w + 32).
    const int w = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int row = 32 * quarter + lane;
    const uint32_t lane_addr = uint32_t(32 * quarter) << 16;
    const int hh = row >> 6, qpos = row & 63;
    const bool valid = hh < nv;
    const int hq = h * a.G + 2 * hp + hh;
    const size_t grow = (size_t(b) * a.Hq + (valid ? hq : h * a.G)) * a.N + size_t(t) * kBlock + qpos;
    const float L2 = valid ? a.lse_o[grow] * kLog2e : 0.f;
    const float Dr = valid ? a.drow[grow] : 0.f;
    const float sc2 = a.scale * kLog2e;
    bool ok = true;
    for (int i = 0; i < nl; ++i) {
      const int sb = i & 1;
      ok = mbar_wait(smem_u32(&bar_s[sb]), (i >> 1) & 1, abort_flag, a.err);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t tS = tmem + lane_addr + sb * 64 + w * 32, tP = tmem + lane_addr + 128 + sb * 64 + w * 32;
      const float off2 = L2 - lam_s[i];
      // Columns this row may use: all 32, none for a missing head, and the causal
      // prefix on the diagonal block.
      int n_ok = valid ? 32 : 0;
      if (valid && i == 0) n_ok = min(32, max(0, qpos + 1 - w * 32));
      uint32_t vs[32], vp[32], dz[16];
      tmem_ld32(tS, vs);
      tmem_ld32(tP, vp);
      tmem_wait_ld();
      float zr[32];
#pragma unroll
      for (int x = 0; x < 32; ++x) zr[x] = fast_exp2(fmaf(__uint_as_float(vs[x]), sc2, -off2));
#pragma unroll
      for (int x = 0; x < 32; ++x) zr[x] = x < n_ok ? zr[x] * (__uint_as_float(vp[x]) - Dr) : 0.f;
#pragma unroll
      for (int x = 0; x < 16; ++x) dz[x] = pack_bf16x2(zr[2 * x], zr[2 * x + 1]);
      tmem_st16(tS, dz);  // packed dZ over this warpgroup's own, already read S columns
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(smem_u32(&bar_p[sb]));
    }
    if (ok) ok = mbar_wait(smem_u32(&bar_fin), 0, abort_flag, a.err);
    ok = __all_sync(0xffffffffu, ok);
    if (ok && valid) {  // rows 64..127 of a one-head tile form whole warps
      tc_fence_after();
      const uint32_t tQ = tmem + lane_addr + 256 + w * 64;
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
                                   const float* rev_lam, float* dl, uint16_t* dq, uint16_t* dk, uint16_t* dv, int* err,
                                   cudaStream_t st) {
  CUtensorMap tq, tk, tv, tdo, tq3, tdo3, tl, td;
  const uint64_t hq = uint64_t(sh.B) * sh.Hq, rq = hq * sh.N, rkv = uint64_t(sh.B) * sh.Hkv * sh.N;
  if (!make_tmap_bf16_2d(&tq, q, rq, 128) || !make_tmap_bf16_2d(&tdo, dO, rq, 128) ||
      !make_tmap_bf16_2d(&tk, k, rkv, 128) || !make_tmap_bf16_2d(&tv, v, rkv, 128) ||
      !make_tmap_bf16_3d_heads(&tq3, q, hq, sh.N) || !make_tmap_bf16_3d_heads(&tdo3, dO, hq, sh.N) ||
      !make_tmap_f32_rows(&tl, lse_o, hq, sh.N) || !make_tmap_f32_rows(&td, drow, hq, sh.N))
    return cudaErrorInvalidValue;
  BwdSm100Args a;
  a.rev_off = rev_off;
  a.rev_list = rev_list;
  a.rev_lam = rev_lam;
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
  bwd_kv_sm100_kernel<<<dim3(sh.NB, sh.Hkv, sh.B), bkv::kThreads, bkv::kSmem, st>>>(tq3, tk, tv, tdo3, tl, td, a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  bwd_q_sm100_kernel<<<dim3(sh.NB, sh.Hkv * a.n_hp, sh.B), bq::kThreads, bq::kSmem, st>>>(tq, tk, tv, tdo, a);
  return cudaGetLastError();
}

}  // namespace sas
