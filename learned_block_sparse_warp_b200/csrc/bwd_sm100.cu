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
//       dP = dO Vᵀ land in a three-deep TMEM ring. The softmax-gradient warps
//       write P and dZ as bf16 rows, 128-byte swizzled, into shared memory.
//       dVᵀ += dOᵀ P and dKᵀ += Qᵀ dZ then accumulate in TMEM as M = 128
//       (d-major) MMAs with MN-major operands, so dK_j and dV_j stay on chip
//       for the whole walk. The CTA is also the only writer of dl[t, slot(j)].
//       With the full workspace it also stores every dZ tile (128 x 64 bf16
//       per query block, attended block and head pair) by TMA.
//   bwd_dq_sm100_kernel  (full workspace) one CTA per (batch, KV head, query
//       block, up to two head pairs): dQ = scale · Σ_j dZ_tj K_j as a gather
//       GEMM over the stored tiles and the attended K blocks, accumulated in
//       TMEM and written once in bf16. It reads each tile once and computes
//       no exponential: HBM-bound.
//   bwd_q_sm100_kernel   (minimal workspace) the same dQ without the stored
//       tiles: the tile's Q and dO rows stay in TMEM as the A operands of S
//       and dP, S and dP per selected block land in TMEM, dZ is written back
//       as bf16 over S, and dQ += dZ K is a TS MMA with K MN-major. It
//       recomputes S and dP (7 GEMM-shaped products instead of 5) in exchange
//       for a workspace without the tiles.
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
  int B, Hq, Hkv, G, N, NB, K, gate, gated, n_hp, n_tp;
  int d;  // head dim, 64 or 128; at 64 the tensor maps zero-fill the second 64-column half of every box
  float scale;
  int spill;            // 1: the KV pass stores every dZ tile and the dQ pass reads them back
  long long dz_slots;   // dZ slots per (batch, KV head): Σ_t (1 + min(K, t))
};

// First dZ slot of query block t: Σ_{t' < t} (1 + min(K, t')). Slot 0 of a query
// block holds its diagonal block, slot 1 + s the block in idx[t][s].
__host__ __device__ __forceinline__ long long dz_slot_base(int t, int K) {
  const long long tt = t, kk = K;
  if (tt <= kk + 1) return tt + tt * (tt - 1) / 2;
  return (kk + 1) + kk * (kk + 1) / 2 + (tt - kk - 1) * (kk + 1);
}

// ===========================================================================
// Pass 1: dK, dV and dl, KV-major
// ===========================================================================
namespace bkv {
constexpr int kSoftWarps = 16;                   // softmax-gradient warps: 4 column groups x 4 TMEM lane quarters
constexpr int kWarpDK = 4 + kSoftWarps;          // 20
constexpr int kWarpProdO = kWarpDK + 1;          // 21
constexpr int kThreads = 32 * (kWarpProdO + 1);  // 704
constexpr int kTile = 32768;                     // 128 rows (two heads) x d 128 bf16, two 16 KB d-halves
constexpr int kHalf = 16384;
constexpr int kHalf64 = 8192;                    // one d-half of the 64-row K or V block
constexpr int kNQ = 3, kNO = 2;                  // Q slots, dO slots
constexpr int kOffK = 0, kOffV = 16384;
constexpr int kOffQ = 32768;                     // kNQ Q tiles
constexpr int kOffO = kOffQ + kNQ * kTile;       // kNO dO tiles
constexpr int kOffP = kOffO + kNO * kTile;       // P: 128 q rows x 64 kv bf16, 128-byte rows, swizzled
constexpr int kOffZ = kOffP + 16384;             // dZ, same layout
constexpr int kOffL = kOffZ + 16384;             // kNQ rows of 128 saved LSEs
constexpr int kOffD = kOffL + kNQ * 512;         // kNO rows of 128 D values
constexpr int kOffCtl = kOffD + kNO * 512;
constexpr int kSmem = kOffCtl + 512;             // 232448 bytes: the whole opt-in shared memory
struct Meta {
  int t, slot, nv;
  float lam2;
};
struct Ctl {
  uint64_t bar_kv, fq[kNQ], eq[kNQ], fo[kNO], eo[kNO], bs[3], bd[3], bp[3], bz[3], pf, zf, fin;
  Meta meta[kNQ];
  float red_s[2][kSoftWarps];
  uint32_t tmem;
  int abort;
};
static_assert(sizeof(Ctl) <= 512, "control block");
static_assert(kSmem == 232448, "shared memory plan");
}  // namespace bkv

// Loads the walk's reverse-index entries 32 at a time into the lanes of a
// warp, one batch ahead: entry e of the walk (e >= 1) is rev_list[e - 1].
struct EntryRing {
  int w_cur, w_nxt;
  float l_cur, l_nxt;
  int batch;
  __device__ void load(const int* lst, const float* lam, int n_ent, int b, int lane, int& w, float& l) {
    const int e = 32 * b + lane;
    w = (e >= 1 && e < n_ent) ? lst[e - 1] : 0;
    l = (e >= 1 && e < n_ent) ? lam[e - 1] : 0.f;
  }
  __device__ void init(const int* lst, const float* lam, int n_ent, int lane) {
    batch = 0;
    load(lst, lam, n_ent, 0, lane, w_cur, l_cur);
    load(lst, lam, n_ent, 1, lane, w_nxt, l_nxt);
  }
  // (t, slot, gate) of entry e; e never decreases between calls, and e < 32 (batch + 2)
  __device__ void get(const int* lst, const float* lam, int n_ent, int lane, int e, int j, int& t, int& slot,
                      float& lam2) {
    while ((e >> 5) > batch) {
      w_cur = w_nxt;
      l_cur = l_nxt;
      ++batch;
      load(lst, lam, n_ent, batch + 1, lane, w_nxt, l_nxt);
    }
    const int w = __shfl_sync(0xffffffffu, w_cur, e & 31);
    lam2 = __shfl_sync(0xffffffffu, l_cur, e & 31);
    t = e == 0 ? j : (w >> kSlotBits);
    slot = e == 0 ? -1 : (w & ((1 << kSlotBits) - 1));
    if (e == 0) lam2 = 0.f;
  }
  // t of entry e of the next batch at most, for prefetching (no state change)
  __device__ int peek_t(int e, int j) const {
    const int src = (e >> 5) == batch ? w_cur : w_nxt;
    const int w = __shfl_sync(0xffffffffu, src, e & 31);
    return e == 0 ? j : (w >> kSlotBits);
  }
};

// tmQ3 / tmDO3 load both heads of a head pair per box; tmL / tmD load their
// saved row LSE and D. The walk's steps are (entry, head pair). Q tiles sit in
// a ring of three slots and dO tiles in a ring of two, each with its own
// producer warp: a Q tile lives from S = Q Kᵀ to dKᵀ += Qᵀ dZ, which spans the
// whole step, so a third slot keeps its load off the step's critical path.
// Four threads issue the MMAs (S, dP, dVᵀ, dKᵀ), so that each product's group
// of eight dependent MMAs, about 800 cycles from first issue to completion,
// overlaps the others instead of queueing behind them on one thread. Sixteen
// softmax-gradient warps (four per SM sub-partition) write P as soon as S
// allows, so dVᵀ starts before dP is consumed, then dZ.
//
// Per step i, with q = i % 3, o = i % 2 and b = i % 3 (the TMEM S/dP buffer):
//   Q producer   waits eq[q] (step i - 3), loads Q, L        -> fq[q]
//   dO producer  waits eo[o] (step i - 2), loads dO, D       -> fo[o]
//   S            waits fq[q], bp[b] (step i - 3)             -> bs[b], eq[q]
//   dP           waits fo[o], bz[b] (step i - 3)             -> bd[b], eo[o]
//   softmax      waits fq[q], fo[o], bs[b], reads L, D and the entry;
//                waits pf (step i - 1), writes P  -> bp[b]
//                waits bd[b] and zf (step i - 1), writes dZ -> bz[b]
//   dVᵀ          waits fo[o], bp[b]                          -> pf, eo[o]
//   dKᵀ          waits fq[q], bz[b]                          -> zf, eq[q]
//                and, when spilling, stores the dZ tile     -> zf (second arrival, once it is read)
// bp and bz are per TMEM buffer because the S and dP issuers wait three steps
// back; with one barrier they could fall phases behind. Every other waiter's
// next phase needs the waiter's own next action first. The three-deep ring
// lets S and dP run up to three steps ahead of the softmax-gradient warps.
// kOut: the gate weights the values after a softmax over the plain logits
// (SAS_GATE_SOFTMAX_OUTSIDE): dVᵀ takes g·P, dZ = P·(g·dP − D) and
// dl = Σ P·g·dP (= g ∂/∂g) instead of Σ dZ.
template <bool kOut>
__global__ void __launch_bounds__(bkv::kThreads, 1)
    bwd_kv_sm100_kernel(const __grid_constant__ CUtensorMap tmQ3, const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO3,
                        const __grid_constant__ CUtensorMap tmL, const __grid_constant__ CUtensorMap tmD,
                        const __grid_constant__ CUtensorMap tmDZ, BwdSm100Args a) {
  using namespace sm100;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t base = smem_u32(smem_raw);
  if (base & 1023u) {  // the swizzled tiles need 1024-byte alignment; there is no room to pad
    if (threadIdx.x == 0) raise_error(a.err, SAS_ERR_CUDA);
    return;
  }
  bkv::Ctl& C = *reinterpret_cast<bkv::Ctl*>(smem_raw + bkv::kOffCtl);
  const uint32_t sK = base + bkv::kOffK, sV = base + bkv::kOffV;
  const uint32_t sQ = base + bkv::kOffQ, sO = base + bkv::kOffO;
  const uint32_t sP = base + bkv::kOffP, sZ = base + bkv::kOffZ;
  const uint32_t sL = base + bkv::kOffL, sD = base + bkv::kOffD;
  const int j = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t bh = size_t(b) * a.Hkv + h;
  const int off0 = a.rev_off[bh * (a.NB + 1) + j];
  const int n_sel = a.rev_off[bh * (a.NB + 1) + j + 1] - off0;
  const int* lst = a.rev_list + bh * size_t(a.NB) * a.K + off0;
  const float* lam_lst = a.rev_lam + bh * size_t(a.NB) * a.K + off0;
  const int n_ent = 1 + n_sel;
  const int n_steps = n_ent * a.n_hp;
  const int hq_base = int(size_t(b) * a.Hq + size_t(h) * a.G);
  volatile int* abort_flag = &C.abort;

  if (threadIdx.x == 0) C.abort = 0;
  if (a.G & 1) {  // keep the rows of a missing head finite: zero every Q and dO tile once
    for (int i = threadIdx.x; i < (bkv::kNQ + bkv::kNO) * bkv::kTile / 16; i += bkv::kThreads)
      asm volatile("st.shared.v4.u32 [%0], {%1,%1,%1,%1};\n" ::"r"(sQ + i * 16), "r"(0));
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&C.tmem), 512);
    if (lane == 0) {
      mbar_init(smem_u32(&C.bar_kv), 1);
      for (int s = 0; s < bkv::kNQ; ++s) {
        mbar_init(smem_u32(&C.fq[s]), 1);
        mbar_init(smem_u32(&C.eq[s]), 2);
      }
      for (int s = 0; s < bkv::kNO; ++s) {
        mbar_init(smem_u32(&C.fo[s]), 1);
        mbar_init(smem_u32(&C.eo[s]), 2);
      }
      for (int r = 0; r < 3; ++r) {
        mbar_init(smem_u32(&C.bs[r]), 1);
        mbar_init(smem_u32(&C.bd[r]), 1);
        mbar_init(smem_u32(&C.bp[r]), bkv::kSoftWarps);
        mbar_init(smem_u32(&C.bz[r]), bkv::kSoftWarps);
      }
      mbar_init(smem_u32(&C.pf), 1);
      mbar_init(smem_u32(&C.zf), a.spill ? 2 : 1);  // dKᵀ's commit, and the dZ store's read when spilling
      mbar_init(smem_u32(&C.fin), 2);
      fence_barrier_init();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = C.tmem;
  // TMEM columns: S buffers 0 / 64 / 128, dP buffers 192 / 256 / 320, dVᵀ 384, dKᵀ 448
  constexpr uint32_t kColDV = 384, kColDK = 448;

  if (warp == 0 || warp == bkv::kWarpProdO) {
    // ------------------------------------------------------------ TMA producers
    // warp 0: Q tiles and L rows; the last warp: dO tiles and D rows. Lane 0
    // issues; the warp holds the walk's entries in its lanes.
    const bool is_q = (warp == 0);
    EntryRing ring;
    ring.init(lst, lam_lst, n_ent, lane);
    if (is_q && lane == 0) {
      tma_prefetch_desc(&tmQ3);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmL);
      const int krow = int(bh * a.N + size_t(j) * kBlock);
      mbar_arrive_expect_tx(smem_u32(&C.bar_kv), 4u * 8192u);
      for (int c = 0; c < 2; ++c) {
        tma_load_2d(sK + c * bkv::kHalf64, &tmK, c * 64, krow, smem_u32(&C.bar_kv));
        tma_load_2d(sV + c * bkv::kHalf64, &tmV, c * 64, krow, smem_u32(&C.bar_kv));
      }
    }
    if (!is_q && lane == 0) {
      tma_prefetch_desc(&tmDO3);
      tma_prefetch_desc(&tmD);
    }
    const int nslot = is_q ? bkv::kNQ : bkv::kNO;
    const CUtensorMap* tm = is_q ? &tmQ3 : &tmDO3;
    const CUtensorMap* tr = is_q ? &tmL : &tmD;
    const uint32_t s_tile = is_q ? sQ : sO, s_row = is_q ? sL : sD;
    int issued = 0;
    bool live = true;
    for (int i = 0; i < n_steps; ++i) {
      const int e = i / a.n_hp, hp = i % a.n_hp;
      int t, slot;
      float lam2;
      ring.get(lst, lam_lst, n_ent, lane, e, j, t, slot, lam2);
      const int i2 = i + 2;  // tiles to warm in L2: two steps ahead, within the entries held
      const int t2 = (i2 < n_steps && (i2 / a.n_hp) < 32 * (ring.batch + 2)) ? ring.peek_t(i2 / a.n_hp, j) : -1;
      if (lane == 0 && live) {
        const int st = i % nslot, use = i / nslot;
        const uint32_t emp = smem_u32(is_q ? &C.eq[st] : &C.eo[st]);
        if (!mbar_wait(emp, (use & 1) ^ 1, abort_flag, a.err)) {
          live = false;
        } else {
          const int nv = min(2, a.G - 2 * hp);
          if (is_q) C.meta[st] = bkv::Meta{t, slot, nv, lam2};
          const uint32_t full = smem_u32(is_q ? &C.fq[st] : &C.fo[st]);
          const int hq0 = hq_base + 2 * hp;
          // a box always holds two heads; for a one-head pair the second head's rows
          // are another head's (or zero-filled past the tensor) and are masked to zero
          mbar_arrive_expect_tx(full, 2u * 16384u + 512u);
          for (int c = 0; c < 2; ++c) tma_load_3d(s_tile + st * bkv::kTile + c * bkv::kHalf, tm, c * 64, t * kBlock, hq0, full);
          tma_load_2d(s_row + st * 512, tr, t * kBlock, hq0, full);
          ++issued;
          if (t2 >= 0) {
            const int hq2 = hq_base + 2 * (i2 % a.n_hp);
            for (int c = 0; c < 2; ++c) tma_prefetch_l2_3d(tm, c * 64, t2 * kBlock, hq2);
          }
        }
      }
      live = __shfl_sync(0xffffffffu, live, 0);
    }
    if (lane == 0 && *abort_flag) {  // let the copies in flight land before the CTA exits
      for (int i = max(0, issued - nslot); i < issued; ++i) {
        const uint32_t full = smem_u32(is_q ? &C.fq[i % nslot] : &C.fo[i % nslot]);
        const long long t0 = clock64();
        while (!mbar_try_wait(full, (i / nslot) & 1) && clock64() - t0 < kWaitCycles) {
        }
      }
    }
  } else if (warp == 1 || warp == 3) {
    // ------------------------------------------------------------ MMA issuers: S = Q Kᵀ (warp 1), dP = dO Vᵀ (warp 3)
    if (lane == 0) {
      const bool is_s = (warp == 1);
      const int nslot = is_s ? bkv::kNQ : bkv::kNO;
      const uint32_t idS = idesc_bf16_f32(128, 64, 0, 0);  // q rows x kv, K = d
      // Descriptors are built once; a slot or K step only moves the start address.
      const uint64_t dA = smem_desc_sw128(is_s ? sQ : sO, 16, 1024);
      const uint64_t dB = smem_desc_sw128(is_s ? sK : sV, 16, 1024);
      const uint32_t tD = tmem + (is_s ? 0u : 192u);
      bool ok = mbar_wait(smem_u32(&C.bar_kv), 0, abort_flag, a.err);
      tc_fence_after();
      for (int i = 0; ok && i < n_steps; ++i) {
        const int st = i % nslot, use = i / nslot, sb = i % 3;
        if (!(ok = mbar_wait(smem_u32(is_s ? &C.fq[st] : &C.fo[st]), use & 1, abort_flag, a.err))) break;
        // the softmax-gradient warps have read S / dP of step i - 3 from this buffer
        if (i >= 3 && !(ok = mbar_wait(smem_u32(is_s ? &C.bp[sb] : &C.bz[sb]), ((i - 3) / 3) & 1, abort_flag, a.err)))
          break;
        tc_fence_after();
        const uint32_t so = st * bkv::kTile;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t oa = (k >> 2) * bkv::kHalf + (k & 3) * 32, ob = (k >> 2) * bkv::kHalf64 + (k & 3) * 32;
          mma_ss(tD + sb * 64, desc_advance(dA, so + oa), desc_advance(dB, ob), idS, k > 0 ? 1u : 0u);
        }
        mma_commit(smem_u32(is_s ? &C.bs[sb] : &C.bd[sb]));
        mma_commit(smem_u32(is_s ? &C.eq[st] : &C.eo[st]));
      }
    }
  } else if (warp == 2 || warp == bkv::kWarpDK) {
    // ------------------------------------------------------------ MMA issuers: dVᵀ += dOᵀ P (warp 2), dKᵀ += Qᵀ dZ
    if (lane == 0) {
      const bool is_v = (warp == 2);
      const int nslot = is_v ? bkv::kNO : bkv::kNQ;
      const uint32_t idG = idesc_bf16_f32(128, 64, 1, 1);  // d x kv, K = q rows, both operands MN-major
      const uint64_t dGa = smem_desc_sw128(is_v ? sO : sQ, bkv::kHalf, 1024);
      const uint64_t dGb = smem_desc_sw128(is_v ? sP : sZ, bkv::kHalf, 1024);
      const uint32_t tG = tmem + (is_v ? kColDV : kColDK);
      bool ok = true;
      for (int i = 0; ok && i < n_steps; ++i) {
        const int st = i % nslot, use = i / nslot, sb = i % 3;
        if (!(ok = mbar_wait(smem_u32(is_v ? &C.fo[st] : &C.fq[st]), use & 1, abort_flag, a.err))) break;
        if (!(ok = mbar_wait(smem_u32(is_v ? &C.bp[sb] : &C.bz[sb]), (i / 3) & 1, abort_flag, a.err))) break;
        tc_fence_after();
        // read before the MMAs: their commit on eq lets the producer refill this Q slot and its meta
        const bkv::Meta m = is_v ? bkv::Meta{0, 0, 0, 0.f} : C.meta[st];
        const uint32_t so = st * bkv::kTile;
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mma_ss(tG, desc_advance(dGa, so + k * 2048), desc_advance(dGb, k * 2048), idG, (i > 0 || k > 0) ? 1u : 0u);
        mma_commit(smem_u32(is_v ? &C.pf : &C.zf));
        mma_commit(smem_u32(is_v ? &C.eo[st] : &C.eq[st]));
        if (!is_v && a.spill) {
          // The dZ tile also goes to the workspace, where the dQ pass reads it back
          // instead of recomputing S and dP. The buffer is released (the second
          // arrival on zf) once the store has read it.
          const long long tile =
              (static_cast<long long>(bh) * a.dz_slots + dz_slot_base(m.t, a.K) + (m.slot + 1)) * a.n_hp + (i % a.n_hp);
          tma_store_3d(&tmDZ, 0, 0, int(tile), sZ);
          bulk_commit_group();
          bulk_wait_read_all();
          mbar_arrive(smem_u32(&C.zf));
        }
      }
      mma_commit(smem_u32(&C.fin));
      if (!is_v && a.spill) bulk_wait_all();
    }
  } else if (warp >= 4 && warp < 4 + bkv::kSoftWarps) {
    // ------------------------------------------------------------ softmax gradient
    // Thread (cg, row): q row `row`, kv columns [16 cg, 16 cg + 16).
    const int sw = warp - 4;
    const int cg = sw >> 2;
    const int quarter = warp & 3;  // the TMEM lane quarter this warp may access
    const int row = 32 * quarter + lane;
    const uint32_t lane_addr = uint32_t(32 * quarter) << 16;
    const int hh = row >> 6, qpos = row & 63;
    const float sc2 = a.scale * kLog2e;
    float dl_part = 0.f;
    bool ok = true;
    // After an abort a warp keeps walking the steps without touching TMEM or
    // shared tiles, so that every softmax warp still meets named barrier 1.
    for (int i = 0; i < n_steps; ++i) {
      const int qs = i % bkv::kNQ, os = i % bkv::kNO, sb = i % 3;
      const int e = i / a.n_hp, hp = i % a.n_hp;
      const bool diag = (e == 0);
      // Everything this step reads from the Q and dO slots (L, D, the entry) is
      // read here: once P is released, dVᵀ may free the dO slot for step i + 2.
      if (ok) {
        ok = mbar_wait(smem_u32(&C.fq[qs]), (i / bkv::kNQ) & 1, abort_flag, a.err);
        ok = ok && mbar_wait(smem_u32(&C.fo[os]), (i / bkv::kNO) & 1, abort_flag, a.err);
        ok = ok && mbar_wait(smem_u32(&C.bs[sb]), (i / 3) & 1, abort_flag, a.err);
        ok = __all_sync(0xffffffffu, ok);
      }
      const bkv::Meta m = C.meta[qs];
      const bool valid = hh < m.nv;  // uniform over the warp: a warp's rows belong to one head
      const int n_ok = valid ? (diag ? min(16, max(0, qpos + 1 - cg * 16)) : 16) : 0;
      float pr[16];
      float Dr = 0.f;
      if (ok) {
        tc_fence_after();
        float L2 = 0.f;
        asm volatile("ld.shared.f32 %0, [%1];\n" : "=f"(L2) : "r"(sL + qs * 512 + row * 4));
        asm volatile("ld.shared.f32 %0, [%1];\n" : "=f"(Dr) : "r"(sD + os * 512 + row * 4));
        L2 = L2 * kLog2e - (kOut ? 0.f : m.lam2);  // P = exp2(S·sc2 − (L·log2e − λ))
        uint32_t vs[16];
        tmem_ld16(tmem + lane_addr + sb * 64 + cg * 16, vs);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          const float pe = fast_exp2(fmaf(__uint_as_float(vs[x]), sc2, -L2));
          pr[x] = x < n_ok ? pe : 0.f;  // none for a missing head, the causal prefix on the diagonal
        }
        // dVᵀ of step i - 1 has read the P buffer
        if (i >= 1) ok = mbar_wait(smem_u32(&C.pf), (i - 1) & 1, abort_flag, a.err);
        ok = __all_sync(0xffffffffu, ok);
      }
      const float gw = kOut ? fast_exp2(m.lam2) : 1.f;  // the gate outside the softmax (1 on the diagonal)
      if (ok) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {  // 16-byte chunk 2 cg + c: 8 kv columns
          const uint32_t off = uint32_t(row * 128 + (((2 * cg + c) ^ (row & 7)) << 4));
          float w8[8];
#pragma unroll
          for (int x = 0; x < 8; ++x) w8[x] = kOut ? pr[8 * c + x] * gw : pr[8 * c + x];  // dVᵀ's weights
          asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(sP + off),
                       "r"(pack_bf16x2(w8[0], w8[1])), "r"(pack_bf16x2(w8[2], w8[3])),
                       "r"(pack_bf16x2(w8[4], w8[5])), "r"(pack_bf16x2(w8[6], w8[7])));
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&C.bp[sb]));
        ok = mbar_wait(smem_u32(&C.bd[sb]), (i / 3) & 1, abort_flag, a.err);
        ok = __all_sync(0xffffffffu, ok);
      }
      if (ok) {
        tc_fence_after();
        uint32_t vp[16];
        tmem_ld16(tmem + lane_addr + 192 + sb * 64 + cg * 16, vp);
        tmem_wait_ld();
        float zr[16];
        float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
        if constexpr (kOut) {
#pragma unroll
          for (int x = 0; x < 16; ++x) {
            const float gdp = gw * __uint_as_float(vp[x]);
            zr[x] = pr[x] * (gdp - Dr);
            const float term = pr[x] * gdp;  // dl's term: P·g·dP
            if ((x & 3) == 0) s0 += term;
            else if ((x & 3) == 1) s1 += term;
            else if ((x & 3) == 2) s2 += term;
            else s3 += term;
          }
        } else {
#pragma unroll
          for (int x = 0; x < 16; ++x) zr[x] = pr[x] * (__uint_as_float(vp[x]) - Dr);  // P is 0 where masked
#pragma unroll
          for (int x = 0; x < 16; x += 4) {
            s0 += zr[x];
            s1 += zr[x + 1];
            s2 += zr[x + 2];
            s3 += zr[x + 3];
          }
        }
        dl_part += (s0 + s1) + (s2 + s3);
        // dKᵀ of step i - 1 has read the dZ buffer
        if (i >= 1) ok = mbar_wait(smem_u32(&C.zf), (i - 1) & 1, abort_flag, a.err);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const uint32_t off = uint32_t(row * 128 + (((2 * cg + c) ^ (row & 7)) << 4));
            asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(sZ + off),
                         "r"(pack_bf16x2(zr[8 * c], zr[8 * c + 1])), "r"(pack_bf16x2(zr[8 * c + 2], zr[8 * c + 3])),
                         "r"(pack_bf16x2(zr[8 * c + 4], zr[8 * c + 5])), "r"(pack_bf16x2(zr[8 * c + 6], zr[8 * c + 7])));
          }
          fence_proxy_async_smem();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(&C.bz[sb]));
        }
      }
      if (hp == a.n_hp - 1) {  // the entry's last head pair: dl[t, slot] has this CTA as its only writer
        if (!diag) {
          const float w = warp_sum(dl_part);
          if (lane == 0) C.red_s[e & 1][sw] = w;
          named_bar_sync(1, 32 * bkv::kSoftWarps);
          if (sw == 0 && lane == 0 && a.gated && !*abort_flag) {
            float tot = 0.f;
#pragma unroll
            for (int k = 0; k < bkv::kSoftWarps; ++k) tot += C.red_s[e & 1][k];
            a.dl[(bh * a.NB + m.t) * a.K + m.slot] = tot;
          }
        }
        dl_part = 0.f;
      }
    }
    // epilogue: column groups 0 / 1 write kv columns 0-31 / 32-63 of dV, groups
    // 2 / 3 those of dK. TMEM lanes are d rows, so each row is transposed
    // through shared memory into [kv][d], in the P and dZ buffers.
    ok = ok && mbar_wait(smem_u32(&C.fin), 0, abort_flag, a.err);
    ok = __all_sync(0xffffffffu, ok);
    const bool is_v = cg < 2;
    const uint32_t stage_buf = is_v ? sP : sZ;  // [64 kv][128 d] bf16, row-major
    if (ok) {
      tc_fence_after();
      const int d = row;
      const float mul = is_v ? 1.f : a.scale;
      uint32_t v[32];
      tmem_ld32(tmem + lane_addr + (is_v ? kColDV : kColDK) + (cg & 1) * 32, v);
      tmem_wait_ld();
#pragma unroll
      for (int x = 0; x < 32; ++x) {
        const __nv_bfloat16 bv = __float2bfloat16_rn(__uint_as_float(v[x]) * mul);
        const uint16_t bits = *reinterpret_cast<const uint16_t*>(&bv);
        asm volatile("st.shared.u16 [%0], %1;\n" ::"r"(stage_buf + ((cg & 1) * 32 + x) * 256 + d * 2), "h"(bits));
      }
    }
    named_bar_sync(2 + (is_v ? 0 : 1), 256);
    if (ok) {  // the staged rows hold 128 d; the first d of them go out
      const int cpr = a.d / 8;  // 16-byte chunks per output row
      uint16_t* dst = (is_v ? a.dv : a.dk) + (bh * a.N + size_t(j) * kBlock) * a.d;
      uint4* g = reinterpret_cast<uint4*>(dst);
      for (int i = (cg & 1) * 128 + row; i < 64 * cpr; i += 256) {
        uint4 x;
        asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n" : "=r"(x.x), "=r"(x.y), "=r"(x.z), "=r"(x.w)
                     : "r"(stage_buf + ((i / cpr) * 16 + i % cpr) * 16));
        g[i] = x;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    if (lane == 0) {
      const long long t0 = clock64();
      while (!mbar_try_wait(smem_u32(&C.fin), 0) && clock64() - t0 < kWaitCycles) {
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
constexpr int kSoftWarps = 16;                // 4 column groups x 4 TMEM lane quarters
constexpr int kThreads = 32 * (4 + kSoftWarps);  // 0 TMA, 1 S, 2 dQ, 3 dP MMA issue, 4-19 softmax gradient
constexpr int kHalfKV = 64 * 128;             // one d-half of a 64-row block
constexpr int kStage = 4 * kHalfKV;           // K and V of one block
constexpr int kStages = 6;
constexpr int kSmem = kStages * kStage + 1024;
}  // namespace bq

// One CTA per (batch, KV head, query block, head pair): 128 rows. The tile's
// Q and dO rows stay in TMEM for the whole walk as the A operands of
// S = Q Kᵀ and dP = dO Vᵀ (TS MMAs), so shared memory only carries the
// gathered K and V blocks, six deep. S and dP of consecutive blocks alternate
// between two TMEM buffers, so the tensor cores compute block i + 1 while the
// softmax-gradient warps work on block i. kOut as in the KV pass: dZ = P·(g·dP − D)
// over the plain logits.
template <bool kOut>
__global__ void __launch_bounds__(bq::kThreads, 1)
    bwd_q_sm100_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                       const uint16_t* __restrict__ q, const uint16_t* __restrict__ dO, BwdSm100Args a) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  __shared__ int list_s[kMaxTopK + 1];
  __shared__ float lam_s[kMaxTopK + 1];
  __shared__ int nlist_s;
  // bar_p is per S/dP buffer: with one barrier the softmax warps could complete
  // two phases before the MMA thread observed the first, and its parity wait
  // would then never return.
  __shared__ __align__(8) uint64_t bar_qo, bar_full[bq::kStages], bar_empty[bq::kStages], bar_s[2], bar_p[2],
      bar_o[2], bar_fin;
  __shared__ uint32_t tmem_s;
  __shared__ int abort_s;

  const uint32_t sKV = (smem_u32(smem_raw) + 1023u) & ~1023u;
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
                     a.lse_s != nullptr ? a.lse_s[row] : 0.f, a.gate, list_s, lam_s, &nlist_s, a.err);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_s), 512);
    if (lane == 0) {
      mbar_init(smem_u32(&bar_qo), bq::kSoftWarps);
      for (int s = 0; s < bq::kStages; ++s) {
        mbar_init(smem_u32(&bar_full[s]), 1);
        mbar_init(smem_u32(&bar_empty[s]), 2);
      }
      for (int r = 0; r < 2; ++r) {
        mbar_init(smem_u32(&bar_s[r]), 2);
        mbar_init(smem_u32(&bar_o[r]), 1);
        mbar_init(smem_u32(&bar_p[r]), bq::kSoftWarps);
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
  // TMEM columns: S buffers at 0 / 64, dP buffers at 128 / 192, dQ at 256, and
  // the tile's Q and dO as bf16 pairs at 384 and 448 (column 8 k + c holds d
  // elements 16 k + 2 c and 16 k + 2 c + 1). The four column groups split the
  // 64 kv columns; each writes its packed dZ over the first 8 of its own 16 S
  // columns, so tokens 16 k .. 16 k + 15 sit at buffer columns 16 k .. 16 k + 7,
  // the A operand of the k-th dQ MMA.
  constexpr uint32_t kColQ = 384, kColDO = 448;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
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
  } else if (warp == 1 || warp == 3) {
    // ------------------------------------------------------------ MMA issuers: S = Q Kᵀ (warp 1), dP = dO Vᵀ (warp 3)
    if (lane == 0) {
      const bool is_s = (warp == 1);
      const uint32_t idS = idesc_bf16_f32(128, 64, 0, 0);
      // Descriptors are built once; a stage or K step only moves the start address.
      const uint64_t dB0 = smem_desc_sw128(sKV + (is_s ? 0u : uint32_t(2 * bq::kHalfKV)), 16, 1024);
      const uint32_t tA = tmem + (is_s ? kColQ : kColDO);
      const uint32_t tD = tmem + (is_s ? 0u : 128u);
      bool ok = mbar_wait(smem_u32(&bar_qo), 0, abort_flag, a.err);
      tc_fence_after();
      for (int i = 0; ok && i < nl; ++i) {
        const int st = i % bq::kStages, use = i / bq::kStages, sb = i & 1;
        if (!(ok = mbar_wait(smem_u32(&bar_full[st]), use & 1, abort_flag, a.err))) break;
        if (i >= 2) {
          // S: dQ(i - 2) read dZ from the S buffer that S(i) overwrites.
          // dP: the softmax warps finished reading dP(i - 2) from this buffer.
          ok = is_s ? mbar_wait(smem_u32(&bar_o[sb]), ((i - 2) >> 1) & 1, abort_flag, a.err)
                    : mbar_wait(smem_u32(&bar_p[sb]), ((i - 2) >> 1) & 1, abort_flag, a.err);
          if (!ok) break;
        }
        tc_fence_after();
        const uint32_t so = st * bq::kStage;
#pragma unroll
        for (int k = 0; k < 8; ++k)
          mma_ts(tD + sb * 64, tA + 8 * k, desc_advance(dB0, so + (k >> 2) * bq::kHalfKV + (k & 3) * 32), idS,
                 k > 0 ? 1u : 0u);
        mma_commit(smem_u32(&bar_s[sb]));
        if (!is_s) mma_commit(smem_u32(&bar_empty[st]));
      }
      if (!is_s) mma_commit(smem_u32(&bar_fin));
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ MMA issuer: dQ
    // A separate thread from S, because one thread issuing both would spend
    // more cycles issuing than the tensor cores spend on the two products.
    if (lane == 0) {
      const uint32_t idQ = idesc_bf16_f32(128, 128, 0, 1);  // dQ: q rows x d, K = kv tokens (K MN-major)
      const uint64_t dKmn0 = smem_desc_sw128(sKV, bq::kHalfKV, 1024);
      bool ok = true;
      for (int i = 0; ok && i < nl; ++i) {
        const int st = i % bq::kStages, use = i / bq::kStages, sb = i & 1;
        // K(i) is in stage st (its phase cannot move on before this MMA releases the stage)
        if (!(ok = mbar_wait(smem_u32(&bar_full[st]), use & 1, abort_flag, a.err))) break;
        // dZ(i) is in the S columns of buffer sb (phase i cannot be overtaken: step i + 2
        // needs bar_o[sb] from this MMA)
        if (!(ok = mbar_wait(smem_u32(&bar_p[sb]), (i >> 1) & 1, abort_flag, a.err))) break;
        tc_fence_after();
        const uint32_t so = st * bq::kStage;
        const uint32_t zb = tmem + sb * 64;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_ts(tmem + 256, zb + k * 16, desc_advance(dKmn0, so + k * 2048), idQ, (i > 0 || k > 0) ? 1u : 0u);
        mma_commit(smem_u32(&bar_o[sb]));
        mma_commit(smem_u32(&bar_empty[st]));
      }
      mma_commit(smem_u32(&bar_fin));
    }
  } else if (warp >= 4 && warp < 4 + bq::kSoftWarps) {
    // ------------------------------------------------------------ softmax gradient
    // Thread (cg, row): row `row` of the tile, kv columns [16 cg, 16 cg + 16).
    const int cg = (warp - 4) >> 2;
    const int quarter = warp & 3;  // the TMEM lane quarter this warp may access
    const int row = 32 * quarter + lane;
    const uint32_t lane_addr = uint32_t(32 * quarter) << 16;
    const int hh = row >> 6, qpos = row & 63;
    const bool valid = hh < nv;  // uniform over the warp
    const int hq = h * a.G + 2 * hp + hh;
    const size_t grow = (size_t(b) * a.Hq + (valid ? hq : h * a.G)) * a.N + size_t(t) * kBlock + qpos;
    {  // this thread's quarter of its row of Q and dO (d [32 cg, 32 cg + 32)) into TMEM; zero for a missing head
      uint32_t qw[16], ow[16];
      const bool in_d = valid && cg * 32 < a.d;  // at d = 64 the upper half of the row is zero
      const uint4* qg = reinterpret_cast<const uint4*>(q + grow * a.d + (in_d ? cg * 32 : 0));
      const uint4* og = reinterpret_cast<const uint4*>(dO + grow * a.d + (in_d ? cg * 32 : 0));
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint4 x = in_d ? qg[c] : make_uint4(0, 0, 0, 0);
        const uint4 y = in_d ? og[c] : make_uint4(0, 0, 0, 0);
        qw[4 * c] = x.x, qw[4 * c + 1] = x.y, qw[4 * c + 2] = x.z, qw[4 * c + 3] = x.w;
        ow[4 * c] = y.x, ow[4 * c + 1] = y.y, ow[4 * c + 2] = y.z, ow[4 * c + 3] = y.w;
      }
      tmem_st16(tmem + lane_addr + kColQ + cg * 16, qw);
      tmem_st16(tmem + lane_addr + kColDO + cg * 16, ow);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bar_qo));
    }
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
      const uint32_t tS = tmem + lane_addr + sb * 64 + cg * 16, tP = tmem + lane_addr + 128 + sb * 64 + cg * 16;
      const float off2 = kOut ? L2 : L2 - lam_s[i];
      const float gw = kOut ? fast_exp2(lam_s[i]) : 1.f;  // the gate outside the softmax (1 on the diagonal)
      uint32_t vs[16], vp[16], dz[8];
      tmem_ld16(tS, vs);
      tmem_ld16(tP, vp);
      tmem_wait_ld();
      float zr[16];
      if (valid && i > 0) {  // every column counts
#pragma unroll
        for (int x = 0; x < 16; ++x)
          zr[x] = fast_exp2(fmaf(__uint_as_float(vs[x]), sc2, -off2)) *
                  (kOut ? fmaf(gw, __uint_as_float(vp[x]), -Dr) : __uint_as_float(vp[x]) - Dr);
      } else {
        // none for a missing head, the causal prefix on the diagonal block
        const int n_ok = valid ? min(16, max(0, qpos + 1 - cg * 16)) : 0;
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          const float z = fast_exp2(fmaf(__uint_as_float(vs[x]), sc2, -off2)) *
                          (kOut ? fmaf(gw, __uint_as_float(vp[x]), -Dr) : __uint_as_float(vp[x]) - Dr);
          zr[x] = x < n_ok ? z : 0.f;
        }
      }
#pragma unroll
      for (int x = 0; x < 8; ++x) dz[x] = pack_bf16x2(zr[2 * x], zr[2 * x + 1]);
      tmem_st8(tS, dz);  // packed dZ over this group's own, already read S columns
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&bar_p[sb]));
    }
    if (ok) ok = mbar_wait(smem_u32(&bar_fin), 0, abort_flag, a.err);
    ok = __all_sync(0xffffffffu, ok);
    if (ok && valid && cg * 32 < a.d) {  // rows 64..127 of a one-head tile form whole warps
      tc_fence_after();
      uint32_t v[32];
      tmem_ld32(tmem + lane_addr + 256 + cg * 32, v);  // d columns [32 cg, 32 cg + 32)
      tmem_wait_ld();
      uint4* og = reinterpret_cast<uint4*>(a.dq + grow * a.d + cg * 32);
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        uint4 o4;
        o4.x = pack_bf16x2(__uint_as_float(v[8 * q4 + 0]) * a.scale, __uint_as_float(v[8 * q4 + 1]) * a.scale);
        o4.y = pack_bf16x2(__uint_as_float(v[8 * q4 + 2]) * a.scale, __uint_as_float(v[8 * q4 + 3]) * a.scale);
        o4.z = pack_bf16x2(__uint_as_float(v[8 * q4 + 4]) * a.scale, __uint_as_float(v[8 * q4 + 5]) * a.scale);
        o4.w = pack_bf16x2(__uint_as_float(v[8 * q4 + 6]) * a.scale, __uint_as_float(v[8 * q4 + 7]) * a.scale);
        og[q4] = o4;
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
// Pass 2 with stored dZ: dQ = scale · Σ_j dZ_tj K_j, query-major
// ===========================================================================
namespace bdq {
constexpr int kThreads = 192;          // 0 TMA, 1 TMEM + MMA issue, 2-5 epilogue
constexpr int kTileZ = 128 * 64 * 2;   // one stored dZ tile: 128 rows (a head pair) x 64 kv bf16
constexpr int kHalfK = 64 * 128;       // one d-half of a 64-row K block
constexpr int kStage = 2 * kHalfK + 2 * kTileZ;  // K block + up to two dZ tiles: 48 KB
constexpr int kStages = 2;             // two CTAs per SM: one's start and end hide under the other's loop
constexpr int kSmem = kStages * kStage + 1024;
}  // namespace bdq

// One CTA per (batch, KV head, query block, up to two head pairs). The list of
// the block's dZ slots is [diagonal, idx[t][0], idx[t][1], ...]. For each,
// the producer brings the K block and the stored dZ tiles of the CTA's head
// pairs into a stage, and one thread issues dQ_r += dZ_r · K as four M = 128,
// N = 128, K = 16 MMAs per tile (dZ K-major, K MN-major), accumulating in TMEM.
// No exponential and no recomputed product: the KV pass derived dZ already.
__global__ void __launch_bounds__(bdq::kThreads, 2)
    bwd_dq_sm100_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmDZ,
                        BwdSm100Args a) {
  using namespace sm100;
  extern __shared__ uint8_t smem_raw[];
  __shared__ int list_s[kMaxTopK + 1];  // (m << kSlotBits) | dZ slot
  __shared__ int nlist_s;
  __shared__ __align__(8) uint64_t bar_full[bdq::kStages], bar_empty[bdq::kStages], bar_fin;
  __shared__ uint32_t tmem_s;
  __shared__ int abort_s;

  const uint32_t sbase = (smem_u32(smem_raw) + 1023u) & ~1023u;
  const int t = a.NB - 1 - int(blockIdx.x);
  const int n_pp = (a.n_hp + 1) / 2;  // CTAs per KV head
  const int h = int(blockIdx.y) / n_pp, pp = int(blockIdx.y) % n_pp;
  const int b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hp0 = 2 * pp;
  const int n_tiles = min(2, a.n_hp - hp0);
  const size_t bh = size_t(b) * a.Hkv + h;
  const long long slot0 = static_cast<long long>(bh) * a.dz_slots + dz_slot_base(t, a.K);
  volatile int* abort_flag = &abort_s;

  if (threadIdx.x == 0) abort_s = 0;
  if (warp == 0) {
    // list: the diagonal (slot 0), then every valid idx entry s (slot s + 1); an entry
    // outside the history is skipped and raised, the first -1 ends the list
    const int n = min(a.K, t);
    const int32_t* row = a.idx + (bh * a.NB + t) * size_t(a.K);
    int cnt = 0;
    bool stop = false;
    for (int base = 0; base < n && !stop; base += 32) {
      const int k = base + lane;
      const int m = k < n ? row[k] : -1;
      const bool end = k < n && m < 0, bad = k < n && m >= t;
      if (bad) raise_error(a.err, SAS_ERR_DEVICE_INDEX);
      const unsigned end_mask = __ballot_sync(0xffffffffu, end);
      const int first_end = end_mask ? __ffs(end_mask) - 1 : 32;
      const bool ok = k < n && !bad && m >= 0 && lane < first_end;
      const unsigned ok_mask = __ballot_sync(0xffffffffu, ok);
      if (ok) list_s[1 + cnt + __popc(ok_mask & ((1u << lane) - 1u))] = (m << kSlotBits) | (k + 1);
      cnt += __popc(ok_mask);
      stop = end_mask != 0;
    }
    if (lane == 0) {
      list_s[0] = t << kSlotBits;
      nlist_s = 1 + cnt;
    }
  } else if (warp == 1) {
    tmem_alloc(smem_u32(&tmem_s), 256);
    if (lane == 0) {
      for (int s = 0; s < bdq::kStages; ++s) {
        mbar_init(smem_u32(&bar_full[s]), 1);
        mbar_init(smem_u32(&bar_empty[s]), 1);
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

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmDZ);
      int issued = 0;
      for (int i = 0; i < nl; ++i) {
        const int st = i % bdq::kStages, use = i / bdq::kStages;
        if (!mbar_wait(smem_u32(&bar_empty[st]), (use & 1) ^ 1, abort_flag, a.err)) break;
        const uint32_t sk = sbase + st * bdq::kStage, sz = sk + 2 * bdq::kHalfK;
        const int w = list_s[i];
        const int krow = int(bh * a.N + size_t(w >> kSlotBits) * kBlock);
        const long long tile = (slot0 + (w & ((1 << kSlotBits) - 1))) * a.n_hp + hp0;
        mbar_arrive_expect_tx(smem_u32(&bar_full[st]), uint32_t(2 * bdq::kHalfK + n_tiles * bdq::kTileZ));
        for (int c = 0; c < 2; ++c) tma_load_2d(sk + c * bdq::kHalfK, &tmK, c * 64, krow, smem_u32(&bar_full[st]));
        for (int r = 0; r < n_tiles; ++r)
          tma_load_3d(sz + r * bdq::kTileZ, &tmDZ, 0, 0, int(tile + r), smem_u32(&bar_full[st]));
        ++issued;
      }
      if (*abort_flag) {  // let the copies in flight land before the CTA exits
        for (int i = max(0, issued - bdq::kStages); i < issued; ++i) {
          const long long t0 = clock64();
          while (!mbar_try_wait(smem_u32(&bar_full[i % bdq::kStages]), (i / bdq::kStages) & 1) &&
                 clock64() - t0 < kWaitCycles) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idQ = idesc_bf16_f32(128, 128, 0, 1);  // q rows x d, K = kv tokens; K block MN-major
      const uint64_t dZ0 = smem_desc_sw128(sbase + 2 * bdq::kHalfK, 16, 1024);
      const uint64_t dK0 = smem_desc_sw128(sbase, bdq::kHalfK, 1024);
      bool ok = true;
      for (int i = 0; ok && i < nl; ++i) {
        const int st = i % bdq::kStages, use = i / bdq::kStages;
        if (!(ok = mbar_wait(smem_u32(&bar_full[st]), use & 1, abort_flag, a.err))) break;
        tc_fence_after();
        const uint32_t so = st * bdq::kStage;
        // K steps outer, tiles inner: consecutive MMAs feed different accumulators
#pragma unroll
        for (int k = 0; k < 4; ++k)
          for (int r = 0; r < n_tiles; ++r)
            mma_ss(tmem + r * 128, desc_advance(dZ0, so + r * bdq::kTileZ + k * 32), desc_advance(dK0, so + k * 2048),
                   idQ, (i > 0 || k > 0) ? 1u : 0u);
        mma_commit(smem_u32(&bar_empty[st]));
      }
      mma_commit(smem_u32(&bar_fin));
    }
  } else {
    // ------------------------------------------------------------ epilogue: dQ rows out of TMEM, bf16
    const int quarter = warp & 3;  // warps 2-5: TMEM lane quarters 2, 3, 0, 1
    const int row = 32 * quarter + lane;
    const uint32_t lane_addr = uint32_t(32 * quarter) << 16;
    bool ok = mbar_wait(smem_u32(&bar_fin), 0, abort_flag, a.err);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
      for (int r = 0; r < n_tiles; ++r) {
        const int g = 2 * (hp0 + r) + (row >> 6);
        const bool valid = g < a.G;  // uniform over the warp: 32 rows of one head
        const size_t grow = (size_t(b) * a.Hq + size_t(h) * a.G + (valid ? g : 0)) * a.N + size_t(t) * kBlock + (row & 63);
        for (int ch = 0; ch < a.d / 32; ++ch) {
          uint32_t v[32];
          tmem_ld32(tmem + lane_addr + r * 128 + ch * 32, v);
          tmem_wait_ld();
          if (valid) {
            uint4* og = reinterpret_cast<uint4*>(a.dq + grow * a.d + ch * 32);
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
              uint4 o4;
              o4.x = pack_bf16x2(__uint_as_float(v[8 * q4 + 0]) * a.scale, __uint_as_float(v[8 * q4 + 1]) * a.scale);
              o4.y = pack_bf16x2(__uint_as_float(v[8 * q4 + 2]) * a.scale, __uint_as_float(v[8 * q4 + 3]) * a.scale);
              o4.z = pack_bf16x2(__uint_as_float(v[8 * q4 + 4]) * a.scale, __uint_as_float(v[8 * q4 + 5]) * a.scale);
              o4.w = pack_bf16x2(__uint_as_float(v[8 * q4 + 6]) * a.scale, __uint_as_float(v[8 * q4 + 7]) * a.scale);
              og[q4] = o4;
            }
          }
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
    tmem_dealloc(tmem, 256);
  }
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
long long bwd_dz_tiles(const Shape& sh) {
  return static_cast<long long>(sh.B) * sh.Hkv * dz_slot_base(sh.NB, sh.K) * ((sh.G + 1) / 2);
}

cudaError_t launch_bwd_passes_sm100(const Shape& sh, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                   const uint16_t* dO, const float* s, const int32_t* idx, const float* lse_s,
                                   const float* lse_o, const float* drow, const int* rev_off, const int* rev_list,
                                   const float* rev_lam, float* dl, uint16_t* dz, uint16_t* dq, uint16_t* dk,
                                   uint16_t* dv, int* err, cudaStream_t st) {
  CUtensorMap tk, tv, tq3, tdo3, tl, td, tdz;
  const uint64_t hq = uint64_t(sh.B) * sh.Hq, rkv = uint64_t(sh.B) * sh.Hkv * sh.N;
  // rows of d = 64 or 128 values: the kernels always load two 64-column boxes; at d = 64 the second
  // lies past the extent and TMA fills it with zeros, which add nothing to any product
  if (!make_tmap_bf16_2d(&tk, k, rkv, sh.d) || !make_tmap_bf16_2d(&tv, v, rkv, sh.d) ||
      !make_tmap_bf16_3d_heads(&tq3, q, hq, sh.N, sh.d) || !make_tmap_bf16_3d_heads(&tdo3, dO, hq, sh.N, sh.d) ||
      !make_tmap_f32_rows(&tl, lse_o, hq, sh.N) || !make_tmap_f32_rows(&td, drow, hq, sh.N))
    return cudaErrorInvalidValue;
  // without a spill region the map is never used; it is encoded over the K cache so that it is valid
  if (!make_tmap_bf16_tiles(&tdz, dz != nullptr ? static_cast<const void*>(dz) : static_cast<const void*>(k),
                            dz != nullptr ? uint64_t(bwd_dz_tiles(sh)) : 1))
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
  a.gate = sh.gate;
  a.gated = sh.gated;
  a.n_hp = (sh.G + 1) / 2;
  a.n_tp = (sh.G + 3) / 4;
  a.d = sh.d;
  a.scale = sh.scale;
  a.spill = dz != nullptr ? 1 : 0;
  a.dz_slots = dz_slot_base(sh.NB, sh.K);
  cudaError_t e;
  auto kv = sh.outside ? bwd_kv_sm100_kernel<true> : bwd_kv_sm100_kernel<false>;
  auto qk = sh.outside ? bwd_q_sm100_kernel<true> : bwd_q_sm100_kernel<false>;
  if ((e = cudaFuncSetAttribute(kv, cudaFuncAttributeMaxDynamicSharedMemorySize, bkv::kSmem)) != cudaSuccess)
    return e;
  kv<<<dim3(sh.NB, sh.Hkv, sh.B), bkv::kThreads, bkv::kSmem, st>>>(tq3, tk, tv, tdo3, tl, td, tdz, a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (a.spill) {  // dQ from the stored dZ tiles
    if ((e = cudaFuncSetAttribute(bwd_dq_sm100_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bdq::kSmem)) !=
        cudaSuccess)
      return e;
    const int n_pp = (a.n_hp + 1) / 2;
    bwd_dq_sm100_kernel<<<dim3(sh.NB, sh.Hkv * n_pp, sh.B), bdq::kThreads, bdq::kSmem, st>>>(tk, tdz, a);
    return cudaGetLastError();
  }
  // dQ recomputing S and dP (the small-workspace form)
  if ((e = cudaFuncSetAttribute(qk, cudaFuncAttributeMaxDynamicSharedMemorySize, bq::kSmem)) != cudaSuccess)
    return e;
  qk<<<dim3(sh.NB, sh.Hkv * a.n_hp, sh.B), bq::kThreads, bq::kSmem, st>>>(tk, tv, q, dO, a);
  return cudaGetLastError();
}

}  // namespace sas
