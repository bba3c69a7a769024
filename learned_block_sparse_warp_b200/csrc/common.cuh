// Shared device helpers for the SAS kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "sas.h"

namespace sas {

constexpr int kBlock = 64;          // tokens per block (b)
constexpr int kMaxTopK = 2048;      // largest K the kernels accept
constexpr int kSlotBits = 12;       // reverse-index entry: (t << kSlotBits) | slot, slot < K <= 4096
constexpr int kMaxDecodeBlocksPerSplit = 64;  // ceil((K + 1) / n_split) fits the decode task list
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Shapes as the kernels see them.
struct Shape {
  int B, Hq, Hkv, G, d, N, NB, K;
  float scale;  // softmax scale (1/sqrt(d) unless given)
  int gate;     // sas_gate_mode
  int gated;    // 1 when a gate applies (every mode but SAS_GATE_NONE)
  int outside;  // 1 when the gate weights the values after the softmax (SAS_GATE_SOFTMAX_OUTSIDE)
};

// λ_m of a selected history block in log2 units, log g_m · log2 e, for the gate
// mode: s_m − LSE(s) (softmax-normalised, inside or outside the softmax),
// log σ(s_m), s_m (raw logit), or 0.
__device__ __forceinline__ float gate_lam2(int gate, float s_m, float lse) {
  switch (gate) {
    case SAS_GATE_LOG_SOFTMAX:
    case SAS_GATE_SOFTMAX_OUTSIDE: return (s_m - lse) * kLog2e;
    case SAS_GATE_LOG_SIGMOID: return (fminf(s_m, 0.f) - log1pf(expf(-fabsf(s_m)))) * kLog2e;
    case SAS_GATE_LOGIT: return s_m * kLog2e;
    default: return 0.f;
  }
}

// First error wins. The word lives in device memory owned by the library
// (one per device) and is read back by sas_get_device_error.
__device__ __forceinline__ void raise_error(int* err, int code) {
  if (err != nullptr) atomicCAS(err, 0, code);
}

__device__ __forceinline__ float bf16_to_f32(uint16_t x) { return __uint_as_float(uint32_t(x) << 16); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ int warp_isum(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------------------
// Warp-level tensor-core helpers (mma.sync m16n8k16, ldmatrix, cp.async)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D += A·B, A 16x16 bf16 (row), B 16x8 bf16 (col), D 16x8 fp32.
__device__ __forceinline__ void mma_bf16_16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void cp_async16(uint32_t smem_addr, const void* gptr) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_addr), "l"(gptr));
}
// Copies `src_bytes` (0 or 16) bytes and zero-fills the rest of the 16-byte chunk.
__device__ __forceinline__ void cp_async16_zfill(uint32_t smem_addr, const void* gptr, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_addr), "l"(gptr), "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }

// Programmatic dependent launch. A kernel launched with programmatic stream
// serialization may start before its predecessor in the stream has finished;
// griddep_wait() blocks until that predecessor has completed and its writes
// are visible, so it must come before the first global access that could
// depend on earlier work. Without that launch attribute it returns at once.
// griddep_launch_dependents() lets the next such kernel begin its launch.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

// Byte offset of 16-byte chunk `c` of row `r` in a [rows][CH] tile of 16-byte
// chunks, XOR-swizzled so that eight consecutive rows at the same logical
// chunk fall into eight different bank groups (ldmatrix is then conflict-free).
template <int CH>
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return uint32_t((r * CH + (c ^ (r & 7))) * 16);
}

// Orderable key of a float score: larger score <=> larger key. -0 and +0
// share a key; NaN gets key 0, below every number.
__device__ __forceinline__ uint32_t score_key(float x) {
  uint32_t u = __float_as_uint(x);
  if ((u & 0x7fffffffu) > 0x7f800000u) return 0u;  // NaN
  if ((u & 0x7fffffffu) == 0u) u = 0u;             // -0 -> +0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Builds the ordered block list [t, I_t...] of one query block in shared
// memory with each block's log2-domain gate. Run by one warp.
__device__ __forceinline__ void build_block_list(const int32_t* __restrict__ idx_row, int K, int t,
                                                 const float* __restrict__ s_row, float lse_t, int gate,
                                                 int* list_s, float* lam_s, int* nlist_s, int* err) {
  const int lane = threadIdx.x & 31;
  const int n = min(K, t);
  int cnt = 0;
  bool stop = false;
  for (int base = 0; base < n && !stop; base += 32) {
    const int k = base + lane;
    const int m = (k < n) ? idx_row[k] : -1;
    const bool end = (k < n) && m < 0;
    const bool bad = (k < n) && m >= t;
    if (bad) raise_error(err, SAS_ERR_DEVICE_INDEX);
    const unsigned end_mask = __ballot_sync(0xffffffffu, end);
    const int first_end = end_mask ? __ffs(end_mask) - 1 : 32;
    const bool ok = (k < n) && !bad && m >= 0 && lane < first_end;
    const unsigned ok_mask = __ballot_sync(0xffffffffu, ok);
    if (ok) {
      const int pos = 1 + cnt + __popc(ok_mask & ((1u << lane) - 1u));
      list_s[pos] = m;
      lam_s[pos] = gate != SAS_GATE_NONE ? gate_lam2(gate, s_row[m], lse_t) : 0.f;
    }
    cnt += __popc(ok_mask);
    stop = end_mask != 0;
  }
  if (lane == 0) {
    list_s[0] = t;
    lam_s[0] = 0.f;
    *nlist_s = 1 + cnt;
  }
}

// Launches `kern` with programmatic stream serialization, so that its launch
// overlaps the tail of the preceding kernel. The kernel must call
// griddep_wait() before its first global access.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

}  // namespace sas
