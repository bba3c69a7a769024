// C ABI of the SAS gated block-sparse attention library: argument checks,
// shape derivation and kernel dispatch. The declarations and the contract of
// every entry point are in include/sas.h.
#include <math.h>
#include <mutex>

#include "common.cuh"

namespace sas {
cudaError_t launch_select(const Shape& sh, const float* s, const int32_t* cache_len, int32_t* idx, float* lse,
                          int* err, cudaStream_t st);
cudaError_t launch_fwd_sm100(const Shape& sh, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                             const float* s, const int32_t* idx, const float* lse_s, uint16_t* o, float* lse_o,
                             int* err, cudaStream_t st);
struct BwdWs;
size_t bwd_ws_layout(const Shape& sh, bool spill, void* base, BwdWs* ws);
bool bwd_can_spill(const Shape& sh);
cudaError_t launch_bwd_mma(const Shape& sh, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                           const uint16_t* o, const uint16_t* dO, const float* s, const int32_t* idx,
                           const float* lse_s, const float* lse_o, uint16_t* dq, uint16_t* dk, uint16_t* dv, float* ds,
                           void* ws, bool spill, int* err, cudaStream_t st);
cudaError_t launch_decode(const Shape& sh, const uint16_t* q, const uint16_t* kc, const uint16_t* vc,
                          const int32_t* cl, const float* s, const int32_t* idx, const float* lse_s, int n_split,
                          float* o_part, float* lse_part, int* err, cudaStream_t st);
cudaError_t launch_decode_paged(const Shape& sh, const uint16_t* q, const uint16_t* kp, const uint16_t* vp,
                                int n_pages, const int32_t* table, const int32_t* cl, const float* s,
                                const int32_t* idx, const float* lse_s, int n_split, float* o_part, float* lse_part,
                                int* err, cudaStream_t st);
cudaError_t launch_decode_combine(const Shape& sh, int n_split, const float* o_part, const float* lse_part,
                                  uint16_t* o, float* lse_o, cudaStream_t st);
bool decode_fused_fits(const Shape& sh);
cudaError_t launch_decode_fused(const Shape& sh, const uint16_t* q, const uint16_t* kc, const uint16_t* vc,
                                const int32_t* table, int n_pages, const int32_t* cl, const float* s, int32_t* idx,
                                float* lse_s, uint16_t* o, float* lse_o, int* err, cudaStream_t st);
cudaError_t launch_wait_timeout(int* err, cudaStream_t st);
}  // namespace sas

using sas::Shape;

// One error word per device. Kernels raise it with atomicCAS(0 -> code), and
// sas_get_device_error reads and clears it.
__device__ int g_sas_device_error;

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_err_mu;
int* g_err_ptr[kMaxDevices];

// Device address of the error word on the current device. Host code cannot
// use the symbol itself as an address, so the address is fetched once per
// device with cudaGetSymbolAddress.
int* device_error_word() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_err_mu);
  if (g_err_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_sas_device_error) != cudaSuccess) return nullptr;
    g_err_ptr[dev] = static_cast<int*>(p);
  }
  return g_err_ptr[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool ok_ptr(const void* p) { return p != nullptr && aligned16(p); }
bool ok_opt(const void* p) { return p == nullptr || aligned16(p); }

// Gate inputs: s for every gate mode but SAS_GATE_NONE, and lse_s for the
// softmax-normalised gate, inside or outside the softmax. The activation
// ablations do not read lse_s (it may be NULL).
bool gate_inputs_ok(const Shape& sh, const float* s, const float* lse_s) {
  if (!sh.gated) return true;
  if (!ok_ptr(s) || !ok_opt(lse_s)) return false;
  return (sh.gate != SAS_GATE_LOG_SOFTMAX && sh.gate != SAS_GATE_SOFTMAX_OUTSIDE) || lse_s != nullptr;
}

// Checks the shared parameters and fills the kernel-side shape.
sas_status make_shape(const sas_params* p, Shape* sh) {
  if (p == nullptr) return SAS_ERR_INVALID_ARG;
  if (p->batch < 1 || p->n_q_heads < 1 || p->n_kv_heads < 1 || p->seq_len < 1 || p->top_k < 1)
    return SAS_ERR_INVALID_ARG;
  if (p->n_q_heads % p->n_kv_heads != 0) return SAS_ERR_INVALID_ARG;
  if (p->gate_mode < SAS_GATE_LOG_SOFTMAX || p->gate_mode > SAS_GATE_SOFTMAX_OUTSIDE) return SAS_ERR_INVALID_ARG;
  if (!(p->softmax_scale >= 0.f) || isinf(p->softmax_scale)) return SAS_ERR_INVALID_ARG;
  if (p->top_k > sas::kMaxTopK) return SAS_ERR_INVALID_ARG;
  static_assert(sas::kMaxTopK <= (1 << sas::kSlotBits), "reverse-index slot field");
  if (p->block != sas::kBlock) return SAS_ERR_UNSUPPORTED;
  if (p->head_dim != 64 && p->head_dim != 128) return SAS_ERR_UNSUPPORTED;
  if (p->seq_len % sas::kBlock != 0) return SAS_ERR_INVALID_ARG;
  if (p->batch > 65535 || p->n_q_heads > 65535) return SAS_ERR_UNSUPPORTED;
  // keep every flattened row index of the scores within int range, and every
  // reverse-index entry (t << kSlotBits) | slot positive
  const long long nb = p->seq_len / sas::kBlock;
  if ((long long)p->batch * p->n_kv_heads * nb > (1LL << 30) || nb > (1LL << (31 - sas::kSlotBits)))
    return SAS_ERR_UNSUPPORTED;
  sh->B = p->batch;
  sh->Hq = p->n_q_heads;
  sh->Hkv = p->n_kv_heads;
  sh->G = p->n_q_heads / p->n_kv_heads;
  sh->d = p->head_dim;
  sh->N = p->seq_len;
  sh->NB = int(nb);
  sh->K = p->top_k;
  sh->scale = p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / sqrtf(float(p->head_dim));
  sh->gate = p->gate_mode;
  sh->gated = p->gate_mode != SAS_GATE_NONE ? 1 : 0;
  sh->outside = p->gate_mode == SAS_GATE_SOFTMAX_OUTSIDE ? 1 : 0;
  return SAS_OK;
}

sas_status from_cuda(cudaError_t e) { return e == cudaSuccess ? SAS_OK : SAS_ERR_CUDA; }

}  // namespace

namespace sas {
// Parameter checks and the device error word, shared with the other
// entry-point files of the library.
sas_status check_params(const sas_params* p, Shape* sh) { return make_shape(p, sh); }
int* error_word() { return device_error_word(); }
}  // namespace sas

extern "C" {

int sas_version(void) { return 100; }

const char* sas_status_string(sas_status status) {
  switch (status) {
    case SAS_OK: return "SAS_OK";
    case SAS_ERR_INVALID_ARG: return "SAS_ERR_INVALID_ARG: a pointer, size or layout rule is broken";
    case SAS_ERR_UNSUPPORTED: return "SAS_ERR_UNSUPPORTED: no kernel for these parameters";
    case SAS_ERR_WORKSPACE: return "SAS_ERR_WORKSPACE: workspace missing or too small";
    case SAS_ERR_CUDA: return "SAS_ERR_CUDA: a CUDA call or launch failed";
    case SAS_ERR_TIMEOUT: return "SAS_ERR_TIMEOUT: a device-side bounded wait expired";
    case SAS_ERR_DEVICE_INDEX: return "SAS_ERR_DEVICE_INDEX: a kernel met a block index outside the history";
  }
  return "unknown sas_status";
}

sas_status sas_topk_select(const sas_params* p, const float* s, const int32_t* cache_len, int32_t* idx,
                           float* lse_s, void* stream) {
  Shape sh;
  sas_status r = make_shape(p, &sh);
  if (r != SAS_OK) return r;
  if (!ok_ptr(s) || !ok_ptr(idx) || !ok_opt(lse_s) || !ok_opt(cache_len)) return SAS_ERR_INVALID_ARG;
  return from_cuda(sas::launch_select(sh, s, cache_len, idx, lse_s, device_error_word(),
                                      static_cast<cudaStream_t>(stream)));
}

sas_status sas_gate_lse(const sas_params* p, const float* s, const int32_t* cache_len, float* lse_s, void* stream) {
  Shape sh;
  sas_status r = make_shape(p, &sh);
  if (r != SAS_OK) return r;
  if (!ok_ptr(s) || !ok_ptr(lse_s) || !ok_opt(cache_len)) return SAS_ERR_INVALID_ARG;
  return from_cuda(sas::launch_select(sh, s, cache_len, nullptr, lse_s, device_error_word(),
                                      static_cast<cudaStream_t>(stream)));
}

sas_status sas_fwd(const sas_params* p, const sas_bf16* q, const sas_bf16* k, const sas_bf16* v, const float* s,
                   const int32_t* idx, const float* lse_s, sas_bf16* o, float* lse_o, void* stream) {
  Shape sh;
  sas_status r = make_shape(p, &sh);
  if (r != SAS_OK) return r;
  if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(idx) || !ok_ptr(o) || !ok_opt(lse_o))
    return SAS_ERR_INVALID_ARG;
  if (!gate_inputs_ok(sh, s, lse_s)) return SAS_ERR_INVALID_ARG;
  // tcgen05 kernel for d = 64 and 128 (at 64 the tensor maps zero-fill the second half of each row box)
  return from_cuda(sas::launch_fwd_sm100(sh, q, k, v, sh.gated ? s : nullptr, idx, sh.gated ? lse_s : nullptr, o,
                                         lse_o, device_error_word(), static_cast<cudaStream_t>(stream)));
}

sas_status sas_bwd_workspace_size(const sas_params* p, size_t* bytes) {
  Shape sh;
  sas_status r = make_shape(p, &sh);
  if (r != SAS_OK) return r;
  if (bytes == nullptr) return SAS_ERR_INVALID_ARG;
  *bytes = sas::bwd_ws_layout(sh, sas::bwd_can_spill(sh), nullptr, nullptr);
  return SAS_OK;
}

sas_status sas_bwd_workspace_size_min(const sas_params* p, size_t* bytes) {
  Shape sh;
  sas_status r = make_shape(p, &sh);
  if (r != SAS_OK) return r;
  if (bytes == nullptr) return SAS_ERR_INVALID_ARG;
  *bytes = sas::bwd_ws_layout(sh, false, nullptr, nullptr);
  return SAS_OK;
}

sas_status sas_bwd(const sas_params* p, const sas_bf16* q, const sas_bf16* k, const sas_bf16* v, const sas_bf16* o,
                   const sas_bf16* dO, const float* s, const int32_t* idx, const float* lse_s, const float* lse_o,
                   sas_bf16* dq, sas_bf16* dk, sas_bf16* dv, float* ds, void* ws, size_t ws_bytes, void* stream) {
  Shape sh;
  sas_status r = make_shape(p, &sh);
  if (r != SAS_OK) return r;
  if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(o) || !ok_ptr(dO) || !ok_ptr(idx) || !ok_ptr(lse_o) ||
      !ok_ptr(dq) || !ok_ptr(dk) || !ok_ptr(dv))
    return SAS_ERR_INVALID_ARG;
  if (!gate_inputs_ok(sh, s, lse_s) || (sh.gated && !ok_ptr(ds))) return SAS_ERR_INVALID_ARG;
  if (!ok_opt(ds)) return SAS_ERR_INVALID_ARG;
  // the full workspace holds the dZ tiles, which spares the dQ pass recomputing S and dP
  const bool spill = sas::bwd_can_spill(sh) && ws_bytes >= sas::bwd_ws_layout(sh, true, nullptr, nullptr);
  const size_t need = sas::bwd_ws_layout(sh, false, nullptr, nullptr);
  if (ws == nullptr || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return SAS_ERR_WORKSPACE;
  return from_cuda(sas::launch_bwd_mma(sh, q, k, v, o, dO, sh.gated ? s : nullptr, idx, sh.gated ? lse_s : nullptr,
                                       lse_o, dq, dk, dv, ds, ws, spill, device_error_word(),
                                       static_cast<cudaStream_t>(stream)));
}

sas_status sas_decode(const sas_params* p, const sas_bf16* q, const sas_bf16* kc, const sas_bf16* vc,
                      const int32_t* cache_len, const float* s, const int32_t* idx, const float* lse_s, int n_split,
                      float* o_part, float* lse_part, void* stream) {
  Shape sh;
  sas_status r = make_shape(p, &sh);
  if (r != SAS_OK) return r;
  if (sh.G > 8) return SAS_ERR_UNSUPPORTED;
  if (!ok_ptr(q) || !ok_ptr(kc) || !ok_ptr(vc) || !ok_ptr(cache_len) || !ok_ptr(idx) || !ok_ptr(o_part) ||
      !ok_ptr(lse_part))
    return SAS_ERR_INVALID_ARG;
  if (!gate_inputs_ok(sh, s, lse_s)) return SAS_ERR_INVALID_ARG;
  if (n_split < 1 || n_split > sh.K + 1 || n_split > 65535) return SAS_ERR_INVALID_ARG;
  if ((sh.K + n_split) / n_split > sas::kMaxDecodeBlocksPerSplit) return SAS_ERR_UNSUPPORTED;
  return from_cuda(sas::launch_decode(sh, q, kc, vc, cache_len, sh.gated ? s : nullptr, idx,
                                      sh.gated ? lse_s : nullptr, n_split, o_part, lse_part, device_error_word(),
                                      static_cast<cudaStream_t>(stream)));
}

sas_status sas_decode_paged(const sas_params* p, const sas_bf16* q, const sas_bf16* k_pages,
                            const sas_bf16* v_pages, int n_pages, const int32_t* block_table,
                            const int32_t* cache_len, const float* s, const int32_t* idx, const float* lse_s,
                            int n_split, float* o_part, float* lse_part, void* stream) {
  Shape sh;
  sas_status r = make_shape(p, &sh);
  if (r != SAS_OK) return r;
  if (sh.G > 8) return SAS_ERR_UNSUPPORTED;
  if (!ok_ptr(q) || !ok_ptr(k_pages) || !ok_ptr(v_pages) || !ok_ptr(block_table) || !ok_ptr(cache_len) ||
      !ok_ptr(idx) || !ok_ptr(o_part) || !ok_ptr(lse_part))
    return SAS_ERR_INVALID_ARG;
  if (n_pages < 1 || int64_t(n_pages) * sh.Hkv > (int64_t(1) << 31) / sas::kBlock) return SAS_ERR_INVALID_ARG;
  if (!gate_inputs_ok(sh, s, lse_s)) return SAS_ERR_INVALID_ARG;
  if (n_split < 1 || n_split > sh.K + 1 || n_split > 65535) return SAS_ERR_INVALID_ARG;
  if ((sh.K + n_split) / n_split > sas::kMaxDecodeBlocksPerSplit) return SAS_ERR_UNSUPPORTED;
  return from_cuda(sas::launch_decode_paged(sh, q, k_pages, v_pages, n_pages, block_table, cache_len,
                                            sh.gated ? s : nullptr, idx, sh.gated ? lse_s : nullptr, n_split, o_part,
                                            lse_part, device_error_word(), static_cast<cudaStream_t>(stream)));
}

sas_status sas_decode_combine(const sas_params* p, int n_split, const float* o_part, const float* lse_part,
                              sas_bf16* o, float* lse_o, void* stream) {
  Shape sh;
  sas_status r = make_shape(p, &sh);
  if (r != SAS_OK) return r;
  if (!ok_ptr(o_part) || !ok_ptr(lse_part) || !ok_ptr(o) || !ok_opt(lse_o)) return SAS_ERR_INVALID_ARG;
  if (n_split < 1 || n_split > sh.K + 1) return SAS_ERR_INVALID_ARG;
  return from_cuda(sas::launch_decode_combine(sh, n_split, o_part, lse_part, o, lse_o,
                                              static_cast<cudaStream_t>(stream)));
}

sas_status sas_decode_fused(const sas_params* p, const sas_bf16* q, const sas_bf16* kc, const sas_bf16* vc,
                            const int32_t* cache_len, const float* s, int32_t* idx, float* lse_s, sas_bf16* o,
                            float* lse_o, void* stream) {
  Shape sh;
  sas_status r = make_shape(p, &sh);
  if (r != SAS_OK) return r;
  if (!sas::decode_fused_fits(sh)) return SAS_ERR_UNSUPPORTED;
  if (!ok_ptr(q) || !ok_ptr(kc) || !ok_ptr(vc) || !ok_ptr(cache_len) || !ok_ptr(s) || !ok_ptr(o) || !ok_opt(idx) ||
      !ok_opt(lse_s) || !ok_opt(lse_o))
    return SAS_ERR_INVALID_ARG;
  return from_cuda(sas::launch_decode_fused(sh, q, kc, vc, nullptr, 0, cache_len, s, idx, lse_s, o, lse_o,
                                            device_error_word(), static_cast<cudaStream_t>(stream)));
}

sas_status sas_decode_fused_paged(const sas_params* p, const sas_bf16* q, const sas_bf16* k_pages,
                                  const sas_bf16* v_pages, int n_pages, const int32_t* block_table,
                                  const int32_t* cache_len, const float* s, int32_t* idx, float* lse_s, sas_bf16* o,
                                  float* lse_o, void* stream) {
  Shape sh;
  sas_status r = make_shape(p, &sh);
  if (r != SAS_OK) return r;
  if (!sas::decode_fused_fits(sh)) return SAS_ERR_UNSUPPORTED;
  if (!ok_ptr(q) || !ok_ptr(k_pages) || !ok_ptr(v_pages) || !ok_ptr(block_table) || !ok_ptr(cache_len) ||
      !ok_ptr(s) || !ok_ptr(o) || !ok_opt(idx) || !ok_opt(lse_s) || !ok_opt(lse_o))
    return SAS_ERR_INVALID_ARG;
  if (n_pages < 1 || int64_t(n_pages) * sh.Hkv > (int64_t(1) << 31) / sas::kBlock) return SAS_ERR_INVALID_ARG;
  return from_cuda(sas::launch_decode_fused(sh, q, k_pages, v_pages, block_table, n_pages, cache_len, s, idx, lse_s,
                                            o, lse_o, device_error_word(), static_cast<cudaStream_t>(stream)));
}

sas_status sas_selftest_wait_timeout(void* stream) {
  int* err = device_error_word();
  if (err == nullptr) return SAS_ERR_CUDA;
  return from_cuda(sas::launch_wait_timeout(err, static_cast<cudaStream_t>(stream)));
}

sas_status sas_get_device_error(void* stream, int* code) {
  if (code == nullptr) return SAS_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return SAS_ERR_CUDA;
  int* w = device_error_word();
  if (w == nullptr) return SAS_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, w, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return SAS_ERR_CUDA;
  if (v != 0 && cudaMemset(w, 0, sizeof(int)) != cudaSuccess) return SAS_ERR_CUDA;
  *code = v;
  return SAS_OK;
}

}  // extern "C"
