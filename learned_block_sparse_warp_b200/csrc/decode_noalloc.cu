// Decode step that allocates nothing: sas_decode_noalloc.
//
// Some callers cannot call cudaMalloc. cudaMalloc synchronises the device, so
// a serving loop with a fixed latency budget may not call it per step. A
// plugin that runs inside a host framework may not be allowed to either: the
// framework's caching allocator may already hold most of HBM, so a direct
// cudaMalloc can fail or fragment memory behind its back. Plain C callers may
// have no device allocator of their own at all. This entry point serves those
// callers. It runs the whole decode step (select, split, merge), and the
// buffers between the kernels live in one file-scope device array of fixed
// size instead of caller-allocated memory. The caller passes only the inputs
// and the outputs o and lse_o.
//
// The array below is SAS_NOALLOC_SCRATCH_BYTES (16 MiB) on every GPU that
// loads this library, and it stays resident until the process exits. Every
// call uses the same array. Two calls that overlap on the GPU (on different
// streams, or from different host threads) race on it and must be serialised
// by the caller. Nothing in it needs to start at zero: each call writes every
// byte it later reads (the index lists with their −1 padding, the gate
// normalisers and every split's partial), so the previous call's contents
// never leak into a result.
#include <mutex>

#include "common.cuh"

namespace sas {
cudaError_t launch_select(const Shape& sh, const float* s, const int32_t* cache_len, int32_t* idx, float* lse,
                          int* err, cudaStream_t st);
cudaError_t launch_decode(const Shape& sh, const uint16_t* q, const uint16_t* kc, const uint16_t* vc,
                          const int32_t* cl, const float* s, const int32_t* idx, const float* lse_s, int n_split,
                          float* o_part, float* lse_part, int* err, cudaStream_t st);
cudaError_t launch_decode_combine(const Shape& sh, int n_split, const float* o_part, const float* lse_part,
                                  uint16_t* o, float* lse_o, cudaStream_t st);
sas_status check_params(const sas_params* p, Shape* sh);
int* error_word();
}  // namespace sas

// The scratch. In host code this name is only a host-side stand-in for the
// symbol, not a device address, so its device address is fetched below.
static __device__ __align__(256) unsigned char g_decode_scratch[SAS_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned char* g_scratch_ptr[kMaxDevices];

size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

// Device address of the scratch on the current device. It is fetched once per
// device, on that device's first call, with the device current.
sas_status scratch_on_current_device(unsigned char** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SAS_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SAS_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    unsigned char* ptr = nullptr;
    if (cudaGetSymbolAddress((void**)&ptr, g_decode_scratch) != cudaSuccess || ptr == nullptr) return SAS_ERR_CUDA;
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return SAS_OK;
}

bool ok16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" sas_status sas_decode_noalloc(const sas_params* p, const sas_bf16* q, const sas_bf16* kc,
                                         const sas_bf16* vc, const int32_t* cache_len, const float* s, sas_bf16* o,
                                         float* lse_o, void* stream) {
  sas::Shape sh;
  sas_status r = sas::check_params(p, &sh);
  if (r != SAS_OK) return r;
  if (sh.G > 8) return SAS_ERR_UNSUPPORTED;
  if (!ok16(q) || !ok16(kc) || !ok16(vc) || !ok16(cache_len) || !ok16(s) || !ok16(o)) return SAS_ERR_INVALID_ARG;
  if (lse_o != nullptr && (reinterpret_cast<uintptr_t>(lse_o) & 15u) != 0) return SAS_ERR_INVALID_ARG;

  // carve the scratch: index lists, gate normalisers, split partials
  const int n_split = sh.K + 1;  // one selected block (or the current block) per split
  const size_t n_idx = size_t(sh.B) * sh.Hkv * sh.K;
  const size_t n_lse = size_t(sh.B) * sh.Hkv;
  const size_t n_opart = size_t(sh.B) * sh.Hq * n_split * sh.d;
  const size_t n_lpart = size_t(sh.B) * sh.Hq * n_split;
  const size_t off_lse = round256(n_idx * sizeof(int32_t));
  const size_t off_opart = off_lse + round256(n_lse * sizeof(float));
  const size_t off_lpart = off_opart + round256(n_opart * sizeof(float));
  const size_t need = off_lpart + round256(n_lpart * sizeof(float));
  if (need > size_t(SAS_NOALLOC_SCRATCH_BYTES)) return SAS_ERR_WORKSPACE;

  unsigned char* base = nullptr;
  if ((r = scratch_on_current_device(&base)) != SAS_OK) return r;
  int32_t* idx = reinterpret_cast<int32_t*>(base);
  float* lse_s = reinterpret_cast<float*>(base + off_lse);
  float* o_part = reinterpret_cast<float*>(base + off_opart);
  float* lse_part = reinterpret_cast<float*>(base + off_lpart);

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int* err = sas::error_word();
  if (sas::launch_select(sh, s, cache_len, idx, lse_s, err, st) != cudaSuccess) return SAS_ERR_CUDA;
  if (sas::launch_decode(sh, q, kc, vc, cache_len, sh.gated ? s : nullptr, idx, sh.gated ? lse_s : nullptr, n_split,
                         o_part, lse_part, err, st) != cudaSuccess)
    return SAS_ERR_CUDA;
  if (sas::launch_decode_combine(sh, n_split, o_part, lse_part, o, lse_o, st) != cudaSuccess) return SAS_ERR_CUDA;
  return SAS_OK;
}
