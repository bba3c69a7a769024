// Training steps end to end from host memory, with the copies of neighbouring
// steps overlapping each step's kernels.
//
// Step i uses device slot i % 2. Its inputs go up on one copy stream, its
// kernels (select + LSE, forward, backward with ds) run on the caller's
// stream, and its outputs come down on a second copy stream. Three kinds of
// event order the work:
//   in[k]    the inputs of the step in slot k have landed;
//   done[k]  the kernels of that step have finished (its inputs may be overwritten);
//   out[k]   its outputs have left the slot (the next step in slot k may write them).
// So the upload of step i + 1 and the download of step i − 1 run while step i
// computes, and the PCIe link is busy in both directions at once. The copy
// streams and events live for one call; the caller's stream waits for the last
// download, so synchronising it covers the whole call.
#include "common.cuh"

namespace sas {
sas_status check_params(const sas_params* p, Shape* sh);
}  // namespace sas

namespace {

bool ok16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Streams and events of one call, released when the call returns (CUDA frees
// them once their pending work completes).
struct CallResources {
  cudaStream_t up = nullptr, down = nullptr;
  cudaEvent_t entry = nullptr, in[2] = {nullptr, nullptr}, done[2] = {nullptr, nullptr}, out[2] = {nullptr, nullptr};
  cudaError_t create() {
    cudaError_t e;
    if ((e = cudaStreamCreateWithFlags(&up, cudaStreamNonBlocking)) != cudaSuccess) return e;
    if ((e = cudaStreamCreateWithFlags(&down, cudaStreamNonBlocking)) != cudaSuccess) return e;
    for (cudaEvent_t* ev : {&entry, &in[0], &in[1], &done[0], &done[1], &out[0], &out[1]})
      if ((e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming)) != cudaSuccess) return e;
    return cudaSuccess;
  }
  ~CallResources() {
    for (cudaEvent_t ev : {entry, in[0], in[1], done[0], done[1], out[0], out[1]})
      if (ev != nullptr) cudaEventDestroy(ev);
    if (up != nullptr) cudaStreamDestroy(up);
    if (down != nullptr) cudaStreamDestroy(down);
  }
};

}  // namespace

extern "C" sas_status sas_train_steps_host(const sas_params* p, int n_steps, const sas_host_step* steps,
                                           const sas_device_slot* slots, void* stream) {
  sas::Shape sh;
  sas_status r = sas::check_params(p, &sh);
  if (r != SAS_OK) return r;
  if (n_steps < 1 || steps == nullptr || slots == nullptr) return SAS_ERR_INVALID_ARG;
  size_t ws_need = 0;
  if ((r = sas_bwd_workspace_size_min(p, &ws_need)) != SAS_OK) return r;
  for (int k = 0; k < 2 && k < n_steps; ++k) {
    const sas_device_slot& d = slots[k];
    if (!ok16(d.q) || !ok16(d.k) || !ok16(d.v) || !ok16(d.s) || !ok16(d.dO) || !ok16(d.idx) || !ok16(d.lse_s) ||
        !ok16(d.o) || !ok16(d.lse_o) || !ok16(d.dq) || !ok16(d.dk) || !ok16(d.dv) || (sh.gated && !ok16(d.ds)))
      return SAS_ERR_INVALID_ARG;
    if (d.ws == nullptr || d.ws_bytes < ws_need || (reinterpret_cast<uintptr_t>(d.ws) & 255u) != 0)
      return SAS_ERR_WORKSPACE;
  }
  for (int i = 0; i < n_steps; ++i) {
    const sas_host_step& h = steps[i];
    if (h.q == nullptr || h.k == nullptr || h.v == nullptr || h.s == nullptr || h.dO == nullptr || h.o == nullptr ||
        h.dq == nullptr || h.dk == nullptr || h.dv == nullptr)
      return SAS_ERR_INVALID_ARG;
    if (h.ds != nullptr && !sh.gated) return SAS_ERR_INVALID_ARG;  // no ds without a gate
  }
  const size_t rows_q = size_t(sh.B) * sh.Hq * sh.N, rows_kv = size_t(sh.B) * sh.Hkv * sh.N;
  const size_t b_q = rows_q * sh.d * 2, b_kv = rows_kv * sh.d * 2, b_lse = rows_q * 4;
  const size_t b_s = size_t(sh.B) * sh.Hkv * sh.NB * sh.NB * 4;

  CallResources cr;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (cr.create() != cudaSuccess) return SAS_ERR_CUDA;
  cudaError_t e = cudaEventRecord(cr.entry, cs);  // nothing of this call starts before the caller's prior work
  if (e == cudaSuccess) e = cudaStreamWaitEvent(cr.up, cr.entry, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(cr.down, cr.entry, 0);
  if (e != cudaSuccess) return SAS_ERR_CUDA;
  const cudaMemcpyKind H2D = cudaMemcpyHostToDevice, D2H = cudaMemcpyDeviceToHost;
  // Every return after this point first makes the caller's stream wait for whatever the copy
  // streams hold, so that no copy is still in flight once the caller's stream has completed.
  auto leave = [&](sas_status status) {
    cudaEvent_t j = nullptr;
    bool joined = cudaEventCreateWithFlags(&j, cudaEventDisableTiming) == cudaSuccess;
    for (cudaStream_t cp : {cr.up, cr.down})
      joined = joined && cudaEventRecord(j, cp) == cudaSuccess && cudaStreamWaitEvent(cs, j, 0) == cudaSuccess;
    if (j != nullptr) cudaEventDestroy(j);
    return joined ? status : (status == SAS_OK ? SAS_ERR_CUDA : status);
  };

  for (int i = 0; i < n_steps; ++i) {
    const int k = i & 1;
    const sas_device_slot& d = slots[k];
    const sas_host_step& h = steps[i];
    // inputs into slot k, once the kernels of step i − 2 have read them
    if (i >= 2 && (e = cudaStreamWaitEvent(cr.up, cr.done[k], 0)) != cudaSuccess) return leave(SAS_ERR_CUDA);
    if ((e = cudaMemcpyAsync(d.q, h.q, b_q, H2D, cr.up)) != cudaSuccess ||
        (e = cudaMemcpyAsync(d.k, h.k, b_kv, H2D, cr.up)) != cudaSuccess ||
        (e = cudaMemcpyAsync(d.v, h.v, b_kv, H2D, cr.up)) != cudaSuccess ||
        (e = cudaMemcpyAsync(d.s, h.s, b_s, H2D, cr.up)) != cudaSuccess ||
        (e = cudaMemcpyAsync(d.dO, h.dO, b_q, H2D, cr.up)) != cudaSuccess ||
        (e = cudaEventRecord(cr.in[k], cr.up)) != cudaSuccess)
      return leave(SAS_ERR_CUDA);
    // kernels, once the inputs have landed and the outputs of step i − 2 have left
    if ((e = cudaStreamWaitEvent(cs, cr.in[k], 0)) != cudaSuccess) return leave(SAS_ERR_CUDA);
    if (i >= 2 && (e = cudaStreamWaitEvent(cs, cr.out[k], 0)) != cudaSuccess) return leave(SAS_ERR_CUDA);
    if ((r = sas_topk_select(p, d.s, nullptr, d.idx, d.lse_s, stream)) != SAS_OK) return leave(r);
    if ((r = sas_fwd(p, d.q, d.k, d.v, d.s, d.idx, d.lse_s, d.o, d.lse_o, stream)) != SAS_OK) return leave(r);
    if ((r = sas_bwd(p, d.q, d.k, d.v, d.o, d.dO, d.s, d.idx, d.lse_s, d.lse_o, d.dq, d.dk, d.dv, d.ds, d.ws,
                     d.ws_bytes, stream)) != SAS_OK)
      return leave(r);
    if ((e = cudaEventRecord(cr.done[k], cs)) != cudaSuccess) return leave(SAS_ERR_CUDA);
    // outputs back to the host
    if ((e = cudaStreamWaitEvent(cr.down, cr.done[k], 0)) != cudaSuccess ||
        (e = cudaMemcpyAsync(h.o, d.o, b_q, D2H, cr.down)) != cudaSuccess ||
        (h.lse_o != nullptr && (e = cudaMemcpyAsync(h.lse_o, d.lse_o, b_lse, D2H, cr.down)) != cudaSuccess) ||
        (e = cudaMemcpyAsync(h.dq, d.dq, b_q, D2H, cr.down)) != cudaSuccess ||
        (e = cudaMemcpyAsync(h.dk, d.dk, b_kv, D2H, cr.down)) != cudaSuccess ||
        (e = cudaMemcpyAsync(h.dv, d.dv, b_kv, D2H, cr.down)) != cudaSuccess ||
        (h.ds != nullptr && (e = cudaMemcpyAsync(h.ds, d.ds, b_s, D2H, cr.down)) != cudaSuccess) ||
        (e = cudaEventRecord(cr.out[k], cr.down)) != cudaSuccess)
      return leave(SAS_ERR_CUDA);
  }
  // the caller's stream completes only after the last downloads
  return leave(SAS_OK);
}
