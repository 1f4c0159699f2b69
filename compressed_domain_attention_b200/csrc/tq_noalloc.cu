// tq_decode_attention_noalloc: decode attention for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc at the point where they decode: code
// running inside a custom allocator or memory pool that must not re-enter
// itself, runtimes that forbid device allocation after start-up (fixed memory
// budgets, pre-planned arenas), and plug-ins handed only the tensors they work
// on. The regular entry point needs a caller-provided split-K workspace; this
// one uses a fixed-size array that lives in the library's own device image
// instead, so the caller passes only inputs and outputs.
//
// The array is a file-scope static device array: every GPU that loads this
// library holds TQ_NOALLOC_WORKSPACE_BYTES of device memory for it until the
// process exits. Host code cannot use the array's name as a device address
// (in host code it names a host-side stand-in), so the first call on each
// device (and in each new context of it) looks up the real address with
// cudaGetSymbolAddress while that device is current, and caches it.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/tq.h"
#include "tq_kernels.h"

namespace {

// The shared scratch. No part of it needs to start at zero: the split-K kernel
// writes every header entry and partial slot that the merge kernel reads in the
// same call, so a call never depends on what an earlier call left behind.
static __device__ __align__(256) unsigned char g_noalloc_ws[TQ_NOALLOC_WORKSPACE_BYTES];

constexpr int kMaxDevices = 64;

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current context (0 if it cannot be read). A
// device's context can be destroyed and made again (cudaDeviceReset, or a caller
// that switches contexts); the array then has a new device address, so the
// cached address is keyed on this id as well as on the device ordinal.
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
  });
  if (get_current == nullptr || get_id == nullptr) return 0;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of g_noalloc_ws for the current device and context, looked up
// (cudaGetSymbolAddress, with that device current) on the first call in each
// context and cached. The runtime makes the device's context current if it is
// not yet, so the id is read after the lookup.
void* ws_address_for_current_device(int* err) {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {nullptr};
  static unsigned long long ctx_of[kMaxDevices] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    *err = (int)e;
    return nullptr;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    *err = (int)cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(mu);
  const unsigned long long ctx = current_context_id();
  if (addr[dev] == nullptr || ctx == 0 || ctx != ctx_of[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_ws);  // with `dev` current
    if (e != cudaSuccess || p == nullptr) {
      *err = (int)(e != cudaSuccess ? e : cudaErrorUnknown);
      return nullptr;
    }
    addr[dev] = p;
    ctx_of[dev] = current_context_id();
  }
  return addr[dev];
}

}  // namespace

extern "C" int tq_decode_attention_noalloc(const tq_layout_t* layout, const void* q, int q_dtype,
                                           const int32_t* d_seq_lens, const uint8_t* k_codes,
                                           const uint16_t* k_scales, const uint8_t* v_codes,
                                           const uint16_t* v_scales, float sm_scale, float* out,
                                           int32_t* d_status, void* stream) {
  if (layout == nullptr) return TQ_ERR_INVALID_ARG;
  if (layout->k_format == TQ_KV_DELEGATED) return TQ_ERR_INVALID_ARG;  // no hot-tail argument here
  if (layout->page_tokens > 0) return TQ_ERR_INVALID_ARG;              // no block-table argument here
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return TQ_ERR_CUDA;
  int sms = 0;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return TQ_ERR_CUDA;
  if (sms > layout->max_ctas) sms = layout->max_ctas;
  // Reject requests whose workspace would not fit, before touching the device (the
  // same workspace arithmetic the decode call checks its workspace size against).
  if (tqk::decode_workspace_bytes(layout->batch, layout->n_q_heads, layout->head_dim, sms, 0) >
      (uint64_t)TQ_NOALLOC_WORKSPACE_BYTES)
    return TQ_ERR_CAPACITY;
  int err = 0;
  void* ws = ws_address_for_current_device(&err);
  if (ws == nullptr) return TQ_ERR_CUDA;
  tq_decode_opts_t opts = {};
  opts.min_split_tokens = 0;
  opts.max_ctas = sms;
  opts.after_split_event = nullptr;
  return tq_decode_attention_ex(layout, q, q_dtype, d_seq_lens, k_codes, k_scales, v_codes, v_scales, sm_scale, out,
                                ws, (size_t)TQ_NOALLOC_WORKSPACE_BYTES, d_status, &opts, stream);
}
