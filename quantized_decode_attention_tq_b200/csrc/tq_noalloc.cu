// Decode attention for callers that cannot allocate device memory.
//
// Some callers are handed device pointers by a host application that owns all
// device memory (an engine plugin inside a server with its own memory pool, a
// component whose memory budget is fixed up front) and are not allowed to call
// cudaMalloc, or cannot afford the device synchronisation it may cause.  They
// cannot provide tq_decode_attention's workspace.  This entry point runs the
// same decode kernels with their scratch taken from a fixed-size array that is
// part of this library on every GPU that loads it.

#include <cuda_runtime.h>

#include <mutex>

#include "../../include/tq.h"
#include "tq_internal.h"

namespace {

// The scratch array.  Every GPU that loads the library holds it until exit.
// In host code `g_scratch` is only a host-side stand-in for the symbol, never
// a device address: the device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_scratch[TQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_ptr[kMaxDevices] = {};

// Device address of g_scratch on the current device (looked up once per
// device, with that device current).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return TQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_scratch) != cudaSuccess || !p) return TQ_ERR_CUDA;
    g_ptr[dev] = p;
  }
  *out = g_ptr[dev];
  return TQ_OK;
}

}  // namespace

extern "C" int tq_decode_attention_noalloc(const tq_kv_desc* desc, const tq_codebook* k_cb,
                                           const tq_codebook* v_cb, int q_heads, const void* q,
                                           int q_dtype, const uint8_t* k_codes,
                                           const uint16_t* k_norms, const uint8_t* v_codes,
                                           const uint16_t* v_norms, const int32_t* seq_lens,
                                           float scale, float sparse_thr, float* out,
                                           uint32_t* dev_status, void* stream) {
  // Every argument check runs before the first CUDA call.
  int st = tq::validate_decode(desc, k_cb, v_cb, q_heads, 1, q, q_dtype, k_codes, k_norms, v_codes,
                               v_norms, seq_lens, scale, sparse_thr, out, dev_status);
  if (st != TQ_OK) return st;
  const size_t need = tq_decode_workspace_size(desc, q_heads, sparse_thr);
  if (need == 0) return TQ_ERR_INVALID_ARG;
  if (need > (size_t)TQ_NOALLOC_SCRATCH_BYTES) return TQ_ERR_SCRATCH_LIMIT;
  void* scratch = nullptr;
  st = scratch_address(&scratch);
  if (st != TQ_OK) return st;
  // The merge counters at the start of the workspace must be zero; the array
  // keeps whatever the previous call left, so clear them on the caller's stream.
  const tq::DecodeWorkspace w = tq::decode_workspace_layout(
      desc->batch, desc->kv_heads, q_heads, desc->head_dim, desc->seq_cap, sparse_thr > 0.0f);
  const size_t counters = w.ml_off - w.tickets_off;
  if (cudaMemsetAsync(static_cast<char*>(scratch) + w.tickets_off, 0, counters,
                      static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return TQ_ERR_CUDA;
  return tq_decode_attention(desc, k_cb, v_cb, q_heads, q, q_dtype, k_codes, k_norms, v_codes,
                             v_norms, seq_lens, scale, sparse_thr, out, scratch,
                             (size_t)TQ_NOALLOC_SCRATCH_BYTES, dev_status, stream);
}
