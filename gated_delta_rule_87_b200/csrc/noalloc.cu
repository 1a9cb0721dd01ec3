// KDA prefill for callers that may not allocate device memory.
//
// kda_chunk_fwd needs a caller-provided workspace.  Some callers cannot get
// one: a host program that hands out every byte of device memory from its
// own pool and does not let libraries allocate, or a code path where a
// cudaMalloc (which can synchronise the device) is not allowed.  This entry
// point runs the same prefill with its scratch in a fixed array that lives in
// this library's device memory, so the call itself allocates nothing.
//
// The array is kNoAllocScratchBytes (64 MiB) per device.  Every device that
// loads this library keeps that memory until the process exits.  All calls on
// a device share the array and it keeps whatever the last call left in it;
// the prefill clears its status word itself at the start of every call and
// overwrites everything else it reads.  Two calls whose kernels overlap on
// the GPU (different streams or host threads) corrupt each other's scratch:
// order them on one stream.
#include <stdio.h>

#include <mutex>

#include "gated_delta.h"
#include "internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {};

// The array's symbol is a host-side stand-in, not a device address: look up
// the real address once per device, with that device current.
kda_status_t scratch_for_current_device(void **addr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return KDA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return KDA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *addr = g_scratch_addr[dev];
  return KDA_OK;
}

}  // namespace

extern "C" {

kda_status_t kda_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const float *g,
                                   const float *beta, void *o, const float *initial_state,
                                   float *final_state, const int32_t *cu_seqlens,
                                   int32_t num_seqs, int32_t B, int32_t T, int32_t H,
                                   int32_t d_k, int32_t d_v, kda_dtype_t io_dtype, void *stream) {
  const size_t need = kda_chunk_fwd_workspace_size(B, T, H, d_k, d_v,
                                                   cu_seqlens ? num_seqs : 0, io_dtype);
  if (need > kNoAllocScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "kda_chunk_fwd_noalloc: this problem needs %zu bytes of scratch but the built-in "
             "scratch holds %zu; use kda_chunk_fwd with a workspace",
             need, kNoAllocScratchBytes);
    gdr::set_last_error(msg);
    return KDA_ERR_WORKSPACE;
  }
  void *scratch = nullptr;
  const kda_status_t st = scratch_for_current_device(&scratch);
  if (st != KDA_OK) {
    gdr::set_last_error("kda_chunk_fwd_noalloc: could not look up the scratch address");
    return st;
  }
  return kda_chunk_fwd(q, k, v, g, beta, o, initial_state, final_state, cu_seqlens, num_seqs, B,
                       T, H, d_k, d_v, io_dtype, scratch, kNoAllocScratchBytes, stream);
}

}  // extern "C"
