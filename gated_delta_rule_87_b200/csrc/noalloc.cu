// KDA prefill for callers that may not allocate device memory.
//
// kda_chunk_fwd needs a caller-provided workspace.  Some callers cannot get
// one: a host program that hands out every byte of device memory from its
// own pool and does not let libraries allocate, or a code path where a
// cudaMalloc (which can synchronise the device) is not allowed.  This entry
// point runs the same prefill with its scratch in a fixed array that lives in
// this library's device memory, so the call itself allocates nothing.
//
// The array is kNoAllocScratchBytes (64 MiB) per device.  It is part of this
// file's device module, which holds no kernels: under CUDA's default lazy
// module loading the module, and with it the 64 MiB, is loaded on a device
// when the first call on that device looks the array's address up (with
// CUDA_MODULE_LOADING=EAGER, when the library is loaded).  A host that lets a
// pool claim the device's memory should make one call first (a call with
// T = 0 computes nothing and only does the lookup); the memory then stays
// reserved until the process exits or the context is destroyed.  If the
// module cannot be loaded the call returns KDA_ERR_CUDA and kda_last_error()
// says so.
//
// All calls on a device share the array and it keeps whatever the last call
// left in it; the prefill clears its status word itself at the start of every
// call and overwrites everything else it reads.  Two calls whose kernels
// overlap on the GPU (different streams or host threads) corrupt each other's
// scratch: order them on one stream.
#include <cudaTypedefs.h>
#include <stdio.h>

#include <mutex>

#include "gated_delta.h"
#include "internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Identity of the calling thread's current context (driver API, looked up
// through the runtime; no allocation).  False when it cannot be told.
bool current_context_id(unsigned long long *id) {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  CUcontext ctx = nullptr;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

struct ScratchAddr {
  unsigned long long ctx_id;  // context the address belongs to
  void *addr;                 // nullptr: not looked up yet
};

std::mutex g_mu;
ScratchAddr g_scratch[kMaxDevices] = {};

// The array's symbol is a host-side stand-in, not a device address: look the
// real address up with the device current, once per device and context (a
// device reset creates a new context, whose copy of the array lives
// elsewhere, so a changed context triggers a new lookup).
kda_status_t scratch_for_current_device(void **addr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    gdr::set_last_error("kda_chunk_fwd_noalloc: no usable current device");
    return KDA_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  unsigned long long id = 0;
  if (g_scratch[dev].addr && current_context_id(&id) && id == g_scratch[dev].ctx_id) {
    *addr = g_scratch[dev].addr;
    return KDA_OK;
  }
  void *p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess || !p) {
    cudaGetLastError();  // a failed module load must not surface at the next launch check
    char msg[256];
    snprintf(msg, sizeof(msg),
             "kda_chunk_fwd_noalloc: the %zu-byte built-in scratch could not be mapped on device "
             "%d (%s); make the first call before device memory is handed to a pool",
             kNoAllocScratchBytes, dev, cudaGetErrorString(e));
    gdr::set_last_error(msg);
    return KDA_ERR_CUDA;
  }
  // cache only when the context can be told apart; otherwise look up every call
  g_scratch[dev] = current_context_id(&id) ? ScratchAddr{id, p} : ScratchAddr{0, nullptr};
  *addr = p;
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
  if (st != KDA_OK) return st;
  return kda_chunk_fwd(q, k, v, g, beta, o, initial_state, final_state, cu_seqlens, num_seqs, B,
                       T, H, d_k, d_v, io_dtype, scratch, kNoAllocScratchBytes, stream);
}

}  // extern "C"
