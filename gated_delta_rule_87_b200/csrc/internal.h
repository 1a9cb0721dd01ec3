// Internal launch interfaces between the C ABI layer (api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace gdr {

// Records the device time of the enclosed launch(es) on `s` when tracing is
// enabled (kda_trace_enable); does nothing otherwise.
class TraceScope {
 public:
  TraceScope(const char *name, cudaStream_t s);
  ~TraceScope();
  TraceScope(const TraceScope &) = delete;
  TraceScope &operator=(const TraceScope &) = delete;

 private:
  const char *name_;
  cudaStream_t stream_;
  void *start_ = nullptr;
  void *stop_ = nullptr;
};

// Sets the text kda_last_error() returns on the calling host thread.
void set_last_error(const char *msg);

// Multiprocessor count of the current device.
int sm_count();

// Bounds-checked build: violations counted by each translation unit's
// kernels since the last read (0 in the normal build; ~0u if unreadable).
unsigned int oob_count_prefill_tc();
unsigned int oob_count_prefill_simt();
unsigned int oob_count_decode();
unsigned int oob_count_api();

// Token-by-token form: T tokens for each of N sequences ([N, T, H, d]
// layout), state updated in place.  T = 1 is one decode step.
struct DecodeArgs {
  const void *q, *k, *v;
  const float *g, *beta;
  void *o;
  float *state;
  const int32_t *slots;  // device [N] state-pool slots, or nullptr (slot n = n)
  int64_t num_slots;     // pool capacity; slots outside [0, num_slots) are padding
  int N, T, H_qk, H_v, d_k, d_v;
  bool channel_gate;  // KDA (per-channel) or Gated DeltaNet (scalar)
  bool decay_first;   // decay before the erase (KDA only)
  bool bf16;          // io dtype
};

cudaError_t launch_recurrent(const DecodeArgs &a, cudaStream_t stream);

// dst[dst_slots[n]] = src[src_slots[n]] for n < N, per_seq_floats floats per
// entry (a multiple of 4, 16-byte aligned buffers); NULL slots = identity.
// A source slot outside [0, src_limit) copies zeros (as does src == NULL); a
// destination slot outside [0, dst_limit) is skipped.
cudaError_t launch_state_copy(const float *src, const int32_t *src_slots, int64_t src_limit,
                              float *dst, const int32_t *dst_slots, int64_t dst_limit, int N,
                              int64_t per_seq_floats, cudaStream_t stream);

// One bounded on-device wait that expires: writes KDA_DEVICE_TIMEOUT to *status.
cudaError_t launch_wait_timeout(int32_t *status, uint32_t max_polls, cudaStream_t stream);

// Chunk length of the prefill kernels (tokens per chunk).
constexpr int kChunk = 64;

struct PrefillArgs {
  const void *q, *k, *v;
  const float *g, *beta;
  void *o;
  const float *initial_state;
  float *final_state;
  const int32_t *state_slots;  // device [num_seqs] pool slots of the states, or nullptr
  int64_t num_slots;           // pool capacity (slots outside [0, num_slots): no state)
  const int32_t *cu_seqlens;  // device, or nullptr (dense)
  int num_seqs;               // N
  int B, T, H_qk, H_v, d_k, d_v;
  bool channel_gate;
  bool decay_first;  // decay before the erase (KDA only)
  bool bf16;
  // workspace (device); status word at offset 0
  void *workspace;
  size_t workspace_bytes;
  // chunks: an upper bound on the total number of chunks over all sequences
  int64_t max_chunks;
};

// Bytes of workspace a prefill call needs (includes the 256-byte status block).
size_t prefill_workspace_bytes(int T, int H_v, int d_k, int d_v, int num_seqs, bool bf16);

cudaError_t launch_prefill_f32(const PrefillArgs &a, cudaStream_t stream);
cudaError_t launch_prefill_tc(const PrefillArgs &a, cudaStream_t stream);

// Device-side check of cu_seqlens; writes KDA_DEVICE_BAD_CU_SEQLENS into the
// status word on failure (kernels then skip all work).
cudaError_t launch_check_cu_seqlens(const int32_t *cu, int num_seqs, int T, int32_t *status,
                                    cudaStream_t stream);

}  // namespace gdr
