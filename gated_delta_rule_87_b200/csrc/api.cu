// C ABI of the gated delta-rule library: argument validation, workspace
// sizing and dispatch to the kernels.  See include/gated_delta.h.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <mutex>
#include <string>
#include <vector>

#include "common.cuh"
#include "gated_delta.h"
#include "internal.h"

namespace {

thread_local std::string g_last_error;

kda_status_t fail(kda_status_t st, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

kda_status_t cuda_fail(cudaError_t e, const char *where) {
  return fail(KDA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

bool head_dim_ok(int d) { return d == 64 || d == 128; }

constexpr size_t kStatusBytes = 256;


// Validation shared by both prefill entry points.
kda_status_t check_prefill(const gdr::PrefillArgs &a) {
  const bool empty = (int64_t)a.B * a.T == 0;  // no tokens: data pointers may be NULL
  if (!empty && (!a.q || !a.k || !a.v || !a.g || !a.beta || !a.o))
    return fail(KDA_ERR_INVALID_ARG, "q, k, v, g, beta and o must be non-NULL");
  if (a.B <= 0 || a.T < 0 || a.H_qk <= 0 || a.H_v <= 0)
    return fail(KDA_ERR_INVALID_ARG, "need B > 0, T >= 0, H > 0 (B=%d T=%d H_qk=%d H_v=%d)", a.B,
                a.T, a.H_qk, a.H_v);
  if (a.H_v % a.H_qk != 0)
    return fail(KDA_ERR_INVALID_ARG, "H_v (%d) must be a multiple of H_qk (%d)", a.H_v, a.H_qk);
  if (!head_dim_ok(a.d_k) || !head_dim_ok(a.d_v))
    return fail(KDA_ERR_UNSUPPORTED, "d_k and d_v must be 64 or 128 (got %d, %d)", a.d_k, a.d_v);
  const void *ptrs16[] = {a.q, a.k, a.v, a.g, a.o, a.initial_state, a.final_state};
  for (const void *p : ptrs16)
    if (p && !aligned16(p)) return fail(KDA_ERR_INVALID_ARG, "pointer %p is not 16-byte aligned", p);
  if ((a.beta && !aligned4(a.beta)) || (a.cu_seqlens && !aligned4(a.cu_seqlens)) ||
      (a.state_slots && !aligned4(a.state_slots)))
    return fail(KDA_ERR_INVALID_ARG, "beta, cu_seqlens and state_slots must be 4-byte aligned");
  if (a.state_slots && a.num_slots < 0)
    return fail(KDA_ERR_INVALID_ARG, "num_slots must be >= 0");
  if (a.cu_seqlens) {
    if (a.B != 1) return fail(KDA_ERR_INVALID_ARG, "packed sequences (cu_seqlens) need B == 1");
    if (a.num_seqs < 0) return fail(KDA_ERR_INVALID_ARG, "num_seqs must be >= 0");
  }
  if ((int64_t)a.B * a.T > INT32_MAX)
    return fail(KDA_ERR_INVALID_ARG, "B*T must fit in int32");
  if (!empty && (a.o == a.q || a.o == a.k || a.o == a.v))
    return fail(KDA_ERR_INVALID_ARG, "o must not alias q, k or v");
  if (!a.workspace) return fail(KDA_ERR_WORKSPACE, "workspace is NULL");
  if (reinterpret_cast<uintptr_t>(a.workspace) & 255u)
    return fail(KDA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  const size_t need = gdr::prefill_workspace_bytes(a.B * a.T, a.H_v, a.d_k, a.d_v, a.num_seqs, a.bf16);
  if (a.workspace_bytes < need)
    return fail(KDA_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", a.workspace_bytes, need);
  return KDA_OK;
}

bool use_tensor_core_path(const gdr::PrefillArgs &a) {
  return a.bf16 && a.d_k == 128 && a.d_v == 128;
}

// reset_status false: a later piece of one streamed prefill, which keeps the
// status word its first piece reset (so that an error of any piece stays
// recorded, and the kernels of the pieces after it skip their work).
kda_status_t run_prefill(gdr::PrefillArgs &a, cudaStream_t s, bool reset_status = true) {
  kda_status_t st = check_prefill(a);
  if (st != KDA_OK) return st;
  int32_t *status = reinterpret_cast<int32_t *>(a.workspace);
  cudaError_t e = reset_status ? cudaMemsetAsync(status, 0, kStatusBytes, s) : cudaSuccess;
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(status)");
  if (!a.cu_seqlens) a.num_seqs = a.B;
  if (!a.state_slots) a.num_slots = a.num_seqs;
  const bool tc = use_tensor_core_path(a);
  if (a.cu_seqlens && !tc) {  // the tensor-core path validates in its planning kernel
    e = gdr::launch_check_cu_seqlens(a.cu_seqlens, a.num_seqs, a.T, status, s);
    if (e != cudaSuccess) return cuda_fail(e, "cu_seqlens check launch");
  }
  if (a.num_seqs == 0 || a.T == 0) {
    // nothing to compute; final state = initial state
    const int64_t per_seq = (int64_t)a.H_v * a.d_k * a.d_v;
    if (a.final_state && a.state_slots) {
      if (a.final_state != a.initial_state) {
        e = gdr::launch_state_copy(a.initial_state, a.state_slots, a.num_slots, a.final_state,
                                   a.state_slots, a.num_slots, a.num_seqs, per_seq, s);
        if (e != cudaSuccess) return cuda_fail(e, "final state copy");
      }
    } else if (a.final_state) {
      const size_t bytes = (size_t)a.num_seqs * a.H_v * a.d_k * a.d_v * sizeof(float);
      if (bytes) {
        e = a.initial_state ? cudaMemcpyAsync(a.final_state, a.initial_state, bytes,
                                              cudaMemcpyDeviceToDevice, s)
                            : cudaMemsetAsync(a.final_state, 0, bytes, s);
        if (e != cudaSuccess) return cuda_fail(e, "final state copy");
      }
    }
    return KDA_OK;
  }
  a.max_chunks = (int64_t)(a.B * (int64_t)a.T) / gdr::kChunk + a.num_seqs;
  e = tc ? gdr::launch_prefill_tc(a, s) : gdr::launch_prefill_f32(a, s);
  if (e != cudaSuccess) return cuda_fail(e, "prefill launch");
  return KDA_OK;
}

// ---- prefill from host memory, copies overlapped with the kernels ----
// Streams and events of the streamed prefill, per device, created once.
struct HostStreams {
  cudaStream_t h2d = nullptr, d2h = nullptr;
  std::vector<cudaEvent_t> ev;
};
constexpr int kMaxHostDevices = 64;
constexpr int kMaxPieces = 64;
std::mutex g_host_mu;
HostStreams g_host_streams[kMaxHostDevices];

cudaError_t host_streams(int dev, size_t n_events, HostStreams **out) {
  HostStreams &h = g_host_streams[dev];
  cudaError_t e = cudaSuccess;
  if (!h.h2d) e = cudaStreamCreateWithFlags(&h.h2d, cudaStreamNonBlocking);
  if (e == cudaSuccess && !h.d2h) e = cudaStreamCreateWithFlags(&h.d2h, cudaStreamNonBlocking);
  while (e == cudaSuccess && h.ev.size() < n_events) {
    cudaEvent_t ev;
    e = cudaEventCreateWithFlags(&ev, cudaEventDisableTiming);
    if (e == cudaSuccess) h.ev.push_back(ev);
  }
  *out = &h;
  return e;
}

size_t up256(size_t x) { return (x + 255) / 256 * 256; }

// Device buffer of the streamed prefill: the workspace of one piece first (its
// status word at offset 0), then q, k, v, g, beta and o with the pieces one
// after the other ([B, piece length, H, d] each), the initial state and two
// states the pieces hand over through.
struct HostLayout {
  int piece, pieces;
  size_t q, k, v, g, beta, o, s0, st0, st1, total;
};
HostLayout host_layout(int B, int T, int H, int d_k, int d_v, bool bf16, int pieces) {
  HostLayout L{};
  const int per = (T + pieces - 1) / pieces;
  L.piece = (per + gdr::kChunk - 1) / gdr::kChunk * gdr::kChunk;
  L.pieces = (T + L.piece - 1) / L.piece;
  const size_t e = bf16 ? 2 : 4, rows = (size_t)B * T * H;
  const size_t state = (size_t)B * H * d_k * d_v * 4;
  size_t off = up256(gdr::prefill_workspace_bytes(B * L.piece, H, d_k, d_v, B, bf16));
  L.q = off; off = up256(off + rows * d_k * e);
  L.k = off; off = up256(off + rows * d_k * e);
  L.v = off; off = up256(off + rows * d_v * e);
  L.g = off; off = up256(off + rows * d_k * 4);
  L.beta = off; off = up256(off + rows * 4);
  L.o = off; off = up256(off + rows * d_v * e);
  L.s0 = off; off = up256(off + state);
  L.st0 = off; off = up256(off + state);
  L.st1 = off; off = up256(off + state);
  L.total = off;
  return L;
}

int host_pieces(int32_t pieces) { return pieces <= 0 ? 4 : pieces; }

}  // namespace

namespace gdr {

void set_last_error(const char *msg) { g_last_error = msg; }

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

__global__ void check_cu_seqlens_kernel(const int32_t *__restrict__ cu, int num_seqs, int T,
                                        int32_t *status) {
  bool bad = false;
  for (int i = threadIdx.x; i <= num_seqs; i += blockDim.x) {
    const int32_t x = cu[i];
    if (i == 0 && x != 0) bad = true;
    if (i == num_seqs && x != T) bad = true;
    if (i < num_seqs && cu[i + 1] < x) bad = true;
  }
  if (__syncthreads_or(bad) && threadIdx.x == 0) *status = KDA_DEVICE_BAD_CU_SEQLENS;
}

GDR_DEFINE_OOB_COUNTER(oob_count_api)

cudaError_t launch_check_cu_seqlens(const int32_t *cu, int num_seqs, int T, int32_t *status,
                                    cudaStream_t stream) {
  check_cu_seqlens_kernel<<<1, 256, 0, stream>>>(cu, num_seqs, T, status);
  return cudaGetLastError();
}

}  // namespace gdr

extern "C" {

int32_t kda_abi_version(void) { return KDA_ABI_VERSION; }

const char *kda_status_string(kda_status_t s) {
  switch (s) {
    case KDA_OK: return "ok";
    case KDA_ERR_INVALID_ARG: return "invalid argument";
    case KDA_ERR_UNSUPPORTED: return "unsupported configuration";
    case KDA_ERR_CUDA: return "CUDA error";
    case KDA_ERR_DEVICE_CHECK: return "device-side check failed";
    case KDA_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

const char *kda_last_error(void) { return g_last_error.c_str(); }

size_t kda_chunk_fwd_workspace_size(int32_t B, int32_t T, int32_t H, int32_t d_k, int32_t d_v,
                                    int32_t num_seqs, kda_dtype_t io_dtype) {
  const int n = num_seqs > 0 ? num_seqs : B;
  return gdr::prefill_workspace_bytes(B * T, H, d_k, d_v, n, io_dtype == KDA_BF16);
}

size_t gdn_chunk_fwd_workspace_size(int32_t B, int32_t T, int32_t H_qk, int32_t H_v, int32_t d_k,
                                    int32_t d_v, int32_t num_seqs, kda_dtype_t io_dtype) {
  (void)H_qk;
  const int n = num_seqs > 0 ? num_seqs : B;
  return gdr::prefill_workspace_bytes(B * T, H_v, d_k, d_v, n, io_dtype == KDA_BF16);
}

kda_status_t kda_chunk_fwd_ex(const void *q, const void *k, const void *v, const float *g,
                              const float *beta, void *o, const float *initial_state,
                              float *final_state, const int32_t *state_slots, int64_t num_slots,
                              const int32_t *cu_seqlens, int32_t num_seqs, int32_t B, int32_t T,
                              int32_t H, int32_t d_k, int32_t d_v, kda_order_t order,
                              kda_dtype_t io_dtype, void *workspace, size_t workspace_bytes,
                              void *stream) {
  if (io_dtype != KDA_F32 && io_dtype != KDA_BF16)
    return fail(KDA_ERR_INVALID_ARG, "io_dtype must be KDA_F32 or KDA_BF16");
  if (order != KDA_ERASE_THEN_DECAY && order != KDA_DECAY_THEN_ERASE)
    return fail(KDA_ERR_INVALID_ARG, "order must be KDA_ERASE_THEN_DECAY or KDA_DECAY_THEN_ERASE");
  gdr::PrefillArgs a{};
  a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.o = o;
  a.initial_state = initial_state; a.final_state = final_state;
  a.state_slots = state_slots; a.num_slots = num_slots;
  a.cu_seqlens = cu_seqlens; a.num_seqs = cu_seqlens ? num_seqs : B;
  a.B = B; a.T = T; a.H_qk = H; a.H_v = H; a.d_k = d_k; a.d_v = d_v;
  a.channel_gate = true; a.decay_first = (order == KDA_DECAY_THEN_ERASE);
  a.bf16 = (io_dtype == KDA_BF16);
  a.workspace = workspace; a.workspace_bytes = workspace_bytes;
  return run_prefill(a, static_cast<cudaStream_t>(stream));
}

kda_status_t kda_chunk_fwd(const void *q, const void *k, const void *v, const float *g,
                           const float *beta, void *o, const float *initial_state,
                           float *final_state, const int32_t *cu_seqlens, int32_t num_seqs,
                           int32_t B, int32_t T, int32_t H, int32_t d_k, int32_t d_v,
                           kda_dtype_t io_dtype, void *workspace, size_t workspace_bytes,
                           void *stream) {
  return kda_chunk_fwd_ex(q, k, v, g, beta, o, initial_state, final_state, nullptr, 0,
                          cu_seqlens, num_seqs, B, T, H, d_k, d_v, KDA_ERASE_THEN_DECAY, io_dtype,
                          workspace, workspace_bytes, stream);
}

size_t kda_chunk_fwd_host_buffer_size(int32_t B, int32_t T, int32_t H, int32_t d_k, int32_t d_v,
                                      kda_dtype_t io_dtype, int32_t pieces) {
  if (B <= 0 || T <= 0 || H <= 0 || pieces > kMaxPieces) return 0;
  return host_layout(B, T, H, d_k, d_v, io_dtype == KDA_BF16, host_pieces(pieces)).total;
}

kda_status_t kda_chunk_fwd_host(const void *q, const void *k, const void *v, const float *g,
                                const float *beta, void *o, const float *initial_state,
                                float *final_state, int32_t B, int32_t T, int32_t H, int32_t d_k,
                                int32_t d_v, kda_dtype_t io_dtype, int32_t pieces,
                                void *device_buffer, size_t device_buffer_bytes, void *stream) {
  if (io_dtype != KDA_F32 && io_dtype != KDA_BF16)
    return fail(KDA_ERR_INVALID_ARG, "io_dtype must be KDA_F32 or KDA_BF16");
  if (B <= 0 || T <= 0 || H <= 0)
    return fail(KDA_ERR_INVALID_ARG, "need B > 0, T > 0, H > 0 (B=%d T=%d H=%d)", B, T, H);
  if (!head_dim_ok(d_k) || !head_dim_ok(d_v))
    return fail(KDA_ERR_UNSUPPORTED, "d_k and d_v must be 64 or 128 (got %d, %d)", d_k, d_v);
  if (pieces > kMaxPieces) return fail(KDA_ERR_INVALID_ARG, "pieces must be <= %d", kMaxPieces);
  if (!q || !k || !v || !g || !beta || !o)
    return fail(KDA_ERR_INVALID_ARG, "q, k, v, g, beta and o must be non-NULL");
  const bool bf16 = io_dtype == KDA_BF16;
  const HostLayout L = host_layout(B, T, H, d_k, d_v, bf16, host_pieces(pieces));
  if (!device_buffer || (reinterpret_cast<uintptr_t>(device_buffer) & 255u) ||
      device_buffer_bytes < L.total)
    return fail(KDA_ERR_WORKSPACE,
                "device_buffer must be 256-byte aligned and hold kda_chunk_fwd_host_buffer_size() "
                "= %zu bytes (got %zu)", L.total, device_buffer_bytes);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxHostDevices) return fail(KDA_ERR_INVALID_ARG, "device %d", dev);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned char *buf = static_cast<unsigned char *>(device_buffer);
  const size_t e_io = bf16 ? 2 : 4, state = (size_t)B * H * d_k * d_v * 4;
  const size_t rq = (size_t)H * d_k * e_io, rv = (size_t)H * d_v * e_io, rg = (size_t)H * d_k * 4,
               rb = (size_t)H * 4;  // bytes per token row

  std::lock_guard<std::mutex> lk(g_host_mu);
  HostStreams *hs = nullptr;
  e = host_streams(dev, 2 * (size_t)L.pieces + 2, &hs);
  if (e != cudaSuccess) return cuda_fail(e, "creating the copy streams");
  cudaEvent_t start = hs->ev[0], end = hs->ev[1];
  // copies start after the work already queued on the caller's stream
  e = cudaEventRecord(start, s);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(hs->h2d, start, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(hs->d2h, start, 0);
  if (e != cudaSuccess) return cuda_fail(e, "ordering the copy streams");
  // one piece's token rows [t0, t0 + len) of every sequence, host [B, T, row] <-> device [B, len, row]
  // (one sequence: a plain copy; several: one strided copy)
  auto h2d = [&](size_t dst_off, const void *src, size_t row, int t0, int len) {
    unsigned char *dst = buf + dst_off + (size_t)B * t0 * row;
    const unsigned char *from = static_cast<const unsigned char *>(src) + (size_t)t0 * row;
    if (B == 1) return cudaMemcpyAsync(dst, from, (size_t)len * row, cudaMemcpyHostToDevice, hs->h2d);
    return cudaMemcpy2DAsync(dst, (size_t)len * row, from, (size_t)T * row, (size_t)len * row, B,
                             cudaMemcpyHostToDevice, hs->h2d);
  };
  if (initial_state) {
    e = cudaMemcpyAsync(buf + L.s0, initial_state, state, cudaMemcpyHostToDevice, hs->h2d);
    if (e != cudaSuccess) return cuda_fail(e, "initial state copy");
  }
  for (int p = 0; p < L.pieces; ++p) {
    const int t0 = p * L.piece, len = T - t0 < L.piece ? T - t0 : L.piece;
    cudaEvent_t in = hs->ev[2 + 2 * p], done = hs->ev[3 + 2 * p];
    e = h2d(L.q, q, rq, t0, len);
    if (e == cudaSuccess) e = h2d(L.k, k, rq, t0, len);
    if (e == cudaSuccess) e = h2d(L.v, v, rv, t0, len);
    if (e == cudaSuccess) e = h2d(L.g, g, rg, t0, len);
    if (e == cudaSuccess) e = h2d(L.beta, beta, rb, t0, len);
    if (e == cudaSuccess) e = cudaEventRecord(in, hs->h2d);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, in, 0);
    if (e != cudaSuccess) return cuda_fail(e, "input copy");
    gdr::PrefillArgs a{};
    const size_t r0 = (size_t)B * t0;
    a.q = buf + L.q + r0 * rq; a.k = buf + L.k + r0 * rq; a.v = buf + L.v + r0 * rv;
    a.g = reinterpret_cast<const float *>(buf + L.g + r0 * rg);
    a.beta = reinterpret_cast<const float *>(buf + L.beta + r0 * rb);
    a.o = buf + L.o + r0 * rv;
    a.initial_state = p > 0 ? reinterpret_cast<const float *>(buf + ((p - 1) & 1 ? L.st1 : L.st0))
                      : initial_state ? reinterpret_cast<const float *>(buf + L.s0) : nullptr;
    a.final_state = reinterpret_cast<float *>(buf + (p & 1 ? L.st1 : L.st0));
    a.num_seqs = B;
    a.B = B; a.T = len; a.H_qk = H; a.H_v = H; a.d_k = d_k; a.d_v = d_v;
    a.channel_gate = true; a.bf16 = bf16;
    a.workspace = buf; a.workspace_bytes = L.q;
    const kda_status_t st = run_prefill(a, s, p == 0);
    if (st != KDA_OK) return st;
    e = cudaEventRecord(done, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(hs->d2h, done, 0);
    if (e == cudaSuccess && B == 1)
      e = cudaMemcpyAsync(static_cast<unsigned char *>(o) + (size_t)t0 * rv, buf + L.o + r0 * rv,
                          (size_t)len * rv, cudaMemcpyDeviceToHost, hs->d2h);
    else if (e == cudaSuccess)
      e = cudaMemcpy2DAsync(static_cast<unsigned char *>(o) + (size_t)t0 * rv, (size_t)T * rv,
                            buf + L.o + r0 * rv, (size_t)len * rv, (size_t)len * rv, B,
                            cudaMemcpyDeviceToHost, hs->d2h);
    if (e != cudaSuccess) return cuda_fail(e, "output copy");
  }
  if (final_state) {
    e = cudaMemcpyAsync(final_state, buf + ((L.pieces - 1) & 1 ? L.st1 : L.st0), state,
                        cudaMemcpyDeviceToHost, hs->d2h);
    if (e != cudaSuccess) return cuda_fail(e, "final state copy");
  }
  // the caller's stream continues once every copy has landed
  e = cudaEventRecord(end, hs->d2h);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s, end, 0);
  if (e == cudaSuccess) e = cudaEventRecord(end, hs->h2d);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(s, end, 0);
  if (e != cudaSuccess) return cuda_fail(e, "joining the copy streams");
  return KDA_OK;
}

kda_status_t gdn_chunk_fwd_ex(const void *q, const void *k, const void *v, const float *g,
                              const float *beta, void *o, const float *initial_state,
                              float *final_state, const int32_t *state_slots, int64_t num_slots,
                              const int32_t *cu_seqlens, int32_t num_seqs, int32_t B, int32_t T,
                              int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v,
                              kda_dtype_t io_dtype, void *workspace, size_t workspace_bytes,
                              void *stream) {
  if (io_dtype != KDA_F32 && io_dtype != KDA_BF16)
    return fail(KDA_ERR_INVALID_ARG, "io_dtype must be KDA_F32 or KDA_BF16");
  gdr::PrefillArgs a{};
  a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.o = o;
  a.initial_state = initial_state; a.final_state = final_state;
  a.state_slots = state_slots; a.num_slots = num_slots;
  a.cu_seqlens = cu_seqlens; a.num_seqs = cu_seqlens ? num_seqs : B;
  a.B = B; a.T = T; a.H_qk = H_qk; a.H_v = H_v; a.d_k = d_k; a.d_v = d_v;
  a.channel_gate = false; a.bf16 = (io_dtype == KDA_BF16);
  a.workspace = workspace; a.workspace_bytes = workspace_bytes;
  return run_prefill(a, static_cast<cudaStream_t>(stream));
}

kda_status_t gdn_chunk_fwd(const void *q, const void *k, const void *v, const float *g,
                           const float *beta, void *o, const float *initial_state,
                           float *final_state, const int32_t *cu_seqlens, int32_t num_seqs,
                           int32_t B, int32_t T, int32_t H_qk, int32_t H_v, int32_t d_k,
                           int32_t d_v, kda_dtype_t io_dtype, void *workspace,
                           size_t workspace_bytes, void *stream) {
  return gdn_chunk_fwd_ex(q, k, v, g, beta, o, initial_state, final_state, nullptr, 0,
                          cu_seqlens, num_seqs, B, T, H_qk, H_v, d_k, d_v, io_dtype, workspace,
                          workspace_bytes, stream);
}

static kda_status_t decode_common(gdr::DecodeArgs &a, kda_dtype_t io_dtype, void *stream) {
  if (io_dtype != KDA_F32 && io_dtype != KDA_BF16)
    return fail(KDA_ERR_INVALID_ARG, "io_dtype must be KDA_F32 or KDA_BF16");
  a.bf16 = (io_dtype == KDA_BF16);
  if (a.N < 0 || a.T < 0 || a.H_qk <= 0 || a.H_v <= 0)
    return fail(KDA_ERR_INVALID_ARG, "need N >= 0, T >= 0 and H > 0");
  if (a.N == 0 || a.T == 0) return KDA_OK;  // no tokens: nothing to do
  if (!a.q || !a.k || !a.v || !a.g || !a.beta || !a.o || !a.state)
    return fail(KDA_ERR_INVALID_ARG, "q, k, v, g, beta, o and state must be non-NULL");
  if (a.slots && (!aligned4(a.slots) || a.num_slots < 0))
    return fail(KDA_ERR_INVALID_ARG, "state_slots must be 4-byte aligned and num_slots >= 0");
  if (!a.slots) a.num_slots = a.N;
  if ((int64_t)a.N * a.T > INT32_MAX)
    return fail(KDA_ERR_INVALID_ARG, "N*T must fit in int32");
  if (a.H_v % a.H_qk != 0)
    return fail(KDA_ERR_INVALID_ARG, "H_v (%d) must be a multiple of H_qk (%d)", a.H_v, a.H_qk);
  if (!head_dim_ok(a.d_k) || !head_dim_ok(a.d_v))
    return fail(KDA_ERR_UNSUPPORTED, "d_k and d_v must be 64 or 128 (got %d, %d)", a.d_k, a.d_v);
  if ((int64_t)a.N * a.H_v > INT32_MAX)
    return fail(KDA_ERR_INVALID_ARG, "N*H must fit in int32");
  if (!aligned16(a.state))
    return fail(KDA_ERR_INVALID_ARG, "state %p is not 16-byte aligned", (const void *)a.state);
  const size_t esz = a.bf16 ? 2 : 4;
  const void *ptrs[] = {a.q, a.k, a.v, a.o};
  for (const void *p : ptrs)
    if (reinterpret_cast<uintptr_t>(p) % esz)
      return fail(KDA_ERR_INVALID_ARG, "pointer %p is not aligned to its element size", p);
  if (!aligned4(a.g) || !aligned4(a.beta))
    return fail(KDA_ERR_INVALID_ARG, "g and beta must be 4-byte aligned");
  if (a.o == a.q || a.o == a.k || a.o == a.v || a.o == a.state)
    return fail(KDA_ERR_INVALID_ARG, "o must not alias an input or the state");
  cudaError_t e = gdr::launch_recurrent(a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "recurrent launch");
  return KDA_OK;
}

kda_status_t kda_recurrent_fwd(const void *q, const void *k, const void *v, const float *g,
                               const float *beta, void *o, float *state,
                               const int32_t *state_slots, int64_t num_slots, int32_t N,
                               int32_t T, int32_t H, int32_t d_k, int32_t d_v, kda_order_t order,
                               kda_dtype_t io_dtype, void *stream) {
  if (order != KDA_ERASE_THEN_DECAY && order != KDA_DECAY_THEN_ERASE)
    return fail(KDA_ERR_INVALID_ARG, "order must be KDA_ERASE_THEN_DECAY or KDA_DECAY_THEN_ERASE");
  gdr::DecodeArgs a{};
  a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.o = o; a.state = state;
  a.slots = state_slots; a.num_slots = num_slots;
  a.N = N; a.T = T; a.H_qk = H; a.H_v = H; a.d_k = d_k; a.d_v = d_v; a.channel_gate = true;
  a.decay_first = (order == KDA_DECAY_THEN_ERASE);
  return decode_common(a, io_dtype, stream);
}

kda_status_t gdn_recurrent_fwd(const void *q, const void *k, const void *v, const float *g,
                               const float *beta, void *o, float *state,
                               const int32_t *state_slots, int64_t num_slots, int32_t N,
                               int32_t T, int32_t H_qk, int32_t H_v, int32_t d_k, int32_t d_v,
                               kda_dtype_t io_dtype, void *stream) {
  gdr::DecodeArgs a{};
  a.q = q; a.k = k; a.v = v; a.g = g; a.beta = beta; a.o = o; a.state = state;
  a.slots = state_slots; a.num_slots = num_slots;
  a.N = N; a.T = T; a.H_qk = H_qk; a.H_v = H_v; a.d_k = d_k; a.d_v = d_v;
  a.channel_gate = false;
  return decode_common(a, io_dtype, stream);
}

kda_status_t kda_decode_step(const void *q, const void *k, const void *v, const float *g,
                             const float *beta, void *o, float *state, int32_t N, int32_t H,
                             int32_t d_k, int32_t d_v, kda_dtype_t io_dtype, void *stream) {
  return kda_recurrent_fwd(q, k, v, g, beta, o, state, nullptr, 0, N, 1, H, d_k, d_v,
                           KDA_ERASE_THEN_DECAY, io_dtype, stream);
}

kda_status_t gdn_decode_step(const void *q, const void *k, const void *v, const float *g,
                             const float *beta, void *o, float *state, int32_t N, int32_t H_qk,
                             int32_t H_v, int32_t d_k, int32_t d_v, kda_dtype_t io_dtype,
                             void *stream) {
  return gdn_recurrent_fwd(q, k, v, g, beta, o, state, nullptr, 0, N, 1, H_qk, H_v, d_k, d_v,
                           io_dtype, stream);
}

static kda_status_t state_copy_common(const float *src, const int32_t *src_slots,
                                      int64_t src_limit, float *dst, const int32_t *dst_slots,
                                      int64_t dst_limit, int32_t N, int32_t H, int32_t d_k,
                                      int32_t d_v, void *stream) {
  if (N < 0 || H <= 0) return fail(KDA_ERR_INVALID_ARG, "need N >= 0 and H > 0");
  if (!head_dim_ok(d_k) || !head_dim_ok(d_v))
    return fail(KDA_ERR_UNSUPPORTED, "d_k and d_v must be 64 or 128 (got %d, %d)", d_k, d_v);
  if (N == 0) return KDA_OK;
  if (!src || !dst || !(src_slots || dst_slots))
    return fail(KDA_ERR_INVALID_ARG, "pool, slots and the dense buffer must be non-NULL");
  if (!aligned16(src) || !aligned16(dst))
    return fail(KDA_ERR_INVALID_ARG, "state buffers must be 16-byte aligned");
  if ((src_slots && !aligned4(src_slots)) || (dst_slots && !aligned4(dst_slots)))
    return fail(KDA_ERR_INVALID_ARG, "slots must be 4-byte aligned");
  if (src_limit < 0 || dst_limit < 0) return fail(KDA_ERR_INVALID_ARG, "num_slots must be >= 0");
  if (src == dst) return fail(KDA_ERR_INVALID_ARG, "the pool and the dense buffer must differ");
  const int64_t per_seq = (int64_t)H * d_k * d_v;
  cudaError_t e = gdr::launch_state_copy(src, src_slots, src_limit, dst, dst_slots, dst_limit, N,
                                         per_seq, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "state copy launch");
  return KDA_OK;
}

kda_status_t kda_state_gather(const float *pool, const int32_t *state_slots, int64_t num_slots,
                              float *out, int32_t N, int32_t H, int32_t d_k, int32_t d_v,
                              void *stream) {
  return state_copy_common(pool, state_slots, num_slots, out, nullptr, N, N, H, d_k, d_v, stream);
}

kda_status_t kda_state_scatter(const float *src, float *pool, const int32_t *state_slots,
                               int64_t num_slots, int32_t N, int32_t H, int32_t d_k, int32_t d_v,
                               void *stream) {
  return state_copy_common(src, nullptr, N, pool, state_slots, num_slots, N, H, d_k, d_v, stream);
}

kda_status_t kda_selftest_wait_timeout(void *workspace, int32_t max_polls, void *stream) {
  if (!workspace) return fail(KDA_ERR_INVALID_ARG, "workspace is NULL");
  if (max_polls < 1 || max_polls > 4096)
    return fail(KDA_ERR_INVALID_ARG, "max_polls must be in [1, 4096]");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t *status = static_cast<int32_t *>(workspace);
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int32_t), s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(status)");
  e = gdr::launch_wait_timeout(status, (uint32_t)max_polls, s);
  if (e != cudaSuccess) return cuda_fail(e, "wait-timeout launch");
  return KDA_OK;
}

kda_status_t kda_check_device_status(const void *workspace, void *stream, int32_t *device_code) {
  if (!workspace) return fail(KDA_ERR_INVALID_ARG, "workspace is NULL");
  int32_t code = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(&code, workspace, sizeof(code), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device status");
  if (device_code) *device_code = code;
  if (code != KDA_DEVICE_OK)
    return fail(KDA_ERR_DEVICE_CHECK, "device check failed with code %d", code);
  return KDA_OK;
}

int32_t kda_bounds_checked(void) {
#ifdef GDR_BOUNDS_CHECK
  return 1;
#else
  return 0;
#endif
}

kda_status_t kda_bounds_violations(void *stream, uint32_t *count) {
  if (!count) return fail(KDA_ERR_INVALID_ARG, "count is NULL");
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "synchronising before reading the bounds counters");
  const unsigned int parts[] = {gdr::oob_count_prefill_tc(), gdr::oob_count_prefill_simt(),
                                gdr::oob_count_decode(), gdr::oob_count_api()};
  uint64_t total = 0;
  for (unsigned int p : parts) {
    if (p == ~0u) return fail(KDA_ERR_CUDA, "a bounds counter could not be read");
    total += p;
  }
  *count = total > 0xffffffffull ? 0xffffffffu : (uint32_t)total;
  return KDA_OK;
}

}  // extern "C"
