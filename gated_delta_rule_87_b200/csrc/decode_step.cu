// One decode step of the gated delta rule, in place on the fp32 state.
//
// Operator: thethings.ai "The argument, in one page", table "Everything, in
// one table", rows "KDA" / "Gated DeltaNet":
//     S' = Diag(a) (S - beta k (k^T S)) + beta k v^T,   o = S'^T q.
// Expanding the readout through the update lets one pass over the old state
// produce everything:
//     r = S^T k,   p = S^T (a . q)
//     S' = a . (S - beta k r^T) + beta k v^T
//     o  = p - beta (k . (a . q)) r + beta (k . q) v
// so each state element is read once and written once.  The step is bound by
// HBM bandwidth (about 1 flop per byte): the kernel is a streaming copy with
// arithmetic in registers.
//
// Mapping: one CTA of 8 warps per (sequence, head).  Warp w owns rows
// [w*D_K/8, (w+1)*D_K/8) of the d_k x d_v state; lane l owns columns
// [l*D_V/32, (l+1)*D_V/32), loaded with one 16-byte (d_v = 128) or 8-byte
// (d_v = 64) streaming load per row, so every warp load is a contiguous
// 512-byte (256-byte) row.  The column sums r and p are reduced over the
// rows of a warp in registers and across warps through shared memory.
#include "common.cuh"
#include "internal.h"

namespace gdr {
namespace {

template <int CPL> struct vec;
template <> struct vec<4> {
  using T = float4;
  static __device__ __forceinline__ void ld(const float *p, float *x) {
    float4 v = __ldcs(reinterpret_cast<const float4 *>(p));
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
  }
  static __device__ __forceinline__ void st(float *p, const float *x) {
    __stcs(reinterpret_cast<float4 *>(p), make_float4(x[0], x[1], x[2], x[3]));
  }
};
template <> struct vec<2> {
  static __device__ __forceinline__ void ld(const float *p, float *x) {
    float2 v = __ldcs(reinterpret_cast<const float2 *>(p));
    x[0] = v.x; x[1] = v.y;
  }
  static __device__ __forceinline__ void st(float *p, const float *x) {
    __stcs(reinterpret_cast<float2 *>(p), make_float2(x[0], x[1]));
  }
};

constexpr int kWarps = 8;

template <int D_K, int D_V, typename IO, bool CHANNEL_GATE>
__global__ void __launch_bounds__(kWarps * 32, 2)
decode_step_kernel(const IO *__restrict__ q, const IO *__restrict__ k, const IO *__restrict__ v,
                   const float *__restrict__ g, const float *__restrict__ beta,
                   IO *__restrict__ o, float *__restrict__ state, int H_qk, int H_v) {
  constexpr int RPW = D_K / kWarps;  // state rows per warp
  constexpr int CPL = D_V / 32;      // state columns per lane
  static_assert(D_K % (kWarps * 32) == 0 || D_K == 64 || D_K == 128, "d_k");

  const int nh = blockIdx.x;  // n * H_v + h
  const int n = nh / H_v, h = nh - n * H_v;
  const int hk = h / (H_v / H_qk);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  __shared__ float s_k[D_K], s_a[D_K], s_aq[D_K];
  __shared__ float s_red[2][kWarps][D_V];
  __shared__ float s_dot[D_K / 32][2];

  // 1. stream this warp's rows of the state into registers (issued first:
  //    they are >99% of the step's bytes)
  float *S = state + (size_t)nh * D_K * D_V;
  float x[RPW][CPL];
#pragma unroll
  for (int r = 0; r < RPW; ++r) vec<CPL>::ld(S + (warp * RPW + r) * D_V + lane * CPL, x[r]);

  // 2. the token's key, query and gate (one element per thread)
  if (threadIdx.x < D_K) {
    const int i = threadIdx.x;
    const size_t qk_off = ((size_t)n * H_qk + hk) * D_K + i;
    const float kk = io<IO>::load(k + qk_off);
    const float qq = io<IO>::load(q + qk_off);
    const float gg = CHANNEL_GATE ? __ldg(g + (size_t)nh * D_K + i) : __ldg(g + nh);
    const float a = expf(gg);
    s_k[i] = kk;
    s_a[i] = a;
    s_aq[i] = a * qq;
    const float kq = warp_sum(kk * qq);
    const float kaq = warp_sum(kk * a * qq);
    if (lane == 0) {
      s_dot[i >> 5][0] = kq;
      s_dot[i >> 5][1] = kaq;
    }
  }
  const float b = __ldg(beta + nh);
  float vv[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) vv[c] = io<IO>::load(v + (size_t)nh * D_V + lane * CPL + c);
  __syncthreads();

  // 3. partial column sums over this warp's rows: r = S^T k, p = S^T (a.q)
  float rp[CPL], pp[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) rp[c] = pp[c] = 0.f;
#pragma unroll
  for (int r = 0; r < RPW; ++r) {
    const float ki = s_k[warp * RPW + r], aqi = s_aq[warp * RPW + r];
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      rp[c] = fmaf(ki, x[r][c], rp[c]);
      pp[c] = fmaf(aqi, x[r][c], pp[c]);
    }
  }
#pragma unroll
  for (int c = 0; c < CPL; ++c) {
    s_red[0][warp][lane * CPL + c] = rp[c];
    s_red[1][warp][lane * CPL + c] = pp[c];
  }
  __syncthreads();
  float rf[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) {
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) acc += s_red[0][w][lane * CPL + c];
    rf[c] = acc;
  }

  // 4. S' = a . (S - b k r^T) + b k v^T, written back in place
#pragma unroll
  for (int r = 0; r < RPW; ++r) {
    const int i = warp * RPW + r;
    const float a = s_a[i], bk = b * s_k[i];
#pragma unroll
    for (int c = 0; c < CPL; ++c) x[r][c] = fmaf(a, fmaf(-bk, rf[c], x[r][c]), bk * vv[c]);
    vec<CPL>::st(S + i * D_V + lane * CPL, x[r]);
  }

  // 5. o = p - b (k.(a.q)) r + b (k.q) v
  if (warp == 0) {
    float kq = 0.f, kaq = 0.f;
#pragma unroll
    for (int w = 0; w < D_K / 32; ++w) {
      kq += s_dot[w][0];
      kaq += s_dot[w][1];
    }
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      float p = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) p += s_red[1][w][lane * CPL + c];
      const float out = p - b * kaq * rf[c] + b * kq * vv[c];
      io<IO>::store(o + (size_t)nh * D_V + lane * CPL + c, out);
    }
  }
}

template <int D_K, int D_V, typename IO>
cudaError_t launch_dv(const DecodeArgs &a, cudaStream_t s) {
  const unsigned grid = (unsigned)((int64_t)a.N * a.H_v);
  if (a.channel_gate)
    decode_step_kernel<D_K, D_V, IO, true><<<grid, kWarps * 32, 0, s>>>(
        (const IO *)a.q, (const IO *)a.k, (const IO *)a.v, a.g, a.beta, (IO *)a.o, a.state,
        a.H_qk, a.H_v);
  else
    decode_step_kernel<D_K, D_V, IO, false><<<grid, kWarps * 32, 0, s>>>(
        (const IO *)a.q, (const IO *)a.k, (const IO *)a.v, a.g, a.beta, (IO *)a.o, a.state,
        a.H_qk, a.H_v);
  return cudaGetLastError();
}

template <typename IO>
cudaError_t launch_io(const DecodeArgs &a, cudaStream_t s) {
  if (a.d_k == 128 && a.d_v == 128) return launch_dv<128, 128, IO>(a, s);
  if (a.d_k == 128 && a.d_v == 64) return launch_dv<128, 64, IO>(a, s);
  if (a.d_k == 64 && a.d_v == 128) return launch_dv<64, 128, IO>(a, s);
  return launch_dv<64, 64, IO>(a, s);
}

}  // namespace

cudaError_t launch_decode_step(const DecodeArgs &a, cudaStream_t stream) {
  if (a.N == 0) return cudaSuccess;
  TraceScope tr("decode_step_kernel", stream);
  if (a.bf16) return launch_io<__nv_bfloat16>(a, stream);
  return launch_io<float>(a, stream);
}

}  // namespace gdr
