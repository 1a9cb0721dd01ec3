// Token-by-token (recurrent) form of the gated delta rule, in place on the
// fp32 state: one decode step (T = 1) or a few tokens per sequence (T > 1:
// speculative decoding, chunked prefill in small pieces).
//
// Operator: thethings.ai "The argument, in one page", table "Everything, in
// one table", rows "KDA" / "Gated DeltaNet":
//     S' = Diag(a) (S - beta k (k^T S)) + beta k v^T,   o = S'^T q.
// Expanding the readout through the update lets one pass over the old state
// produce everything a token needs:
//     r = S^T k,   p = S^T (a . q)
//     S' = a . (S - beta k r^T) + beta k v^T
//     o  = p - beta (k . (a . q)) r + beta (k . q) v
// With the decay applied before the erase (the variant order, S' = (I - beta k
// k^T) Diag(a) S + beta k v^T) the same pass reads r = S^T (a . k) instead:
//     S' = a . S - beta k r^T + beta k v^T,   o = p - beta (k . q) r + beta (k . q) v.
// Both orders are one template: per token and state row i the kernel keeps
//     kr_i  the direction recall is read along   (k_i, or a_i k_i)
//     e_i   the erase coefficient of row i        (beta a_i k_i, or beta k_i)
// and c_r, the coefficient of r in the readout (beta k.(a.q), or beta k.q).
//
// The state is read from HBM once and written once per call, whatever T; the
// T tokens are applied to it in registers.  A single step is bound by HBM
// bandwidth (about 1 flop per byte): a streaming copy with arithmetic.
//
// Mapping: one CTA of 8 warps per (sequence, head).  Warp w owns rows
// [w*D_K/8, (w+1)*D_K/8) of the d_k x d_v state; lane l owns columns
// [l*D_V/32, (l+1)*D_V/32), loaded with one 16-byte (d_v = 128) or 8-byte
// (d_v = 64) streaming load per row, so every warp load is a contiguous
// 512-byte (256-byte) row.  The column sums r and p are reduced over the
// rows of a warp in registers and across warps through shared memory; each
// warp then writes the readout of its own slice of the columns.  Tokens are
// taken in blocks of 8: one warp per token stages its vectors (decay,
// recall and erase directions, the readout coefficients) into shared memory
// while L2 is asked for the next block's rows, so the per-token chain has one
// block barrier and no global-memory round trip; the cross-warp partial sums
// are double-buffered by token parity.
//
// State pool: with a slot array the state of sequence n is pool[slots[n]]
// (checkpointed recurrent states for serving, inferencex.semianalysis.com
// "Linear attention", "Why it matters": a dropped state can only be rebuilt
// by replaying its sequence); a negative slot marks a padding entry whose outputs
// are written as zeros and whose state is not touched (as is a slot past the
// pool's end).
#include "common.cuh"
#include "internal.h"

namespace gdr {
namespace {

template <int CPL> struct vec;
template <> struct vec<4> {
  static __device__ __forceinline__ void sts(float *p, const float *x) {
    *reinterpret_cast<float4 *>(p) = make_float4(x[0], x[1], x[2], x[3]);
  }
  static __device__ __forceinline__ void lds(const float *p, float *x) {
    const float4 v = *reinterpret_cast<const float4 *>(p);
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
  }
  static __device__ __forceinline__ void ld(const float *p, float *x) {
    float4 v = __ldcs(reinterpret_cast<const float4 *>(p));
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
  }
  static __device__ __forceinline__ void st(float *p, const float *x) {
    __stcs(reinterpret_cast<float4 *>(p), make_float4(x[0], x[1], x[2], x[3]));
  }
};
template <> struct vec<2> {
  static __device__ __forceinline__ void sts(float *p, const float *x) {
    *reinterpret_cast<float2 *>(p) = make_float2(x[0], x[1]);
  }
  static __device__ __forceinline__ void lds(const float *p, float *x) {
    const float2 v = *reinterpret_cast<const float2 *>(p);
    x[0] = v.x; x[1] = v.y;
  }
  static __device__ __forceinline__ void ld(const float *p, float *x) {
    float2 v = __ldcs(reinterpret_cast<const float2 *>(p));
    x[0] = v.x; x[1] = v.y;
  }
  static __device__ __forceinline__ void st(float *p, const float *x) {
    __stcs(reinterpret_cast<float2 *>(p), make_float2(x[0], x[1]));
  }
};

constexpr int kWarps = 8;

// Per-token vectors of a block of up to TB tokens, staged one warp per token.
template <int D_K, int D_V, int TB> struct BlockVecs {
  float kr[TB][D_K];   // recall direction
  float aq[TB][D_K];   // a . q
  float a[TB][D_K];    // decay
  float e[TB][D_K];    // erase coefficient (beta folded in)
  float bk[TB][D_K];   // write coefficient beta k
  float v[TB][D_V];    // value
  float coef[TB][2];   // c_r, c_v = beta k.q
};

__device__ __forceinline__ void prefetch_l2(const void *p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// SINGLE: exactly one token (a decode step), known at compile time, so each
// state row goes back to HBM as soon as it is updated.
template <int D_K, int D_V, typename IO, bool CHANNEL_GATE, bool DECAY_FIRST, bool SINGLE>
__global__ void __launch_bounds__(kWarps * 32, 2)
recurrent_kernel(const IO *__restrict__ q, const IO *__restrict__ k, const IO *__restrict__ v,
                 const float *__restrict__ g, const float *__restrict__ beta,
                 IO *__restrict__ o, float *__restrict__ state,
                 const int32_t *__restrict__ slots, int64_t num_slots, int T_arg, int H_qk,
                 int H_v) {
  const int T = SINGLE ? 1 : T_arg;
  constexpr int TB = SINGLE ? 1 : kWarps;  // tokens per staged block
  constexpr int RPW = D_K / kWarps;        // state rows per warp
  constexpr int CPL = D_V / 32;            // state columns per lane
  // readout: warp w writes columns [w*CW, (w+1)*CW); NP lanes share a column,
  // each summing the partials of WPP warps
  constexpr int CW = D_V / kWarps, NP = 32 / CW, WPP = kWarps / NP;
  static_assert(D_K == 64 || D_K == 128, "d_k");

  const int nh = blockIdx.x;  // n * H_v + h
  const int n = nh / H_v, h = nh - n * H_v;
  const int hk = h / (H_v / H_qk);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  __shared__ __align__(16) BlockVecs<D_K, D_V, TB> bv;
  __shared__ __align__(16) float s_red[2][2][kWarps][D_V];  // [token parity][r | p][warp][column]

  // extents of the token rows (the bounds-checked build compares against them)
  const int64_t tokens = (int64_t)(gridDim.x / H_v) * T;
  (void)tokens;
  const int64_t slot = slots ? (int64_t)__ldg(slots + n) : (int64_t)n;
  if (slot < 0 || slot >= num_slots) {  // padding entry: zero outputs, state untouched
    for (int e = threadIdx.x; e < T * D_V; e += kWarps * 32) {
      const int t = e / D_V, c = e - t * D_V;
      if (GDR_IN_BOUNDS((int64_t)n * T + t < tokens))
        io<IO>::store(o + (((size_t)n * T + t) * H_v + h) * D_V + c, 0.f);
    }
    return;
  }

  // 1. stream this warp's rows of the state into registers (issued first:
  //    for a single step they are >99% of the bytes)
  float *S = state + ((size_t)slot * H_v + h) * D_K * D_V;
  float x[RPW][CPL];
#pragma unroll
  for (int r = 0; r < RPW; ++r) vec<CPL>::ld(S + (warp * RPW + r) * D_V + lane * CPL, x[r]);

  auto token_base = [&](int t) { return (size_t)n * T + t; };
  // One warp stages token t into block entry tt: the row vectors, the value
  // and the readout coefficients (k.q and k.(a.q) by a warp reduction).
  auto stage = [&](int tt, int t) {
    const size_t tok = GDR_IN_BOUNDS((int64_t)token_base(t) < tokens) ? token_base(t) : 0;
    const float b = __ldg(beta + tok * H_v + h);
    const float gsc = CHANNEL_GATE ? 0.f : __ldg(g + tok * H_v + h);
    float kq = 0.f, kaq = 0.f;
#pragma unroll
    for (int j = 0; j < D_K / 32; ++j) {
      const int i = lane + 32 * j;
      const size_t qk_off = (tok * H_qk + hk) * D_K + i;
      const float kk = io<IO>::load(k + qk_off), qq = io<IO>::load(q + qk_off);
      const float a = expf(CHANNEL_GATE ? __ldg(g + (tok * H_v + h) * D_K + i) : gsc);
      const float aq = a * qq;
      bv.kr[tt][i] = DECAY_FIRST ? a * kk : kk;
      bv.aq[tt][i] = aq;
      bv.a[tt][i] = a;
      bv.e[tt][i] = DECAY_FIRST ? b * kk : b * a * kk;
      bv.bk[tt][i] = b * kk;
      kq = fmaf(kk, qq, kq);
      kaq = fmaf(kk, aq, kaq);
    }
#pragma unroll
    for (int j = 0; j < D_V / 32; ++j)
      bv.v[tt][lane + 32 * j] = io<IO>::load(v + (tok * H_v + h) * D_V + lane + 32 * j);
    kq = warp_sum(kq);
    kaq = DECAY_FIRST ? 0.f : warp_sum(kaq);
    if (lane == 0) {
      bv.coef[tt][0] = b * (DECAY_FIRST ? kq : kaq);
      bv.coef[tt][1] = b * kq;
    }
  };
  // One warp asks L2 for token t's input rows (128-byte lines).
  auto prefetch_token = [&](int t) {
    const size_t tok = token_base(t);
    auto rows = [&](const void *p, int bytes) {
      for (int off = lane * 128; off < bytes; off += 32 * 128)
        prefetch_l2(static_cast<const char *>(p) + off);
    };
    rows(k + (tok * H_qk + hk) * D_K, D_K * (int)sizeof(IO));
    rows(q + (tok * H_qk + hk) * D_K, D_K * (int)sizeof(IO));
    rows(v + (tok * H_v + h) * D_V, D_V * (int)sizeof(IO));
    if (CHANNEL_GATE) rows(g + (tok * H_v + h) * D_K, D_K * 4);
  };

  const int ocol = warp * CW + (lane % CW), opart = lane / CW;
  for (int t0 = 0; t0 < T; t0 += TB) {
    const int nt = (T - t0) < TB ? (T - t0) : TB;
    if (!SINGLE) __syncthreads();  // the previous block's vectors are no longer read
    if (warp < nt) stage(warp, t0 + warp);
    if (!SINGLE && t0 + TB + warp < T) prefetch_token(t0 + TB + warp);
    __syncthreads();

    for (int tt = 0; tt < nt; ++tt) {
      const int par = (t0 + tt) & 1;
      // 2. partial column sums over this warp's rows: r = S^T kr, p = S^T (a.q)
      float rp[CPL], pp[CPL];
#pragma unroll
      for (int c = 0; c < CPL; ++c) rp[c] = pp[c] = 0.f;
#pragma unroll
      for (int r = 0; r < RPW; ++r) {
        const float ki = bv.kr[tt][warp * RPW + r], aqi = bv.aq[tt][warp * RPW + r];
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          rp[c] = fmaf(ki, x[r][c], rp[c]);
          pp[c] = fmaf(aqi, x[r][c], pp[c]);
        }
      }
      vec<CPL>::sts(&s_red[par][0][warp][lane * CPL], rp);
      vec<CPL>::sts(&s_red[par][1][warp][lane * CPL], pp);
      __syncthreads();

      float rf[CPL], vv[CPL];
#pragma unroll
      for (int c = 0; c < CPL; ++c) rf[c] = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        float part[CPL];
        vec<CPL>::lds(&s_red[par][0][w][lane * CPL], part);
#pragma unroll
        for (int c = 0; c < CPL; ++c) rf[c] += part[c];
      }
      vec<CPL>::lds(&bv.v[tt][lane * CPL], vv);

      // 3. S' = a . S - e r^T + beta k v^T (e folds the order), in registers
#pragma unroll
      for (int r = 0; r < RPW; ++r) {
        const int i = warp * RPW + r;
        const float a = bv.a[tt][i], e = bv.e[tt][i], bk = bv.bk[tt][i];
#pragma unroll
        for (int c = 0; c < CPL; ++c) x[r][c] = fmaf(a, x[r][c], fmaf(-e, rf[c], bk * vv[c]));
        if (SINGLE) vec<CPL>::st(S + i * D_V + lane * CPL, x[r]);
      }

      // 4. o = p - c_r r + c_v v, every warp a slice of the columns
      float ps = 0.f, rs = 0.f;
#pragma unroll
      for (int w = 0; w < WPP; ++w) {
        ps += s_red[par][1][opart * WPP + w][ocol];
        rs += s_red[par][0][opart * WPP + w][ocol];
      }
#pragma unroll
      for (int off = CW; off < 32; off <<= 1) {
        ps += __shfl_xor_sync(0xffffffffu, ps, off);
        rs += __shfl_xor_sync(0xffffffffu, rs, off);
      }
      if (opart == 0 && GDR_IN_BOUNDS((int64_t)token_base(t0 + tt) < tokens))
        io<IO>::store(o + (token_base(t0 + tt) * H_v + h) * D_V + ocol,
                      ps - bv.coef[tt][0] * rs + bv.coef[tt][1] * bv.v[tt][ocol]);
    }
  }

  // 5. the state goes back once, in place
  if (!SINGLE) {
#pragma unroll
    for (int r = 0; r < RPW; ++r) vec<CPL>::st(S + (warp * RPW + r) * D_V + lane * CPL, x[r]);
  }
}

template <int D_K, int D_V, typename IO>
cudaError_t launch_dv(const DecodeArgs &a, cudaStream_t s) {
  const unsigned grid = (unsigned)((int64_t)a.N * a.H_v);
  const dim3 block(kWarps * 32);
#define GDR_RECURRENT_ARGS                                                                  \
  (const IO *)a.q, (const IO *)a.k, (const IO *)a.v, a.g, a.beta, (IO *)a.o, a.state, a.slots, \
      a.num_slots, a.T, a.H_qk, a.H_v
  if (a.T == 1) {
    if (!a.channel_gate)
      recurrent_kernel<D_K, D_V, IO, false, false, true><<<grid, block, 0, s>>>(GDR_RECURRENT_ARGS);
    else if (a.decay_first)
      recurrent_kernel<D_K, D_V, IO, true, true, true><<<grid, block, 0, s>>>(GDR_RECURRENT_ARGS);
    else
      recurrent_kernel<D_K, D_V, IO, true, false, true><<<grid, block, 0, s>>>(GDR_RECURRENT_ARGS);
  } else {
    if (!a.channel_gate)
      recurrent_kernel<D_K, D_V, IO, false, false, false><<<grid, block, 0, s>>>(GDR_RECURRENT_ARGS);
    else if (a.decay_first)
      recurrent_kernel<D_K, D_V, IO, true, true, false><<<grid, block, 0, s>>>(GDR_RECURRENT_ARGS);
    else
      recurrent_kernel<D_K, D_V, IO, true, false, false><<<grid, block, 0, s>>>(GDR_RECURRENT_ARGS);
  }
#undef GDR_RECURRENT_ARGS
  return cudaGetLastError();
}

template <typename IO>
cudaError_t launch_io(const DecodeArgs &a, cudaStream_t s) {
  if (a.d_k == 128 && a.d_v == 128) return launch_dv<128, 128, IO>(a, s);
  if (a.d_k == 128 && a.d_v == 64) return launch_dv<128, 64, IO>(a, s);
  if (a.d_k == 64 && a.d_v == 128) return launch_dv<64, 128, IO>(a, s);
  return launch_dv<64, 64, IO>(a, s);
}

// dst[dst slot of n] = src[src slot of n] (zeros where the source slot is
// negative; nothing where the destination slot is negative), one float4 per
// thread-iteration.  A NULL slot array is the identity.
__global__ void state_copy_kernel(const float4 *__restrict__ src, const int32_t *__restrict__ src_slots,
                                  int64_t src_limit, float4 *__restrict__ dst,
                                  const int32_t *__restrict__ dst_slots, int64_t dst_limit, int N,
                                  int64_t per_seq4) {
  const int64_t total = (int64_t)N * per_seq4;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int n = (int)(idx / per_seq4);
    const int64_t e = idx - (int64_t)n * per_seq4;
    const int64_t ds = dst_slots ? (int64_t)__ldg(dst_slots + n) : n;
    if (ds < 0 || ds >= dst_limit) continue;
    const int64_t ss = src_slots ? (int64_t)__ldg(src_slots + n) : n;
    const float4 val = (src && ss >= 0 && ss < src_limit) ? __ldcs(src + ss * per_seq4 + e) : make_float4(0.f, 0.f, 0.f, 0.f);
    __stcs(dst + ds * per_seq4 + e, val);
  }
}

}  // namespace

GDR_DEFINE_OOB_COUNTER(oob_count_decode)

cudaError_t launch_recurrent(const DecodeArgs &a, cudaStream_t stream) {
  if (a.N == 0) return cudaSuccess;
  TraceScope tr("recurrent_kernel", stream);
  if (a.bf16) return launch_io<__nv_bfloat16>(a, stream);
  return launch_io<float>(a, stream);
}

cudaError_t launch_state_copy(const float *src, const int32_t *src_slots, int64_t src_limit,
                              float *dst, const int32_t *dst_slots, int64_t dst_limit, int N,
                              int64_t per_seq_floats, cudaStream_t stream) {
  if (N == 0 || per_seq_floats == 0) return cudaSuccess;
  const int64_t per_seq4 = per_seq_floats / 4;
  const int64_t total = (int64_t)N * per_seq4;
  const int threads = 256;
  int64_t blocks = (total + threads - 1) / threads;
  const int64_t cap = (int64_t)sm_count() * 8;
  if (blocks > cap) blocks = cap;
  TraceScope tr("state_copy_kernel", stream);
  state_copy_kernel<<<(unsigned)blocks, threads, 0, stream>>>(
      reinterpret_cast<const float4 *>(src), src_slots, src_limit,
      reinterpret_cast<float4 *>(dst), dst_slots, dst_limit, N, per_seq4);
  return cudaGetLastError();
}

}  // namespace gdr
