// Chunked prefill of the gated delta rule in fp32 on the CUDA cores.
//
// This is the all-fp32 path (io dtype fp32) and the path for head sizes the
// tensor-core kernel does not cover.  It computes the same chunkwise form as
// the tensor-core kernel, in fp32 throughout:
//
// Within a chunk of L tokens with in-chunk cumulative log-decay G_t (G_0 = 0)
// and Gp_t = G_{t-1}, the token recurrence (row "KDA" of the table
// "Everything, in one table", thethings.ai "The argument, in one page";
// erase, then decay, then the undecayed write) is equivalent to
//
//   recalls   R = T^{-1} [ (K.e^{Gp}) S_0 + tril_{-1}(A_w) diag(beta) V ]
//             T = I + tril_{-1}(A_e) diag(beta)
//   outputs   o = (Q.e^{G}) S_0 + tril(B_w) diag(beta) V - tril(B_e) diag(beta) R
//   state     S_L = e^{G_L} . S_0 + (K.e^{G_L - G})^T beta V - (K.e^{G_L - Gp})^T beta R
//
// with the in-chunk Gram matrices (per-channel factors inside the sums)
//   A_w[i][j] = sum_c k_ic k_jc e^{Gp_ic - G_jc}      A_e: e^{Gp_ic - Gp_jc}
//   B_w[i][j] = sum_c q_ic k_jc e^{G_ic - G_jc}       B_e: e^{G_ic - Gp_jc}
// (row "Chunkwise / WY": one C x C triangular solve per chunk, the result
// unchanged).  Every pair factor here is formed directly as one exp of a
// difference that is <= 0, so no factor exceeds 1 and no range limit applies
// to g.
//
// With the decay applied before the erase (DECAY_FIRST, the variant order
// (I - beta k k^T) Diag(a) S), recall reads the state along a_t . k_t, so the
// erase direction equals the write direction: every Gp above becomes G, and
// the rest of the computation is unchanged.
//
// Mapping: one CTA per (sequence, v-head, slice of NS state columns); the
// CTA walks its sequence's chunks in order with the state slice in shared
// memory.  The d_v columns of the state evolve independently (the update
// multiplies S from the left), so slices need no communication.
#include "common.cuh"
#include "internal.h"

namespace gdr {
namespace {

constexpr int C = kChunk;
constexpr int NS = 32;        // state columns per CTA
constexpr int kThreads = 256;

template <int D_K>
struct SimtSmem {
  static constexpr int LD = D_K + 1;  // padded row stride of token x channel tiles
  float K[C][LD];
  float Q[C][LD];
  float G[C][LD];      // in-chunk cumulative log-decay G_t (t = 1..L -> rows 0..L-1)
  float Aw[C][C + 1];
  float Ae[C][C + 1];  // later overwritten by T^{-1}
  float Bw[C][C + 1];
  float Be[C][C + 1];
  float S[D_K][NS];
  float V[C][NS];
  float R[C][NS];
  float Rhs[C][NS];
  float beta[C];
};

template <int D_K, int D_V, typename IO, bool CHANNEL_GATE, bool DECAY_FIRST>
__global__ void __launch_bounds__(kThreads, 1)
prefill_simt_kernel(const IO *__restrict__ q, const IO *__restrict__ k, const IO *__restrict__ v,
                    const float *__restrict__ g, const float *__restrict__ beta,
                    IO *__restrict__ o, const float *s0, float *sT,
                    const int32_t *__restrict__ state_slots, int64_t num_slots,
                    const int32_t *__restrict__ cu,
                    int T, int H_qk, int H_v, const int32_t *__restrict__ status) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  using Sm = SimtSmem<D_K>;
  Sm &sm = *reinterpret_cast<Sm *>(smem_raw);

  if (status && *status != KDA_DEVICE_OK) return;

  constexpr int NSLICE = D_V / NS;
  const int slice = blockIdx.x % NSLICE;
  const int h = (blockIdx.x / NSLICE) % H_v;
  const int n = blockIdx.x / (NSLICE * H_v);
  const int hk = h / (H_v / H_qk);
  const int tid = threadIdx.x;
  const int col0 = slice * NS;

  // token rows of the whole batch (the bounds-checked build compares against it)
  const int nseqs = (int)(gridDim.x / (NSLICE * H_v));
  const int64_t T_total = cu ? (int64_t)cu[nseqs] : (int64_t)nseqs * T;
  (void)T_total;
  int64_t bos, eos;
  if (cu) {
    bos = cu[n];
    eos = cu[n + 1];
  } else {
    bos = (int64_t)n * T;
    eos = bos + T;
  }

  // initial state slice (a negative pool slot: zeros in, nothing out)
  const int64_t slot = state_slots ? (int64_t)state_slots[n] : (int64_t)n;
  if (slot < 0 || slot >= num_slots) {
    s0 = nullptr;
    sT = nullptr;
  }
  const size_t state_off = ((size_t)slot * H_v + h) * D_K * D_V;
  for (int e = tid; e < D_K * NS; e += kThreads) {
    const int i = e / NS, j = e % NS;
    sm.S[i][j] = s0 ? s0[state_off + (size_t)i * D_V + col0 + j] : 0.f;
  }

  for (int64_t c0 = bos; c0 < eos; c0 += C) {
    const int L = (int)((eos - c0) < C ? (eos - c0) : C);
    __syncthreads();  // previous chunk done with every tile

    // 1. load the chunk (rows >= L are zero: no key, no write, no decay)
    for (int e = tid; e < C * D_K; e += kThreads) {
      const int t = e / D_K, c = e % D_K;
      float kk = 0.f, qq = 0.f, gg = 0.f;
      if (t < L && GDR_IN_BOUNDS(c0 + t < T_total)) {
        const size_t off = ((size_t)(c0 + t) * H_qk + hk) * D_K + c;
        kk = io<IO>::load(k + off);
        qq = io<IO>::load(q + off);
        gg = CHANNEL_GATE ? __ldg(g + ((size_t)(c0 + t) * H_v + h) * D_K + c)
                          : __ldg(g + (size_t)(c0 + t) * H_v + h);
      }
      sm.K[t][c] = kk;
      sm.Q[t][c] = qq;
      sm.G[t][c] = gg;
    }
    for (int e = tid; e < C * NS; e += kThreads) {
      const int t = e / NS, j = e % NS;
      sm.V[t][j] = (t < L && GDR_IN_BOUNDS(c0 + t < T_total))
                       ? io<IO>::load(v + ((size_t)(c0 + t) * H_v + h) * D_V + col0 + j) : 0.f;
    }
    if (tid < C)
      sm.beta[tid] = (tid < L && GDR_IN_BOUNDS(c0 + tid < T_total))
                         ? __ldg(beta + (size_t)(c0 + tid) * H_v + h) : 0.f;
    __syncthreads();

    // 2. in-chunk cumulative sum of the log-decay, in token order
    if (tid < D_K) {
      float acc = 0.f;
      for (int t = 0; t < C; ++t) {
        acc += sm.G[t][tid];
        sm.G[t][tid] = acc;
      }
    }
    __syncthreads();

    // 3. Gram matrices with directly formed pair factors
    for (int e = tid; e < C * C; e += kThreads) {
      const int i = e / C, j = e % C;
      float aw = 0.f, ae = 0.f, bw = 0.f, be = 0.f;
      if (j <= i) {
        for (int c = 0; c < D_K; ++c) {
          const float Gi = sm.G[i][c], Gpi = DECAY_FIRST ? Gi : (i > 0) ? sm.G[i - 1][c] : 0.f;
          const float Gj = sm.G[j][c], Gpj = DECAY_FIRST ? Gj : (j > 0) ? sm.G[j - 1][c] : 0.f;
          const float kj = sm.K[j][c];
          const float qk = sm.Q[i][c] * kj;
          bw = fmaf(qk, expf(Gi - Gj), bw);
          be = fmaf(qk, expf(Gi - Gpj), be);
          if (j < i) {
            const float kk = sm.K[i][c] * kj;
            aw = fmaf(kk, expf(Gpi - Gj), aw);
            ae = fmaf(kk, expf(Gpi - Gpj), ae);
          }
        }
      }
      sm.Aw[i][j] = aw;
      sm.Ae[i][j] = ae;
      sm.Bw[i][j] = bw;
      sm.Be[i][j] = be;
    }
    __syncthreads();

    // 4. T^{-1} for T = I + tril_{-1}(A_e) diag(beta), by forward substitution,
    //    one column per thread:  X[i][col] = delta_{i,col} - sum_{col<=j<i} A_e[i][j] beta_j X[j][col]
    {
      float X[C];
      if (tid < C) {
        const int col = tid;
        for (int i = 0; i < C; ++i) {
          float acc = (i == col) ? 1.f : 0.f;
          if (i > col)
            for (int j = col; j < i; ++j) acc = fmaf(-sm.Ae[i][j] * sm.beta[j], X[j], acc);
          X[i] = (i >= col) ? acc : 0.f;
        }
      }
      __syncthreads();  // every column has read A_e
      if (tid < C)
        for (int i = 0; i < C; ++i) sm.Ae[i][tid] = X[i];
    }
    __syncthreads();

    // 5. rhs = (K.e^{Gp}) S_0 + tril_{-1}(A_w) beta V, then R = T^{-1} rhs
    for (int e = tid; e < C * NS; e += kThreads) {
      const int i = e / NS, j = e % NS;
      float acc = 0.f;
      for (int c = 0; c < D_K; ++c) {
        const float Gpi = DECAY_FIRST ? sm.G[i][c] : (i > 0) ? sm.G[i - 1][c] : 0.f;
        acc = fmaf(sm.K[i][c] * expf(Gpi), sm.S[c][j], acc);
      }
      for (int jj = 0; jj < i; ++jj) acc = fmaf(sm.Aw[i][jj] * sm.beta[jj], sm.V[jj][j], acc);
      sm.Rhs[i][j] = acc;
    }
    __syncthreads();
    for (int e = tid; e < C * NS; e += kThreads) {
      const int i = e / NS, j = e % NS;
      float acc = 0.f;
      for (int jj = 0; jj <= i; ++jj) acc = fmaf(sm.Ae[i][jj], sm.Rhs[jj][j], acc);
      sm.R[i][j] = acc;
    }
    __syncthreads();

    // 6. outputs o = (Q.e^{G}) S_0 + tril(B_w) beta V - tril(B_e) beta R
    for (int e = tid; e < C * NS; e += kThreads) {
      const int i = e / NS, j = e % NS;
      if (i >= L || !GDR_IN_BOUNDS(c0 + i < T_total)) continue;
      float acc = 0.f;
      for (int c = 0; c < D_K; ++c) acc = fmaf(sm.Q[i][c] * expf(sm.G[i][c]), sm.S[c][j], acc);
      for (int jj = 0; jj <= i; ++jj)
        acc = fmaf(sm.beta[jj], fmaf(sm.Bw[i][jj], sm.V[jj][j], -sm.Be[i][jj] * sm.R[jj][j]), acc);
      io<IO>::store(o + ((size_t)(c0 + i) * H_v + h) * D_V + col0 + j, acc);
    }
    __syncthreads();

    // 7. state S <- e^{G_L} . S + (K.e^{G_L - G})^T beta V - (K.e^{G_L - Gp})^T beta R
    for (int e = tid; e < D_K * NS; e += kThreads) {
      const int c = e / NS, j = e % NS;
      const float GL = sm.G[C - 1][c];  // rows >= L carry g = 0, so this is G_L
      float acc = expf(GL) * sm.S[c][j];
      for (int t = 0; t < L; ++t) {
        const float Gt = sm.G[t][c], Gpt = DECAY_FIRST ? Gt : (t > 0) ? sm.G[t - 1][c] : 0.f;
        const float bk = sm.beta[t] * sm.K[t][c];
        acc = fmaf(bk * expf(GL - Gt), sm.V[t][j], acc);
        acc = fmaf(-bk * expf(GL - Gpt), sm.R[t][j], acc);
      }
      sm.S[c][j] = acc;  // each (c, j) is read and written by one thread only
    }
  }
  __syncthreads();
  if (sT) {
    for (int e = tid; e < D_K * NS; e += kThreads) {
      const int i = e / NS, j = e % NS;
      sT[state_off + (size_t)i * D_V + col0 + j] = sm.S[i][j];
    }
  }
}

template <int D_K, int D_V, typename IO, bool CG>
cudaError_t launch_cfg(const PrefillArgs &a, cudaStream_t s) {
  auto kern = (CG && a.decay_first) ? prefill_simt_kernel<D_K, D_V, IO, CG, true>
                                    : prefill_simt_kernel<D_K, D_V, IO, CG, false>;
  const int smem = (int)sizeof(SimtSmem<D_K>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)((int64_t)a.num_seqs * a.H_v * (D_V / NS));
  if (grid == 0) return cudaSuccess;
  TraceScope tr("prefill_simt_kernel", s);
  kern<<<grid, kThreads, smem, s>>>((const IO *)a.q, (const IO *)a.k, (const IO *)a.v, a.g,
                                   a.beta, (IO *)a.o, a.initial_state, a.final_state,
                                   a.state_slots, a.num_slots, a.cu_seqlens, a.T, a.H_qk, a.H_v,
                                   (const int32_t *)a.workspace);
  return cudaGetLastError();
}

template <typename IO, bool CG>
cudaError_t launch_io(const PrefillArgs &a, cudaStream_t s) {
  if (a.d_k == 128 && a.d_v == 128) return launch_cfg<128, 128, IO, CG>(a, s);
  if (a.d_k == 128 && a.d_v == 64) return launch_cfg<128, 64, IO, CG>(a, s);
  if (a.d_k == 64 && a.d_v == 128) return launch_cfg<64, 128, IO, CG>(a, s);
  return launch_cfg<64, 64, IO, CG>(a, s);
}

}  // namespace

GDR_DEFINE_OOB_COUNTER(oob_count_prefill_simt)

cudaError_t launch_prefill_f32(const PrefillArgs &a, cudaStream_t stream) {
  if (a.bf16) {
    return a.channel_gate ? launch_io<__nv_bfloat16, true>(a, stream)
                          : launch_io<__nv_bfloat16, false>(a, stream);
  }
  return a.channel_gate ? launch_io<float, true>(a, stream) : launch_io<float, false>(a, stream);
}

}  // namespace gdr
