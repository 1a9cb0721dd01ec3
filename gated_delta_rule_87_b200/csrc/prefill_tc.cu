// Chunked prefill on the sm_100a tensor cores (tcgen05, TMEM, TMA), bf16
// q/k/v with d_k = d_v = 128, fp32 gate/beta/state, chunks of C = 64 tokens.
//
// The chunkwise form (row "Chunkwise / WY" of the table "Everything, in one
// table", thethings.ai "The argument, in one page": one C x C triangular
// solve per chunk, result unchanged) of the recurrence in row "KDA"
// (S <- Diag(a)(I - beta k k^T) S + beta k v^T, erase then decay, o = S^T q)
// is written per chunk as an affine map of the incoming state S_0:
//
//     o   = Q' S_0 + O_intra                 (C x d_v)
//     S_L = P  S_0 + Qc                      (d_k x d_v)
//
// with, for in-chunk cumulative log-decay G_t (G_0 = 0), Gp_t = G_{t-1},
//     T     = I + tril_{-1}(A_e) diag(beta)
//     W     = T^{-1} (K . e^{Gp})            U = T^{-1} tril_{-1}(A_w) diag(beta) V
//     Q'    = Q . e^{G} - tril(B_e) diag(beta) W
//     O_intra = tril(B_w) diag(beta) V - tril(B_e) diag(beta) U
//     P     = Diag(e^{G_L}) - (K . e^{G_L - Gp})^T diag(beta) W
//     Qc    = (K . e^{G_L - G})^T diag(beta) V - (K . e^{G_L - Gp})^T diag(beta) U
// and Gram matrices A_w[i][j] = sum_c k_ic k_jc e^{Gp_ic - G_jc},
// A_e: e^{Gp_ic - Gp_jc}, B_w = q.k e^{G_ic - G_jc}, B_e: e^{G_ic - Gp_jc}.
// P is the product of the chunk's transition matrices in WY form.
//
// Per-channel decay factors inside the Gram sums ("numerical range -- needs
// sub-chunking", row "KDA") are split at the end E_J of the key's 16-token
// sub-chunk J:  e^{x_i - G_j} = e^{x_i - E_J} * e^{E_J - G_j}.  The key-side
// factor is <= 1; the query/key-row factor is <= 1 for rows in later
// sub-chunks and at most e^{16 |g|max} inside the diagonal sub-chunk, which
// stays in fp32/bf16 range for per-token log-decays g >= -5.
//
// Two kernels (plus a one-CTA planning kernel):
//   prep  -- one CTA per (chunk, v-head), all chunks in parallel: loads
//            q/k/v/g tiles with TMA, builds every S-independent factor above
//            with tcgen05 MMAs (bf16 operands, fp32 accumulators in TMEM) and
//            a blocked fp32 triangular inverse, and writes P, Q', Qc,
//            O_intra (bf16) into a workspace slot laid out as the scan's
//            shared-memory operand images.
//   scan  -- one CTA per (sequence, v-head, 32-column slice of the state),
//            walks the chunks in order with the fp32 state slice in
//            registers: one MMA P S (128x32x128) and one Q' S (64x32x128)
//            per chunk, then S <- P S + Qc and o = Q' S + O_intra.  The
//            state columns evolve independently, so slices never talk.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace gdr {
namespace {
using namespace tc;

constexpr int C = kChunk;  // 64 tokens
constexpr int DK = 128;
constexpr int NS = 32;  // scan: state columns per CTA
constexpr int NSL = DK / NS;

// ---- workspace: header, per-sequence chunk offsets, chunk table, slots ----
struct ChunkEntry {
  int32_t seq, start, len, pad;
};
constexpr size_t kHeaderBytes = 256;  // [0] status word, [1] number of chunks
constexpr uint32_t SLOT_P = 0;        // 32 KB  P, K-major A image [i][c]
constexpr uint32_t SLOT_QP = 32768;   // 16 KB  Q', MN-major A image [c][t]
constexpr uint32_t SLOT_QC = 49152;   // 32 KB  Qc, bf16 [slice][i][n mod 32]
constexpr uint32_t SLOT_OI = 81920;   // 16 KB  O_intra, bf16 [slice][t][n mod 32]
constexpr uint32_t SLOT_BYTES = 98304;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct WsLayout {
  size_t seq_off, tab, slots, total;
};
WsLayout ws_layout(int64_t T_total, int num_seqs) {
  WsLayout L;
  const int64_t max_chunks = T_total / C + num_seqs;
  L.seq_off = kHeaderBytes;
  L.tab = align_up(L.seq_off + sizeof(int32_t) * ((size_t)num_seqs + 1), 256);
  L.slots = align_up(L.tab + sizeof(ChunkEntry) * (size_t)max_chunks, 1024);
  L.total = L.slots;  // + slots, added by the caller (depends on H_v)
  return L;
}

// ---------------------------------------------------------------------------
// planning: chunk table and per-sequence chunk offsets (also validates
// cu_seqlens)
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(1024, 1)
plan_kernel(const int32_t *__restrict__ cu, int num_seqs, int T, int T_total, int32_t *hdr,
            int32_t *seq_off, ChunkEntry *tab) {
  __shared__ int32_t warp_tot[32];
  __shared__ int32_t s_running;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  bool bad = false;
  if (cu) {
    for (int i = tid; i <= num_seqs; i += blockDim.x) {
      const int32_t x = cu[i];
      if (i == 0 && x != 0) bad = true;
      if (i == num_seqs && x != T_total) bad = true;
      if (i < num_seqs && cu[i + 1] < x) bad = true;
    }
  }
  if (__syncthreads_or(bad)) {
    for (int i = tid; i <= num_seqs; i += blockDim.x) seq_off[i] = 0;
    if (tid == 0) {
      hdr[0] = KDA_DEVICE_BAD_CU_SEQLENS;
      hdr[1] = 0;
    }
    return;
  }
  if (tid == 0) s_running = 0;
  __syncthreads();
  for (int base = 0; base < num_seqs; base += blockDim.x) {
    const int n = base + tid;
    int bos = 0, len = 0;
    if (n < num_seqs) {
      bos = cu ? cu[n] : n * T;
      len = cu ? cu[n + 1] - bos : T;
    }
    const int cnt = (len + C - 1) / C;
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int t = (lane < (int)(blockDim.x >> 5)) ? warp_tot[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, t, o);
        if (lane >= o) t += y;
      }
      warp_tot[lane] = t;  // inclusive over warps
    }
    __syncthreads();
    const int running = s_running;
    const int excl = incl - cnt + (warp > 0 ? warp_tot[warp - 1] : 0);
    if (n < num_seqs) {
      const int first = running + excl;
      seq_off[n] = first;
      for (int j = 0; j < cnt; ++j) {
        ChunkEntry e;
        e.seq = n;
        e.start = bos + j * C;
        e.len = min(C, len - j * C);
        e.pad = 0;
        tab[first + j] = e;
      }
    }
    __syncthreads();
    if (tid == 0) s_running = running + warp_tot[(blockDim.x >> 5) - 1];
    __syncthreads();
  }
  if (tid == 0) {
    seq_off[num_seqs] = s_running;
    hdr[1] = s_running;
  }
}

// ---------------------------------------------------------------------------
// prep kernel
// ---------------------------------------------------------------------------
constexpr int kPrepThreads = 256;

// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t OFF_Q = 0;         // q tile, two K-major SW128 [64 t][64 c] blocks
constexpr uint32_t OFF_K = 16384;     // k tile
constexpr uint32_t OFF_V = 32768;     // v tile (MN-major operand, 64-wide blocks 8 KB apart)
constexpr uint32_t OFF_G = 49152;     // g / G fp32 [64][128]
constexpr uint32_t OFF_X = 81920;     // 112 KB phase-dependent region
constexpr uint32_t OFF_MISC = 196608;
constexpr uint32_t MISC_BETA = 0;      // f32[64]
constexpr uint32_t MISC_E = 256;       // f32[4][128] sub-chunk-end G
constexpr uint32_t MISC_GSC = 2304;    // f32[64] scalar gate
constexpr uint32_t MISC_BAR = 2560;    // 2 x u64
constexpr uint32_t MISC_TSLOT = 2576;  // u32
constexpr uint32_t PREP_SMEM = OFF_MISC + 3072 + 1024;

// X region, gram phase
constexpr uint32_t X_R = 0;           // 32 KB, K-major B [128 rows][128], blocks 16 KB apart
constexpr uint32_t X_LEFT = 32768;    // 80 KB, four overlapped K-major A tiles
constexpr uint32_t LEFT_BLOCK = 40960;
__device__ __forceinline__ uint32_t left_off(int J) {
  return J == 0 ? 0u : (J == 1 ? 12288u : (J == 2 ? 20480u : 24576u));
}
// X region, after the Gram MMAs
constexpr uint32_t X_AWBW = 0;        // 16 KB K-major B [128 i'][64 j]
constexpr uint32_t X_BE = 16384;      // 8 KB  K-major B [64 i][64 j]
constexpr uint32_t X_TINVB = 24576;   // 8 KB  K-major B [64 i][64 j]; scratch before
constexpr uint32_t X_NAE = 32768;     // 16 KB f32 [64][64]
constexpr uint32_t X_TINVF = 49152;   // 16 KB f32 [64][64]
constexpr uint32_t X_KP = 65536;      // 16 KB MN-major [t][c]
constexpr uint32_t X_KAB = 81920;     // 16 KB MN-major [t][i]
constexpr uint32_t X_KBB = 98304;     // 16 KB MN-major [t][i]
constexpr uint32_t X_W = 32768;       // after T2: K-major [c][t]
constexpr uint32_t X_Y = 49152;       // after T2: K-major [n][t]
constexpr uint32_t X_U = 65536;       // after T3: K-major [n][t]
constexpr uint32_t X_OST = 0;         // after T4: bf16 [64 t][128 n]

// TMEM columns
constexpr uint32_t TM_GRAM = 0, TM_P = 0, TM_W = 128, TM_QC = 128, TM_YB = 192, TM_OI = 256,
                   TM_U = 320, TM_X = 384;

__device__ __forceinline__ float ld_bf16(const unsigned char *base, uint32_t off) {
  return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(base + off));
}

// 8 consecutive bf16 of a K-major SW128 tile row (c multiple of 8)
__device__ __forceinline__ void ld8_kmajor(const unsigned char *tile, int r, int c, float (&x)[8]) {
  const uint4 u = *reinterpret_cast<const uint4 *>(tile + (c >> 6) * 8192 + kmajor_off(r, c & 63));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = bf16_lo(w[i]);
    x[2 * i + 1] = bf16_hi(w[i]);
  }
}

__device__ __forceinline__ uint4 pack8(const float (&x)[8]) {
  return make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                    pack_bf16x2(x[6], x[7]));
}

__device__ __forceinline__ void st16(unsigned char *p, uint4 v) { *reinterpret_cast<uint4 *>(p) = v; }

template <bool CHANNEL>
__global__ void __launch_bounds__(kPrepThreads, 1)
chunk_prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                  const float *__restrict__ g_scalar, const float *__restrict__ beta, int H_qk,
                  int H_v, int32_t *hdr, const ChunkEntry *__restrict__ tab,
                  unsigned char *__restrict__ slots) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char *sm = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  unsigned char *sQ = sm + OFF_Q, *sK = sm + OFF_K, *sV = sm + OFF_V;
  float *sG = reinterpret_cast<float *>(sm + OFF_G);
  unsigned char *sX = sm + OFF_X;
  float *sBeta = reinterpret_cast<float *>(sm + OFF_MISC + MISC_BETA);
  float *sE = reinterpret_cast<float *>(sm + OFF_MISC + MISC_E);
  float *sGsc = reinterpret_cast<float *>(sm + OFF_MISC + MISC_GSC);
  uint64_t *bar_tma = reinterpret_cast<uint64_t *>(sm + OFF_MISC + MISC_BAR);
  uint64_t *bar_mma = bar_tma + 1;
  uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + OFF_MISC + MISC_TSLOT);

  if (hdr[0] != KDA_DEVICE_OK) return;
  const int chunk = blockIdx.x;
  if (chunk >= hdr[1]) return;
  const int h = blockIdx.y;
  const int hk = h / (H_v / H_qk);
  const ChunkEntry ce = tab[chunk];
  const int L = ce.len, t0 = ce.start;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  unsigned char *slot = slots + ((size_t)chunk * H_v + h) * SLOT_BYTES;

  if (warp == 0) {
    tmem_alloc(tslot, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(bar_tma, 1);
    mbar_init(bar_mma, 1);
    mbar_fence_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *tslot;

  // ---- 1. TMA loads of the chunk's q, k, v (bf16, swizzled) and g (fp32) ----
  if (tid == 0) {
    mbar_arrive_expect_tx(bar_tma, 3 * 16384 + (CHANNEL ? 32768 : 0));
#pragma unroll
    for (int cb = 0; cb < 2; ++cb) {
      tma_load_3d(sQ + cb * 8192, &tm_q, cb * 64, hk, t0, bar_tma);
      tma_load_3d(sK + cb * 8192, &tm_k, cb * 64, hk, t0, bar_tma);
      tma_load_3d(sV + cb * 8192, &tm_v, cb * 64, h, t0, bar_tma);
    }
    if (CHANNEL) tma_load_3d(sG, &tm_g, 0, h, t0, bar_tma);
  }
  if (tid < C) {
    sBeta[tid] = (tid < L) ? __ldg(beta + (size_t)(t0 + tid) * H_v + h) : 0.f;
    if (!CHANNEL) sGsc[tid] = (tid < L) ? __ldg(g_scalar + (size_t)(t0 + tid) * H_v + h) : 0.f;
  }
  mbar_wait(bar_tma, 0, hdr, KDA_DEVICE_TIMEOUT);
  __syncthreads();

  // ---- 2. in-chunk cumulative log-decay, rows >= L carry no decay ----
  if (tid < DK) {
    const int c = tid;
    float acc = 0.f;
    for (int t = 0; t < C; ++t) {
      const float gv = (t < L) ? (CHANNEL ? sG[t * DK + c] : sGsc[t]) : 0.f;
      acc += gv;
      sG[t * DK + c] = acc;
      if ((t & 15) == 15) sE[(t >> 4) * DK + c] = acc;
    }
  }
  __syncthreads();

  // ---- 3. Gram operands: R (keys scaled to their sub-chunk end), Left^(J) ----
  // R row rho = 32J + s: s < 16 -> k_j e^{E_J - G_j}, s >= 16 -> k_j e^{E_J - Gp_j}, j = 16J + s%16
  for (int item = tid; item < 128 * 16; item += kPrepThreads) {
    const int rho = item >> 4, c = (item & 15) * 8;
    const int J = rho >> 5, s = rho & 31, j = 16 * J + (s & 15);
    float x[8];
    if (j < L) {
      ld8_kmajor(sK, j, c, x);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float gj = (s < 16) ? sG[j * DK + c + e] : (j > 0 ? sG[(j - 1) * DK + c + e] : 0.f);
        x[e] *= expf(sE[J * DK + c + e] - gj);
      }
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = 0.f;
    }
    st16(sX + X_R + (c >> 6) * 16384 + kmajor_off(rho, c & 63), pack8(x));
  }
  // Left^(J) row lambda = 32I + s (I >= J): s < 16 -> k_i e^{Gp_i - E_J} (i = 16I + s),
  //                                         s >= 16 -> q_i e^{G_i - E_J} (i = 16I + s - 16)
  for (int item = tid; item < 320 * 16; item += kPrepThreads) {
    int r = item >> 4;
    const int c = (item & 15) * 8;
    int J = 0;
    while (r >= 128 - 32 * J) {
      r -= 128 - 32 * J;
      ++J;
    }
    const int lambda = 32 * J + r;
    const int I = lambda >> 5, s = lambda & 31;
    const bool isK = s < 16;
    const int i = 16 * I + (s & 15);
    float x[8];
    if (i < L) {
      ld8_kmajor(isK ? sK : sQ, i, c, x);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float gi = isK ? (i > 0 ? sG[(i - 1) * DK + c + e] : 0.f) : sG[i * DK + c + e];
        x[e] *= expf(gi - sE[J * DK + c + e]);
      }
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = 0.f;
    }
    st16(sX + X_LEFT + left_off(J) + (c >> 6) * LEFT_BLOCK + kmajor_off(lambda, c & 63), pack8(x));
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // ---- 4. Gram MMAs: for each key sub-chunk J, [K;Q] rows x 32 key columns ----
  if (tid == 0) {
    constexpr uint32_t ID = idesc_bf16(128, 32, false, false);
    const uint32_t r_base = smem_u32(sX + X_R);
#pragma unroll
    for (int J = 0; J < 4; ++J) {
      const uint32_t a_base = smem_u32(sX + X_LEFT + left_off(J));
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16(tm + TM_GRAM + 32 * J, desc_kmajor(a_base, 16 * kk, LEFT_BLOCK),
                 desc_kmajor(r_base + 4096 * J, 16 * kk, 16384), ID, kk > 0);
    }
    mma_commit(bar_mma);
  }
  __syncwarp();
  mbar_wait(bar_mma, 0, hdr, KDA_DEVICE_TIMEOUT);
  tc_fence_after();

  const int quad = warp & 3, half = warp >> 2;
  const int lane_row = 32 * quad + lane;  // TMEM lane this thread reads

  // ---- 5. Gram readback: masked, beta-scaled, into the next operands ----
  {
    const int I = quad, s = lane;
    const bool isK = s < 16;
    const int i = 16 * I + (s & 15);
    float* nae = reinterpret_cast<float *>(sX + X_NAE);
#pragma unroll
    for (int part = 0; part < 2; ++part) {
      const int J = 2 * half + part;
      float v[32];
      tmem_ld32(taddr(tm, 32 * quad, TM_GRAM + 32 * J), v);
      tmem_ld_wait();
      float w[16], e[16];
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int j = 16 * J + u;
        const bool ok = (J <= I) && (i < L) && (j < L) && (isK ? (j < i) : (j <= i));
        w[u] = ok ? v[u] * sBeta[j] : 0.f;
        e[u] = ok ? v[16 + u] * sBeta[j] : 0.f;
      }
      const int row_w = isK ? i : 64 + i;
#pragma unroll
      for (int hseg = 0; hseg < 2; ++hseg) {
        float x[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) x[u] = w[8 * hseg + u];
        st16(sX + X_AWBW + kmajor_off(row_w, 16 * J + 8 * hseg), pack8(x));
      }
      if (isK) {
#pragma unroll
        for (int u = 0; u < 16; u += 4)
          *reinterpret_cast<float4 *>(nae + i * 64 + 16 * J + u) =
              make_float4(e[u], e[u + 1], e[u + 2], e[u + 3]);
      } else {
#pragma unroll
        for (int hseg = 0; hseg < 2; ++hseg) {
          float x[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) x[u] = e[8 * hseg + u];
          st16(sX + X_BE + kmajor_off(i, 16 * J + 8 * hseg), pack8(x));
        }
      }
    }
  }
  // K . e^{Gp}, beta K . e^{G_L - G}, beta K . e^{G_L - Gp}  (MN-major [t][c])
  for (int item = tid; item < 64 * 16; item += kPrepThreads) {
    const int t = item >> 4, c = (item & 15) * 8;
    float kp[8], ka[8], kb[8];
    if (t < L) {
      float kx[8];
      ld8_kmajor(sK, t, c, kx);
      const float b = sBeta[t];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float G = sG[t * DK + c + e];
        const float Gp = t > 0 ? sG[(t - 1) * DK + c + e] : 0.f;
        const float GL = sE[3 * DK + c + e];
        kp[e] = kx[e] * expf(Gp);
        ka[e] = b * kx[e] * expf(GL - G);
        kb[e] = b * kx[e] * expf(GL - Gp);
      }
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) kp[e] = ka[e] = kb[e] = 0.f;
    }
    const uint32_t off = mnmajor_off(t, c, 8192);
    st16(sX + X_KP + off, pack8(kp));
    st16(sX + X_KAB + off, pack8(ka));
    st16(sX + X_KBB + off, pack8(kb));
  }
  __syncthreads();

  // ---- 6. T^{-1}, T = I + N, N = tril_{-1}(A_e) diag(beta) (blocked, fp32) ----
  {
    const float *nae = reinterpret_cast<const float *>(sX + X_NAE);
    float *tinv = reinterpret_cast<float *>(sX + X_TINVF);
    float *tmp = reinterpret_cast<float *>(sX + X_TINVB);  // 16 x 64 f32 scratch
    if (tid < 64) {  // diagonal 16x16 blocks, one column per thread
      const int I = tid >> 4, cc = tid & 15;
      float x[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        float acc = (r == cc) ? 1.f : 0.f;
#pragma unroll
        for (int s2 = 0; s2 < r; ++s2)
          if (s2 >= cc) acc = fmaf(-nae[(16 * I + r) * 64 + 16 * I + s2], x[s2], acc);
        x[r] = (r >= cc) ? acc : 0.f;
      }
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        tinv[(16 * I + r) * 64 + 16 * I + cc] = x[r];
#pragma unroll
        for (int J = 0; J < 4; ++J)
          if (J > I) tinv[(16 * I + r) * 64 + 16 * J + cc] = 0.f;
      }
    }
    __syncthreads();
    const int r = tid >> 4, cc = tid & 15;
    for (int I = 1; I < 4; ++I) {
      for (int J = 0; J < I; ++J) {
        float acc = 0.f;
        for (int K2 = J; K2 < I; ++K2)
#pragma unroll
          for (int s2 = 0; s2 < 16; ++s2)
            acc = fmaf(nae[(16 * I + r) * 64 + 16 * K2 + s2], tinv[(16 * K2 + s2) * 64 + 16 * J + cc], acc);
        tmp[r * 64 + 16 * J + cc] = acc;
      }
      __syncthreads();
      for (int J = 0; J < I; ++J) {
        float acc = 0.f;
#pragma unroll
        for (int s2 = 0; s2 < 16; ++s2)
          acc = fmaf(tinv[(16 * I + r) * 64 + 16 * I + s2], tmp[s2 * 64 + 16 * J + cc], acc);
        tinv[(16 * I + r) * 64 + 16 * J + cc] = -acc;
      }
      __syncthreads();
    }
    // bf16 copy, K-major [i][j]
    for (int item = tid; item < 64 * 8; item += kPrepThreads) {
      const int i = item >> 3, j = (item & 7) * 8;
      float x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) x[u] = tinv[i * 64 + j + u];
      st16(sX + X_TINVB + kmajor_off(i, j), pack8(x));
    }
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // ---- 7. W^T = (K e^{Gp})^T T^{-T};  [Y^T | (B_w beta V)^T] = V^T [(A_w beta)^T | (B_w beta)^T] ----
  if (tid == 0) {
    const uint32_t tinvb = smem_u32(sX + X_TINVB);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_bf16(tm + TM_W, desc_mnmajor(smem_u32(sX + X_KP), 16 * kk, 8192),
               desc_kmajor(tinvb, 16 * kk, 0), idesc_bf16(128, 64, true, false), kk > 0);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_bf16(tm + TM_YB, desc_mnmajor(smem_u32(sV), 16 * kk, 8192),
               desc_kmajor(smem_u32(sX + X_AWBW), 16 * kk, 0), idesc_bf16(128, 128, true, false),
               kk > 0);
    mma_commit(bar_mma);
  }
  __syncwarp();
  mbar_wait(bar_mma, 1, hdr, KDA_DEVICE_TIMEOUT);
  tc_fence_after();

  // readback W (lanes c, cols i) -> K-major [c][t]; Y (lanes n, cols i) -> K-major [n][t]
  {
    float v[32];
    tmem_ld32(taddr(tm, 32 * quad, TM_W + 32 * half), v);
    tmem_ld_wait();
#pragma unroll
    for (int seg = 0; seg < 4; ++seg) {
      float x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) x[u] = v[8 * seg + u];
      st16(sX + X_W + kmajor_off(lane_row, 32 * half + 8 * seg), pack8(x));
    }
    tmem_ld32(taddr(tm, 32 * quad, TM_YB + 32 * half), v);
    tmem_ld_wait();
#pragma unroll
    for (int seg = 0; seg < 4; ++seg) {
      float x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) x[u] = v[8 * seg + u];
      st16(sX + X_Y + kmajor_off(lane_row, 32 * half + 8 * seg), pack8(x));
    }
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // ---- 8. U^T = Y^T T^{-T};  K_b^T beta W (for P);  X = W^T (B_e beta)^T (for Q') ----
  if (tid == 0) {
    const uint32_t tinvb = smem_u32(sX + X_TINVB), wsm = smem_u32(sX + X_W);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_bf16(tm + TM_U, desc_kmajor(smem_u32(sX + X_Y), 16 * kk, 0), desc_kmajor(tinvb, 16 * kk, 0),
               idesc_bf16(128, 64, false, false), kk > 0);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_bf16(tm + TM_P, desc_mnmajor(smem_u32(sX + X_KBB), 16 * kk, 8192), desc_kmajor(wsm, 16 * kk, 0),
               idesc_bf16(128, 128, true, false), kk > 0);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_bf16(tm + TM_X, desc_kmajor(wsm, 16 * kk, 0), desc_kmajor(smem_u32(sX + X_BE), 16 * kk, 0),
               idesc_bf16(128, 64, false, false), kk > 0);
    mma_commit(bar_mma);
  }
  __syncwarp();
  mbar_wait(bar_mma, 0, hdr, KDA_DEVICE_TIMEOUT);
  tc_fence_after();

  {
    float v[32];
    // U (lanes n, cols t) -> K-major [n][t]
    tmem_ld32(taddr(tm, 32 * quad, TM_U + 32 * half), v);
    tmem_ld_wait();
#pragma unroll
    for (int seg = 0; seg < 4; ++seg) {
      float x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) x[u] = v[8 * seg + u];
      st16(sX + X_U + kmajor_off(lane_row, 32 * half + 8 * seg), pack8(x));
    }
    // P = Diag(e^{G_L}) - K_b^T beta W (lanes i, cols c) -> slot, K-major A image
    const int i = lane_row;
    const float gl = expf(sE[3 * DK + i]);
#pragma unroll
    for (int part = 0; part < 2; ++part) {
      const int c0 = 64 * half + 32 * part;
      tmem_ld32(taddr(tm, 32 * quad, TM_P + c0), v);
      tmem_ld_wait();
#pragma unroll
      for (int seg = 0; seg < 4; ++seg) {
        float x[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int c = c0 + 8 * seg + u;
          x[u] = (c == i ? gl : 0.f) - v[8 * seg + u];
        }
        const int c = c0 + 8 * seg;
        st16(slot + SLOT_P + (c >> 6) * 16384 + kmajor_off(i, c & 63), pack8(x));
      }
    }
    // Q'[t][c] = q_tc e^{G_tc} - X[c][t] (lanes c, cols t) -> slot, MN-major A image [c][t]
    const int c = lane_row;
    tmem_ld32(taddr(tm, 32 * quad, TM_X + 32 * half), v);
    tmem_ld_wait();
#pragma unroll
    for (int seg = 0; seg < 4; ++seg) {
      float x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int t = 32 * half + 8 * seg + u;
        const float qv = ld_bf16(sQ, (c >> 6) * 8192 + kmajor_off(t, c & 63));
        x[u] = (t < L) ? qv * expf(sG[t * DK + c]) - v[8 * seg + u] : 0.f;
      }
      st16(slot + SLOT_QP + sw128((uint32_t)(c * 128 + (32 * half + 8 * seg) * 2)), pack8(x));
    }
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // ---- 9. O_intra^T -= U^T (B_e beta)^T;  Qc = (K_a beta)^T V - (K_b beta)^T U ----
  if (tid == 0) {
    const uint32_t usm = smem_u32(sX + X_U);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_bf16(tm + TM_OI, desc_kmajor(usm, 16 * kk, 0), desc_kmajor(smem_u32(sX + X_BE), 16 * kk, 0),
               idesc_bf16(128, 64, false, false, true), 1);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_bf16(tm + TM_QC, desc_mnmajor(smem_u32(sX + X_KAB), 16 * kk, 8192),
               desc_mnmajor(smem_u32(sV), 16 * kk, 8192), idesc_bf16(128, 128, true, true), kk > 0);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_bf16(tm + TM_QC, desc_mnmajor(smem_u32(sX + X_KBB), 16 * kk, 8192), desc_kmajor(usm, 16 * kk, 0),
               idesc_bf16(128, 128, true, false, true), 1);
    mma_commit(bar_mma);
  }
  __syncwarp();
  mbar_wait(bar_mma, 1, hdr, KDA_DEVICE_TIMEOUT);
  tc_fence_after();

  {
    float v[32];
    // O_intra (lanes n, cols t) -> staging [t][n]
    const int n = lane_row;
    tmem_ld32(taddr(tm, 32 * quad, TM_OI + 32 * half), v);
    tmem_ld_wait();
    __nv_bfloat16 *ost = reinterpret_cast<__nv_bfloat16 *>(sX + X_OST);
#pragma unroll
    for (int u = 0; u < 32; ++u) ost[(32 * half + u) * DK + n] = __float2bfloat16_rn(v[u]);
    // Qc (lanes i, cols n) -> slot [slice][i][n mod 32]
    const int i = lane_row;
#pragma unroll
    for (int part = 0; part < 2; ++part) {
      const int n0 = 64 * half + 32 * part;  // one 32-wide slice
      tmem_ld32(taddr(tm, 32 * quad, TM_QC + n0), v);
      tmem_ld_wait();
      const int sl = n0 / NS;
#pragma unroll
      for (int seg = 0; seg < 4; ++seg) {
        float x[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) x[u] = v[8 * seg + u];
        st16(slot + SLOT_QC + ((sl * DK + i) * NS + 8 * seg) * 2, pack8(x));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  // staging -> slot [slice][t][n mod 32]
  for (int item = tid; item < 64 * 16; item += kPrepThreads) {
    const int t = item >> 4, n8 = (item & 15) * 8;
    const uint4 u = *reinterpret_cast<const uint4 *>(sX + X_OST + (t * DK + n8) * 2);
    const int sl = n8 / NS;
    *reinterpret_cast<uint4 *>(slot + SLOT_OI + ((sl * C + t) * NS + (n8 % NS)) * 2) = u;
  }
  if (warp == 0) tmem_dealloc(tm, 512);
}

// ---------------------------------------------------------------------------
// scan kernel
// ---------------------------------------------------------------------------
constexpr int kScanThreads = 128;
constexpr uint32_t ST_P = 0, ST_QP = 32768, ST_QC = 49152, ST_OI = 57344, ST_BYTES = 65536;
constexpr uint32_t SC_SB = 2 * ST_BYTES;  // 8 KB S operand, K-major [n][i] (two 4 KB blocks)
constexpr uint32_t SC_MISC = SC_SB + 8192;
constexpr uint32_t SCAN_SMEM = SC_MISC + 128 + 1024;
constexpr uint32_t STAGE_TX = 32768 + 16384 + 8192 + 4096;

__global__ void __launch_bounds__(kScanThreads, 1)
chunk_scan_kernel(const int32_t *hdr, const int32_t *__restrict__ seq_off,
                  const ChunkEntry *__restrict__ tab, const unsigned char *__restrict__ slots,
                  __nv_bfloat16 *__restrict__ o, const float *__restrict__ s0,
                  float *__restrict__ sT, int H_v, int32_t *err) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char *sm = reinterpret_cast<unsigned char *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint64_t *full = reinterpret_cast<uint64_t *>(sm + SC_MISC);
  uint64_t *mma_bar = full + 2;
  uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + SC_MISC + 64);
  unsigned char *sb = sm + SC_SB;

  if (hdr[0] != KDA_DEVICE_OK) return;
  const int n = blockIdx.x / NSL, sl = blockIdx.x % NSL, h = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c_begin = seq_off[n], c_end = seq_off[n + 1];
  const int nch = c_end - c_begin;

  if (warp == 0) {
    tmem_alloc(tslot, 64);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&full[0], 1);
    mbar_init(&full[1], 1);
    mbar_init(mma_bar, 1);
    mbar_fence_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *tslot;

  auto load_stage = [&](int u) {
    const int st = u & 1;
    const unsigned char *slot = slots + ((size_t)(c_begin + u) * H_v + h) * SLOT_BYTES;
    unsigned char *dst = sm + st * ST_BYTES;
    mbar_arrive_expect_tx(&full[st], STAGE_TX);
    bulk_g2s(dst + ST_P, slot + SLOT_P, 32768, &full[st]);
    bulk_g2s(dst + ST_QP, slot + SLOT_QP, 16384, &full[st]);
    bulk_g2s(dst + ST_QC, slot + SLOT_QC + sl * (DK * NS * 2), DK * NS * 2, &full[st]);
    bulk_g2s(dst + ST_OI, slot + SLOT_OI + sl * (C * NS * 2), C * NS * 2, &full[st]);
  };
  if (tid == 0) {
    if (nch > 0) load_stage(0);
    if (nch > 1) load_stage(1);
  }

  // state row i = tid, columns [sl*32, sl*32 + 32)
  const int i = tid;
  float S[NS];
  const size_t soff = ((size_t)n * H_v + h) * DK * DK + (size_t)i * DK + sl * NS;
#pragma unroll
  for (int u = 0; u < NS; u += 4) {
    float4 x = s0 ? *reinterpret_cast<const float4 *>(s0 + soff + u) : make_float4(0.f, 0.f, 0.f, 0.f);
    S[u] = x.x; S[u + 1] = x.y; S[u + 2] = x.z; S[u + 3] = x.w;
  }

  for (int u = 0; u < nch; ++u) {
    const int st = u & 1;
    const uint32_t ph = (u >> 1) & 1;
    const unsigned char *stage = sm + st * ST_BYTES;
    // S (bf16) -> K-major B operand [n][i]
#pragma unroll
    for (int nn = 0; nn < NS; ++nn)
      *reinterpret_cast<__nv_bfloat16 *>(sb + (i >> 6) * 4096 + kmajor_off(nn, i & 63)) =
          __float2bfloat16_rn(S[nn]);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    mbar_wait(&full[st], ph, err, KDA_DEVICE_TIMEOUT);
    if (tid == 0) {
      tc_fence_after();
      const uint32_t pa = smem_u32(stage + ST_P), qa = smem_u32(stage + ST_QP), sbb = smem_u32(sb);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16(tm, desc_kmajor(pa, 16 * kk, 16384), desc_kmajor(sbb, 16 * kk, 4096),
                 idesc_bf16(128, NS, false, false), kk > 0);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_bf16(tm + 32, desc_mnmajor(qa, 16 * kk, 0), desc_kmajor(sbb, 16 * kk, 4096),
                 idesc_bf16(64, NS, true, false), kk > 0);
      mma_commit(mma_bar);
    }
    __syncwarp();
    mbar_wait(mma_bar, u & 1, err, KDA_DEVICE_TIMEOUT);
    tc_fence_after();

    // S <- P S + Qc
    float v[32];
    tmem_ld32(taddr(tm, 32 * warp, 0), v);
    tmem_ld_wait();
    const uint4 *qc = reinterpret_cast<const uint4 *>(stage + ST_QC + i * NS * 2);
#pragma unroll
    for (int seg = 0; seg < NS / 8; ++seg) {
      const uint4 w = qc[seg];
      const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        S[8 * seg + 2 * e] = v[8 * seg + 2 * e] + bf16_lo(ww[e]);
        S[8 * seg + 2 * e + 1] = v[8 * seg + 2 * e + 1] + bf16_hi(ww[e]);
      }
    }
    // o = Q' S + O_intra  (M = 64 accumulator: row t in lane 32*(t/16) + t%16)
    tmem_ld32(taddr(tm, 32 * warp, 32), v);
    tmem_ld_wait();
    const ChunkEntry ce = tab[c_begin + u];
    const int t = 16 * warp + lane;
    if (lane < 16 && t < ce.len) {
      const uint4 *oi = reinterpret_cast<const uint4 *>(stage + ST_OI + t * NS * 2);
      __nv_bfloat16 *dst = o + ((size_t)(ce.start + t) * H_v + h) * DK + sl * NS;
#pragma unroll
      for (int seg = 0; seg < NS / 8; ++seg) {
        const uint4 w = oi[seg];
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
        float x[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          x[2 * e] = v[8 * seg + 2 * e] + bf16_lo(ww[e]);
          x[2 * e + 1] = v[8 * seg + 2 * e + 1] + bf16_hi(ww[e]);
        }
        *reinterpret_cast<uint4 *>(dst + 8 * seg) = pack8(x);
      }
    }
    tc_fence_before();
    __syncthreads();  // stage, TMEM and the S operand are free again
    if (tid == 0 && u + 2 < nch) load_stage(u + 2);
  }

  if (sT) {
#pragma unroll
    for (int u = 0; u < NS; u += 4)
      *reinterpret_cast<float4 *>(sT + soff + u) = make_float4(S[u], S[u + 1], S[u + 2], S[u + 3]);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tm, 64);
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3-D map over a [T_total, H, 128] tensor (innermost first), box {inner, 1, 64}
bool make_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int esize, int H,
              int64_t T_total, int box_inner, CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)DK, (cuuint64_t)H, (cuuint64_t)T_total};
  cuuint64_t strides[2] = {(cuuint64_t)DK * esize, (cuuint64_t)H * DK * esize};
  cuuint32_t box[3] = {(cuuint32_t)box_inner, 1, (cuuint32_t)C};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, dt, 3, const_cast<void *>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

size_t prefill_workspace_bytes(int T, int H_v, int d_k, int d_v, int num_seqs, bool bf16) {
  if (!(bf16 && d_k == DK && d_v == DK))
    return kHeaderBytes + align_up(sizeof(int32_t) * ((size_t)num_seqs + 1), 256);
  const WsLayout L = ws_layout(T, num_seqs);
  const int64_t max_chunks = (int64_t)T / C + num_seqs;
  return L.slots + (size_t)max_chunks * H_v * SLOT_BYTES;
}

cudaError_t launch_prefill_tc(const PrefillArgs &a, cudaStream_t stream) {
  const int64_t T_total = (int64_t)a.B * a.T;
  const WsLayout L = ws_layout(T_total, a.num_seqs);
  unsigned char *ws = static_cast<unsigned char *>(a.workspace);
  int32_t *hdr = reinterpret_cast<int32_t *>(ws);
  int32_t *seq_off = reinterpret_cast<int32_t *>(ws + L.seq_off);
  ChunkEntry *tab = reinterpret_cast<ChunkEntry *>(ws + L.tab);
  unsigned char *slots = ws + L.slots;
  const int64_t max_chunks = T_total / C + a.num_seqs;

  CUtensorMap mq, mk, mv, mg;
  if (!make_map(&mq, a.q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.H_qk, T_total, 64,
                CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&mk, a.k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.H_qk, T_total, 64,
                CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&mv, a.v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.H_v, T_total, 64,
                CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (a.channel_gate) {
    if (!make_map(&mg, a.g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, a.H_v, T_total, 128,
                  CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
  } else {
    mg = mv;  // unused
  }

  {
    TraceScope tr("plan_kernel", stream);
    plan_kernel<<<1, 1024, 0, stream>>>(a.cu_seqlens, a.num_seqs, a.T, (int)T_total, hdr,
                                        seq_off, tab);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  auto prep = a.channel_gate ? chunk_prep_kernel<true> : chunk_prep_kernel<false>;
  e = cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize, PREP_SMEM);
  if (e != cudaSuccess) return e;
  dim3 gp((unsigned)max_chunks, (unsigned)a.H_v);
  {
    TraceScope tr("chunk_prep_kernel", stream);
    prep<<<gp, kPrepThreads, PREP_SMEM, stream>>>(mq, mk, mv, mg, a.channel_gate ? nullptr : a.g,
                                                 a.beta, a.H_qk, a.H_v, hdr, tab, slots);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  e = cudaFuncSetAttribute(chunk_scan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SCAN_SMEM);
  if (e != cudaSuccess) return e;
  dim3 gs((unsigned)(a.num_seqs * NSL), (unsigned)a.H_v);
  {
    TraceScope tr("chunk_scan_kernel", stream);
    chunk_scan_kernel<<<gs, kScanThreads, SCAN_SMEM, stream>>>(
        hdr, seq_off, tab, slots, (__nv_bfloat16 *)a.o, a.initial_state, a.final_state, a.H_v, hdr);
  }
  return cudaGetLastError();
}

}  // namespace gdr
