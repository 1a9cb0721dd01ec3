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
// sub-chunking", row "KDA") are split at an anchor, the cumulative log-decay
// E_1 at the end of the chunk's second 16-token sub-chunk:
// e^{x_i - G_j} = e^{x_i - E_1} * e^{E_1 - G_j}.  A row factor is at most the
// inverse decay product of the two sub-chunks up to the anchor, a key factor
// that of the two after it; bf16 and fp32 rounding is relative, so the scaled
// operands lose nothing as long as they stay in range.  A chunk with a 16-token
// log-decay sum below -32 in some channel (so that a 32-token one could fall
// below -64) takes its Grams from directly formed pair factors instead (fp32,
// every factor <= 1, out of line), so no gate strength leaves the fp32/bf16
// range.
//
// With the decay applied before the erase (the variant order (I - beta k
// k^T) Diag(a) S), recall reads the state along a_t . k_t: the erase
// direction equals the write direction, every Gp above becomes G, and only
// the operand scale factors change (template flag DECAY_FIRST).
//
// Two kernels (plus a one-CTA planning kernel):
//   prep  -- persistent, one CTA per SM looping over (chunk, v-head) items,
//            all chunks in parallel: loads q/k/v/g tiles with TMA (the next
//            item's loads overlap the current item's last products), builds
//            every S-independent factor above with tcgen05 MMAs (bf16
//            operands, fp32 accumulators in TMEM) and a blocked fp32
//            triangular inverse, and writes P, Q', Qc, O_intra (bf16) into a
//            workspace slot laid out as the scan's shared-memory operand
//            images.
//   scan  -- one CTA per (sequence, v-head, 32- or 64-column slice of the
//            state), walking the chunks in order: the fp32 state rows in
//            registers of 4 chain warps, its bf16 copy in shared memory as
//            the MN-major B operand; per chunk one MMA P S (M = 128, N = the
//            slice width, K = 128) and one Q' S (M = 64), then
//            S <- P S + Qc and o = Q' S + O_intra, with a load warp
//            streaming the slots through 2-3 stages and 4 output warps.
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

// ---- workspace: header, per-sequence chunk offsets, chunk table, slots ----
struct ChunkEntry {
  int32_t seq, start, len, pad;
};
constexpr size_t kHeaderBytes = 256;  // [0] status word, [1] number of chunks
constexpr uint32_t SLOT_P = 0;        // 32 KB  P, K-major A image [i][c]
constexpr uint32_t SLOT_QP = 32768;   // 16 KB  Q', MN-major A image [c][t]
constexpr uint32_t SLOT_QC = 49152;   // 32 KB  Qc, four 32-column slices [s][i][32 j] (slice_off)
constexpr uint32_t SLOT_OI = 81920;   // 16 KB  O_intra, four 32-column slices [s][t][32 j] (slice_off)
constexpr uint32_t SLOT_BYTES = 98304;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct WsLayout {
  size_t seq_off, order, tab, slots, total;
};
WsLayout ws_layout(int64_t T_total, int num_seqs) {
  WsLayout L;
  const int64_t max_chunks = T_total / C + num_seqs;
  L.seq_off = kHeaderBytes;
  L.order = align_up(L.seq_off + sizeof(int32_t) * ((size_t)num_seqs + 1), 256);
  L.tab = align_up(L.order + sizeof(int32_t) * (size_t)num_seqs, 256);
  L.slots = align_up(L.tab + sizeof(ChunkEntry) * (size_t)max_chunks, 1024);
  L.total = L.slots;  // + slots, added by the caller (depends on H_v)
  return L;
}

// Where a kernel finds its chunks: for a dense batch (B sequences of T tokens)
// they follow from the chunk index; for packed sequences from the planning
// kernel's table, per-sequence offsets and scan order.
struct Chunks {
  const ChunkEntry *tab;
  const int32_t *seq_off, *order;
  int dense_T;  // > 0: dense batch of sequences of this length (no table)
  int per_seq;  // dense: chunks per sequence
  int64_t T_total, max_chunks;  // extents of the token rows and of the chunk table / slots
  __device__ __forceinline__ ChunkEntry entry(int ck) const {
    if (dense_T > 0) {
      const int n = ck / per_seq, j = ck - n * per_seq;
      return ChunkEntry{n, n * dense_T + j * C, min(C, dense_T - j * C), 0};
    }
    return GDR_IN_BOUNDS(ck >= 0 && ck < max_chunks) ? tab[ck] : ChunkEntry{0, 0, 0, 0};
  }
  __device__ __forceinline__ int first(int n) const { return dense_T > 0 ? n * per_seq : seq_off[n]; }
  __device__ __forceinline__ int seq(int r) const { return dense_T > 0 ? r : order[r]; }
  // total chunks: dense from the shape, packed from the plan's header word
  __device__ __forceinline__ int total(const int32_t *hdr, int num_seqs) const {
    return dense_T > 0 ? num_seqs * per_seq : hdr[1];
  }
};

// ---------------------------------------------------------------------------
// planning: chunk table, per-sequence chunk offsets and the order in which
// the scan takes the sequences (also validates cu_seqlens)
// ---------------------------------------------------------------------------
constexpr int kSortMax = 512;  // packed batches up to this size are scanned longest first
__global__ void __launch_bounds__(1024, 1)
plan_kernel(const int32_t *__restrict__ cu, int num_seqs, int T, int T_total, int32_t *hdr,
            int32_t *seq_off, int32_t *order, ChunkEntry *tab) {
  __shared__ int32_t warp_tot[32];
  __shared__ int32_t s_len[kSortMax];
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
  if (__syncthreads_or(bad)) {  // every table entry stays in bounds
    for (int i = tid; i <= num_seqs; i += blockDim.x) seq_off[i] = 0;
    for (int i = tid; i < num_seqs; i += blockDim.x) order[i] = i;
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
        if (GDR_IN_BOUNDS(first + j < (int64_t)T_total / C + num_seqs)) tab[first + j] = e;
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
  // scan order: decreasing length (ties by index), so the longest chains start first
  if (cu && num_seqs <= kSortMax) {
    for (int i = tid; i < num_seqs; i += blockDim.x) s_len[i] = cu[i + 1] - cu[i];
    __syncthreads();
    for (int i = tid; i < num_seqs; i += blockDim.x) {
      const int li = s_len[i];
      int r = 0;
      for (int m = 0; m < num_seqs; ++m) {
        const int lm = s_len[m];
        r += (lm > li) || (lm == li && m < i);
      }
      order[r] = i;
    }
  } else {
    for (int i = tid; i < num_seqs; i += blockDim.x) order[i] = i;
  }
}

// ---------------------------------------------------------------------------
// prep kernel
// ---------------------------------------------------------------------------
constexpr int kPrepThreads = 512;
constexpr int kIoThread = 480;  // issues the TMA loads and image stores (lane 0 of the last warp)

// shared memory map (bytes from a 1024-aligned base)
constexpr uint32_t OFF_Q = 0;         // q tile, two K-major SW128 [64 t][64 c] blocks; later q.e^{G}
constexpr uint32_t OFF_K = 16384;     // k tile; later K.e^{Gp} (same bytes: MN-major [t][c])
constexpr uint32_t OFF_V = 32768;     // v tile (MN-major operand, 64-wide blocks 8 KB apart)
constexpr uint32_t OFF_KAB = 49152;   // beta K.e^{G_L-G}
constexpr uint32_t OFF_KBB = 65536;   // beta K.e^{G_L-Gp}
constexpr uint32_t OFF_G = 81920;     // g fp32 [64][128]; the next item's lands once the decays are taken
constexpr uint32_t OFF_X = 114688;    // 96 KB phase-dependent region
constexpr uint32_t OFF_MISC = 212992;
constexpr uint32_t MISC_BETA = 0;      // f32[64]
constexpr uint32_t MISC_GSC = 256;     // f32[64] scalar gate
constexpr uint32_t MISC_PBLK = 512;    // f32[4][128] product of a over each sub-chunk
constexpr uint32_t MISC_GSUM = 2560;   // f32[4][128] sum of g over each sub-chunk
constexpr uint32_t MISC_GLE = 4608;    // f32[128] e^{G_L}
constexpr uint32_t MISC_BAR = 5120;    // 5 x u64; the drain barrier at +48, two failure flags at +56
constexpr uint32_t MISC_TSLOT = 5160;  // u32; the exact-Gram flag at +4
constexpr uint32_t MISC_GBAR = 5184;   // u64: the gate tile's own TMA barrier (per-channel gate)
constexpr uint32_t MISC_XP = 6144;     // f32[4][2][128] product of a over each half sub-chunk
constexpr uint32_t MISC_XS = 10240;    // f32[4][2][128] sum of g over each half sub-chunk
constexpr uint32_t PREP_SMEM = OFF_MISC + 14336 + 1024;

// X region, gram phase
constexpr uint32_t X_R = 0;           // 32 KB, K-major B [128 rows][128], blocks 16 KB apart
constexpr uint32_t X_LEFT = 32768;    // 48 KB, K-major A tile [128 rows][128] ([K; Q] scaled to the anchor)
constexpr uint32_t LEFT_BLOCK = 24576;  // its 64-column blocks (16 KB used of each)
// X region, after the Gram MMAs
constexpr uint32_t X_AWBW = 0;        // 16 KB K-major B [128 i'][64 j]
constexpr uint32_t X_BE = 16384;      // 8 KB  K-major B [64 i][64 j]
constexpr uint32_t X_TINVB = 24576;   // 8 KB  K-major B [64 i][64 j]; scratch before
constexpr int LDN = 68;               // padded row stride (floats) of the fp32 64x64 tiles
constexpr uint32_t X_GEXACT = 50176;  // exact Gram only: f32 [65][kLdG] cumulative log-decay
constexpr int kLdG = 129;             // its padded row stride (floats)
// The Gram's operands grow by at most e^{-(a 32-token log-decay sum)}; this is
// the bound on that sum (e^{64} leaves e^{24} of headroom below the fp32/bf16
// maximum for q, k).  An item with a 16-token sum below half of it (so that a
// 32-token one may fall below it) takes the exact Gram.
constexpr float kExactBound = -64.f;
constexpr uint32_t X_NAE = 32768;     // 17 KB f32 [64][LDN]  (N = tril(A_e) diag(beta))
constexpr uint32_t X_TINVF = 50176;   // 17 KB f32 [64][LDN]  (T^{-1}); both dead after step 6
constexpr uint32_t X_Y = 69632;       // while T^{-1} is built: K-major [n][t]
constexpr uint32_t X_W = 32768;       // after T^{-1}: K-major [c][t]
constexpr uint32_t X_U = 49152;       // after T^{-1}: K-major [n][t]
// slot images, staged in shared memory and bulk-copied to the workspace; the
// copies' reads of these bytes only have to finish before the next item's
// operand build
constexpr uint32_t X_QPI = 0;         // after P and X: Q' image (16 KB)
constexpr uint32_t X_PI = 65536;      // after P and X: P image (32 KB)
constexpr uint32_t X_OII = 16384;     // after the last products: O_intra image (16 KB)
constexpr uint32_t X_QCI = 32768;     // after the last products: Qc image (32 KB)

// TMEM columns (W, Y die at their readback, U at its readback)
// Rounds of products: the Gram; Y, the first O_intra term and the first Qc
// term (issued before T^{-1} is built, which none of them needs; the last
// products that read v); W and U; then P and X (one thread) beside the second
// O_intra and Qc terms (another).
constexpr uint32_t TM_GRAM = 0, TM_Y = 320, TM_OI = 128, TM_W = 256, TM_U = 0, TM_P = 0,
                   TM_QC = 384, TM_X = 256;

__device__ __forceinline__ float ld_bf16(const unsigned char *base, uint32_t off) {
  return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(base + off));
}

// Column-slice images read one row per thread (Qc, O_intra): 32 value columns
// of bf16 per row (64 bytes), the 16-byte chunks swizzled as in the SW64
// operand layout so that the 8 threads of a shared-memory phase hit distinct
// banks.  Byte offset of chunk `ch` (columns 8 ch .. 8 ch + 7) of row r:
__device__ __forceinline__ uint32_t slice_off(int r, int ch) {
  return sw64((uint32_t)(r * 64 + ch * 16));
}
constexpr uint32_t QC_SLICE_BYTES = 128 * 64;  // d_k rows
constexpr uint32_t OI_SLICE_BYTES = 64 * 64;   // C rows

__device__ __forceinline__ uint4 pack8(const float (&x)[8]) {
  return make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                    pack_bf16x2(x[6], x[7]));
}

__device__ __forceinline__ void st16(unsigned char *p, uint4 v) { *reinterpret_cast<uint4 *>(p) = v; }


// ---- warp-level tf32 MMA (m16n8k8) for the small block products of T^{-1} ----
constexpr int LDT = 40;  // row stride (floats) of the fp32 scratch: conflict-free B fragments

__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}

// d (16x8 fp32, per-lane fragment) += A[0..16)[k] * B[k][n0 .. n0+8) over k in [k_lo, k_hi)
// (multiples of 8, at most 8 NSTEP).  A and B are row-major fp32 in shared
// memory with row strides lda, ldb; A points at row 0 / column 0 of the tile,
// B at row 0 and column n0 is given separately.  Fragments follow the
// m16n8k8 layout: lane = 4 g + t holds A (g, t), (g+8, t), (g, t+4), (g+8, t+4),
// B (t, g), (t+4, g) and D (g, 2t), (g, 2t+1), (g+8, 2t), (g+8, 2t+1).  The
// k-steps are unrolled: every operand load of the first 8 NSTEP columns of A
// and rows of B (all inside the tiles) is issued up front, and only the
// products of steps in [k_lo, k_hi) run (a warp-uniform test), so no load
// waits on the previous product.
template <int NSTEP>
__device__ __forceinline__ void warp_mma_tf32_range(float (&d)[4], const float *A, int lda,
                                                    const float *B, int ldb, int n0, int k_lo,
                                                    int k_hi, int lane) {
  const int g = lane >> 2, t = lane & 3;
  uint32_t a[NSTEP][4], b[NSTEP][2];
#pragma unroll
  for (int s = 0; s < NSTEP; ++s) {
    const int k0 = 8 * s;
    a[s][0] = to_tf32(A[g * lda + k0 + t]);
    a[s][1] = to_tf32(A[(g + 8) * lda + k0 + t]);
    a[s][2] = to_tf32(A[g * lda + k0 + t + 4]);
    a[s][3] = to_tf32(A[(g + 8) * lda + k0 + t + 4]);
    b[s][0] = to_tf32(B[(k0 + t) * ldb + n0 + g]);
    b[s][1] = to_tf32(B[(k0 + t + 4) * ldb + n0 + g]);
  }
#pragma unroll
  for (int s = 0; s < NSTEP; ++s) {
    if (8 * s < k_lo || 8 * s >= k_hi) continue;
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[s][0]), "r"(a[s][1]), "r"(a[s][2]), "r"(a[s][3]), "r"(b[s][0]), "r"(b[s][1]));
  }
}

// K-extent K from 0, B already offset to its column n0 (so n0 = 0 inside)
template <int K>
__device__ __forceinline__ void warp_mma_tf32(float (&d)[4], const float *A, int lda, const float *B,
                                              int ldb, int lane) {
  warp_mma_tf32_range<K / 8>(d, A, lda, B, ldb, 0, 0, K, lane);
}

// Writes a 16x8 fp32 fragment to row-major shared memory at P (row stride ld).
__device__ __forceinline__ void store_frag(float *P, int ld, const float (&d)[4], int lane) {
  const int g = lane >> 2, t = lane & 3;
  *reinterpret_cast<float2 *>(P + g * ld + 2 * t) = make_float2(d[0], d[1]);
  *reinterpret_cast<float2 *>(P + (g + 8) * ld + 2 * t) = make_float2(d[2], d[3]);
}

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// ---- exact Gram of one per-channel item (step 2a), all 512 threads ----
// Every pair factor is formed directly from the in-chunk cumulative
// log-decay G as one exp of a difference <= 0, in fp32 on the CUDA cores, so
// nothing overflows whatever g is; the results go into the same images
// (A_w beta, B_w beta, B_e beta in bf16, N = A_e beta in fp32) as the Gram
// readback.  Reads the raw q, k and g tiles and the decay step's sub-chunk
// and half-sub-chunk sums; ends with a block barrier after its last write.
// Kept out of line: only items with a steep sub-chunk run it.
template <bool DECAY_FIRST>
__device__ __noinline__ void exact_gram(unsigned char *sm, int L) {
  const int tid = threadIdx.x, bI = tid >> 7, rh = (tid >> 6) & 1, c2 = (tid & 63) * 2;
  unsigned char *sX = sm + OFF_X;
  const unsigned char *sQ = sm + OFF_Q, *sK = sm + OFF_K;
  const float *sG = reinterpret_cast<const float *>(sm + OFF_G);
  const float *sGsum = reinterpret_cast<const float *>(sm + OFF_MISC + MISC_GSUM);
  const float *sBeta = reinterpret_cast<const float *>(sm + OFF_MISC + MISC_BETA);
  float *Gt = reinterpret_cast<float *>(sX + X_GEXACT);  // Gt[t + 1][c] = G_t, Gt[0][c] = 0
  {
    const float *xs = reinterpret_cast<const float *>(sm + OFF_MISC + MISC_XS);
    float b0 = rh ? xs[(2 * bI) * DK + c2] : 0.f, b1 = rh ? xs[(2 * bI) * DK + c2 + 1] : 0.f;
    for (int J = 0; J < bI; ++J) {
      b0 += sGsum[J * DK + c2];
      b1 += sGsum[J * DK + c2 + 1];
    }
    if (bI == 0 && rh == 0) Gt[c2] = Gt[c2 + 1] = 0.f;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int t = 16 * bI + 8 * rh + r;
      if (t < L) {
        const float2 gg = *reinterpret_cast<const float2 *>(sG + t * DK + c2);
        b0 += gg.x;
        b1 += gg.y;
      }
      Gt[(t + 1) * kLdG + c2] = b0;
      Gt[(t + 1) * kLdG + c2 + 1] = b1;
    }
  }
  __syncthreads();
  // thread (row, chunk of 8 keys): key row i = row against keys j < i (A_w,
  // A_e), query row t = row against keys j <= t (B_w, B_e)
  const int row = tid >> 3, j0 = 8 * (tid & 7);
  float aw[8], ae[8], bw[8], be[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) aw[u] = ae[u] = bw[u] = be[u] = 0.f;
  if (j0 <= row && row < L) {
    // keys in two halves of four (fewer live accumulators per channel loop)
#pragma unroll
    for (int hv = 0; hv < 2; ++hv) {
#pragma unroll 1
      for (int c = 0; c < DK; ++c) {
        const uint32_t cb = (uint32_t)(c >> 6) * 8192;
        const float Gi = Gt[(row + 1) * kLdG + c], Gpi = Gt[row * kLdG + c];
        const float qv = ld_bf16(sQ, cb + kmajor_off(row, c & 63));
        const float kv = ld_bf16(sK, cb + kmajor_off(row, c & 63));
        const float arow = __expf(Gi - Gpi);  // a of the row's own token
#pragma unroll
        for (int u = 4 * hv; u < 4 * hv + 4; ++u) {
          const int j = j0 + u;
          if (j > row) continue;
          const float Gj = Gt[(j + 1) * kLdG + c], Gpj = Gt[j * kLdG + c];
          const float kj = ld_bf16(sK, cb + kmajor_off(j, c & 63));
          const float qk = qv * kj, kk = kv * kj;
          if (j == row) {  // the query's own key: e^{G_t - G_t} = 1, e^{G_t - Gp_t} = a_t
            bw[u] += qk;
            be[u] = fmaf(qk, DECAY_FIRST ? 1.f : arow, be[u]);
          } else {
            // K row: e^{Gp_i - G_j} (<= 1 for j < i); the rest follow by
            // multiplying with a_i, a_j <= 1
            const float faw = __expf((DECAY_FIRST ? Gi : Gpi) - Gj);
            const float aj = DECAY_FIRST ? 1.f : __expf(Gj - Gpj);
            const float fbw = DECAY_FIRST ? faw : faw * arow;  // e^{G_i - G_j}
            aw[u] = fmaf(kk, faw, aw[u]);
            ae[u] = fmaf(kk, faw * aj, ae[u]);
            bw[u] = fmaf(qk, fbw, bw[u]);
            be[u] = fmaf(qk, fbw * aj, be[u]);
          }
        }
      }
    }
  }
  __syncthreads();  // every read of the tables and tiles is done
  {
    float xw[8], xb[8], xe[8], xn[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int j = j0 + u;
      const float bj = sBeta[j];  // 0 past the chunk's length
      const bool key = row < L && j < row, qry = row < L && j <= row;
      xw[u] = key ? aw[u] * bj : 0.f;
      xn[u] = key ? ae[u] * bj : 0.f;
      xb[u] = qry ? bw[u] * bj : 0.f;
      xe[u] = qry ? be[u] * bj : 0.f;
    }
    float *nae = reinterpret_cast<float *>(sX + X_NAE);
    st16(sX + X_AWBW + kmajor_off(row, j0), pack8(xw));
    st16(sX + X_AWBW + kmajor_off(64 + row, j0), pack8(xb));
    st16(sX + X_BE + kmajor_off(row, j0), pack8(xe));
    *reinterpret_cast<float4 *>(nae + row * LDN + j0) = make_float4(xn[0], xn[1], xn[2], xn[3]);
    *reinterpret_cast<float4 *>(nae + row * LDN + j0 + 4) = make_float4(xn[4], xn[5], xn[6], xn[7]);
  }
  __syncthreads();
}

template <bool CHANNEL, bool DECAY_FIRST>
__global__ void __launch_bounds__(kPrepThreads, 1)
chunk_prep_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                  const float *__restrict__ g_scalar, const float *__restrict__ beta, int H_qk,
                  int H_v, int32_t *hdr, const Chunks chunks, int num_seqs,
                  unsigned char *__restrict__ slots) {
  extern __shared__ unsigned char smem_raw[];
  // 1024-byte aligned base, derived by pointer arithmetic on the shared array so
  // that the compiler keeps shared-memory addressing for every access
  unsigned char *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  // q and k tiles: two K-major SW128 blocks of 64 channels each.  Per-channel
  // gate: the q blocks, then the k blocks.  Scalar gate: each 16 KB block holds
  // 64 k rows then 64 q rows, so that [K; Q] is one 128-row MMA operand.
  constexpr uint32_t QK_CB = CHANNEL ? 8192 : 16384;  // bytes between 64-channel blocks
  unsigned char *sQ = sm + (CHANNEL ? OFF_Q : OFF_Q + 8192), *sK = sm + (CHANNEL ? OFF_K : OFF_Q);
  unsigned char *sV = sm + OFF_V;
  // k e^{Gp} and q e^{G} as the later products read them (64-channel blocks
  // 8 KB apart): in place per-channel, in the g buffer with a scalar gate
  unsigned char *sKd = CHANNEL ? sK : sm + OFF_G, *sQd = CHANNEL ? sQ : sm + OFF_G + 16384;
  float *sG = reinterpret_cast<float *>(sm + OFF_G);
  unsigned char *sX = sm + OFF_X;
  float *sBeta = reinterpret_cast<float *>(sm + OFF_MISC + MISC_BETA);
  float *sGsc = reinterpret_cast<float *>(sm + OFF_MISC + MISC_GSC);
  float *sPblk = reinterpret_cast<float *>(sm + OFF_MISC + MISC_PBLK);
  float *sGsum = reinterpret_cast<float *>(sm + OFF_MISC + MISC_GSUM);
  float *sGLe = reinterpret_cast<float *>(sm + OFF_MISC + MISC_GLE);
  uint64_t *bar_tma = reinterpret_cast<uint64_t *>(sm + OFF_MISC + MISC_BAR);
  uint64_t *bar_mma = bar_tma + 1;   // the Gram, then W and U (two commits each)
  uint64_t *bar_yo = bar_tma + 2;    // Y and the first O_intra term (two commits)
  uint64_t *bar_px = bar_tma + 3;    // P and X (one commit)
  uint64_t *bar_oq = bar_tma + 4;    // the second O_intra term and Qc (one commit)
  uint64_t *bar_drain = bar_tma + 6;  // after an expired wait: every issuing thread's last MMAs
  // the gate tile lands on a barrier of its own, so that an item's decays can
  // start while its q, k, v tiles are still on their way
  uint64_t *bar_g = reinterpret_cast<uint64_t *>(sm + OFF_MISC + MISC_GBAR);
  uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + OFF_MISC + MISC_TSLOT);
  volatile uint32_t *s_exact = reinterpret_cast<volatile uint32_t *>(sm + OFF_MISC + MISC_TSLOT + 4);
  volatile uint32_t *s_fail = reinterpret_cast<volatile uint32_t *>(sm + OFF_MISC + MISC_BAR + 56);

  if (hdr[0] != KDA_DEVICE_OK) return;
  // persistent: this CTA walks (chunk, v-head) work items blockIdx.x,
  // blockIdx.x + gridDim.x, ...; the next item's tiles are loaded while the
  // current one finishes.
  const int total = chunks.total(hdr, num_seqs) * H_v;
  int work = blockIdx.x;
  if (work >= total) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (warp == 0) {
    tmem_alloc(tslot, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(bar_tma, 1);
    mbar_init(bar_g, 1);
    mbar_init(bar_mma, 2);
    mbar_init(bar_yo, 2);
    mbar_init(bar_px, 1);
    mbar_init(bar_oq, 1);
    mbar_init(bar_drain, 4);
    *s_exact = 0u;
    s_fail[0] = s_fail[1] = 0u;
    mbar_fence_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *tslot;

  // ---- 1. TMA loads of an item's q, k, v (bf16, swizzled) and g (fp32) ----
  // Items' chunk-table entries are read one item ahead of their use, so no
  // thread waits on a global load between phases.
  auto entry = [&](int w) { return w < total ? chunks.entry(w / H_v) : ChunkEntry{0, 0, 0, 0}; };
  // Each tile of the next item loads as soon as the current one is done with
  // its buffer: g once the decays are taken, v once the products before T^{-1}
  // have run, q and k once their last reader has run (the raw-tile Gram and
  // the image pass with a scalar gate, before v; Q' with a per-channel gate,
  // after v).  The gate tile completes a phase of its own barrier, waited for at
  // the top of the item; of the q, k, v loads every one but the last adds its
  // bytes to the phase without an arrival and the last one arrives, so that
  // phase completes only when all three have landed.  It is waited for after
  // the decays, which need the gate alone: the q/k load issued late in the
  // previous item (after its Q' readback) lands meanwhile.  All from thread
  // kIoThread, in program order.
  // TMA phases armed by kIoThread (loads whose last one carried the arrival)
  // and whether loads of a phase not yet armed are in flight: an aborted CTA
  // completes and waits out every such phase before it exits.
  // (bar_g: every gate load is a phase of its own, g_armed of them so far)
  int tma_armed = 0, tma_done = 0, g_armed = 0, g_done = 0;
  bool tma_partial = false;
  auto load_g = [&](int w, const ChunkEntry &e) {
    if (CHANNEL) {
      ++g_armed;
      fence_async_smem();
      mbar_arrive_expect_tx(bar_g, 32768);
      tma_load_3d(sG, &tm_g, 0, w % H_v, e.start, bar_g);
    }
  };
  auto load_qk = [&](int w, const ChunkEntry &e, bool arrive) {
    const int hkk = (w % H_v) / (H_v / H_qk);
    tma_armed += arrive ? 1 : 0;
    tma_partial = !arrive;
    fence_async_smem();
    if (arrive)
      mbar_arrive_expect_tx(bar_tma, 2 * 16384);
    else
      mbar_expect_tx(bar_tma, 2 * 16384);
#pragma unroll
    for (int cb = 0; cb < 2; ++cb) {
      tma_load_3d(sQ + cb * QK_CB, &tm_q, cb * 64, hkk, e.start, bar_tma);
      tma_load_3d(sK + cb * QK_CB, &tm_k, cb * 64, hkk, e.start, bar_tma);
    }
  };
  auto load_v = [&](int w, const ChunkEntry &e, bool arrive) {
    tma_armed += arrive ? 1 : 0;
    tma_partial = !arrive;
    fence_async_smem();
    if (arrive)
      mbar_arrive_expect_tx(bar_tma, 16384);
    else
      mbar_expect_tx(bar_tma, 16384);
#pragma unroll
    for (int cb = 0; cb < 2; ++cb) tma_load_3d(sV + cb * 8192, &tm_v, cb * 64, w % H_v, e.start, bar_tma);
  };
  auto prefetch_l2 = [&](int w, const ChunkEntry &e) {  // kIoThread: a later item's tiles into L2
    const int ck = w / H_v, hh = w - ck * H_v, hkk = hh / (H_v / H_qk);
    const int ts = e.start;
    (void)ck;
#pragma unroll
    for (int cb = 0; cb < 2; ++cb) {
      tma_prefetch_l2_3d(&tm_q, cb * 64, hkk, ts);
      tma_prefetch_l2_3d(&tm_k, cb * 64, hkk, ts);
      tma_prefetch_l2_3d(&tm_v, cb * 64, hh, ts);
    }
    if (CHANNEL) tma_prefetch_l2_3d(&tm_g, 0, hh, ts);
  };
  // beta (and the scalar gate) of an item, one token per thread tid < C
  auto load_beta = [&](int w, const ChunkEntry &e, float &b, float &gs) {
    const int hh = w % H_v;
    const bool in = tid < e.len && GDR_IN_BOUNDS((int64_t)e.start + tid < chunks.T_total);
    b = in ? __ldg(beta + (size_t)(e.start + tid) * H_v + hh) : 0.f;
    gs = (!CHANNEL && in) ? __ldg(g_scalar + (size_t)(e.start + tid) * H_v + hh) : 0.f;
  };
  float nbeta = 0.f, ngsc = 0.f;  // the coming item's, loaded one item ahead
  ChunkEntry ce = entry(work), ce_next = entry(work + gridDim.x);
  if (tid == kIoThread) {
    load_g(work, ce);
    load_v(work, ce, false);
    load_qk(work, ce, true);
    if (work + (int)gridDim.x < total) prefetch_l2(work + gridDim.x, ce_next);
  }
  if (tid < C) load_beta(work, ce, nbeta, ngsc);

  // A bounded wait that expires (the status word then holds
  // KDA_DEVICE_TIMEOUT) raises the item's failure flag; at the top of the
  // next item all threads take one verdict and leave the work loop together,
  // so an expired wait costs at most one bound per wait site of one item,
  // not one per item.  (Skipping a thread's later waits once one expired
  // measured 8 % slower on the scalar-gate path.)
  bool failed = false, aborted = false;
  int it = 0;
  auto wait_bar = [&](uint64_t *bar, uint32_t parity, int32_t *err, int32_t code) {
    if (!mbar_wait(bar, parity, err, code)) {
      failed = true;
      s_fail[it & 1] = 1u;
    }
  };
  for (; work < total; ++it, work += gridDim.x) {
  const int chunk = work / H_v, h = work - chunk * H_v;
  const int L = ce.len;
  unsigned char *slot = slots + ((size_t)chunk * H_v + h) * SLOT_BYTES;
  const int next = work + gridDim.x;
  const ChunkEntry ce_next2 = entry(next + gridDim.x);  // used by the next item's prefetch

  if (tid < C) {
    sBeta[tid] = nbeta;
    if (!CHANNEL) sGsc[tid] = ngsc;
    // the next item's, a whole item ahead of their use
    if (next < total) load_beta(next, ce_next, nbeta, ngsc);
  }
  if constexpr (CHANNEL) {  // the gate tile; q, k, v are waited for after the decays
    wait_bar(bar_g, it & 1, hdr, KDA_DEVICE_TIMEOUT);
    if (!failed) g_done = it + 1;
  } else {
    wait_bar(bar_tma, it & 1, hdr, KDA_DEVICE_TIMEOUT);
    if (!failed) tma_done = it + 1;
  }
  // One CTA-wide verdict per item: a wait that expired anywhere in the
  // previous item ends the work loop on every thread.  Item i's waits raise
  // flag i & 1, read by all threads after the next item's first barrier and
  // cleared by thread 0 after a later barrier of that item, before any wait
  // of item i + 2 can raise it again.
  __syncthreads();
  if (s_fail[(it + 1) & 1]) {
    aborted = true;
    break;
  }
  // readbacks: warp (quad, qtr) reads TMEM lanes 32*quad .. +31, column quarter qtr
  const int quad = warp & 3, qtr = warp >> 2;
  const int lane_row = 32 * quad + lane;

  if constexpr (CHANNEL) {
  // ---- 2. per-token decays a = e^{g} (rows >= L: no decay), sub-chunk sums ----
  // Thread (I, h, p) owns channels c = 2p, 2p+1 of tokens 8h .. 8h+7 of
  // sub-chunk I; a warp spans 64 channels of the same rows, so its 4-byte
  // stores below fill whole 128-byte rows (no bank conflicts).  The two
  // halves of a sub-chunk exchange their partial products through shared
  // memory.  Every
  // in-chunk factor is a product of these a's: with G the in-chunk cumulative
  // log-decay and E_I its value at the end of sub-chunk I,
  //   e^{G_t - E_{I-1}} = prefix product of a in sub-chunk I up to t   (<= 1)
  //   e^{E_I - G_t}     = suffix product after t                       (<= 1)
  // and factors across sub-chunks are products of whole-sub-chunk products.
  const int bI = tid >> 7, rh = (tid >> 6) & 1, c2 = (tid & 63) * 2;
  float a0[8], a1[8];
  float pre0, pre1, suf0, suf1;  // product of a before / after this thread's rows
  {
    float s0 = 0.f, s1 = 0.f, p0 = 1.f, p1 = 1.f;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int t = 16 * bI + 8 * rh + r;
      float g0 = 0.f, g1 = 0.f;
      if (t < L) {
        if (CHANNEL) {
          const float2 gg = *reinterpret_cast<const float2 *>(sG + t * DK + c2);
          g0 = gg.x;
          g1 = gg.y;
        } else {
          g0 = g1 = sGsc[t];
        }
      }
      a0[r] = __expf(g0);  // the intrinsic: its error is far below the bf16 rounding of every operand
      a1[r] = __expf(g1);
      s0 += g0;
      s1 += g1;
      p0 *= a0[r];
      p1 *= a1[r];
    }
    float *xp = reinterpret_cast<float *>(sm + OFF_MISC + MISC_XP);
    float *xs = reinterpret_cast<float *>(sm + OFF_MISC + MISC_XS);
    *reinterpret_cast<float2 *>(xp + (2 * bI + rh) * DK + c2) = make_float2(p0, p1);
    *reinterpret_cast<float2 *>(xs + (2 * bI + rh) * DK + c2) = make_float2(s0, s1);
    __syncthreads();
    const float2 op = *reinterpret_cast<const float2 *>(xp + (2 * bI + (rh ^ 1)) * DK + c2);
    const float2 os = *reinterpret_cast<const float2 *>(xs + (2 * bI + (rh ^ 1)) * DK + c2);
    const float op0 = op.x, op1 = op.y, os0 = os.x, os1 = os.y;
    pre0 = rh ? op0 : 1.f;
    pre1 = rh ? op1 : 1.f;
    suf0 = rh ? 1.f : op0;
    suf1 = rh ? 1.f : op1;
    if (rh == 0) {
      sPblk[bI * DK + c2] = p0 * op0;
      sPblk[bI * DK + c2 + 1] = p1 * op1;
      sGsum[bI * DK + c2] = s0 + os0;
      sGsum[bI * DK + c2 + 1] = s1 + os1;
    }
    // The Gram scales operands by up to the inverse decay product of two
    // 16-token sub-chunks; a sub-chunk whose log-decay sum is below half of
    // kExactBound could push them past the fp32/bf16 range: such an item takes
    // the exact Gram below instead.
    const bool steep = rh == 0 && (s0 + os0 < 0.5f * kExactBound || s1 + os1 < 0.5f * kExactBound);
    if (__any_sync(0xffffffffu, steep) && lane == 0) *s_exact = 1u;  // every writer writes 1
  }
  // the previous item's image copies must have read the X region before it is rebuilt
  if (tid == kIoThread) bulk_wait_read0();
  __syncthreads();  // g is consumed: the next item's lands there
  wait_bar(bar_tma, it & 1, hdr, KDA_DEVICE_TIMEOUT);  // q, k, v
  if (!failed) tma_done = it + 1;
  const bool exact = *s_exact != 0;  // CTA-uniform; reset after the operand pass
  if (tid == kIoThread && next < total && !exact) {
    load_g(next, ce_next);
    if (next + (int)gridDim.x < total) prefetch_l2(next + gridDim.x, ce_next2);
  }

  // ---- 2a. exact Gram (items with a steep sub-chunk only; slower than the
  //          tensor-core Gram: ~2 exps per key pair and channel) ----
  if (exact) {
    exact_gram<DECAY_FIRST>(sm, L);
    if (tid == kIoThread && next < total) {  // g is consumed
      load_g(next, ce_next);
      if (next + (int)gridDim.x < total) prefetch_l2(next + gridDim.x, ce_next2);
    }
  }

  // ---- 3. one pass builds every operand of the chunk ----
  {
    // The Gram's anchor is E_1.  A row of sub-chunk I takes e^{E_{I-1} - E_1}
    // on top of its prefix product (1/(PB_0 PB_1), 1/PB_1, 1, PB_2 for
    // I = 0 .. 3), a key of sub-chunk I takes e^{E_1 - E_I} on top of its
    // suffix product (PB_1, 1, 1/PB_2, 1/(PB_2 PB_3)); PB_J is a channel's
    // decay product over sub-chunk J.
    float ei0 = 1.f, ei1 = 1.f, ge0 = 1.f, ge1 = 1.f;  // e^{E_{I-1}}, e^{G_L - E_I}
#pragma unroll
    for (int J = 0; J < 4; ++J) {
      if (J < bI) {
        ei0 *= sPblk[J * DK + c2];
        ei1 *= sPblk[J * DK + c2 + 1];
      }
      if (J > bI) {
        ge0 *= sPblk[J * DK + c2];
        ge1 *= sPblk[J * DK + c2 + 1];
      }
    }
    float fa0, fa1, rf0, rf1;
    if (bI == 0) {
      fa0 = __expf(-(sGsum[c2] + sGsum[DK + c2]));
      fa1 = __expf(-(sGsum[c2 + 1] + sGsum[DK + c2 + 1]));
      rf0 = sPblk[DK + c2];
      rf1 = sPblk[DK + c2 + 1];
    } else if (bI == 1) {
      fa0 = __expf(-sGsum[DK + c2]);
      fa1 = __expf(-sGsum[DK + c2 + 1]);
      rf0 = rf1 = 1.f;
    } else if (bI == 2) {
      fa0 = fa1 = 1.f;
      rf0 = __expf(-sGsum[2 * DK + c2]);
      rf1 = __expf(-sGsum[2 * DK + c2 + 1]);
    } else {
      fa0 = sPblk[2 * DK + c2];
      fa1 = sPblk[2 * DK + c2 + 1];
      rf0 = __expf(-(sGsum[2 * DK + c2] + sGsum[3 * DK + c2]));
      rf1 = __expf(-(sGsum[2 * DK + c2 + 1] + sGsum[3 * DK + c2 + 1]));
    }
    if (bI == 0 && rh == 0) {
      sGLe[c2] = ge0 * sPblk[c2];  // e^{G_L}: product over all four sub-chunks
      sGLe[c2 + 1] = ge1 * sPblk[c2 + 1];
    }
    // suffix products e^{E_I - G_t}
    float w0[8], w1[8];
    w0[7] = suf0;
    w1[7] = suf1;
#pragma unroll
    for (int r = 6; r >= 0; --r) {
      w0[r] = w0[r + 1] * a0[r + 1];
      w1[r] = w1[r + 1] * a1[r + 1];
    }
    // Channel pairs in packed fp32x2 arithmetic.  Every operand row written
    // here has the same residue mod 8 as t, so the SW128 position of channel
    // pair c2 within a 128-byte row is one offset per row.
    const float2 fa = make_float2(fa0, fa1), rf = make_float2(rf0, rf1);
    const float2 ei = make_float2(ei0, ei1), ge = make_float2(ge0, ge1);
    const uint32_t cblk = (uint32_t)(c2 >> 6), cpos = (uint32_t)(c2 & 63) * 2;  // byte in the row
    unsigned char *const rbase = sX + X_R + cblk * 16384;
    unsigned char *const lbase = sX + X_LEFT + cblk * LEFT_BLOCK;
    unsigned char *const kbase = sK + cblk * 8192, *const qbase = sQ + cblk * 8192;
    unsigned char *const abase = sm + OFF_KAB + cblk * 8192, *const bbase = sm + OFF_KBB + cblk * 8192;
    auto st4 = [](unsigned char *p, float2 x) {
      *reinterpret_cast<uint32_t *>(p) = pack_bf16x2(x.x, x.y);
    };
    float2 pq = make_float2(pre0, pre1);  // prefix product through t-1: e^{Gp_t - E_{I-1}}
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int t = 16 * bI + 8 * rh + r;
      const uint32_t x = (cpos ^ ((uint32_t)(t & 7) << 4));  // swizzled byte within a row
      const uint32_t koff = (uint32_t)t * 128 + x;
      const uint32_t kraw = *reinterpret_cast<const uint32_t *>(kbase + koff);
      const uint32_t qraw = *reinterpret_cast<const uint32_t *>(qbase + koff);
      const bool ok = t < L;
      const float2 k = ok ? make_float2(bf16_lo(kraw), bf16_hi(kraw)) : make_float2(0.f, 0.f);
      const float2 q = ok ? make_float2(bf16_lo(qraw), bf16_hi(qraw)) : make_float2(0.f, 0.f);
      const float b = sBeta[t];
      const float2 a = make_float2(a0[r], a1[r]);
      const float2 bq = __fmul2_rn(pq, a);                    // e^{G_t - E_{I-1}}
      const float2 bk = DECAY_FIRST ? bq : pq;                // e^{Gp_t - E_{I-1}}
      const float2 rw = make_float2(w0[r], w1[r]);            // e^{E_I - G_t}
      const float2 re = DECAY_FIRST ? rw : __fmul2_rn(rw, a); // e^{E_I - Gp_t}
      pq = bq;
      const float2 kw = __fmul2_rn(k, rw), ke = __fmul2_rn(k, re);
      const float2 kb = __fmul2_rn(k, bk), qb = __fmul2_rn(q, bq);
      const uint32_t rowK = (uint32_t)(32 * bI + 8 * rh + r) * 128 + x, rowQ = rowK + 16 * 128;
      if (!exact) {  // the exact Gram's images occupy this region
        // Gram right operand (keys scaled to the anchor)
        st4(rbase + rowK, __fmul2_rn(kw, rf));
        st4(rbase + rowQ, __fmul2_rn(ke, rf));
        // Gram left operand (rows scaled to the anchor)
        st4(lbase + rowK, __fmul2_rn(kb, fa));
        st4(lbase + rowQ, __fmul2_rn(qb, fa));
      }
      // K e^{Gp} over k, q e^{G} over q (same element, same owner), beta K e^{G_L - G|Gp}
      st4(kbase + koff, __fmul2_rn(kb, ei));
      st4(qbase + koff, __fmul2_rn(qb, ei));
      const float2 bge = __fmul2_rn(make_float2(b, b), ge);
      st4(abase + koff, __fmul2_rn(kw, bge));
      st4(bbase + koff, __fmul2_rn(ke, bge));
    }
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // ---- 4. Gram MMA: [K;Q] rows x 128 key columns (w and e of the four key
  //         sub-chunks), one M = 128, N = 128 product (the two anchors of an
  //         earlier form needed two N = 64 products: 8 more issues, prep 4.5 %
  //         slower) ----
  if (tid == 0) *s_exact = 0u;  // every thread holds its copy of the flag
  if ((tid == 0 || tid == 32) && exact) {
    mbar_arrive(bar_mma);  // the phase completes with no product: the exact Gram is written
  } else if (tid == 0) {
    constexpr uint32_t ID = idesc_bf16(128, 128, false, false);
    const uint32_t a_base = smem_u32(sX + X_LEFT), r_base = smem_u32(sX + X_R);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
      mma_bf16(tm + TM_GRAM, desc_kmajor(a_base, 16 * kk, LEFT_BLOCK),
               desc_kmajor(r_base, 16 * kk, 16384), ID, kk > 0);
    mma_commit(bar_mma);
    mma_commit(bar_mma);  // the phase counts two commits
  }
  __syncwarp();
  wait_bar(bar_mma, 0, hdr, KDA_DEVICE_TIMEOUT);
  tc_fence_after();

  // ---- 5. Gram readback: masked, beta-scaled, into the next operands ----
  // Warp (I = quad, J = qtr) holds rows of query/key sub-chunk I against keys of
  // sub-chunk J.  Blocks with J > I are zero; inside J == I the strict (keys) or
  // inclusive (queries) lower triangle survives.  Rows and keys past the chunk's
  // length are zero already (k = q = beta = 0 there).
  if (!exact) {
    const int I = quad, J = qtr, s = lane;
    const bool isK = s < 16;
    const int i = 16 * I + (s & 15);
    float* nae = reinterpret_cast<float *>(sX + X_NAE);
    float w[16], e[16];
    if (J <= I) {  // warp-uniform
      float v[32];
      tmem_ld32(taddr(tm, 32 * quad, TM_GRAM + 32 * J), v);
      float bj[16];
#pragma unroll
      for (int u = 0; u < 16; u += 4) {
        const float4 b4 = *reinterpret_cast<const float4 *>(sBeta + 16 * J + u);
        bj[u] = b4.x; bj[u + 1] = b4.y; bj[u + 2] = b4.z; bj[u + 3] = b4.w;
      }
      tmem_ld_wait();
      const int lim = J < I ? 16 : (isK ? (s & 15) : (s & 15) + 1);  // keys u < lim survive
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        w[u] = u < lim ? v[u] * bj[u] : 0.f;
        e[u] = u < lim ? v[16 + u] * bj[u] : 0.f;
      }
    } else {
#pragma unroll
      for (int u = 0; u < 16; ++u) w[u] = e[u] = 0.f;
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
      if (J <= I) {  // T^{-1} reads N only on and below the diagonal blocks
#pragma unroll
        for (int u = 0; u < 16; u += 4)
          *reinterpret_cast<float4 *>(nae + i * LDN + 16 * J + u) =
              make_float4(e[u], e[u + 1], e[u + 2], e[u + 3]);
      }
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
  fence_async_smem();  // the images are operands of the next products
  __syncthreads();
  } else {
  // ---- 2'. scalar gate: every decay factor is a per-token scalar, so the Gram
  //          products take the raw tiles and the factors are applied to the
  //          64 x 64 results.  [K; Q] K^T is issued as soon as the tiles land ----
  if (tid == 0) {
    tc_fence_after();
    constexpr uint32_t ID = idesc_bf16(128, 64, false, false);
    const uint32_t kq = smem_u32(sK);  // rows 0..63: k, rows 64..127: q
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
      mma_bf16(tm + TM_GRAM, desc_kmajor(kq, 16 * kk, QK_CB), desc_kmajor(kq, 16 * kk, QK_CB), ID,
               kk > 0);
    mma_commit(bar_mma);
    mma_commit(bar_mma);  // the phase counts two commits
  }
  // Per-token tables, warp 1 (lane: tokens 2 lane, 2 lane + 1).  G_t is the
  // in-chunk cumulative log-decay through t, Gp_t through t - 1, E_J its value
  // at the end of 16-token block J, G_L at the end of the chunk (g = 0 past
  // the chunk's length).  Every factor is e^{x} with x <= 0:
  //   a_t = e^{g_t}; e^{Gp_t} (K for W); e^{G_t} (q for Q');
  //   beta_t e^{G_L - G_t}, beta_t e^{G_L - Gp_t} (K_a, K_b);
  //   beta_t e^{E_J - G_t} (key column factor of the Gram blocks left of the diagonal).
  // Rows past the chunk's length get 0 in the tile factors.  (The exponentials
  // use the intrinsic: its error is far below the bf16 rounding every factor
  // meets in the operands.)
  float *tG = sPblk, *tGp = sPblk + 64, *tA = sPblk + 128, *tCW = sPblk + 192, *tE = sPblk + 256;
  float *tFK = sGsum, *tFQ = sGsum + 64, *tFA = sGsum + 128, *tFB = sGsum + 192;
  // diagonal-block factors [4 blocks][16 rows][kLdD] (the per-channel path's
  // half-sub-chunk scratch; no image copy reads it)
  constexpr int kLdD = 20;  // padded row: two-way bank conflicts at most
  float *tD = reinterpret_cast<float *>(sm + OFF_MISC + MISC_XP);
  if (warp == 1) {
    const int t0 = 2 * lane, t1 = t0 + 1;
    const float g0 = sGsc[t0], g1 = sGsc[t1];  // 0 past the chunk's length
    float incl = g0 + g1;  // inclusive scan of token pairs over the lanes
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    float excl = __shfl_up_sync(0xffffffffu, incl, 1);
    if (lane == 0) excl = 0.f;
    const float G0 = excl + g0, G1 = G0 + g1;
    const float GL = __shfl_sync(0xffffffffu, G1, 31);
    const float EJ = __shfl_sync(0xffffffffu, G1, lane | 7);  // end of this lane's 16-token block
    const float gle = __expf(GL);
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const int t = t0 + h2;
      const float Gt = h2 ? G1 : G0, Gpt = h2 ? G0 : excl, at = __expf(h2 ? g1 : g0);
      const bool ok = t < L;
      const float b = sBeta[t];  // 0 past the chunk's length
      const float fa = b * __expf(GL - Gt);
      tG[t] = Gt;
      tGp[t] = Gpt;
      tA[t] = at;
      tCW[t] = b * __expf(EJ - Gt);
      tFK[t] = ok ? __expf(Gpt) : 0.f;
      tFQ[t] = ok ? __expf(Gt) : 0.f;
      tFA[t] = fa;
      tFB[t] = fa * at;  // e^{G_L - Gp_t} = e^{G_L - G_t} e^{g_t}
      sGLe[t] = gle;
      sGLe[t + C] = gle;
    }
    if ((lane & 7) == 7) tE[lane >> 3] = G1;
  } else if (warp == 2 || warp == 3) {
    // Diagonal Gram blocks, row a of 16-token block I (thread 16 I + a; a
    // half-warp per block): D[I][a][b] = e^{Gp_{16I+a} - G_{16I+b}}, the product
    // of the decays a_s of tokens b < s < a (1 for b = a - 1, 0 for b >= a).
    // Products of factors <= 1: none overflows.
    const int I = (tid - 64) >> 4, a = (tid - 64) & 15;
    const float own = __expf(sGsc[16 * I + a]);  // a_{16I+a}
    float as[16];
#pragma unroll
    for (int s2 = 0; s2 < 16; ++s2) as[s2] = __shfl_sync(0xffffffffu, own, (lane & 16) | s2);
    float d[16], prod = 1.f;
    d[15] = 0.f;
#pragma unroll
    for (int b2 = 14; b2 >= 0; --b2) {
      prod = (b2 + 1 < a) ? prod * as[b2 + 1] : 1.f;
      d[b2] = (b2 < a) ? prod : 0.f;
    }
    float4 *row = reinterpret_cast<float4 *>(tD + (16 * I + a) * kLdD);
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) row[q4] = make_float4(d[4 * q4], d[4 * q4 + 1], d[4 * q4 + 2], d[4 * q4 + 3]);
  }
  __syncthreads();
  if (tid == kIoThread && next < total) {
    load_g(next, ce_next);
    if (next + (int)gridDim.x < total) prefetch_l2(next + gridDim.x, ce_next2);
  }
  // ---- 3'. while the Gram runs: the row-scaled tiles the later products read,
  //          in the per-channel path's layout: k e^{Gp} and q e^{G} (in the g
  //          buffer, which a scalar gate does not use), beta k e^{G_L - G} and
  //          beta k e^{G_L - Gp}.  Thread: channels c4 .. c4 + 3 (8 bytes,
  //          inside one swizzled 16-byte chunk), rows 4 rg .. +3; a warp covers
  //          one whole 256-byte row ----
  {
    const int c4 = (tid & 31) * 4, rg = tid >> 5;
    const uint32_t cblk = (uint32_t)(c4 >> 6), cpos = (uint32_t)(c4 & 63) * 2;
    const unsigned char *const kr = sK + cblk * QK_CB, *const qr = sQ + cblk * QK_CB;
    unsigned char *const kd = sm + OFF_G + cblk * 8192, *const qd = sm + OFF_G + 16384 + cblk * 8192;
    unsigned char *const ab = sm + OFF_KAB + cblk * 8192, *const bb = sm + OFF_KBB + cblk * 8192;
    auto scaled = [](float2 x0, float2 x1, float f) {
      const float2 ff = make_float2(f, f);
      const float2 y0 = __fmul2_rn(x0, ff), y1 = __fmul2_rn(x1, ff);
      return make_uint2(pack_bf16x2(y0.x, y0.y), pack_bf16x2(y1.x, y1.y));
    };
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int t = 4 * rg + r;
      const uint32_t koff = (uint32_t)t * 128 + (cpos ^ ((uint32_t)(t & 7) << 4));
      const uint2 kraw = *reinterpret_cast<const uint2 *>(kr + koff);
      const uint2 qraw = *reinterpret_cast<const uint2 *>(qr + koff);
      const float2 k0 = make_float2(bf16_lo(kraw.x), bf16_hi(kraw.x));
      const float2 k1 = make_float2(bf16_lo(kraw.y), bf16_hi(kraw.y));
      const float2 q0 = make_float2(bf16_lo(qraw.x), bf16_hi(qraw.x));
      const float2 q1 = make_float2(bf16_lo(qraw.y), bf16_hi(qraw.y));
      *reinterpret_cast<uint2 *>(kd + koff) = scaled(k0, k1, tFK[t]);
      *reinterpret_cast<uint2 *>(qd + koff) = scaled(q0, q1, tFQ[t]);
      *reinterpret_cast<uint2 *>(ab + koff) = scaled(k0, k1, tFA[t]);
      *reinterpret_cast<uint2 *>(bb + koff) = scaled(k0, k1, tFB[t]);
    }
  }
  __syncwarp();
  wait_bar(bar_mma, 0, hdr, KDA_DEVICE_TIMEOUT);
  // The readback is the first to rebuild the X region (the tables and tiles
  // above live elsewhere): only now must the previous item's image copies have
  // read it, so their reads overlap this item's tables and image pass.
  if (tid == kIoThread) bulk_wait_read0();
  __syncthreads();
  tc_fence_after();

  // ---- 5'. Gram readback: TMEM lane r < 64 is key row i = r, lane 64 + t query
  //          row t; column j is key j.  Warp (quad, qtr) takes 32 rows and key
  //          columns 16 qtr .. +15 (block J = qtr).  With the row term Gp_i
  //          (keys) or G_t (queries):
  //            w = raw beta_j e^{row - G_j}   (A_w beta, B_w beta)
  //            e = raw beta_j e^{row - Gp_j} = w a_j   (A_e beta, B_e beta)
  //          keys j < i, queries j <= t, rows past the chunk's length zero.
  //          Left of the diagonal block the factor splits at E_J into a row
  //          and a column factor, both <= 1; inside it each factor is one exp.
  //          The same images and N as the per-channel path ----
  {
    const bool isQ = quad >= 2;
    const int r = 32 * (quad & 1) + lane, J = qtr, I = r >> 4;
    float *nae = reinterpret_cast<float *>(sX + X_NAE);
    float w[16], e[16];
    if (J <= 2 * (quad & 1) + 1) {  // warp-uniform: some row of the warp reaches block J
      float v[16], cf[16], aj[16];
      tmem_ld16(taddr(tm, 32 * quad, TM_GRAM + 16 * J), v);
      const bool diag = J == I;
#pragma unroll
      for (int u = 0; u < 16; u += 4) {
        // diagonal block: beta_j and G_j; left of it: beta_j e^{E_J - G_j}
        const float4 c4 = *reinterpret_cast<const float4 *>((diag ? sBeta : tCW) + 16 * J + u);
        const float4 a4 = *reinterpret_cast<const float4 *>(tA + 16 * J + u);
        cf[u] = c4.x; cf[u + 1] = c4.y; cf[u + 2] = c4.z; cf[u + 3] = c4.w;
        aj[u] = a4.x; aj[u + 1] = a4.y; aj[u + 2] = a4.z; aj[u + 3] = a4.w;
      }
      const float rowg = isQ ? tG[r] : tGp[r];
      const bool rowok = r < L && J <= I;
      const float rowf = (rowok && !diag) ? __expf(rowg - tE[J]) : 0.f;
      tmem_ld_wait();
      if (diag) {
        // keys: beta_j D[a][u]; queries: beta_j D[a][u] a_t for u < a, beta_t at u = a
        const int a = r & 15;
        const float4 *drow = reinterpret_cast<const float4 *>(tD + r * kLdD);
        const float rf = !rowok ? 0.f : isQ ? tA[r] : 1.f;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const float4 d4 = drow[q4];
          const float dd[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const int u = 4 * q4 + k4;
            const float f = (isQ && u == a) ? (rowok ? 1.f : 0.f) : dd[k4] * rf;
            w[u] = v[u] * cf[u] * f;
            e[u] = w[u] * aj[u];
          }
        }
      } else {
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          w[u] = v[u] * rowf * cf[u];
          e[u] = w[u] * aj[u];
        }
      }
    } else {
#pragma unroll
      for (int u = 0; u < 16; ++u) w[u] = e[u] = 0.f;
    }
    const int row_w = isQ ? 64 + r : r;
#pragma unroll
    for (int hseg = 0; hseg < 2; ++hseg) {
      float x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) x[u] = w[8 * hseg + u];
      st16(sX + X_AWBW + kmajor_off(row_w, 16 * J + 8 * hseg), pack8(x));
    }
    if (!isQ) {
      if (J <= I) {  // T^{-1} reads N only on and below the diagonal blocks
#pragma unroll
        for (int u = 0; u < 16; u += 4)
          *reinterpret_cast<float4 *>(nae + r * LDN + 16 * J + u) =
              make_float4(e[u], e[u + 1], e[u + 2], e[u + 3]);
      }
    } else {
#pragma unroll
      for (int hseg = 0; hseg < 2; ++hseg) {
        float x[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) x[u] = e[8 * hseg + u];
        st16(sX + X_BE + kmajor_off(r, 16 * J + 8 * hseg), pack8(x));
      }
    }
  }
  fence_async_smem();  // the images are operands of the next products
  __syncthreads();
  // the raw q, k tiles are consumed (Gram and image pass): the next item's load now
  if (tid == kIoThread && next < total) load_qk(next, ce_next, false);
  }  // scalar gate

  if (tid == 0) s_fail[(it + 1) & 1] = 0u;  // the previous item's flag, read by now
  // ---- 6. products that need no T^{-1}, issued before it is built:
  //         Y^T = V^T (A_w beta)^T;  O_intra = tril(B_w) beta V (rows t < 64 of an
  //         M = 128 product whose upper 64 rows read the bytes after the operand
  //         and are discarded);  Qc = (beta K e^{G_L-G})^T V.  With these v is
  //         read for the last time ----
  if (tid == 256) {
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_bf16(tm + TM_Y, desc_mnmajor(smem_u32(sV), 16 * kk, 8192),
               desc_kmajor(smem_u32(sX + X_AWBW), 16 * kk, 0), idesc_bf16(128, 64, true, false),
               kk > 0);
    mma_commit(bar_yo);
  } else if (tid == 288) {
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_bf16(tm + TM_OI, desc_kmajor(smem_u32(sX + X_AWBW + 64 * 128), 16 * kk, 0),
               desc_mnmajor(smem_u32(sV), 16 * kk, 8192), idesc_bf16(128, 128, false, true),
               kk > 0);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_bf16(tm + TM_QC, desc_mnmajor(smem_u32(sm + OFF_KAB), 16 * kk, 8192),
               desc_mnmajor(smem_u32(sV), 16 * kk, 8192), idesc_bf16(128, 128, true, true),
               kk > 0);
    mma_commit(bar_yo);
  }

  if (warp < 8) {
    // ---- 7. T^{-1}, T = I + N, N = tril_{-1}(A_e) diag(beta) (blocked, fp32), warps 0-7 ----
    // Unit lower triangular, so T^{-1} is built block by block:
    //   diagonal 16x16 blocks by forward substitution (fp32, one thread per column);
    //   T^{-1}[h][l] = -T^{-1}[h][h] N[h][l] T^{-1}[l][l] for the 16x16 blocks below
    //   the diagonal pairs, then for the lower-left 32x32 block.  The block
    //   products are warp-level tf32 MMAs with fp32 accumulation: too small for
    //   the CTA-wide tensor-core path, and tf32 (10-bit mantissa) keeps them well
    //   inside the bf16 rounding every T^{-1} entry gets afterwards.
    constexpr int kTinvBar = 2, kTinvThreads = 256;
    const float *nae = reinterpret_cast<const float *>(sX + X_NAE);
    float *tinv = reinterpret_cast<float *>(sX + X_TINVF);
    float *tmp = reinterpret_cast<float *>(sX + X_TINVB);  // fp32 scratch, row stride LDT
    // (a) column c of the inverse of diagonal block b: x_i = [i == c] - sum_{j<i} N_ij x_j
    if (tid < 64) {
      const int b = tid >> 4, c = tid & 15;
      const float *nb = nae + 16 * b * LDN + 16 * b;
      float x[16];
      x[0] = (c == 0) ? 1.f : 0.f;
#pragma unroll
      for (int i = 1; i < 16; ++i) {
        float row[16];
#pragma unroll
        for (int q4 = 0; q4 < (i + 3) / 4; ++q4) {
          const float4 r4 = *reinterpret_cast<const float4 *>(nb + i * LDN + 4 * q4);
          row[4 * q4] = r4.x; row[4 * q4 + 1] = r4.y; row[4 * q4 + 2] = r4.z; row[4 * q4 + 3] = r4.w;
        }
        float acc = (i == c) ? 1.f : 0.f;
#pragma unroll
        for (int j = 0; j < i - 1; ++j) acc = fmaf(-row[j], x[j], acc);
        x[i] = fmaf(-row[i - 1], x[i - 1], acc);  // the newest term last: short chain
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) tinv[(16 * b + i) * LDN + 16 * b + c] = x[i];
    }
    named_bar_sync(kTinvBar, kTinvThreads);
    // (b) the two 16x16 blocks T^{-1}[16p+16][16p] (p = 0, 2): warp w < 4 owns
    //     pair w >> 1 and 8 output columns (w & 1)
    if (warp < 4) {
      const int R0 = 32 * (warp >> 1) + 16, C0 = R0 - 16, n0 = 8 * (warp & 1);
      float *tp = tmp + (warp >> 1) * 16 * LDT;
      float d[4] = {0.f, 0.f, 0.f, 0.f};
      warp_mma_tf32<16>(d, nae + R0 * LDN + C0, LDN, tinv + C0 * LDN + C0 + n0, LDN, lane);
      store_frag(tp + n0, LDT, d, lane);
      named_bar_sync(1, 128);
      float e[4] = {0.f, 0.f, 0.f, 0.f};
      warp_mma_tf32<16>(e, tinv + R0 * LDN + R0, LDN, tp + n0, LDT, lane);
      e[0] = -e[0]; e[1] = -e[1]; e[2] = -e[2]; e[3] = -e[3];
      store_frag(tinv + R0 * LDN + C0 + n0, LDN, e, lane);
    }
    named_bar_sync(kTinvBar, kTinvThreads);
    // (c) the lower-left 32x32 block: warp w < 8 owns rows 16 (w >> 2) .. +16 and
    //     columns 8 (w & 3) .. +8; zero blocks of the triangular factors are skipped
    {
      const int m0 = 16 * (warp >> 2), n0 = 8 * (warp & 3);
      float d[4] = {0.f, 0.f, 0.f, 0.f};
      // tmp = N[32..63][0..31] T^{-1}[0..31][0..31]: rows k < n0 of the right factor are 0
      warp_mma_tf32_range<4>(d, nae + (32 + m0) * LDN, LDN, tinv, LDN, n0, n0 & ~7, 32, lane);
      store_frag(tmp + m0 * LDT + n0, LDT, d, lane);
      named_bar_sync(kTinvBar, kTinvThreads);
      float e[4] = {0.f, 0.f, 0.f, 0.f};
      // T^{-1}[32..63][32..63] tmp: columns k >= m0 + 16 of the left factor are 0
      warp_mma_tf32_range<4>(e, tinv + (32 + m0) * LDN + 32, LDN, tmp, LDT, n0, 0, m0 + 16, lane);
      e[0] = -e[0]; e[1] = -e[1]; e[2] = -e[2]; e[3] = -e[3];
      store_frag(tinv + (32 + m0) * LDN + n0, LDN, e, lane);
    }
    named_bar_sync(kTinvBar, kTinvThreads);
    // bf16 copy, K-major [i][j]; blocks above the diagonal are zero.  Thread
    // (i, j8): row i, columns 8 j8 .. +7 (rows are 16-byte aligned: LDN = 68)
    for (int item = tid; item < 64 * 8; item += kTinvThreads) {
      const int i = item & 63, j = (item >> 6) * 8;
      const bool upper = (j >> 4) > (i >> 4);
      const float4 *src = reinterpret_cast<const float4 *>(tinv + i * LDN + j);
      const float4 x0 = upper ? make_float4(0.f, 0.f, 0.f, 0.f) : src[0];
      const float4 x1 = upper ? make_float4(0.f, 0.f, 0.f, 0.f) : src[1];
      st16(sX + X_TINVB + kmajor_off(i, j),
           make_uint4(pack_bf16x2(x0.x, x0.y), pack_bf16x2(x0.z, x0.w), pack_bf16x2(x1.x, x1.y),
                      pack_bf16x2(x1.z, x1.w)));
    }
  } else {
    // warps 8-15, meanwhile: Y (lanes n, cols i) -> K-major [n][t]
    wait_bar(bar_yo, it & 1, hdr, KDA_DEVICE_TIMEOUT);
    // the step-6 products were the last to read v: the next item's v tile now
    if (tid == kIoThread && next < total) load_v(next, ce_next, !CHANNEL);
    tc_fence_after();
    const int cg = (warp >> 2) - 2;  // column group: 32 cg .. +31
    float v[32];
    tmem_ld32(taddr(tm, 32 * quad, TM_Y + 32 * cg), v);
    tmem_ld_wait();
#pragma unroll
    for (int seg = 0; seg < 4; ++seg) {
      float x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) x[u] = v[8 * seg + u];
      st16(sX + X_Y + kmajor_off(lane_row, 32 * cg + 8 * seg), pack8(x));
    }
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // ---- 8. W^T = (K e^{Gp})^T T^{-T};  U^T = Y^T T^{-T} ----
  if (tid == 0) {
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_bf16(tm + TM_W, desc_mnmajor(smem_u32(sKd), 16 * kk, 8192),
               desc_kmajor(smem_u32(sX + X_TINVB), 16 * kk, 0), idesc_bf16(128, 64, true, false),
               kk > 0);
    mma_commit(bar_mma);
  } else if (tid == 32) {
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_bf16(tm + TM_U, desc_kmajor(smem_u32(sX + X_Y), 16 * kk, 0),
               desc_kmajor(smem_u32(sX + X_TINVB), 16 * kk, 0), idesc_bf16(128, 64, false, false),
               kk > 0);
    mma_commit(bar_mma);
  }
  __syncwarp();
  wait_bar(bar_mma, 1, hdr, KDA_DEVICE_TIMEOUT);
  tc_fence_after();
  {
    // W (lanes c, cols t) -> K-major [c][t]; U (lanes n, cols t) -> K-major [n][t]
    float v[16], v2[16];
    tmem_ld16(taddr(tm, 32 * quad, TM_W + 16 * qtr), v);
    tmem_ld16(taddr(tm, 32 * quad, TM_U + 16 * qtr), v2);
    tmem_ld_wait();
#pragma unroll
    for (int seg = 0; seg < 2; ++seg) {
      float x[8], y[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        x[u] = v[8 * seg + u];
        y[u] = v2[8 * seg + u];
      }
      st16(sX + X_W + kmajor_off(lane_row, 16 * qtr + 8 * seg), pack8(x));
      st16(sX + X_U + kmajor_off(lane_row, 16 * qtr + 8 * seg), pack8(y));
    }
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  // ---- 9. one thread, in this order: K_b^T beta W (for P), X = W^T (B_e beta)^T
  //         (for Q'), then O_intra -= tril(B_e) beta U (M = 128 as in step 6) and
  //         Qc -= (beta K e^{G_L-Gp})^T U (lanes i, columns j).  Products issue one
  //         at a time whatever thread issues them, so a single issuer puts P and
  //         X, whose readback comes first, ahead of the other two (from two
  //         threads they interleave: prep 1.2-2.7 % slower) ----
  if (tid == 32) {
    const uint32_t wsm = smem_u32(sX + X_W), usm = smem_u32(sX + X_U);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_bf16(tm + TM_P, desc_mnmajor(smem_u32(sm + OFF_KBB), 16 * kk, 8192), desc_kmajor(wsm, 16 * kk, 0),
               idesc_bf16(128, 128, true, false), kk > 0);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_bf16(tm + TM_X, desc_kmajor(wsm, 16 * kk, 0), desc_kmajor(smem_u32(sX + X_BE), 16 * kk, 0),
               idesc_bf16(128, 64, false, false), kk > 0);
    mma_commit(bar_px);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_bf16(tm + TM_OI, desc_kmajor(smem_u32(sX + X_BE), 16 * kk, 0), desc_kmajor(usm, 16 * kk, 0),
               idesc_bf16(128, 128, false, false, true), 1);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk)
      mma_bf16(tm + TM_QC, desc_mnmajor(smem_u32(sm + OFF_KBB), 16 * kk, 8192),
               desc_kmajor(usm, 16 * kk, 0), idesc_bf16(128, 128, true, false, true), 1);
    mma_commit(bar_oq);
  }
  __syncwarp();
  wait_bar(bar_px, it & 1, hdr, KDA_DEVICE_TIMEOUT);
  tc_fence_after();
  // P and Q' leave TMEM for the slot while the last products run (disjoint columns)
  {
    float v[32], x16[16];
    tmem_ld32(taddr(tm, 32 * quad, TM_P + 32 * qtr), v);
    tmem_ld16(taddr(tm, 32 * quad, TM_X + 16 * qtr), x16);
    tmem_ld_wait();
    // P = Diag(e^{G_L}) - K_b^T beta W (lanes i, cols c) -> K-major A image [i][c]
    const int i = lane_row;
    const float gl = sGLe[i];
#pragma unroll
    for (int seg = 0; seg < 4; ++seg) {
      float x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int c = 32 * qtr + 8 * seg + u;
        x[u] = (c == i ? gl : 0.f) - v[8 * seg + u];
      }
      const int c = 32 * qtr + 8 * seg;
      st16(sX + X_PI + (c >> 6) * 16384 + kmajor_off(i, c & 63), pack8(x));
    }
    // Q'[t][c] = q_tc e^{G_tc} - X[c][t] (lanes c, cols t) -> MN-major A image [c][t]
    const int c = lane_row;
#pragma unroll
    for (int seg = 0; seg < 2; ++seg) {
      float x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int t = 16 * qtr + 8 * seg + u;
        const float qg = ld_bf16(sQd, (c >> 6) * 8192 + kmajor_off(t, c & 63));  // q e^{G}
        x[u] = (t < L) ? qg - x16[8 * seg + u] : 0.f;
      }
      st16(sX + X_QPI + sw128((uint32_t)(c * 128 + (16 * qtr + 8 * seg) * 2)), pack8(x));
    }
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();  // the P / Q' images are written
  tc_fence_after();
  const bool slot_ok = tid != kIoThread || GDR_IN_BOUNDS(chunk < chunks.max_chunks);
  if (tid == kIoThread && slot_ok) {  // P and Q' images -> workspace slot
    bulk_s2g(slot + SLOT_P, sX + X_PI, 32768);
    bulk_s2g(slot + SLOT_QP, sX + X_QPI, 16384);
  }
  if (tid == kIoThread) {
    bulk_commit();
    if (CHANNEL && next < total) load_qk(next, ce_next, true);  // Q' has read the q tile
  }
  wait_bar(bar_oq, it & 1, hdr, KDA_DEVICE_TIMEOUT);
  tc_fence_after();
  {
    // warp (quad, qtr) holds rows 32 quad + lane, value columns 32 qtr .. +31,
    // i.e. one row of column slice qtr
    float v[32];
    tmem_ld32(taddr(tm, 32 * quad, TM_QC + 32 * qtr), v);
    tmem_ld_wait();
#pragma unroll
    for (int seg = 0; seg < 4; ++seg) {  // Qc rows i
      float x[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) x[u] = v[8 * seg + u];
      st16(sX + X_QCI + qtr * QC_SLICE_BYTES + slice_off(lane_row, seg), pack8(x));
    }
    if (quad < 2) {  // O_intra rows t < 64 (lanes 64..127 hold the discarded rows)
      tmem_ld32(taddr(tm, 32 * quad, TM_OI + 32 * qtr), v);
      tmem_ld_wait();
#pragma unroll
      for (int seg = 0; seg < 4; ++seg) {
        float x[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) x[u] = v[8 * seg + u];
        st16(sX + X_OII + qtr * OI_SLICE_BYTES + slice_off(lane_row, seg), pack8(x));
      }
    }
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (tid == kIoThread && slot_ok) {  // Qc and O_intra images -> workspace slot
    bulk_s2g(slot + SLOT_QC, sX + X_QCI, 32768);
    bulk_s2g(slot + SLOT_OI, sX + X_OII, 16384);
    bulk_commit();
  }
  ce = ce_next;
  ce_next = ce_next2;
  }  // work items

  // a wait in the last item may have expired after the final verdict
  aborted = __syncthreads_or(aborted || failed) != 0;
  if (aborted) {
    // Nothing may still write this CTA's shared memory or TMEM when it exits:
    // the issuing threads' last products finish (a commit arrives once every
    // earlier tcgen05 op of its thread is done), and every TMA phase kIoThread
    // armed (or began to fill without arming) lands.  All waits stay bounded.
    if (tid == 0 || tid == 32 || tid == 256 || tid == 288) mma_commit(bar_drain);
    if (tid == kIoThread) {
      if (tma_partial) {
        mbar_arrive(bar_tma);
        ++tma_armed;
      }
      // phases before tma_done (g_done) were waited for in their items
      for (int ph = tma_done; ph < tma_armed; ++ph)
        mbar_wait(bar_tma, ph & 1, hdr, KDA_DEVICE_TIMEOUT);
      for (int ph = g_done; ph < g_armed; ++ph)
        mbar_wait(bar_g, ph & 1, hdr, KDA_DEVICE_TIMEOUT);
    }
    mbar_wait(bar_drain, 0, hdr, KDA_DEVICE_TIMEOUT);
  }
  if (tid == kIoThread) bulk_wait0();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tm, 512);
}

// ---------------------------------------------------------------------------
// scan kernel
// ---------------------------------------------------------------------------
// The columns of the state never interact (every chunk map multiplies S from
// the left), so a (sequence, v-head) chain is split into 128 / NS column
// slices, one CTA each.  Per chunk u a CTA computes, for its NS columns,
//     S_{u+1} = P_u S_u + Qc_u        o_u = Q'_u S_u + O_intra_u
// with S_u in bf16 as the MN-major B operand in shared memory, P_u (K-major,
// M = 128) and Q'_u (MN-major, M = 64) as A operands, fp32 accumulators in
// TMEM and the fp32 state in registers of the chain warps.  Roles, connected
// by mbarriers:
//   chain warps 0-3 : S_{u+1} = (P S)_u + Qc_u, row i = TMEM lane i
//   output warps 4-7: o_u = (Q' S)_u + O_intra_u; an M = 64 product leaves
//                     rows 16 q .. 16 q + 15 in TMEM lanes 32 q .. 32 q + 15,
//                     so warp 4 + q (lane quarter q) stores them from lanes 0-15
//   MMA warp 8      : the two products of each chunk
//   load warp 9     : chunk slots into kStages stages (bulk copies)
template <int NS>
struct ScanCfg {
  static constexpr int kSlices = NS / 32;   // 32-column image slices per CTA
  static constexpr int kStages = NS == 32 ? 3 : 2;
  static constexpr uint32_t QC_BYTES = QC_SLICE_BYTES * kSlices;
  static constexpr uint32_t OI_BYTES = OI_SLICE_BYTES * kSlices;
  static constexpr uint32_t ST_P = 0, ST_QP = 32768, ST_QC = 49152, ST_OI = ST_QC + QC_BYTES;
  static constexpr uint32_t ST_BYTES = ST_OI + OI_BYTES;  // 60 KB / 72 KB
  static constexpr uint32_t SB_BYTES = 128 * NS * 2;     // bf16 state operand [c][NS]
  static constexpr uint32_t OFF_SB = kStages * ST_BYTES;  // two state operand buffers
  static constexpr uint32_t OFF_MISC = OFF_SB + 2 * SB_BYTES;
  static constexpr uint32_t SMEM = OFF_MISC + 256 + 1024;
  static constexpr uint32_t TD_S = 0, TD_O = NS;          // TMEM columns: (P S), (Q' S) x 2
  static constexpr uint32_t TMEM_COLS = NS == 32 ? 128 : 256;
};
constexpr int kScanThreads = 320;
constexpr int kScanMmaWarp = 8, kScanLoadWarp = 9;
constexpr uint32_t kScanEmptyCount = 128 + 128 + 1;  // chain + output threads + MMA commit

// byte offset of the 16-byte chunk `ch` of state-operand row c (MN-major, NS columns)
template <int NS>
__device__ __forceinline__ uint32_t sop_off(int c, int ch) {
  return NS == 32 ? sw64((uint32_t)(c * 64 + ch * 16)) : sw128((uint32_t)(c * 128 + ch * 16));
}
template <int NS>
__device__ __forceinline__ uint64_t sop_desc(uint32_t base, int kk) {
  return NS == 32 ? desc_mnmajor32(base, 16 * kk) : desc_mnmajor(base, 16 * kk, 16384);
}

template <int NS>
__global__ void __launch_bounds__(kScanThreads, 1)
chunk_scan_kernel(const int32_t *hdr, const Chunks chunks, const unsigned char *__restrict__ slots, __nv_bfloat16 *__restrict__ o,
                  const float *s0, float *sT, const int32_t *__restrict__ state_slots,
                  int64_t num_slots, int H_v, int32_t *err) {
  using Cfg = ScanCfg<NS>;
  constexpr int NSL = 128 / NS;  // CTAs per (sequence, v-head)
  constexpr int S = Cfg::kStages;
  extern __shared__ unsigned char smem_raw[];
  unsigned char *sm = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t *full = reinterpret_cast<uint64_t *>(sm + Cfg::OFF_MISC);  // [S] loads landed
  uint64_t *empty = full + S;         // [S] stage consumed (chain, output, MMA commit)
  uint64_t *sb_ready = empty + S;     // [2] state operand written (chain)
  uint64_t *ds_full = sb_ready + 2;   // (P S) done (commit)
  uint64_t *do_full = ds_full + 1;    // [2] (Q' S) done (commit)
  uint64_t *do_free = do_full + 2;    // [2] (Q' S) read (output)
  uint64_t *drain = do_free + 2;      // final commit of the MMA warp
  uint32_t *tslot = reinterpret_cast<uint32_t *>(sm + Cfg::OFF_MISC + 192);

  if (hdr[0] != KDA_DEVICE_OK) return;
  const int cid = blockIdx.x;
  const int sl = cid % NSL, h = (cid / NSL) % H_v;
  const int n = chunks.seq(cid / (NSL * H_v));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c_begin = chunks.first(n), nch = chunks.first(n + 1) - c_begin;

  if (warp == 0) {
    tmem_alloc(tslot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    for (int st = 0; st < S; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], kScanEmptyCount);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sb_ready[b], 128);
      mbar_init(&do_full[b], 1);
      mbar_init(&do_free[b], 128);
    }
    mbar_init(ds_full, 1);
    mbar_init(drain, 1);
    mbar_fence_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = *tslot;
  // the state's pool slot; a slot outside the pool starts from zeros and keeps no final state
  const int64_t sslot = state_slots ? (int64_t)state_slots[n] : (int64_t)n;
  if (sslot < 0 || sslot >= num_slots) {
    s0 = nullptr;
    sT = nullptr;
  }
  const size_t state_base = ((size_t)sslot * H_v + h) * DK * DK + (size_t)sl * NS;
  auto slot_of = [&](int u) {  // (slot 0 in place of one outside the table: counted, not read)
    const bool ok = GDR_IN_BOUNDS((int64_t)c_begin + u < chunks.max_chunks);
    return slots + (ok ? ((size_t)(c_begin + u) * H_v + h) * SLOT_BYTES : 0);
  };

  if (warp == kScanLoadWarp) {
    // ---------------- loads ----------------
    if (lane == 0) {
      // chunks prefetched into L2 ahead of their stage load: 2 measured best
      // (further ahead, many chains' prefetches evict each other from L2)
      constexpr int kAhead = 2;
      auto prefetch = [&](int u) {
        const unsigned char *src = slot_of(u);
        bulk_prefetch_l2(src + SLOT_P, 49152);  // P and Q'
        bulk_prefetch_l2(src + SLOT_QC + sl * Cfg::QC_BYTES, Cfg::QC_BYTES);
        bulk_prefetch_l2(src + SLOT_OI + sl * Cfg::OI_BYTES, Cfg::OI_BYTES);
      };
      for (int u = 0; u < kAhead && u < nch; ++u) prefetch(u);
      int issued = 0;
      for (int u = 0; u < nch; ++u) {
        const int st = u % S;
        if (u + kAhead < nch) prefetch(u + kAhead);
        if (u >= S && !mbar_wait(&empty[st], ((u / S) - 1) & 1, err, KDA_DEVICE_TIMEOUT)) break;
        unsigned char *dst = sm + st * Cfg::ST_BYTES;
        const unsigned char *src = slot_of(u);
        mbar_arrive_expect_tx(&full[st], Cfg::ST_BYTES);
        bulk_g2s(dst + Cfg::ST_P, src + SLOT_P, 49152, &full[st]);
        bulk_g2s(dst + Cfg::ST_QC, src + SLOT_QC + sl * Cfg::QC_BYTES, Cfg::QC_BYTES, &full[st]);
        bulk_g2s(dst + Cfg::ST_OI, src + SLOT_OI + sl * Cfg::OI_BYTES, Cfg::OI_BYTES, &full[st]);
        issued = u + 1;
      }
      // no copy may still be writing this CTA's shared memory when it exits
      for (int u = (issued > S ? issued - S : 0); u < issued; ++u)
        mbar_wait(&full[u % S], (u / S) & 1, err, KDA_DEVICE_TIMEOUT);
    }
  } else if (warp == kScanMmaWarp) {
    // ---------------- tensor-core issue ----------------
    // The whole warp runs the loop and computes the operand descriptors
    // (warp-uniform values); one elected lane issues the products.
    constexpr uint32_t idS = idesc_bf16(128, NS, false, true);  // P K-major, S MN-major
    constexpr uint32_t idO = idesc_bf16(64, NS, true, true);    // Q' MN-major, S MN-major, M = 64
    // descriptors of K-slice 0 for every stage and operand buffer, built once;
    // K-slice kk adds its byte offset / 16 to the start-address field
    uint64_t dP[S], dQ[S], dS[2];
#pragma unroll
    for (int st = 0; st < S; ++st) {
      const uint32_t stage = smem_u32(sm + st * Cfg::ST_BYTES);
      dP[st] = desc_kmajor(stage + Cfg::ST_P, 0, 16384);
      dQ[st] = desc_mnmajor(stage + Cfg::ST_QP, 0, 16384);
    }
#pragma unroll
    for (int b = 0; b < 2; ++b) dS[b] = sop_desc<NS>(smem_u32(sm + Cfg::OFF_SB + b * Cfg::SB_BYTES), 0);
    constexpr uint32_t kSOp = NS == 32 ? 64 : 128;  // state operand: 16-byte units per K-slice
    for (int u = 0; u < nch; ++u) {
      const int st = u % S, b = u & 1;
      if (!mbar_wait_warp(&full[st], (u / S) & 1, err, KDA_DEVICE_TIMEOUT)) break;
      if (!mbar_wait_warp(&sb_ready[b], (u >> 1) & 1, err, KDA_DEVICE_TIMEOUT)) break;
      tc_fence_after();
      const uint64_t p0 = st == 0 ? dP[0] : (st == 1 ? dP[1] : dP[S - 1]);
      const uint64_t q0 = st == 0 ? dQ[0] : (st == 1 ? dQ[1] : dQ[S - 1]);
      const uint64_t s0d = b ? dS[1] : dS[0];
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16(tm + Cfg::TD_S, p0 + (uint64_t)((kk >> 2) * 1024 + (kk & 3) * 2),
                   s0d + (uint64_t)(kk * kSOp), idS, kk > 0);
        mma_commit(ds_full);
      }
      __syncwarp();
      if (u >= 2 && !mbar_wait_warp(&do_free[b], ((u - 2) >> 1) & 1, err, KDA_DEVICE_TIMEOUT)) break;
      tc_fence_after();
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_bf16(tm + Cfg::TD_O + NS * b, q0 + (uint64_t)(kk * 128), s0d + (uint64_t)(kk * kSOp),
                   idO, kk > 0);
        mma_commit(&do_full[b]);
        mma_commit(&empty[st]);
      }
      __syncwarp();
    }
    // every issued product has finished before TMEM is released
    if (elect_one()) mma_commit(drain);
    __syncwarp();
    mbar_wait_warp(drain, 0, err, KDA_DEVICE_TIMEOUT);
  } else if (warp < 4) {
    // ---------------- the state chain: row i, NS columns ----------------
    const int i = 32 * warp + lane;
    float Sr[NS];
    if (s0) {
#pragma unroll
      for (int j = 0; j < NS; j += 4) {
        const float4 x = *reinterpret_cast<const float4 *>(s0 + state_base + (size_t)i * DK + j);
        Sr[j] = x.x; Sr[j + 1] = x.y; Sr[j + 2] = x.z; Sr[j + 3] = x.w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < NS; ++j) Sr[j] = 0.f;
    }
    auto write_operand = [&](int b) {  // row i of S in bf16 -> MN-major B operand
      unsigned char *sb = sm + Cfg::OFF_SB + b * Cfg::SB_BYTES;
#pragma unroll
      for (int ch = 0; ch < NS / 8; ++ch) {
        float x[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = Sr[8 * ch + e];
        st16(sb + sop_off<NS>(i, ch), pack8(x));
      }
      fence_async_smem();
    };
    if (nch > 0) {
      write_operand(0);
      mbar_arrive(&sb_ready[0]);
    }
    for (int u = 0; u < nch; ++u) {
      const int st = u % S;
      // this chunk's Qc rows, read while the product runs
      if (!mbar_wait(&full[st], (u / S) & 1, err, KDA_DEVICE_TIMEOUT)) break;
      uint4 qv[NS / 8];
      const unsigned char *qc = sm + st * Cfg::ST_BYTES + Cfg::ST_QC;
#pragma unroll
      for (int p = 0; p < NS / 32; ++p)
#pragma unroll
        for (int ch = 0; ch < 4; ++ch)
          qv[4 * p + ch] = *reinterpret_cast<const uint4 *>(qc + p * QC_SLICE_BYTES + slice_off(i, ch));
      if (!mbar_wait(ds_full, u & 1, err, KDA_DEVICE_TIMEOUT)) break;
      tc_fence_after();
      float v[NS];
#pragma unroll
      for (int p = 0; p < NS / 32; ++p)
        tmem_ld32(taddr(tm, 32 * warp, Cfg::TD_S + 32 * p), *reinterpret_cast<float(*)[32]>(&v[32 * p]));
      tmem_ld_wait();
      tc_fence_before();
#pragma unroll
      for (int c8 = 0; c8 < NS / 8; ++c8) {
        const uint32_t ww[4] = {qv[c8].x, qv[c8].y, qv[c8].z, qv[c8].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          Sr[8 * c8 + 2 * e] = v[8 * c8 + 2 * e] + bf16_lo(ww[e]);
          Sr[8 * c8 + 2 * e + 1] = v[8 * c8 + 2 * e + 1] + bf16_hi(ww[e]);
        }
      }
      if (u + 1 < nch) {
        write_operand((u + 1) & 1);
        mbar_arrive(&sb_ready[(u + 1) & 1]);
      }
      mbar_arrive(&empty[st]);
    }
    if (sT) {
#pragma unroll
      for (int j = 0; j < NS; j += 4)
        *reinterpret_cast<float4 *>(sT + state_base + (size_t)i * DK + j) =
            make_float4(Sr[j], Sr[j + 1], Sr[j + 2], Sr[j + 3]);
    }
  } else if (warp < 8) {
    // ---------------- outputs: row t of o = Q' S + O_intra ----------------
    // M = 64 product: rows 16 q4 .. +15 in TMEM lanes 32 q4 .. +15 (lane quarter q4 = warp % 4)
    const int q4 = warp - 4;
    const bool row_lane = lane < 16;
    const int t = 16 * q4 + (row_lane ? lane : 0);
    ChunkEntry ce = nch > 0 ? chunks.entry(c_begin) : ChunkEntry{0, 0, 0, 0};
    for (int u = 0; u < nch; ++u) {
      const int st = u % S, b = u & 1;
      const ChunkEntry ce_next = (u + 1 < nch) ? chunks.entry(c_begin + u + 1) : ce;
      if (!mbar_wait(&do_full[b], (u >> 1) & 1, err, KDA_DEVICE_TIMEOUT)) break;
      tc_fence_after();
      float v[NS];
#pragma unroll
      for (int p = 0; p < NS / 32; ++p) {
        float w32[32];
        tmem_ld32(taddr(tm, 32 * q4, Cfg::TD_O + NS * b + 32 * p), w32);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) v[32 * p + e] = w32[e];
      }
      tc_fence_before();
      mbar_arrive(&do_free[b]);
      if (!mbar_wait(&full[st], (u / S) & 1, err, KDA_DEVICE_TIMEOUT)) break;
      const unsigned char *oi = sm + st * Cfg::ST_BYTES + Cfg::ST_OI;
      uint4 out[NS / 8];
#pragma unroll
      for (int p = 0; p < NS / 32; ++p) {
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          const uint4 w = *reinterpret_cast<const uint4 *>(oi + p * OI_SLICE_BYTES + slice_off(t, ch));
          const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
          float x[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            x[2 * e] = v[32 * p + 8 * ch + 2 * e] + bf16_lo(ww[e]);
            x[2 * e + 1] = v[32 * p + 8 * ch + 2 * e + 1] + bf16_hi(ww[e]);
          }
          out[4 * p + ch] = pack8(x);
        }
      }
      mbar_arrive(&empty[st]);
      if (row_lane && t < ce.len && GDR_IN_BOUNDS((int64_t)ce.start + t < chunks.T_total)) {
        uint4 *dst = reinterpret_cast<uint4 *>(o + ((size_t)(ce.start + t) * H_v + h) * DK + sl * NS);
#pragma unroll
        for (int q = 0; q < NS / 8; ++q) dst[q] = out[q];
      }
      ce = ce_next;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tm, Cfg::TMEM_COLS);
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

GDR_DEFINE_OOB_COUNTER(oob_count_prefill_tc)

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
  int32_t *order = reinterpret_cast<int32_t *>(ws + L.order);
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

  // a dense batch needs no planning: its chunks follow from the shape
  Chunks chunks{tab, seq_off, order, 0, 0, T_total, max_chunks};
  cudaError_t e = cudaSuccess;
  if (a.cu_seqlens) {
    TraceScope tr("plan_kernel", stream);
    plan_kernel<<<1, 1024, 0, stream>>>(a.cu_seqlens, a.num_seqs, a.T, (int)T_total, hdr,
                                        seq_off, order, tab);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  } else {
    chunks.dense_T = a.T;
    chunks.per_seq = (a.T + C - 1) / C;
  }

  auto prep = !a.channel_gate ? chunk_prep_kernel<false, false>
               : a.decay_first ? chunk_prep_kernel<true, true>
                               : chunk_prep_kernel<true, false>;
  e = cudaFuncSetAttribute(prep, cudaFuncAttributeMaxDynamicSharedMemorySize, PREP_SMEM);
  if (e != cudaSuccess) return e;
  const int64_t items = (a.cu_seqlens ? max_chunks : (int64_t)a.num_seqs * chunks.per_seq) * a.H_v;
  dim3 gp((unsigned)(items < sm_count() ? items : sm_count()));
  {
    TraceScope tr("chunk_prep_kernel", stream);
    prep<<<gp, kPrepThreads, PREP_SMEM, stream>>>(mq, mk, mv, mg, a.channel_gate ? nullptr : a.g,
                                                 a.beta, a.H_qk, a.H_v, hdr, chunks, a.num_seqs,
                                                 slots);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  // Four 32-column slices per chain while they fit on the SMs in one wave,
  // else two 64-column slices (twice the work per CTA, half the re-reads of P, Q').
  const int64_t chains = (int64_t)a.num_seqs * a.H_v;
  const bool narrow = chains * 4 <= sm_count();
  auto scan = narrow ? chunk_scan_kernel<32> : chunk_scan_kernel<64>;
  const uint32_t scan_smem = narrow ? ScanCfg<32>::SMEM : ScanCfg<64>::SMEM;
  e = cudaFuncSetAttribute(scan, cudaFuncAttributeMaxDynamicSharedMemorySize, scan_smem);
  if (e != cudaSuccess) return e;
  dim3 gs((unsigned)(chains * (narrow ? 4 : 2)));
  {
    TraceScope tr("chunk_scan_kernel", stream);
    scan<<<gs, kScanThreads, scan_smem, stream>>>(
        hdr, chunks, slots, (__nv_bfloat16 *)a.o, a.initial_state, a.final_state,
        a.state_slots, a.num_slots, a.H_v, hdr);
  }
  return cudaGetLastError();
}

}  // namespace gdr
