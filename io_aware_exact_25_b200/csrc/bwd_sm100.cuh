// bwd_sm100.cuh -- fused attention backward for sm_100a.
//
// Recomputes S and P tile by tile from Q, K, V and the saved logsumexp
// instead of storing them ("How FlashAttention Optimizes GPU Memory for Fast
// AI Training", Recomputation in the Backward Pass; "FlashAttention for
// Efficient Training" section 2, Forward Pass with Recomputation).  With
// Pd = P * Z / (1 - p) the dropped probabilities (Z the keep mask):
//   dV = Pd^T dO                 ("FlashAttention for Efficient Training",
//                                 section 3.2, Integration with Autograd)
//   dP = (dO V^T) * Z / (1 - p)
//   D_i = sum_j P_ij dP_ij = dO_i . O_i
//   dS = P * (dP - D)
//   dQ = scale * dS K,  dK = scale * dS^T Q      (chain rule)
// The pages' printed dQ formulas are garbled; the expressions above follow
// from the attention definition and are what the fp64 oracle checks.
//
// Three launches:
//  1. row pass: D_i = dO_i . O_i and lse2_i = lse_i * log2(e) per row (rows
//     padded to a multiple of 128 get lse2 = +inf so their P is 0), and a
//     zeroed fp32 dQ accumulator;
//  2. the fused recompute kernel, whose work item is a 128-key tile K_j, V_j
//     of a head: a persistent grid (one CTA per SM) takes items from a
//     counter in head-grouped order (one CTA per item with dropout,
//     variable lengths or a block mask), and each item loops over the
//     128-row query tiles i that see it (i >= j when causal).  Per step it
//     computes, in tensor memory with keys on the lanes,
//     S^T = K_j Q_i^T and dP^T = V_j dO_i^T, forms P^T and dS^T in registers,
//     accumulates dV += P^T dO_i (P^T from tensor memory) and dK += dS^T Q_i
//     (dS from shared memory) in tensor memory, and
//     computes the dQ_i partial dS K_j, which a warpgroup adds into the fp32
//     accumulator (d = 64: from registers with vector reductions; d = 128:
//     staged in shared memory, one 8 KB bulk reduction per piece);
//  3. dQ = scale * accumulator, rounded to bf16.
// Variable-length mode ("FlashAttention for Efficient Training" section 5.2):
// sequences stored token-major at offsets cu_seqlens; a CTA's item is a key
// tile of one sequence and head, it loops over that sequence's query tiles
// only, and items past a sequence's real length do nothing.
// Block-sparse mode ("FlashAttention for Efficient Training" section 3.2,
// Block-Sparse Attention Support): the CTA of key tile j loops only over
// the query tiles whose mask entry for j is nonzero (a bit set in shared
// memory built by the producer warp); a key tile no query tile sees writes
// dK = dV = 0, and dQ rows nobody reaches keep the zeroed accumulator.
// Warp roles of the fused kernel:
//   warps 0-3   P/dS for query columns 0-63 of the step   (TMEM lanes = keys)
//   warps 4-7   P/dS for query columns 64-127
//   warps 8-11  dQ read-out and accumulation               (TMEM lanes = queries)
//   warp  12    tcgen05 MMA issue (one thread)
//   warp  13    TMA producer (+ dropout row keys)
//   warps 14-15 idle (they complete warpgroup 3 for the register split)
// Tensor memory (512 columns): R_S [0,128) S^T fp32, then P^T bf16 in
// [0,32) and [64,96); R_dP [128,256) dP^T fp32, then (d = 128) the dQ
// partial (fp32, D columns); dV at 256, dK at 256 + D; at d = 64 the dQ
// partial has its own columns at 384.  dS goes to shared memory only.  MMA
// order per step: dP(i), dV(i), S(i+1), dQ(i), dK(i); dP(i) runs while the
// softmax warps form P(i), S(i+1) while they form dS(i), and the dQ read-out
// of one step overlaps dK and the next step's P.
#pragma once

#include "debug_check.cuh"
#include "dropout_hash.cuh"
#include "sm100.cuh"

namespace fa {

struct BwdArgs {
  int B, H, N;
  float scale;       // softmax scale
  float scale_log2;  // scale * log2(e)
  uint32_t drop_threshold;
  float drop_scale;
  uint64_t seed;
  // bf16 [B,H,N,D] tensors with element strides (batch, head, row); D is
  // contiguous
  const __nv_bfloat16* o;
  long long o_sb, o_sh, o_sn;
  const __nv_bfloat16* dout;
  long long do_sb, do_sh, do_sn;
  const float* lse;  // [BH, N] contiguous, natural log
  __nv_bfloat16* dq;
  long long dq_sb, dq_sh, dq_sn;
  __nv_bfloat16* dk;
  long long dk_sb, dk_sh, dk_sn;
  __nv_bfloat16* dv;
  long long dv_sb, dv_sh, dv_sn;
  float* dq_acc;  // [BH, N, D] fp32 scratch
  float* lse2;    // [BH, Npad] scratch: lse * log2(e), +inf on padded rows
  float* drow;    // [BH, Npad] scratch: D_i, 0 on padded rows
  int* sched;     // scratch: the persistent grid's item counter and done count
                  // (zeroed by the row pass; the kernel leaves them zero)
  int* err;
  // block-sparse (SPARSE kernels only): bmask[hm][qt][kt] != 0 lets query
  // tile qt see key tile kt; hm = 0 when bmask_heads == 1, else the head
  const uint8_t* bmask;
  int bmask_heads;
  // variable-length (VARLEN kernels; the row pass and dQ conversion test
  // cu_seqlens at run time): token offsets [B+1], optional used lengths [B],
  // token count T; N holds the largest slot size; lse is [H, T]
  const int* cu_seqlens;
  const int* seqused;
  int total_tokens;
  // key window: only key tiles [kv_lo, kv_hi) are processed (a rank's key
  // chunk); the K, V, dK, dV tensors hold key rows from kv_row_off on, and
  // the dQ accumulator receives the partial over those keys only
  int kv_lo, kv_hi, kv_row_off;
};

__host__ __device__ inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Workspace: the fp32 dQ accumulator over N rounded up to 128 rows, stored
// tile by tile -- for each head and 128-row query tile one contiguous block of
// 128 x D floats.  At d = 64 the block is chunk-major: the four columns
// 4c..4c+3 of row r at (c * 128 + r) * 4.  At d = 128 it is eight 16-column
// pieces of 8 KB, each 128 rows x 16 columns with its 16-byte chunks permuted
// by the 64-byte swizzle (chunk k of row r at k ^ ((r >> 1) & 3)).  Then the
// scaled lse and D row vectors, then the item counter.
inline size_t bwd_workspace_bytes(int BH, int N, int d) {
  const size_t npad = round_up((size_t)N, 128);
  return round_up((size_t)BH * npad * d * 4, 256) + 2 * round_up((size_t)BH * npad * 4, 256) + 256;
}

inline void bwd_workspace_split(void* ws, int BH, int N, int d, float** dq_acc, float** lse2, float** drow,
                                int** sched) {
  const size_t npad = round_up((size_t)N, 128);
  char* p = static_cast<char*>(ws);
  *dq_acc = reinterpret_cast<float*>(p);
  p += round_up((size_t)BH * npad * d * 4, 256);
  *lse2 = reinterpret_cast<float*>(p);
  p += round_up((size_t)BH * npad * 4, 256);
  *drow = reinterpret_cast<float*>(p);
  p += round_up((size_t)BH * npad * 4, 256);
  *sched = reinterpret_cast<int*>(p);
}

// ------------------------------------------------------------ row pass

// D_i = sum_c dO_ic O_ic in fp32 and lse2_i for every (padded) row, then the
// whole dQ accumulator is set to zero.  HBM-bound: a row is read by D / 8
// lanes with 16-byte loads, and each warp keeps four groups of rows in flight.
template <int D>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const BwdArgs a, int BH, int npad) {
  constexpr int kTpr = D * 2 / 16;  // lanes per row
  constexpr int kRpw = 32 / kTpr;   // rows per warp per group
  constexpr int kU = 4;             // groups in flight
  const long long rows = (long long)BH * npad;
  // buffer extents for the bounds-checking build (unused otherwise)
  const bool vl = a.cu_seqlens != nullptr;
  const long long rows_t = vl ? a.total_tokens : a.N;
  const long long o_lim = extent4(vl ? 1 : a.B, a.H, rows_t, D, a.o_sb, a.o_sh, a.o_sn);
  const long long do_lim = extent4(vl ? 1 : a.B, a.H, rows_t, D, a.do_sb, a.do_sh, a.do_sn);
  const long long lse_lim = vl ? (long long)a.H * a.total_tokens : (long long)BH * a.N;
  (void)o_lim, (void)do_lim, (void)lse_lim;
  const int lane = threadIdx.x & 31;
  const int sub = lane / kTpr, part = lane - sub * kTpr;
  const long long warp0 = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  for (long long r0 = warp0 * (kRpw * kU); r0 < rows; r0 += nwarps * (kRpw * kU)) {
    uint4 ov[kU], dv[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      ov[u] = make_uint4(0u, 0u, 0u, 0u);
      dv[u] = make_uint4(0u, 0u, 0u, 0u);
      const long long r = r0 + u * kRpw + sub;
      if (r < rows) {
        const int bh = (int)(r / npad);
        const int i = (int)(r - (long long)bh * npad);
        const int b_ = bh / a.H, h_ = bh - b_ * a.H;
        int len = a.N, row0 = 0;
        if (a.cu_seqlens) {
          const SeqSpan sp = varlen_span(a.cu_seqlens, a.seqused, b_, a.total_tokens, a.N, nullptr, false);
          len = sp.len;
          row0 = sp.row0;
        }
        if (i < len) {
          const long long row = row0 + i;
          const long long ooff = b_ * a.o_sb + h_ * a.o_sh + row * a.o_sn + 8 * part;
          const long long doff = b_ * a.do_sb + h_ * a.do_sh + row * a.do_sn + 8 * part;
          if (FA_IN(kSiteBwdPreRow, ooff, 8, o_lim, a.err) && FA_IN(kSiteBwdPreRow, doff, 8, do_lim, a.err)) {
            ov[u] = *reinterpret_cast<const uint4*>(a.o + ooff);
            dv[u] = *reinterpret_cast<const uint4*>(a.dout + doff);
          }
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const uint32_t o4[4] = {ov[u].x, ov[u].y, ov[u].z, ov[u].w};
      const uint32_t d4[4] = {dv[u].x, dv[u].y, dv[u].z, dv[u].w};
      float acc = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) acc += bf16_lo(o4[e]) * bf16_lo(d4[e]) + bf16_hi(o4[e]) * bf16_hi(d4[e]);
#pragma unroll
      for (int s = kTpr / 2; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
      const long long r = r0 + u * kRpw + sub;
      if (part == 0 && r < rows) {
        const int bh = (int)(r / npad);
        const int i = (int)(r - (long long)bh * npad);
        int len = a.N;
        long long lse_at = (long long)bh * a.N + i;
        if (a.cu_seqlens) {
          const int b_ = bh / a.H, h_ = bh - b_ * a.H;
          const SeqSpan sp = varlen_span(a.cu_seqlens, a.seqused, b_, a.total_tokens, a.N, nullptr, false);
          len = sp.len;
          lse_at = (long long)h_ * a.total_tokens + sp.row0 + i;
        }
        a.drow[r] = i < len ? acc : 0.f;
        const bool l_ok = i >= len || FA_IN(kSiteBwdPreLse, lse_at, 1, lse_lim, a.err);
        a.lse2[r] = i < len && l_ok ? a.lse[lse_at] * 1.4426950408889634f : INFINITY;
      }
    }
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    a.sched[0] = 0;  // items drawn
    a.sched[1] = 0;  // CTAs done drawing
  }
  const long long n4 = (long long)BH * npad * D / 4;
  float4* acc4 = reinterpret_cast<float4*>(a.dq_acc);
  for (long long u = blockIdx.x * (long long)blockDim.x + threadIdx.x; u < n4; u += (long long)gridDim.x * blockDim.x)
    acc4[u] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// dQ = scale * accumulator.  Each thread converts 8 columns (two 4-column
// chunks) of one row.  d = 64 (chunk-major tiles): a warp takes 32
// consecutive rows of one chunk pair, so its reads are two contiguous
// 512-byte runs.  d = 128 (swizzled 16-column pieces): consecutive threads
// take consecutive chunk pairs of one row, so its writes are contiguous.
template <int D>
__global__ void __launch_bounds__(256) bwd_post_kernel(const float* __restrict__ acc, __nv_bfloat16* __restrict__ dq,
                                                       int BH, int H, int N, long long sb, long long sh, long long sn,
                                                       float scale, const int* cu_seqlens, const int* seqused,
                                                       int total_tokens, int* err) {
  constexpr bool kChunkMajor = D == 64;
  const int nT = (N + 127) >> 7;
  constexpr int kC8 = D / 8;  // chunk pairs per row
  const long long n = (long long)BH * nT * 128 * kC8;
  // buffer extents for the bounds-checking build (unused otherwise)
  const long long acc_lim = (long long)BH * nT * 128 * D;
  const long long dq_lim = extent4(cu_seqlens ? 1 : BH / H, H, cu_seqlens ? total_tokens : N, D, sb, sh, sn);
  (void)acc_lim, (void)dq_lim, (void)err;
  for (long long u = blockIdx.x * (long long)blockDim.x + threadIdx.x; u < n;
       u += (long long)gridDim.x * blockDim.x) {
    int c8, r, tile, bh;
    if (kChunkMajor) {  // (bh, tile, row group, chunk pair, lane)
      const int j = (int)(u & 31);
      long long v = u >> 5;
      c8 = (int)(v % kC8);
      v /= kC8;
      r = (int)(v & 3) * 32 + j;
      v >>= 2;
      tile = (int)(v % nT);
      bh = (int)(v / nT);
    } else {  // (bh, tile, row, chunk pair)
      c8 = (int)(u % kC8);
      long long v = u / kC8;
      r = (int)(v & 127);
      v >>= 7;
      tile = (int)(v % nT);
      bh = (int)(v / nT);
    }
    const int i = tile * 128 + r;
    const int b_ = bh / H, h_ = bh - b_ * H;
    long long row = i;
    int len = N;
    if (cu_seqlens) {
      const SeqSpan sp = varlen_span(cu_seqlens, seqused, b_, total_tokens, N, nullptr, false);
      len = sp.len;  // padding rows are filled separately
      row = sp.row0 + i;
    }
    if (i >= len) continue;
    const long long blk_off = ((long long)bh * nT + tile) * (128 * D);
    const long long dq_off = b_ * sb + h_ * sh + row * sn + 8 * c8;
    if (!FA_IN(kSiteBwdPost, blk_off, 128 * D, acc_lim, err) || !FA_IN(kSiteBwdPost, dq_off, 8, dq_lim, err)) continue;
    const float* blk = acc + blk_off;
    float4 x, y;
    if (kChunkMajor) {
      x = *reinterpret_cast<const float4*>(blk + ((2 * c8) * 128 + r) * 4);
      y = *reinterpret_cast<const float4*>(blk + ((2 * c8 + 1) * 128 + r) * 4);
    } else {
      const int piece = c8 >> 1;    // 16-column piece
      const int k0 = (c8 & 1) * 2;  // first of the two 4-column chunks
      const int sw = (r >> 1) & 3;
      const float* pr = blk + piece * 2048 + r * 16;
      x = *reinterpret_cast<const float4*>(pr + ((k0 ^ sw) << 2));
      y = *reinterpret_cast<const float4*>(pr + (((k0 + 1) ^ sw) << 2));
    }
    uint4 w;
    w.x = pack_bf16x2(x.x * scale, x.y * scale);
    w.y = pack_bf16x2(x.z * scale, x.w * scale);
    w.z = pack_bf16x2(y.x * scale, y.y * scale);
    w.w = pack_bf16x2(y.z * scale, y.w * scale);
    *reinterpret_cast<uint4*>(dq + dq_off) = w;
  }
}

// ------------------------------------------------------- fused kernel

template <int D, bool DROPOUT>
struct BwdLayout {
  // 16 warps: P/dS warpgroups 0-1, dQ warpgroup 2, and warpgroup 3 (MMA
  // issue, TMA producer, two idle warps) so that every warpgroup is whole for
  // the register reallocation: launched at 128 registers a thread (the whole
  // register file), then for the P/dS warpgroups, dQ and warpgroup 3
  // 152 / 112 / 88 without dropout, 160 / 112 / 80 with it at d = 128 and
  // 160 / 104 / 80 with it at d = 64 (2*128*R_ps + 128*R_dq + 128*R_ctl =
  // 64512, 65536 and 64512 <= 65536).  At 128 registers for every warp the
  // dropout kernels spilled 220-280 bytes a thread; with these splits no
  // kernel spills (ptxas).  Without dropout the long8k backward is 1.7 %
  // faster than at 160/104/80, which spilled 48 bytes; at d = 128 with
  // dropout 160/104/80 spilled 12-16 bytes and 160/112/72 4, and 160/112/80
  // spills none at d = 128 but 4-28 bytes at d = 64.
  static constexpr int kThreads = 512;
  static constexpr uint32_t kRegsPS = DROPOUT ? 160 : 152, kRegsDQ = DROPOUT ? (D == 128 ? 112 : 104) : 112,
                            kRegsCtl = DROPOUT ? 80 : 88;
  static_assert(2 * 128 * kRegsPS + 128 * kRegsDQ + 128 * kRegsCtl <= 512 * 128, "register split");
  static constexpr uint32_t kHalf = 128u * 128u;
  static constexpr uint32_t kTile = 128u * D * 2u;
  static constexpr int kQStages = 2;
  static constexpr int kDoStages = D == 128 ? 1 : 2;
  static constexpr uint32_t kOffK = 0;
  static constexpr uint32_t kOffV = kOffK + kTile;
  static constexpr uint32_t kOffQ = kOffV + kTile;
  static constexpr uint32_t kOffDO = kOffQ + kQStages * kTile;
  static constexpr uint32_t kOffDS = kOffDO + kDoStages * kTile;  // dS, 128 x 128 bf16, MN-major halves
  static constexpr uint32_t kRowStage = (DROPOUT ? 3u : 2u) * 128u * 4u;  // lse2, D (, dropout row keys)
  // double-buffered row statistics, except where shared memory runs out
  static constexpr int kRowStages = (D == 128 && DROPOUT) ? 1 : 2;
  static constexpr uint32_t kOffRow = kOffDS + 2u * kHalf;
  // dQ accumulation: at d = 64 straight from registers (vector reductions);
  // at d = 128 through shared memory: 128-row x 16-column fp32 pieces
  // (64-byte rows, 64-byte swizzle), each the source of one 8 KB bulk
  // reduction (measured: direct reductions win 4% at d = 64 and lose 1% at
  // d = 128, where they also make the dQ conversion's writes strided)
  static constexpr bool kDqDirect = D == 64;
  static constexpr uint32_t kDqPiece = 128u * 64u;
  static constexpr int kDqBufs = kDqDirect ? 0 : 4;
  static constexpr uint32_t kOffDQ = (kOffRow + kRowStages * kRowStage + 1023u) & ~1023u;
  static constexpr uint32_t kOffBar = kOffDQ + kDqBufs * kDqPiece;
  // kv, q_full[2], q_empty[2], do_full[2], do_empty[2], row_full[2],
  // row_empty[2], s, dp, p, ds, kv_free, dk, dq, dq_free, drain, acc_free,
  // item_full[2], item_empty[2]
  static constexpr int kNumBars = 1 + 12 + 10 + 4;
  // after the barriers: TMEM address, abort flag, dQ-warpgroup flag, two item
  // slots
  static constexpr uint32_t kSmem = kOffBar + kNumBars * 8 + 32;
  // block-sparse: the query-tile bit set and its count after the barriers
  static constexpr uint32_t kOffBits = (kSmem + 15u) & ~15u;
  static constexpr uint32_t kSmemSparse = kOffBits + kSparseWords * 4u + 16u;
  static_assert(kOffDQ % 1024 == 0, "staging tiles must be swizzle-aligned");
  static_assert(kSmemSparse <= 232448, "shared memory budget");
  static constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 256 + D;
  // d = 64 leaves 128 columns free: the dQ partial gets its own, so dP(i+1)
  // need not wait for the dQ(i) read-out; at d = 128 it shares dP's columns
  static constexpr bool kOwnDQ = D == 64;
  static constexpr uint32_t kColDQ = kOwnDQ ? 256 + 2 * D : kColDP;
};

// TMEM column of the packed bf16 P^T slice kk (16 queries) written by the
// two P/dS warpgroups: queries 0-63 at [0,32), 64-127 at [64,96).
__device__ __forceinline__ uint32_t packed_col(int kk) { return kk < 4 ? 8u * kk : 64u + 8u * (kk - 4); }

// Visit each work item's query tiles from a rotated start (see q_tile).
// Measured within noise (+1.3% on long8k, -1% on train2k) and it changes the
// dK/dV summation order against the one-item-per-CTA kernels; off.
constexpr bool kRotateQueryTiles = false;

// Of every 8 pairs of recomputed probabilities, this many take the
// exponential on the FMA pipe (polynomial), the rest on MUFU.  Measured: 2 of
// 8 is 1.4% faster at d = 128 (3.6% with dropout) and 2-4% slower at d = 64.
template <int D>
__host__ __device__ constexpr int bwd_poly_pairs_of8() { return D == 128 ? 2 : 0; }

template <int D, bool CAUSAL, bool DROPOUT, bool SPARSE, bool VARLEN>
__global__ void __launch_bounds__(512, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
               const BwdArgs a) {
  using L = BwdLayout<D, DROPOUT>;
  static_assert(D == 64 || D == 128, "head dim");
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* bar_kv = bars;
  uint64_t* bar_q_full = bars + 1;
  uint64_t* bar_q_empty = bars + 3;
  uint64_t* bar_do_full = bars + 5;
  uint64_t* bar_do_empty = bars + 7;
  uint64_t* bar_row_full = bars + 9;
  uint64_t* bar_row_empty = bars + 11;
  uint64_t* bar_s = bars + 13;
  uint64_t* bar_dp = bars + 14;
  uint64_t* bar_p = bars + 15;
  uint64_t* bar_ds = bars + 16;
  uint64_t* bar_kv_free = bars + 17;  // K/V buffers no longer read (last MMA of an item)
  uint64_t* bar_dk = bars + 18;
  uint64_t* bar_dq = bars + 19;
  uint64_t* bar_dq_free = bars + 20;
  uint64_t* bar_drain = bars + 21;
  uint64_t* bar_acc_free = bars + 22;  // dV/dK accumulators read out by the epilogue
  uint64_t* bar_item_full = bars + 23;   // [2] the producer published the next item
  uint64_t* bar_item_empty = bars + 25;  // [2] every role has read it (13 arrivals)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + L::kNumBars);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);  // [0] abort, [1] dQ warpgroup flag
  int* item_slot = abort_flag + 2;                           // [2] published item indices
  const uint32_t sbase = smem_u32(smem);

  const int BH = a.B * a.H;
  const int nT = (a.N + 127) >> 7;
  const int npad = nT * 128;
  // buffer extents for the bounds-checking build (unused otherwise)
  const long long rows_q = VARLEN ? a.total_tokens : a.N;
  const long long rows_k = VARLEN ? a.total_tokens : min((long long)a.N, (long long)a.kv_hi * 128) - a.kv_row_off;
  const long long acc_lim = (long long)BH * nT * 128 * D;
  const long long row_lim = (long long)BH * npad;
  const long long dk_lim = extent4(VARLEN ? 1 : a.B, a.H, rows_k, D, a.dk_sb, a.dk_sh, a.dk_sn);
  const long long dv_lim = extent4(VARLEN ? 1 : a.B, a.H, rows_k, D, a.dv_sb, a.dv_sh, a.dv_sn);
  (void)rows_q, (void)rows_k, (void)acc_lim, (void)row_lim, (void)dk_lim, (void)dv_lim;
  // Work items are (key tile, head) pairs.  Their order groups the heads, hg
  // at a time, and within a group
  // puts the key tiles in ascending order with the group's heads interleaved:
  // longest first when causal.  CTAs take items in this order -- the
  // persistent grid from a counter in the workspace, one-item-per-CTA grids
  // by block index, which the hardware dispatches in order -- so the items
  // running at any time belong to a few heads, whose Q, dO and fp32 dQ
  // accumulator stay in L2, and the short items of a group fill the time its
  // long items leave.  In the persistent grid the next item's first products
  // overlap the last item's dQ reductions and dK/dV write-out.
  const int kt_hi = min(a.kv_hi, nT), kt_lo = min(a.kv_lo, kt_hi);
  const int nTr = kt_hi - kt_lo;  // key tiles in the window
  const int n_items = BH * nTr;
  // Group size: a group holds about one CTA's share of the running items'
  // work per SM (hg >= SMs / average item length, in query tiles); the heads
  // left over join the last group, so the last group -- whose long items
  // start last -- always holds at least that much work and the tail stays
  // short.
  uint32_t n_sm;
  asm("mov.u32 %0, %%nsmid;" : "=r"(n_sm));
  const int avg_len = max(1, CAUSAL ? nT - (kt_lo + kt_hi - 1) / 2 : nT);
  const int hg = min(BH, max(1, ((int)n_sm + avg_len - 1) / avg_len));
  const int n_groups = max(1, BH / hg);
  // An item's sequence: real rows [0, len) at tokens row0.. of the tensors,
  // batch coordinate wc of the tensor maps (variable-length: 0).
  struct Item {
    int jt, bh, bb, hh, i_begin, n_steps, row0, len, wc, rot;
  };
  auto item_of = [&](int w) {
    const int grp = min(w / (hg * nTr), n_groups - 1);
    const int h0 = grp * hg;
    const int nh = grp == n_groups - 1 ? BH - h0 : hg;  // the last group takes the rest
    const int r = w - h0 * nTr;
    const int jl = r / nh;  // key tile within the window
    Item t;
    t.jt = kt_lo + jl;
    t.bh = h0 + (r - jl * nh);
    t.bb = t.bh / a.H;
    t.hh = t.bh - t.bb * a.H;
    t.i_begin = CAUSAL ? t.jt : 0;
    t.n_steps = nT - t.i_begin;
    t.row0 = 0;
    t.len = a.N;
    t.wc = t.bb;
    if (VARLEN) {
      const SeqSpan sp = varlen_span(a.cu_seqlens, a.seqused, t.bb, a.total_tokens, a.N, a.err, t.jt == 0);
      t.row0 = sp.row0;
      t.len = sp.len;
      t.wc = 0;
      const int nTb = (sp.len + 127) >> 7;
      t.n_steps = t.jt < nTb ? nTb - t.i_begin : 0;
    }
    // The item visits its query tiles starting at a rotation of its own, so
    // items of one head that run at the same time reduce their dQ partials
    // into different accumulator tiles instead of all into the same one.
    t.rot = t.n_steps > 1 ? (int)(((uint32_t)t.jt * 2654435761u + (uint32_t)t.bh * 40503u) % (uint32_t)t.n_steps) : 0;
    return t;
  };
  // query tile of step `it` of item t (dense items; block-sparse ones walk
  // their bit set in order)
  auto q_tile = [&](const Item& t, int it) {
    int s = it + (kRotateQueryTiles ? t.rot : 0);
    if (s >= t.n_steps) s -= t.n_steps;
    return t.i_begin + s;
  };
  uint32_t* qbits = reinterpret_cast<uint32_t*>(smem + L::kOffBits);  // SPARSE: query tiles that see jt
  int* sparse_cnt = reinterpret_cast<int*>(qbits + kSparseWords);
  const int nwords = (nT + 31) >> 5;

  if (threadIdx.x == 0) {
    mbar_init(bar_kv, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar_q_full[s], 1);
      mbar_init(&bar_q_empty[s], 1);
      mbar_init(&bar_do_full[s], 1);
      mbar_init(&bar_do_empty[s], 1);
      mbar_init(&bar_row_full[s], 1);
      mbar_init(&bar_row_empty[s], 256);
    }
    mbar_init(bar_s, 1);
    mbar_init(bar_dp, 1);
    mbar_init(bar_p, 256);
    mbar_init(bar_ds, 256);
    mbar_init(bar_kv_free, 1);
    mbar_init(bar_acc_free, 256);
    mbar_init(bar_dk, 1);
    mbar_init(bar_dq, 1);
    mbar_init(bar_dq_free, 128);
    mbar_init(bar_drain, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bar_item_full[s], 1);
      mbar_init(&bar_item_empty[s], 13);  // MMA thread, 4 dQ warps, 8 P/dS warps
    }
    const bool misaligned = (sbase & 1023u) != 0u;
    *abort_flag = misaligned ? 1 : 0;
    if (misaligned && a.err) atomicCAS(a.err, kDevOk, kDevMisaligned);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (SPARSE && warp == 13) {
    // column jt of the mask: entry (i, jt) for i in [i_begin, nT)
    const Item t = item_of(blockIdx.x);
    const int hm = a.bmask_heads == 1 ? 0 : t.hh;
    const uint8_t* col = a.bmask + (size_t)hm * nT * nT + t.jt;
    const int3 c = build_bit_sets(col, nT, nullptr, 0, t.i_begin, nT, nwords, qbits, nullptr, lane);
    if (lane == 0) sparse_cnt[0] = c.x;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Abort ab{abort_flag, a.err};
  const bool run = *abort_flag == 0;
  // Dropout, variable-length and block-sparse kernels run one item per CTA
  // (see the launch); for them the loops below make a single pass.
  constexpr bool PERSIST = !SPARSE && !DROPOUT && !VARLEN;
  // Item r of this CTA for a consuming role: the persistent grid reads the
  // slot the producer published (the caller then arrives on
  // bar_item_empty[r & 1]); n_items ends the loop.
  auto peek_item = [&](int r, bool& ok_) -> int {
    if (!PERSIST) return r == 0 ? (int)blockIdx.x : n_items;
    if (!mbar_wait(&bar_item_full[r & 1], (uint32_t)(r >> 1) & 1u, ab)) {
      ok_ = false;
      return n_items;
    }
    return *reinterpret_cast<volatile int*>(&item_slot[r & 1]);
  };
  // the items of this CTA, with the block-sparse step count
  auto item_at = [&](int w) {
    Item t = item_of(w);
    if (SPARSE) t.n_steps = sparse_cnt[0];
    return t;
  };

  // Each warpgroup sets its register budget at the top of its branch (every
  // thread of the warpgroup, whatever its role or the abort state).
  if (warp >= 12) {
  regs_dec<L::kRegsCtl>();
  if (run && warp == 13) {
    // ------------------------------------------------------ TMA producer
    const uint64_t pol_keep = policy_evict_last();
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      prefetch_tmap(&tm_do);
    }
    // All 32 lanes run these loops (they compute the dropout row keys); the
    // waits are made warp-uniform with __all_sync, lane 0 issues the copies.
    // g counts query-tile steps over all items of the CTA and drives the
    // rings' stages and phases.
    int q_issued = 0, do_issued = 0, kv_issued = 0;
    int g = 0;
    bool ok = true;
    for (int r = 0; ok; ++r) {
      int w = 0;
      if (PERSIST) {
        // take the next item from the counter and publish it to the other roles
        if (!__all_sync(0xffffffffu, mbar_wait(&bar_item_empty[r & 1], ((uint32_t)(r >> 1) & 1u) ^ 1u, ab))) {
          ok = false;
          break;
        }
        if (lane == 0) {
          w = min(atomicAdd(a.sched, 1), n_items);
          item_slot[r & 1] = w;
          mbar_arrive(&bar_item_full[r & 1]);
        }
        w = __shfl_sync(0xffffffffu, w, 0);
      } else {
        w = r == 0 ? (int)blockIdx.x : n_items;
      }
      if (w >= n_items) {
        // The last CTA to draw the end of the items resets the counter (and
        // this count), so the next launch on the workspace starts from zero
        // without a row pass: every CTA has drawn its last value by then.
        if (PERSIST && lane == 0 && atomicAdd(a.sched + 1, 1) == (int)gridDim.x - 1) {
          atomicExch(a.sched, 0);
          atomicExch(a.sched + 1, 0);
        }
        break;
      }
      const Item t = item_at(w);
      if (lane == 0) {
        (void)FA_IN(kSiteBwdItem, t.jt - kt_lo, 1, nTr, a.err);
        (void)FA_IN(kSiteBwdItem, t.bh, 1, BH, a.err);
        if (!SPARSE) (void)FA_IN(kSiteBwdItem, t.i_begin, t.n_steps, nT, a.err);
      }
      if (t.n_steps == 0) continue;  // (a key tile no query tile sees loads nothing)
      auto load_kv = [&]() {
        if (lane == 0) {
          mbar_arrive_expect_tx(bar_kv, 2 * L::kTile);
          (void)FA_IN(kSiteBwdTile, t.row0 + t.jt * 128 - a.kv_row_off, 1, rows_k, a.err);
          for (int h = 0; h < D / 64; ++h) {
            const int krow = t.row0 + t.jt * 128 - a.kv_row_off;
            tma_load_4d(smem + L::kOffK + h * L::kHalf, &tm_k, 64 * h, krow, t.hh, t.wc, bar_kv, pol_keep);
            tma_load_4d(smem + L::kOffV + h * L::kHalf, &tm_v, 64 * h, krow, t.hh, t.wc, bar_kv, pol_keep);
          }
        }
        ++kv_issued;
      };
      if (!PERSIST) load_kv();  // one item per CTA: K/V first
      BitWalk walk(qbits, qbits, nwords);
      for (int it = 0; it < t.n_steps; ++it) {
        const int gs = g + it;
        const int i = SPARSE ? walk.next() : q_tile(t, it);
        // Q_i and dO_i: re-read by every key tile of the head -> keep in L2
        const int qs = gs & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&bar_q_empty[qs], ((gs >> 1) & 1) ^ 1u, ab))) {
          ok = false;
          break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(&bar_q_full[qs], L::kTile);
          (void)FA_IN(kSiteBwdTile, t.row0 + i * 128, 1, rows_q, a.err);
          for (int h = 0; h < D / 64; ++h)
            tma_load_4d(smem + L::kOffQ + qs * L::kTile + h * L::kHalf, &tm_q, 64 * h, t.row0 + i * 128, t.hh,
                        t.wc, &bar_q_full[qs], pol_keep);
        }
        ++q_issued;
        const int ds_ = gs % L::kDoStages;
        if (!__all_sync(0xffffffffu, mbar_wait(&bar_do_empty[ds_], ((gs / L::kDoStages) & 1) ^ 1u, ab))) {
          ok = false;
          break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(&bar_do_full[ds_], L::kTile);
          for (int h = 0; h < D / 64; ++h)
            tma_load_4d(smem + L::kOffDO + ds_ * L::kTile + h * L::kHalf, &tm_do, 64 * h, t.row0 + i * 128, t.hh,
                        t.wc, &bar_do_full[ds_], pol_keep);
        }
        ++do_issued;
        // row statistics of query tile i
        const int rs = gs % L::kRowStages;
        if (!__all_sync(0xffffffffu, mbar_wait(&bar_row_empty[rs], ((gs / L::kRowStages) & 1) ^ 1u, ab))) {
          ok = false;
          break;
        }
        uint8_t* rowbuf = smem + L::kOffRow + rs * L::kRowStage;
        if (DROPOUT) {
          uint32_t* keys = reinterpret_cast<uint32_t*>(rowbuf + 2 * 512);
          for (int c = lane; c < 128; c += 32)
            keys[c] = dropout_row_key(a.seed, (uint32_t)t.bb, (uint32_t)t.hh, (uint32_t)(i * 128 + c));
          __syncwarp();
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(&bar_row_full[rs], 1024);
          long long roff = (long long)t.bh * npad + i * 128;
          if (!FA_IN(kSiteBwdRow, roff, 128, row_lim, a.err)) roff = 0;  // (debug build: record, read row 0)
          bulk_load(rowbuf, a.lse2 + roff, 512, &bar_row_full[rs]);
          bulk_load(rowbuf + 512, a.drow + roff, 512, &bar_row_full[rs]);
        }
        __syncwarp();
        if (PERSIST && it == 0) {
          // K_j, V_j, after the item's first Q/dO/row loads (which only need
          // ring slots): the previous item's last product must have read them
          if (kv_issued > 0 && !__all_sync(0xffffffffu, mbar_wait(bar_kv_free, (kv_issued - 1) & 1, ab))) {
            ok = false;
            break;
          }
          load_kv();
        }
      }
      g += t.n_steps;
    }
    if (lane == 0) {
      // Every load issued must land before the CTA may exit.
      if (kv_issued > 0) mbar_wait_drain(bar_kv, (kv_issued - 1) & 1);
      for (int n = q_issued > 2 ? q_issued - 2 : 0; n < q_issued; ++n) mbar_wait_drain(&bar_q_full[n & 1], (n >> 1) & 1);
      for (int n = do_issued > L::kDoStages ? do_issued - L::kDoStages : 0; n < do_issued; ++n)
        mbar_wait_drain(&bar_do_full[n % L::kDoStages], (n / L::kDoStages) & 1);
    }
  } else if (run && warp == 12) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t kIdKK = idesc_bf16(128, 128, false, false);  // S^T, dP^T: both operands K-major
      constexpr uint32_t kIdTM = idesc_bf16(128, D, false, true);     // dV, dK: A K-major, B MN-major
      constexpr uint32_t kIdMM = idesc_bf16(128, D, true, true);      // dQ: both MN-major
      const uint32_t sK = sbase + L::kOffK, sV = sbase + L::kOffV, sDS = sbase + L::kOffDS;
      bool ok = true;
      bool issued_any = false;
      int g = 0, kv_used = 0;
      // Per step: dP(i), dV(i), S(i+1), dQ(i), dK(i).  At d = 128 dP(i)
      // overwrites the dQ(i-1) partial and waits for the dQ warpgroup to have
      // read it (at d = 64 dQ(i) waits instead); dP(i) then runs while the
      // softmax warps form P(i).  S(i+1) overwrites the columns
      // holding P^T(i), which dV(i) reads; it is queued behind its reader and
      // the tensor core executes one thread's MMAs in order, so it needs no
      // wait.  S(i+1) goes right behind dV(i) so it runs while the softmax
      // warps form dS(i), and P(i+1) can start as soon as dS(i) is done.  dQ(i)
      // and dK(i) both read dS from shared memory (dS^T for dK is the same tile
      // read K-major); dQ(i) goes first so its read-out, which gates dP(i+1),
      // starts while dK(i) runs.  Across items the same order holds: the next
      // item's S(0) is queued behind the last dK, its first dV and dK (which
      // overwrite the accumulators) wait for the epilogue to have read them.
      for (int r = 0; ok; ++r) {
        const int w = peek_item(r, ok);
        if (PERSIST && ok) mbar_arrive(&bar_item_empty[r & 1]);
        if (w >= n_items) break;
        const Item t = item_at(w);
        if (t.n_steps == 0) continue;
        ok = mbar_wait(bar_kv, kv_used & 1, ab) && mbar_wait(&bar_q_full[g & 1], (g >> 1) & 1, ab);
        if (!ok) break;
        tc_fence_after();
        {
          const uint32_t sQ0 = sbase + L::kOffQ + (g & 1) * L::kTile;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ss(tmem + L::kColS, desc_kmajor(sK, kk, L::kHalf), desc_kmajor(sQ0, kk, L::kHalf), kIdKK,
                   kk > 0 ? 1u : 0u);
          mma_commit(bar_s);
          issued_any = true;
        }
        for (int it = 0; it < t.n_steps && ok; ++it) {
          const int gs = g + it;
          const uint32_t ph = gs & 1;
          const int qs = gs & 1;
          const int ds_ = gs % L::kDoStages;
          const uint32_t sQ = sbase + L::kOffQ + qs * L::kTile;
          const uint32_t sDO = sbase + L::kOffDO + ds_ * L::kTile;
          // dP^T = V dO_i^T into R_dP
          if (!mbar_wait(&bar_do_full[ds_], (gs / L::kDoStages) & 1, ab) ||
              (!L::kOwnDQ && gs > 0 && !mbar_wait(bar_dq_free, ph ^ 1u, ab))) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ss(tmem + L::kColDP, desc_kmajor(sV, kk, L::kHalf), desc_kmajor(sDO, kk, L::kHalf), kIdKK,
                   kk > 0 ? 1u : 0u);
          mma_commit(bar_dp);
          // dV += P^T dO_i; the item's first one overwrites the accumulator
          if (!mbar_wait(bar_p, ph, ab) || (it == 0 && kv_used > 0 && !mbar_wait(bar_acc_free, (kv_used - 1) & 1, ab))) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tmem + L::kColDV, tmem + L::kColS + packed_col(kk), desc_mnmajor(sDO, kk, L::kHalf), kIdTM,
                   (it > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&bar_do_empty[ds_]);
          // S^T for the next step (behind dV, which reads P^T from R_S)
          if (it + 1 < t.n_steps) {
            const int qn = (gs + 1) & 1;
            if (!mbar_wait(&bar_q_full[qn], ((gs + 1) >> 1) & 1, ab)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sQn = sbase + L::kOffQ + qn * L::kTile;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
              mma_ss(tmem + L::kColS, desc_kmajor(sK, kk, L::kHalf), desc_kmajor(sQn, kk, L::kHalf), kIdKK,
                     kk > 0 ? 1u : 0u);
            mma_commit(bar_s);
          }
          // dQ_i partial = dS K_j (the softmax warps have read dP^T(i)); with
          // its own columns it waits for the previous partial's read-out here
          if (!mbar_wait(bar_ds, ph, ab) || (L::kOwnDQ && gs > 0 && !mbar_wait(bar_dq_free, ph ^ 1u, ab))) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(tmem + L::kColDQ, desc_mnmajor(sDS, kk, L::kHalf), desc_mnmajor(sK, kk, L::kHalf), kIdMM,
                   kk > 0 ? 1u : 0u);
          mma_commit(bar_dq);
          // dK += dS^T Q_i, A = the shared dS tile read K-major (rows = keys)
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(tmem + L::kColDK, desc_kmajor(sDS, kk, L::kHalf), desc_mnmajor(sQ, kk, L::kHalf), kIdTM,
                   (it > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar_dk);
          mma_commit(&bar_q_empty[qs]);
        }
        if (!ok) break;
        mma_commit(bar_kv_free);  // the item's products have read K_j and V_j
        ++kv_used;
        g += t.n_steps;
      }
      if (issued_any) {
        mma_commit(bar_drain);
        mbar_wait_drain(bar_drain, 0);
      }
    }
  }
  } else if (warp >= 8) {
  regs_dec<L::kRegsDQ>();
  if (run) {
    // ------------------------------------------ dQ read-out + accumulate
    // The partial dQ_i (128 rows x D fp32, query rows on the TMEM lanes) is
    // added into the fp32 accumulator.  At d = 64 straight from registers
    // with vector reductions (red.global.add.v4.f32), each warp instruction
    // covering 512 contiguous bytes of the chunk-major accumulator tile.  At
    // d = 128 in 16-column pieces: every thread writes its row of a piece
    // into a 64-byte-swizzled staging tile and one thread adds each 8 KB tile
    // with a bulk reduction; with four staging tiles the first 64 columns are
    // staged while the rest is read from TMEM.  Either way the TMEM columns
    // are released as soon as the whole row is in registers or shared
    // memory.  The loop is uniform over the warpgroup (named barriers are
    // reached by every thread).
    const int quad = warp & 3;
    const int row = quad * 32 + lane;  // query within the tile == TMEM lane
    const uint32_t tQ = tmem + ((uint32_t)(quad * 32) << 16) + L::kColDQ;
    const bool leader = warp == 8 && lane == 0;
    volatile int* dq_flag = abort_flag + 1;
    // (d = 64) add 32 columns (8 four-column chunks from chunk c0) of this row
    // into the chunk-major accumulator tile: chunk c of row r at
    // (c * 128 + r) * 4 floats, so a warp's 32 rows of a chunk are 512
    // contiguous bytes
    auto add32 = [&](float* tile, const uint32_t (&v)[32], int c0) {
#pragma unroll
      for (int k = 0; k < 8; ++k)
        red_add_v4_f32(tile + ((c0 + k) * 128 + row) * 4, v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
    };
    // (d = 128) stage 32 columns (two 16-column pieces) of this row into
    // staging tiles t, t+1 (64-byte swizzle)
    const uint32_t sw = (uint32_t)(row >> 1) & 3u;
    auto stage = [&](const uint32_t (&v)[32], int t) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t rbase = sbase + L::kOffDQ + (uint32_t)(t + h) * L::kDqPiece + (uint32_t)row * 64u;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
          st_shared_v4(rbase + (((uint32_t)q4 ^ sw) << 4), v[16 * h + 4 * q4], v[16 * h + 4 * q4 + 1],
                       v[16 * h + 4 * q4 + 2], v[16 * h + 4 * q4 + 3]);
      }
    };
    // (d = 128) after a named barrier: add staging tiles 0..n-1 into the
    // tile's 16-column pieces p0..p0+n-1 (8 KB bulk reductions)
    auto reduce = [&](float* tile, int p0, int n) {
      if (leader) {
        for (int t = 0; t < n; ++t)
          bulk_reduce_add_f32(tile + (p0 + t) * 2048, sbase + L::kOffDQ + (uint32_t)t * L::kDqPiece, L::kDqPiece);
        bulk_commit();
      }
    };
    int g = 0;
    bool ok = true;
    for (int r = 0; ok; ++r) {
      const int w = peek_item(r, ok);
      __syncwarp();
      if (PERSIST && ok && lane == 0) mbar_arrive(&bar_item_empty[r & 1]);
      // the warpgroup leaves together: one flag for the whole loop
      if (!L::kDqDirect) {
        if (leader) *dq_flag = (ok && w < n_items) ? 1 : 0;
        named_bar_sync(1, 128);
        const int go = *dq_flag;
        named_bar_sync(1, 128);
        if (!go) break;
      } else if (!ok || w >= n_items) {
        break;
      }
    const Item t = item_at(w);
    BitWalk walk(qbits, qbits, nwords);
    for (int it = 0; it < t.n_steps; ++it) {
      const int i = SPARSE ? walk.next() : q_tile(t, it);
      const long long tile_off = ((long long)t.bh * nT + i) * (128 * D);
      // (debug build: a tile outside the accumulator is recorded and tile 0 takes its adds)
      float* tile = a.dq_acc + (FA_IN(kSiteBwdAcc, tile_off, 128 * D, acc_lim, a.err) ? tile_off : 0);
      if (L::kDqDirect) {
        if (!mbar_wait(bar_dq, (g + it) & 1, ab)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t v0[32], v1[32];
        tmem_ld32(tQ, v0);
        tmem_ld32(tQ + 32u, v1);
        tmem_ld_wait();
        reg_fence(v0);
        reg_fence(v1);
        // the whole partial is in registers: release its columns first
        tc_fence_before();
        mbar_arrive(bar_dq_free);
        add32(tile, v0, 0);
        add32(tile, v1, 8);
      } else {
        // the staging tiles are free once the previous step's reductions
        // have read them; one thread waits, a named barrier shares the outcome
        if (leader) {
          bulk_wait_read<0>();
          *dq_flag = mbar_wait(bar_dq, (g + it) & 1, ab) ? 1 : 0;
        }
        named_bar_sync(1, 128);
        if (*dq_flag == 0) {
          ok = false;
          break;
        }
        tc_fence_after();
        {
          uint32_t v0[32], v1[32];
          tmem_ld32(tQ, v0);
          tmem_ld32(tQ + 32u, v1);
          tmem_ld_wait();
          reg_fence(v0);
          reg_fence(v1);
          stage(v0, 0);
          stage(v1, 2);
        }
        uint32_t v2[32], v3[32];
        tmem_ld32(tQ + 64u, v2);
        tmem_ld32(tQ + 96u, v3);
        tmem_ld_wait();
        reg_fence(v2);
        reg_fence(v3);
        tc_fence_before();
        mbar_arrive(bar_dq_free);
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        reduce(tile, 0, 4);
        if (leader) bulk_wait_read<0>();
        named_bar_sync(1, 128);
        stage(v2, 0);
        stage(v3, 2);
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        reduce(tile, 4, 4);
      }
    }
    g += t.n_steps;
    }
    if (!L::kDqDirect && leader) bulk_wait_all();
  }
  } else {
  regs_inc<L::kRegsPS>();
  if (run) {
    // --------------------------------------------------------- P and dS
    const int wg = warp >> 2;
    const int quad = warp & 3;
    const int jr = quad * 32 + lane;  // key within the tile == TMEM lane
    const int col0 = 64 * wg;         // this warpgroup's query columns
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tmem + lane_off + L::kColS + col0;
    const uint32_t tDP = tmem + lane_off + L::kColDP + col0;
    const uint32_t tPst = tmem + lane_off + L::kColS + 64u * wg;   // packed P^T (32 columns)
    const uint32_t sDSrow = sbase + L::kOffDS + wg * L::kHalf + jr * 128;
    const float sl2 = a.scale_log2;
    bool ok = true;
    int g = 0;
    for (int r = 0; ok; ++r) {
      const int w = peek_item(r, ok);
      __syncwarp();
      if (PERSIST && ok && lane == 0) mbar_arrive(&bar_item_empty[r & 1]);
      if (!ok || w >= n_items) break;
    const Item t = item_at(w);
    const int jt = t.jt, bb = t.bb, hh = t.hh;
    const int key = jt * 128 + jr;
    const bool key_ok = key < t.len;
    BitWalk walk(qbits, qbits, nwords);
    for (int it = 0; it < t.n_steps; ++it) {
      const int i = SPARSE ? walk.next() : q_tile(t, it);
      const int gs = g + it;
      const uint32_t ph = gs & 1;
      const int rs = gs % L::kRowStages;
      const uint32_t rowbuf = sbase + L::kOffRow + rs * L::kRowStage;
      if (!mbar_wait(bar_s, ph, ab) || !mbar_wait(&bar_row_full[rs], (gs / L::kRowStages) & 1, ab)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t u[2][32];
      tmem_ld32(tS, u[0]);
      tmem_ld32(tS + 32u, u[1]);
      tmem_ld_wait();
      reg_fence(u[0]);
      reg_fence(u[1]);
      // P^T_jq = 2^(s * scale * log2 e - lse2_q); padded queries have lse2 = +inf.
      // Scale/subtract on the packed f32x2 pipe; of every 8 pairs,
      // bwd_poly_pairs_of8 take the exponential on the FMA pipe
      // (polynomial), the rest on MUFU.
      float p[64];
      const uint64_t sl2x2 = f2_pack(sl2, sl2);
#pragma unroll
      for (int c4 = 0; c4 < 16; ++c4) {
        const float4 l4 = ld_shared_f4(rowbuf + 4u * (col0 + 4 * c4));
#pragma unroll
        for (int e2 = 0; e2 < 2; ++e2) {
          const int c = 4 * c4 + 2 * e2;
          const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(u[c >> 5][c & 31]), __uint_as_float(u[c >> 5][(c + 1) & 31])),
                                     sl2x2, f2_pack(e2 ? -l4.z : -l4.x, e2 ? -l4.w : -l4.y));
          if (((c >> 1) & 7) < bwd_poly_pairs_of8<D>()) {
            exp2_poly_x2(x2, p[c], p[c + 1]);
          } else {
            float x0, x1;
            f2_unpack(x2, x0, x1);
            p[c] = ex2(x0);
            p[c + 1] = ex2(x1);
          }
        }
      }
      if (!key_ok) {
#pragma unroll
        for (int c = 0; c < 64; ++c) p[c] = 0.f;
      }
      if (CAUSAL && i == jt) {
        // diagonal tile: query 128 i + col0 + c sees key 128 i + jr iff col0 + c >= jr
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (col0 + c < jr) p[c] = 0.f;
      }
      uint32_t keep_bits[2] = {0xffffffffu, 0xffffffffu};
      if (DROPOUT) {
        // Key pair u = key >> 1 is decided by one hash per query; the even
        // key reads its low 16 bits and the odd key its high 16 bits:
        // (w & 0xffff) >= T for the even key, and w >= T * 2^16, which is
        // (w >> 16) >= T, for the odd key -- one mask and one compare.
        // (Sharing each hash between the two lanes of a pair by a shuffle was
        // measured at twice the kernel time.)
        const bool odd = (jr & 1) != 0;
        const uint32_t u = (uint32_t)key >> 1;
        const uint32_t lane_mask = odd ? 0xffffffffu : 0xffffu;
        const uint32_t lane_thr = odd ? (a.drop_threshold << 16) : a.drop_threshold;
        if (a.drop_threshold >= 65536u) {
          keep_bits[0] = keep_bits[1] = 0u;  // p so close to 1 that every element is dropped
        } else {
#pragma unroll
          for (int c4 = 0; c4 < 16; ++c4) {
            const float4 k4 = ld_shared_f4(rowbuf + 1024u + 4u * (col0 + 4 * c4));
            const uint32_t kv[4] = {__float_as_uint(k4.x), __float_as_uint(k4.y), __float_as_uint(k4.z),
                                    __float_as_uint(k4.w)};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c = 4 * c4 + e;
              if ((dropout_hash(kv[e], u) & lane_mask) < lane_thr) keep_bits[c >> 5] &= ~(1u << (c & 31));
            }
          }
        }
      }
      {
        uint32_t pk[2][16];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          float p0 = p[2 * c], p1 = p[2 * c + 1];
          if (DROPOUT) {
            p0 = ((keep_bits[(2 * c) >> 5] >> ((2 * c) & 31)) & 1u) ? p0 * a.drop_scale : 0.f;
            p1 = ((keep_bits[(2 * c + 1) >> 5] >> ((2 * c + 1) & 31)) & 1u) ? p1 * a.drop_scale : 0.f;
          }
          pk[c >> 4][c & 15] = pack_bf16x2(p0, p1);
        }
        tmem_st16(tPst, pk[0]);
        tmem_st16(tPst + 16u, pk[1]);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar_p);
      }
      // the undropped P^T for dS, as fp16 pairs (relative error 2^-11, below
      // the bf16 rounding dS itself gets): frees registers so both dP halves
      // load with one wait
      uint32_t ph16[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        __half2 hv = __floats2half2_rn(p[2 * c], p[2 * c + 1]);
        ph16[c] = *reinterpret_cast<uint32_t*>(&hv);
      }
      // dS^T = P^T * (dP^T * Z / (1 - p) - D)
      if (!mbar_wait(bar_dp, ph, ab)) {
        ok = false;
        break;
      }
      // dQ(i-1) and dK(i-1) read sDS; wait for the later one before overwriting
      if (gs > 0 && !mbar_wait(bar_dk, ph ^ 1u, ab)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t g[2][32];
      tmem_ld32(tDP, g[0]);
      tmem_ld32(tDP + 32u, g[1]);
      tmem_ld_wait();
      reg_fence(g[0]);
      reg_fence(g[1]);
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t pk[16];
#pragma unroll
        for (int c2 = 0; c2 < 8; ++c2) {
          const float4 d4 = ld_shared_f4(rowbuf + 512u + 4u * (col0 + 32 * hf + 4 * c2));
#pragma unroll
          for (int e2 = 0; e2 < 2; ++e2) {
            const int c = 32 * hf + 4 * c2 + 2 * e2;
            float dp0 = __uint_as_float(g[hf][4 * c2 + 2 * e2]), dp1 = __uint_as_float(g[hf][4 * c2 + 2 * e2 + 1]);
            if (DROPOUT) {
              dp0 = ((keep_bits[c >> 5] >> (c & 31)) & 1u) ? dp0 * a.drop_scale : 0.f;
              dp1 = ((keep_bits[(c + 1) >> 5] >> ((c + 1) & 31)) & 1u) ? dp1 * a.drop_scale : 0.f;
            }
            // dS = P * (dP - D) = P * dP - P * D on the packed pipe
            const float2 pf = __half22float2(*reinterpret_cast<const __half2*>(&ph16[c >> 1]));
            const uint64_t p2 = f2_pack(pf.x, pf.y);
            const uint64_t pd = f2_mul(p2, f2_pack(e2 ? -d4.z : -d4.x, e2 ? -d4.w : -d4.y));
            float ds0, ds1;
            f2_unpack(f2_fma(p2, f2_pack(dp0, dp1), pd), ds0, ds1);
            pk[2 * c2 + e2] = pack_bf16x2(ds0, ds1);
          }
        }
        // dS into shared memory (A operand of dQ = dS K and, read K-major, of
        // dK = dS^T Q): row jr of this half, 16-byte chunks XOR-swizzled by
        // (jr mod 8)
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          const uint32_t chunk = (uint32_t)(4 * hf + q8);
          st_shared_v4(sDSrow + ((chunk ^ (uint32_t)(jr & 7)) << 4), pk[4 * q8], pk[4 * q8 + 1], pk[4 * q8 + 2],
                       pk[4 * q8 + 3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar_ds);
      mbar_arrive(&bar_row_empty[rs]);
    }
    // epilogue: warpgroup 0 writes dV, warpgroup 1 writes dK = scale * acc,
    // then both release the accumulators to the next item's first products
    if (!ok) break;
    if (SPARSE && t.n_steps == 0) {
      // no query tile sees this key tile
      const long long zrow = t.row0 + key - a.kv_row_off;
      const long long zoff = wg == 0 ? bb * a.dv_sb + hh * a.dv_sh + zrow * a.dv_sn
                                     : bb * a.dk_sb + hh * a.dk_sh + zrow * a.dk_sn;
      __nv_bfloat16* dst = (wg == 0 ? a.dv : a.dk) + zoff;
      if (key_ok && FA_IN(kSiteBwdKV, zoff, D, wg == 0 ? dv_lim : dk_lim, a.err)) {
#pragma unroll
        for (int c = 0; c < D; c += 8) st_global_v4(dst + c, 0u, 0u, 0u, 0u);
      }
    } else if (t.n_steps > 0) {
      if (!mbar_wait(bar_dk, (g + t.n_steps - 1) & 1, ab)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t src = tmem + lane_off + (wg == 0 ? L::kColDV : L::kColDK);
      const float mul = wg == 0 ? 1.f : a.scale;
      const long long krow = t.row0 + (key_ok ? key : jt * 128) - a.kv_row_off;
      const long long koff = wg == 0 ? bb * a.dv_sb + hh * a.dv_sh + krow * a.dv_sn
                                     : bb * a.dk_sb + hh * a.dk_sh + krow * a.dk_sn;
      const bool k_in = !key_ok || FA_IN(kSiteBwdKV, koff, D, wg == 0 ? dv_lim : dk_lim, a.err);
      __nv_bfloat16* dst = (wg == 0 ? a.dv : a.dk) + koff;
#pragma unroll
      for (int c4 = 0; c4 < D / 32; ++c4) {
        uint32_t v[32];
        tmem_ld32_sync(src + 32u * c4, v);
        uint32_t w[16];
#pragma unroll
        for (int k = 0; k < 16; ++k)
          w[k] = pack_bf16x2(__uint_as_float(v[2 * k]) * mul, __uint_as_float(v[2 * k + 1]) * mul);
        if (key_ok && k_in) {
#pragma unroll
          for (int v4 = 0; v4 < 4; ++v4)
            st_global_v4(dst + 32 * c4 + 8 * v4, w[4 * v4], w[4 * v4 + 1], w[4 * v4 + 2], w[4 * v4 + 3]);
        }
      }
      tc_fence_before();
      mbar_arrive(bar_acc_free);
    }
    g += t.n_steps;
    }
  }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D, bool CAUSAL, bool DROPOUT, bool SPARSE, bool VARLEN>
cudaError_t launch_bwd_main(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                            const CUtensorMap& mdo, const BwdArgs& a, cudaStream_t st) {
  using L = BwdLayout<D, DROPOUT>;
  auto kern = bwd_kernel<D, CAUSAL, DROPOUT, SPARSE, VARLEN>;
  const int smem = (int)(SPARSE ? L::kSmemSparse : L::kSmem);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // One CTA per SM looping over the work items.  Block-sparse, variable-length
  // and dropout kernels run one CTA per item: block-sparse and variable-length
  // items differ in length in ways only device data knows, and with dropout
  // (one row-statistics stage at d = 128) the persistent grid measured 10%
  // slower on N = 65536.
  const int nT = (a.N + 127) / 128;
  const int kt_hi = a.kv_hi < nT ? a.kv_hi : nT, kt_lo = a.kv_lo < kt_hi ? a.kv_lo : kt_hi;
  long long grid = (long long)a.B * a.H * (kt_hi - kt_lo);
  if (grid == 0) return cudaSuccess;
  if (!SPARSE && !DROPOUT && !VARLEN) {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && sms > 0 && grid > sms)
      grid = sms;
  }
  kern<<<(unsigned)grid, L::kThreads, smem, st>>>(mq, mk, mv, mdo, a);
  return cudaGetLastError();
}

// Blocks for a grid-stride kernel of 256 threads: enough for `units` of work
// at `per_block` units a block, at most 8 per SM.
inline unsigned small_grid(long long units, long long per_block) {
  const long long b = (units + per_block - 1) / per_block;
  return (unsigned)(b < 1 ? 1 : (b > 148 * 8 ? 148 * 8 : b));
}

inline cudaError_t launch_bwd_prepare(const BwdArgs& a, int d, cudaStream_t st) {
  const int BH = a.B * a.H;
  const int npad = (a.N + 127) / 128 * 128;
  // a block's 8 warps take 8 * (32 / lanes per row) * 4 rows per pass, and
  // 256 float4 of the accumulator
  const long long rows = (long long)BH * npad;
  const long long rows_per_block = 8LL * (32 / (d * 2 / 16)) * 4;
  const long long n4 = rows * d / 4;
  const unsigned grid = max(small_grid(rows, rows_per_block), small_grid(n4, 256));
  if (d == 64)
    bwd_pre_kernel<64><<<grid, 256, 0, st>>>(a, BH, npad);
  else
    bwd_pre_kernel<128><<<grid, 256, 0, st>>>(a, BH, npad);
  return cudaGetLastError();
}

template <int D, bool SPARSE, bool VARLEN>
cudaError_t launch_bwd_recompute_d(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                                   const CUtensorMap& mdo, const BwdArgs& a, bool causal,
                                   bool dropout, cudaStream_t st) {
  if (causal)
    return dropout ? launch_bwd_main<D, true, true, SPARSE, VARLEN>(mq, mk, mv, mdo, a, st)
                   : launch_bwd_main<D, true, false, SPARSE, VARLEN>(mq, mk, mv, mdo, a, st);
  return dropout ? launch_bwd_main<D, false, true, SPARSE, VARLEN>(mq, mk, mv, mdo, a, st)
                 : launch_bwd_main<D, false, false, SPARSE, VARLEN>(mq, mk, mv, mdo, a, st);
}

inline cudaError_t launch_bwd_recompute(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                                        const CUtensorMap& mdo, const BwdArgs& a, int d,
                                        bool causal, bool dropout, cudaStream_t st) {
  if (a.bmask)
    return d == 64 ? launch_bwd_recompute_d<64, true, false>(mq, mk, mv, mdo, a, causal, dropout, st)
                   : launch_bwd_recompute_d<128, true, false>(mq, mk, mv, mdo, a, causal, dropout, st);
  if (a.cu_seqlens)
    return d == 64 ? launch_bwd_recompute_d<64, false, true>(mq, mk, mv, mdo, a, causal, dropout, st)
                   : launch_bwd_recompute_d<128, false, true>(mq, mk, mv, mdo, a, causal, dropout, st);
  return d == 64 ? launch_bwd_recompute_d<64, false, false>(mq, mk, mv, mdo, a, causal, dropout, st)
                 : launch_bwd_recompute_d<128, false, false>(mq, mk, mv, mdo, a, causal, dropout, st);
}

inline cudaError_t launch_bwd_finalize(const BwdArgs& a, int d, cudaStream_t st) {
  // one thread per 8 columns of a (padded) row
  const unsigned grid = small_grid((long long)a.B * a.H * ((a.N + 127) / 128) * 128 * (d / 8), 256);
  if (d == 64)
    bwd_post_kernel<64><<<grid, 256, 0, st>>>(a.dq_acc, a.dq, a.B * a.H, a.H, a.N, a.dq_sb, a.dq_sh, a.dq_sn,
                                              a.scale, a.cu_seqlens, a.seqused, a.total_tokens, a.err);
  else
    bwd_post_kernel<128><<<grid, 256, 0, st>>>(a.dq_acc, a.dq, a.B * a.H, a.H, a.N, a.dq_sb, a.dq_sh, a.dq_sn,
                                               a.scale, a.cu_seqlens, a.seqused, a.total_tokens, a.err);
  return cudaGetLastError();
}

}  // namespace fa
