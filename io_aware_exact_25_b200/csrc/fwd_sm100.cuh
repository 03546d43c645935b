// fwd_sm100.cuh -- fused attention forward for sm_100a.
//
// O = softmax(scale * Q K^T [+ causal mask]) V with an optional dropout mask
// applied to the probabilities, and lse = logsumexp of each (undropped,
// scaled, masked) score row.  The method is the tiled, fused forward with an
// online softmax: "How FlashAttention Optimizes GPU Memory for Fast AI
// Training" (Tiling, Online Softmax, Kernel Fusion) and "FlashAttention for
// Efficient Training" section 3 (Algorithmic Details: S_ij = Q_i K_j^T /
// sqrt(d_k) per block, running maxima and sums, O written once) and
// section 3.2 (logsumexp, rescaling during accumulation).
//
// One CTA owns 256 query rows of one head as two 128-row tiles Q0, Q1 and
// streams BN-key tiles K_j, V_j through a shared-memory ring: BN = 128, or 64
// for the plain forward at d = 64, where two CTAs share an SM (fwd_bn).  Warp
// roles:
//   warps 0-3   softmax for Q0 (one query row per thread, TMEM lanes 0-127)
//   warps 4-7   softmax for Q1
//   warp  8     tcgen05 MMA issue (one thread)
//   warp  9     TMA producer (one thread)
//   warps 10-11 idle (they complete warpgroup 2 for the register split)
// Tensor memory (4 BN columns): S_t = Q_t K_j^T (fp32, BN columns) at column
// BN t; P_t (bf16 pairs, BN / 2 columns) overwrites the first half of S_t and
// is the A operand of O_t += P_t V_j; O_t (fp32, D columns) at 2 BN + D t.
// The two Q tiles ping-pong: while one tile's softmax runs, the tensor core
// works on the other tile's MMAs.  O_t is only rescaled by its own softmax
// warps, after S_t(j) has completed, which implies that every earlier MMA of
// the issuing thread -- O_t += P_t V(j-1) included -- has completed too.
//
// Block-sparse mode ("FlashAttention for Efficient Training" section 3.2,
// Block-Sparse Attention Support): a byte mask over 128 x 128 blocks says
// which key tiles each query tile sees.  The producer warp turns the CTA's two
// mask rows into bit sets in shared memory; the K/V ring then streams only
// the union of the two sets, each softmax warpgroup walks its own set, and
// the MMA issuer skips the products of a tile its query tile does not see.
// A query tile that sees no key tile writes O = 0 and lse = -inf.
//
// Variable-length mode ("FlashAttention for Efficient Training" section 5.2,
// Handling Variable Sequence Lengths): the B sequences are stored token-major
// and sequence b owns tokens [cu_seqlens[b], cu_seqlens[b+1]), of which the
// first L_b are real (seqused[b], else all of them).  A CTA covers 256 rows of
// one sequence and head; keys at or beyond L_b are masked like the ragged
// last tile of a dense problem, and a CTA whose rows all lie at or beyond L_b
// returns at once, so no work is spent on padding.
//
// Online softmax in base 2: x = s * scale * log2(e); m is a running row
// maximum that is only raised (and O, l rescaled) when the tile maximum
// exceeds it by more than 8, i.e. a factor 256.  Every P and l use the same
// stale m, so the final O / l is exact; P values stay below 256.
#pragma once

#include "debug_check.cuh"
#include "dropout_hash.cuh"
#include "sm100.cuh"

namespace fa {

struct FwdArgs {
  int B, H, N;
  float scale_log2;         // scale * log2(e)
  uint32_t drop_threshold;  // keep iff the key's 16-bit half of the pair hash >= threshold
  float drop_scale;         // 1 / (1 - p)
  uint64_t seed;
  __nv_bfloat16* o;            // [B,H,N,D] with element strides o_sb, o_sh, o_sn
  long long o_sb, o_sh, o_sn;
  float* lse;                  // [B,H,N] contiguous, natural log
  int* err;          // device error word (may be null)
  // split-KV (SPLIT kernels only): each CTA covers key tiles [j0, j1) of its
  // query tiles, split = blockIdx % num_splits, and writes O / l (fp32) and
  // its lse into part_o [split][BH][N][D] and part_lse [split][BH][N]
  int num_splits;
  float* part_o;
  float* part_lse;
  // split-KV key window: only key tiles [kv_lo, kv_hi) are split (and seen);
  // the K/V tensors hold key rows from kv_row_off on (a rank's key chunk)
  int kv_lo, kv_hi, kv_row_off;
  int partial_only;  // host side: split-KV pieces are the output (no combine pass)
  // block-sparse (SPARSE kernels only): bmask[hm][qt][kt] != 0 lets query
  // tile qt see key tile kt; hm = 0 when bmask_heads == 1, else the head
  const uint8_t* bmask;
  int bmask_heads;
  // fault injection for tests: the producer issues no K/V load, so the MMA
  // warp's first wait runs out and the kernel reports a timeout
  int debug_skip_kv;
  // variable-length (VARLEN kernels only): token offsets [B+1], optional used
  // lengths [B], the token count T (q/k/v/o rows; lse is [H, T]); N holds the
  // largest slot size and sizes the grid
  const int* cu_seqlens;
  const int* seqused;
  int total_tokens;
};

// Kernel variants: plain, split-KV, block-sparse, variable-length.
enum FwdMode : int { kFwdPlain = 0, kFwdSplit = 1, kFwdSparse = 2, kFwdVarlen = 3 };

// Of every 8 pairs of probabilities, this many take the exponential on the
// FMA pipe (polynomial) and the rest on the MUFU unit, balancing the two.
constexpr int kPolyPairsOf8 = 0;

// Key tile width: 64 keys for the plain forward at d = 64, 128 otherwise.
// With 64-key tiles a CTA needs 256 TMEM columns and 96 KB of shared memory,
// so two CTAs share an SM and each SMSP runs four softmax warps instead of two
// (at d = 64 the softmax, not the tensor core, bounds the forward).
template <int D, int MODE>
__host__ __device__ constexpr int fwd_bn() { return (D == 64 && MODE == kFwdPlain) ? 64 : 128; }

template <int D, int BN = 128>
struct FwdLayout {
  // 12 warps: softmax warpgroups 0-1, and warpgroup 2 (MMA issue, TMA
  // producer, two idle warps) so that every warpgroup is whole for the
  // register reallocation.  One CTA per SM (128-key tiles): launched at 168
  // registers a thread (3 warps per SMSP x 168 fill its 16K registers), then
  // 200 for the softmax warpgroups and 96 for warpgroup 2: 256 * 200 + 128 *
  // 96 = 63488 <= 384 * 168.  (At 168 for every warp the softmax spilled
  // 48-76 bytes a thread; measured: the forward 2.8 % faster at d = 128, 7.8 %
  // at d = 64.)  Two CTAs per SM (64-key tiles): launched at 80, then 96 for
  // the softmax and 48 for warpgroup 2: 256 * 96 + 128 * 48 = 30720 = 384 * 80.
  static constexpr int kCtasPerSm = BN == 64 ? 2 : 1;
  static constexpr int kThreads = 384;
  static constexpr uint32_t kRegsLaunch = BN == 64 ? 80 : 168;
  static constexpr uint32_t kRegsSoftmax = BN == 64 ? 96 : 200, kRegsCtl = BN == 64 ? 48 : 96;
  static_assert(256 * kRegsSoftmax + 128 * kRegsCtl <= 384 * kRegsLaunch, "register split");
  static constexpr uint32_t kHalf = 128u * 128u;     // one 128-row x 64-column bf16 half tile (Q)
  static constexpr uint32_t kHalfKV = BN * 128u;     // one BN-row x 64-column bf16 half tile (K, V)
  static constexpr uint32_t kTile = 128u * D * 2u;   // one 128 x D bf16 tile (Q)
  static constexpr uint32_t kTileKV = BN * D * 2u;   // one BN x D bf16 tile (K, V)
  static constexpr int kStages = (BN == 64 || D == 64) ? 8 : 4;  // K/V ring depth
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffKV = kOffQ + 2 * kTile;
  static constexpr uint32_t kOffBar = kOffKV + kStages * kTileKV;
  static constexpr int kNumBars = 2 + 2 * kStages + 2 + 2 + 2 + 2 + 1;
  static constexpr uint32_t kSmem = kOffBar + kNumBars * 8 + 16;
  // block-sparse: two key-tile bit sets and three counts after the barriers
  static constexpr uint32_t kOffBits = (kSmem + 15u) & ~15u;
  static constexpr uint32_t kSmemSparse = kOffBits + 2u * kSparseWords * 4u + 16u;
  static constexpr uint32_t kTmemCols = 4u * BN;  // S_0, S_1 (BN columns each), O_0, O_1 (D <= BN each)
  static constexpr uint32_t kColO = 2u * BN;      // O_t at kColO + D * t
  static_assert(D <= BN, "O_t fits in BN columns");
  static_assert(kSmemSparse <= 232448, "shared memory budget");
  static_assert(BN == 128 || kCtasPerSm * (kSmem + 1024) <= 233472, "two CTAs per SM");
};

template <int D, bool CAUSAL, bool DROPOUT, int MODE>
__global__ void __launch_bounds__(384, (fwd_bn<D, MODE>() == 64) ? 2 : 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const FwdArgs a) {
  constexpr int BN = fwd_bn<D, MODE>();  // keys per K/V tile
  using L = FwdLayout<D, BN>;
  constexpr bool SPLIT = MODE == kFwdSplit;
  constexpr bool SPARSE = MODE == kFwdSparse;
  constexpr bool VARLEN = MODE == kFwdVarlen;
  static_assert(D == 64 || D == 128, "head dim");
  extern __shared__ __align__(1024) uint8_t smem[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* bar_q = bars;                               // [2]   Q_t landed
  uint64_t* bar_kv_full = bars + 2;                     // [S]   K/V stage landed
  uint64_t* bar_kv_empty = bar_kv_full + L::kStages;    // [S]   K/V stage consumed
  uint64_t* bar_s = bar_kv_empty + L::kStages;          // [2]   S_t ready in TMEM
  uint64_t* bar_p = bar_s + 2;                          // [2]   P_t written (128 arrivals)
  uint64_t* bar_pv = bar_p + 2;                         // [2]   O_t += P_t V_j done
  uint64_t* bar_p_half = bar_pv + 2;                    // [2]   first half of P_t written
  uint64_t* bar_drain = bar_p_half + 2;                 //       all MMAs retired
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_drain + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  const uint32_t sbase = smem_u32(smem);

  // Work tile.  For the causal mask the CTA with the most key tiles goes
  // first (longest-processing-time order across the grid); heads are
  // interleaved, and the CTAs of a wave sweep the key tiles of their heads in
  // near lockstep, so the K/V tiles they read stay in L2.
  const int BH = a.B * a.H;
  const int n_cta_tiles = (a.N + 255) >> 8;
  const int split = SPLIT ? (int)(blockIdx.x % (unsigned)a.num_splits) : 0;
  const int work = SPLIT ? (int)(blockIdx.x / (unsigned)a.num_splits) : (int)blockIdx.x;
  const int tile_rev = work / BH;
  const int bh = work - tile_rev * BH;
  const int cta_tile = CAUSAL ? (n_cta_tiles - 1 - tile_rev) : tile_rev;
  const int bb = bh / a.H, hh = bh - bb * a.H;  // batch and head of this CTA
  // this CTA's sequence: real rows [0, seq_len) at tokens row0.. of the
  // tensors, batch coordinate wc of the tensor maps
  int seq_len = a.N, row0 = 0, wc = bb;
  long long lse_base = (long long)bh * a.N;
  if (VARLEN) {
    const SeqSpan sp = varlen_span(a.cu_seqlens, a.seqused, bb, a.total_tokens, a.N, a.err, cta_tile == 0);
    seq_len = sp.len;
    row0 = sp.row0;
    wc = 0;
    lse_base = (long long)hh * a.total_tokens + row0;
    if (cta_tile * 256 >= seq_len) return;  // only padding (or nothing) here: no work
  }
  const int n_kv_all = (seq_len + BN - 1) / BN;
  const int qt0 = 2 * cta_tile;
  // buffer extents for the bounds-checking build (unused otherwise)
  const long long rows_q = VARLEN ? a.total_tokens : a.N;
  const long long rows_k = VARLEN ? a.total_tokens : min((long long)a.N, (long long)a.kv_hi * 128) - a.kv_row_off;
  const long long o_lim = extent4(VARLEN ? 1 : a.B, a.H, rows_q, D, a.o_sb, a.o_sh, a.o_sn);
  const long long lse_lim = VARLEN ? (long long)a.H * a.total_tokens : (long long)BH * a.N;
  const long long part_rows = (long long)a.num_splits * BH * a.N;
  (void)rows_q, (void)rows_k, (void)o_lim, (void)lse_lim, (void)part_rows;
  const bool act1 = (qt0 + 1) * 128 < seq_len;
  // key tiles each Q tile sees: [0, end_t)
  const int end0 = CAUSAL ? min(n_kv_all, (qt0 + 1) * (128 / BN)) : n_kv_all;
  const int end1 = act1 ? (CAUSAL ? min(n_kv_all, (qt0 + 2) * (128 / BN)) : n_kv_all) : 0;
  const int end_max = end0 > end1 ? end0 : end1;
  // this CTA's share [j0, j0 + span) of that range; nkv_t counts the tiles
  // tile t processes here, local index jj = j - j0 drives the pipelines
  int j0 = 0, span = end_max;
  if (SPLIT) {
    const int hi = min(a.kv_hi, end_max), lo = min(a.kv_lo, hi);
    const int chunk = (hi - lo + a.num_splits - 1) / a.num_splits;
    j0 = lo + split * chunk;
    span = max(0, min(hi, j0 + chunk) - j0);
  }
  // steps of the K/V stream (nkv_max) and how many of them each Q tile uses
  int nkv0 = max(0, min(end0, j0 + span) - j0);
  int nkv1 = max(0, min(end1, j0 + span) - j0);
  int nkv_max = nkv0 > nkv1 ? nkv0 : nkv1;
  uint32_t* bits0 = reinterpret_cast<uint32_t*>(smem + L::kOffBits);  // SPARSE: key tiles of Q0
  uint32_t* bits1 = bits0 + kSparseWords;                              // SPARSE: key tiles of Q1
  int* sparse_cnt = reinterpret_cast<int*>(bits1 + kSparseWords);
  const int nwords = (n_kv_all + 31) >> 5;

  if (threadIdx.x == 0) {
    mbar_init(&bar_q[0], 1);
    mbar_init(&bar_q[1], 1);
    for (int s = 0; s < L::kStages; ++s) {
      mbar_init(&bar_kv_full[s], 1);
      mbar_init(&bar_kv_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bar_s[t], 1);
      mbar_init(&bar_p[t], 128);
      mbar_init(&bar_pv[t], 1);
      mbar_init(&bar_p_half[t], 128);
    }
    mbar_init(bar_drain, 1);
    const bool misaligned = (sbase & 1023u) != 0u;
    *abort_flag = misaligned ? 1 : 0;
    if (misaligned && a.err) atomicCAS(a.err, kDevOk, kDevMisaligned);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, L::kTmemCols);
    tmem_relinquish();
  }
  if (SPARSE && warp == 9) {
    const int hm = a.bmask_heads == 1 ? 0 : hh;
    const uint8_t* row0 = a.bmask + ((size_t)hm * n_kv_all + qt0) * n_kv_all;
    const int3 c = build_bit_sets(row0, end0, act1 ? row0 + n_kv_all : nullptr, end1, 0, 1, nwords, bits0, bits1, lane);
    if (lane == 0) {
      sparse_cnt[0] = c.x;
      sparse_cnt[1] = c.y;
      sparse_cnt[2] = c.z;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Abort ab{abort_flag, a.err};
  const bool run = *abort_flag == 0;
  if (SPARSE) {
    nkv0 = sparse_cnt[0];
    nkv1 = sparse_cnt[1];
    nkv_max = sparse_cnt[2];
  }

  // Each warpgroup sets its register budget at the top of its branch (every
  // thread of the warpgroup, whatever its role or the abort state).
  if (warp >= 8) {
  regs_dec<L::kRegsCtl>();
  if (run && warp == 9) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      const uint64_t pol_keep = policy_evict_last();   // K/V: re-read by every Q tile of the head
      const uint64_t pol_once = policy_evict_first();  // Q: read once
      // (a CTA with no key tile to visit loads nothing)
      for (int t = 0; t < 2 && nkv_max > 0; ++t) {
        if (t == 1 && !act1) break;
        mbar_arrive_expect_tx(&bar_q[t], L::kTile);
        (void)FA_IN(kSiteFwdTile, row0 + (qt0 + t) * 128, 1, rows_q, a.err);
        for (int h = 0; h < D / 64; ++h)
          tma_load_4d(smem + L::kOffQ + t * L::kTile + h * L::kHalf, &tm_q, 64 * h, row0 + (qt0 + t) * 128, hh,
                      wc, &bar_q[t], pol_once);
      }
      int stage = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      BitWalk walk(bits0, bits1, nwords);
      for (int j = 0; j < nkv_max && ok && !a.debug_skip_kv; ++j) {
        const int kt = SPARSE ? walk.next() : j0 + j;  // key tile of this step
        for (int which = 0; which < 2; ++which) {
          if (!mbar_wait(&bar_kv_empty[stage], phase ^ 1u, ab)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar_kv_full[stage], L::kTileKV);
          const CUtensorMap* m = which ? &tm_v : &tm_k;
          (void)FA_IN(kSiteFwdTile, row0 + kt * BN - a.kv_row_off, 1, rows_k, a.err);
          for (int h = 0; h < D / 64; ++h)
            tma_load_4d(smem + L::kOffKV + stage * L::kTileKV + h * L::kHalfKV, m, 64 * h,
                        row0 + kt * BN - a.kv_row_off, hh, wc, &bar_kv_full[stage], pol_keep);
          ++issued;
          if (++stage == L::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Every load issued must land before the CTA may exit.
      if (nkv_max > 0) {
        mbar_wait_drain(&bar_q[0], 0);
        if (act1) mbar_wait_drain(&bar_q[1], 0);
      }
      const int first = issued > L::kStages ? issued - L::kStages : 0;
      for (int n = first; n < issued; ++n) mbar_wait_drain(&bar_kv_full[n % L::kStages], (n / L::kStages) & 1);
    }
  } else if (run && warp == 8) {
    // ------------------------------------------------------- MMA issuer
    // Issue order for key tile j: O0 += P0 V(j-1), S0(j), O1 += P1 V(j-1),
    // S1(j).  S_t(j) overwrites the TMEM columns that hold P_t(j-1); it is
    // queued directly behind the product that reads P_t(j-1) and the tensor
    // core executes the MMAs of one issuing thread in order, so no wait is
    // needed between them.  The softmax publishes P_t in two halves (keys
    // 0-63, 64-127) so the product starts on the first half early.  K(j)
    // sits at ring position 2j, V(j) at 2j+1; stages are released in ring
    // order.  A Q tile that does not see the key tile of a step (block-sparse)
    // gets neither product for it; its P V product for its previous tile is
    // still issued on the step after that tile.
    if (lane == 0) {
      constexpr uint32_t kIdS = idesc_bf16(128, BN, false, false);  // S = Q K^T, both K-major
      constexpr uint32_t kIdO = idesc_bf16(128, D, false, true);     // O += P V, V is MN-major
      bool ok = nkv_max > 0 && mbar_wait(&bar_q[0], 0, ab) && (!act1 || mbar_wait(&bar_q[1], 0, ab));
      bool issued_any = false;
      auto stage_of = [](int pos) { return pos % L::kStages; };
      auto phase_of = [](int pos) { return (uint32_t)((pos / L::kStages) & 1); };
      auto issue_s = [&](int t, uint32_t sK) {
        const uint32_t sQ = sbase + L::kOffQ + t * L::kTile;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tmem + (uint32_t)BN * t, desc_kmajor(sQ, kk, L::kHalf), desc_kmajor(sK, kk, L::kHalfKV), kIdS,
                 kk > 0 ? 1u : 0u);
        mma_commit(&bar_s[t]);
        issued_any = true;
      };
      auto issue_pv = [&](int t, int j, uint32_t sV) -> bool {
        if (!mbar_wait(&bar_p_half[t], j & 1, ab)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BN / 32; ++kk)
          mma_ts(tmem + L::kColO + D * t, tmem + (uint32_t)BN * t + 8u * kk, desc_mnmajor(sV, kk, L::kHalfKV), kIdO,
                 (j > 0 || kk > 0) ? 1u : 0u);
        if (!mbar_wait(&bar_p[t], j & 1, ab)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = BN / 32; kk < BN / 16; ++kk)
          mma_ts(tmem + L::kColO + D * t, tmem + (uint32_t)BN * t + 8u * kk, desc_mnmajor(sV, kk, L::kHalfKV), kIdO, 1u);
        mma_commit(&bar_pv[t]);
        return true;
      };
      // does Q tile t see the key tile kt of step j?
      auto sees = [&](int t, int j, int kt) -> bool {
        if (SPARSE) return bit_set(t ? bits1 : bits0, kt);
        return j < (t ? nkv1 : nkv0);
      };
      BitWalk walk(bits0, bits1, nwords);
      int pv_count[2] = {0, 0};  // P V products issued per Q tile
      bool prev[2] = {false, false};
      if (nkv_max == 0) {
        ok = false;  // nothing to do in this split / block row
      } else if (ok && mbar_wait(&bar_kv_full[0], 0, ab)) {
        tc_fence_after();
        const uint32_t sK0 = sbase + L::kOffKV;
        const int kt = SPARSE ? walk.next() : j0;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          prev[t] = sees(t, 0, kt);
          if (prev[t]) issue_s(t, sK0);
        }
        mma_commit(&bar_kv_empty[0]);
      } else {
        ok = false;
      }
      for (int j = 1; j < nkv_max && ok; ++j) {
        const int posV = 2 * j - 1, posK = 2 * j;
        if (!mbar_wait(&bar_kv_full[stage_of(posV)], phase_of(posV), ab) ||
            !mbar_wait(&bar_kv_full[stage_of(posK)], phase_of(posK), ab))
          break;
        tc_fence_after();
        const uint32_t sV = sbase + L::kOffKV + stage_of(posV) * L::kTileKV;
        const uint32_t sK = sbase + L::kOffKV + stage_of(posK) * L::kTileKV;
        const int kt = SPARSE ? walk.next() : j0 + j;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (!ok) continue;
          if (prev[t] && !issue_pv(t, pv_count[t]++, sV)) {
            ok = false;
            continue;
          }
          prev[t] = sees(t, j, kt);
          if (prev[t]) issue_s(t, sK);
        }
        if (!ok) break;
        mma_commit(&bar_kv_empty[stage_of(posV)]);  // V(j-1) consumed
        mma_commit(&bar_kv_empty[stage_of(posK)]);  // K(j) consumed
      }
      if (ok && nkv_max > 0) {
        const int j = nkv_max - 1, posV = 2 * j + 1;
        if (mbar_wait(&bar_kv_full[stage_of(posV)], phase_of(posV), ab)) {
          tc_fence_after();
          const uint32_t sV = sbase + L::kOffKV + stage_of(posV) * L::kTileKV;
          bool last_ok = true;
#pragma unroll
          for (int t = 0; t < 2; ++t)
            if (last_ok && prev[t]) last_ok = issue_pv(t, pv_count[t]++, sV);
          mma_commit(&bar_kv_empty[stage_of(posV)]);
        }
      }
      if (issued_any) {
        mma_commit(bar_drain);
        mbar_wait_drain(bar_drain, 0);
      }
    }
  }
  } else {
  regs_inc<L::kRegsSoftmax>();
  if (run) {
    // ---------------------------------------------------------- softmax
    const int t = warp >> 2;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;  // row within the Q tile == TMEM lane
    if (t == 0 || act1) {
      const int nkv = t ? nkv1 : nkv0;
      const int q_row = (qt0 + t) * 128 + r;
      const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
      const uint32_t tS = tmem + lane_off + (uint32_t)BN * t;
      const uint32_t tO = tmem + lane_off + L::kColO + D * t;
      const float sl2 = a.scale_log2;
      float m_used = -INFINITY;  // running maximum (base-2 units) the P values are taken against
      float l = 0.f;             // running sum of undropped P
      uint32_t rkey = 0;
      if (DROPOUT) rkey = dropout_row_key(a.seed, (uint32_t)bb, (uint32_t)hh, (uint32_t)q_row);
      bool ok = true;
      BitWalk walk(t ? bits1 : bits0, t ? bits1 : bits0, nwords);
      for (int j = 0; j < nkv; ++j) {
        const int jg = SPARSE ? walk.next() : j0 + j;  // global key tile
        if (!mbar_wait(&bar_s[t], j & 1, ab)) {
          ok = false;
          break;
        }
        tc_fence_after();
        constexpr int kG = BN / 32;  // 32-column groups of the score tile
        uint32_t u[kG][32];
#pragma unroll
        for (int c4 = 0; c4 < kG; ++c4) tmem_ld32(tS + 32u * c4, u[c4]);
        tmem_ld_wait();
#pragma unroll
        for (int c4 = 0; c4 < kG; ++c4) reg_fence(u[c4]);
        // key BN jg + c is visible to query 128 (qt0 + t) + r iff c < lim;
        // only the diagonal tile(s) (causal) or the ragged last tile mask
        int lim = BN;
        if (CAUSAL) lim = min(BN, (qt0 + t) * 128 + r + 1 - jg * BN);
        if (!CAUSAL && jg == n_kv_all - 1 && (seq_len % BN)) lim = seq_len - jg * BN;
        if (__any_sync(0xffffffffu, lim < BN)) {
#pragma unroll
          for (int c = 0; c < BN; ++c)
            if (c >= lim) u[c >> 5][c & 31] = 0xff800000u;  // -inf
        }
        // row maximum: kG independent 3-input max chains
        float mx4[kG];
#pragma unroll
        for (int g = 0; g < kG; ++g) mx4[g] = __uint_as_float(u[g][0]);
#pragma unroll
        for (int c = 1; c < 31; c += 2)
#pragma unroll
          for (int g = 0; g < kG; ++g)
            mx4[g] = max3(mx4[g], __uint_as_float(u[g][c]), __uint_as_float(u[g][c + 1]));
#pragma unroll
        for (int g = 0; g < kG; ++g) mx4[g] = fmaxf(mx4[g], __uint_as_float(u[g][31]));
        float mx = mx4[0];
#pragma unroll
        for (int g = 1; g < kG; ++g) mx = fmaxf(mx, mx4[g]);
        const float m_new = fmaxf(m_used, mx * sl2);
        if (__any_sync(0xffffffffu, m_new > m_used + 8.0f)) {
          const float alpha = (m_new == -INFINITY) ? 1.f : ex2(m_used - m_new);
          l *= alpha;
          m_used = m_new;
          if (j > 0) {
            // O_t holds the sum over earlier tiles; O_t += P V_{j-1} has
            // retired (it completed before S_t(j) was issued).  The score
            // registers are released for the rescale and reloaded after it.
#pragma unroll
            for (int c4 = 0; c4 < D / 32; ++c4) {
              uint32_t o[32];
              tmem_ld32_sync(tO + 32u * c4, o);
#pragma unroll
              for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
              tmem_st32(tO + 32u * c4, o);
            }
            tmem_st_wait();
#pragma unroll
            for (int c4 = 0; c4 < kG; ++c4) tmem_ld32(tS + 32u * c4, u[c4]);
            tmem_ld_wait();
#pragma unroll
            for (int c4 = 0; c4 < kG; ++c4) reg_fence(u[c4]);
            if (__any_sync(0xffffffffu, lim < BN)) {
#pragma unroll
              for (int c = 0; c < BN; ++c)
                if (c >= lim) u[c >> 5][c & 31] = 0xff800000u;
            }
          }
        }
        const float msub = (m_used == -INFINITY) ? 0.f : m_used;
        // p = 2^(s * scale * log2 e - m): scale/subtract on the packed f32x2
        // pipe, exponentials on MUFU, row sum in four packed accumulators
        const uint64_t mul2 = f2_pack(sl2, sl2);
        const uint64_t sub2 = f2_pack(-msub, -msub);
        uint64_t sum2[4] = {0ull, 0ull, 0ull, 0ull};
        uint32_t pk[kG][16];
#pragma unroll
        for (int c = 0; c < BN / 2; ++c) {
          const uint64_t x2 = f2_fma(f2_pack(__uint_as_float(u[(2 * c) >> 5][(2 * c) & 31]),
                                             __uint_as_float(u[(2 * c + 1) >> 5][(2 * c + 1) & 31])),
                                     mul2, sub2);
          float p0, p1;
          if ((c & 7) < kPolyPairsOf8) {
            exp2_poly_x2(x2, p0, p1);  // FMA pipe
          } else {
            float x0, x1;
            f2_unpack(x2, x0, x1);
            p0 = ex2(x0);  // MUFU
            p1 = ex2(x1);
          }
          sum2[c & 3] = f2_add(sum2[c & 3], f2_pack(p0, p1));
          if (DROPOUT) {
            // keys 2c and 2c+1 of the tile: one pair hash
            const uint32_t w = dropout_hash(rkey, (uint32_t)(jg * (BN / 2) + c));
            p0 = keep_lo(w, a.drop_threshold) ? p0 * a.drop_scale : 0.f;
            p1 = keep_hi(w, a.drop_threshold) ? p1 * a.drop_scale : 0.f;
          }
          pk[c >> 4][c & 15] = pack_bf16x2(p0, p1);
          if (c == BN / 4 - 1) {
            // the first half of the keys done: publish it so O += P V can start
#pragma unroll
            for (int h = 0; h < kG / 2; ++h) tmem_st16(tS + 16u * h, pk[h]);
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&bar_p_half[t]);
          }
        }
        {
          float s0, s1, s2, s3, s4, s5, s6, s7;
          f2_unpack(sum2[0], s0, s1);
          f2_unpack(sum2[1], s2, s3);
          f2_unpack(sum2[2], s4, s5);
          f2_unpack(sum2[3], s6, s7);
          l += ((s0 + s1) + (s2 + s3)) + ((s4 + s5) + (s6 + s7));
        }
#pragma unroll
        for (int h = kG / 2; h < kG; ++h) tmem_st16(tS + 16u * h, pk[h]);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bar_p[t]);
      }
      // epilogue: O = O_t / l, lse = (m + log2 l) ln 2
      const bool in_range = q_row < seq_len;
      if (SPARSE && nkv == 0) {
        // the mask hides every key tile from this query tile
        if (in_range && ok) {
          const long long ooff = bb * a.o_sb + hh * a.o_sh + (long long)q_row * a.o_sn;
          __nv_bfloat16* orow = a.o + ooff;
          if (FA_IN(kSiteFwdO, ooff, D, o_lim, a.err)) {
#pragma unroll
            for (int c = 0; c < D; c += 8) st_global_v4(orow + c, 0u, 0u, 0u, 0u);
          }
          if (FA_IN(kSiteFwdLse, lse_base + q_row, 1, lse_lim, a.err)) a.lse[lse_base + q_row] = -INFINITY;
        }
      } else if (SPLIT && nkv == 0) {
        // this split holds no key tile of this query tile: an empty partial
        const long long prow_i = ((long long)split * BH + bh) * a.N + q_row;
        if (in_range && ok && FA_IN(kSiteFwdPart, prow_i, 1, part_rows, a.err)) {
          float* prow = a.part_o + prow_i * D;
#pragma unroll
          for (int c = 0; c < D; c += 4) *reinterpret_cast<float4*>(prow + c) = make_float4(0.f, 0.f, 0.f, 0.f);
          a.part_lse[prow_i] = -INFINITY;
        }
      } else if (ok && mbar_wait(&bar_pv[t], (nkv - 1) & 1, ab)) {
        tc_fence_after();
        const float inv_l = 1.f / l;
        const float lse_row = (m_used + log2f(l)) * 0.69314718055994531f;
        if (SPLIT) {
          const long long prow_i = ((long long)split * BH + bh) * a.N + (in_range ? q_row : 0);
          const bool p_ok = FA_IN(kSiteFwdPart, prow_i, 1, part_rows, a.err);
          float* prow = a.part_o + prow_i * D;
#pragma unroll
          for (int c4 = 0; c4 < D / 32; ++c4) {
            uint32_t o[32];
            tmem_ld32_sync(tO + 32u * c4, o);
            if (in_range && p_ok) {
#pragma unroll
              for (int v4 = 0; v4 < 8; ++v4)
                *reinterpret_cast<float4*>(prow + 32 * c4 + 4 * v4) =
                    make_float4(__uint_as_float(o[4 * v4]) * inv_l, __uint_as_float(o[4 * v4 + 1]) * inv_l,
                                __uint_as_float(o[4 * v4 + 2]) * inv_l, __uint_as_float(o[4 * v4 + 3]) * inv_l);
            }
          }
          if (in_range && p_ok) a.part_lse[prow_i] = lse_row;
        } else {
          const long long ooff = bb * a.o_sb + hh * a.o_sh + (long long)(row0 + (in_range ? q_row : 0)) * a.o_sn;
          const bool o_ok = FA_IN(kSiteFwdO, ooff, D, o_lim, a.err);
          __nv_bfloat16* orow = a.o + ooff;
#pragma unroll
          for (int c4 = 0; c4 < D / 32; ++c4) {
            uint32_t o[32];
            tmem_ld32_sync(tO + 32u * c4, o);
            uint32_t w[16];
#pragma unroll
            for (int k = 0; k < 16; ++k)
              w[k] = pack_bf16x2(__uint_as_float(o[2 * k]) * inv_l, __uint_as_float(o[2 * k + 1]) * inv_l);
            if (in_range && o_ok) {
#pragma unroll
              for (int v4 = 0; v4 < 4; ++v4)
                st_global_v4(orow + 32 * c4 + 8 * v4, w[4 * v4], w[4 * v4 + 1], w[4 * v4 + 2], w[4 * v4 + 3]);
            }
          }
          if (in_range && FA_IN(kSiteFwdLse, lse_base + q_row, 1, lse_lim, a.err)) a.lse[lse_base + q_row] = lse_row;
        }
      }
    }
  }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, L::kTmemCols);
  }
}

// Merge the split-KV partials: per row lse = ln sum_s exp(lse_s) and
// O = sum_s exp(lse_s - lse) O_s, the exact combination of softmax pieces over
// disjoint key ranges; a row whose pieces are all -inf gets O = 0 and
// lse = -inf.  A warp takes G rows at a time: lane l < G reduces the pieces'
// logsumexps of row l (consecutive lanes read consecutive rows of each
// piece), then the warp combines the rows four at a time, each lane d/32
// floats of a row, so that four rows' loads of a piece are in flight
// together.  G is the largest power of two up to 32 that still gives every
// warp of the grid a group, so a problem of few rows (one long sequence of
// one head) keeps the whole grid busy.  Memory-bound: every piece is read
// once and O written once.
template <int D>
__global__ void __launch_bounds__(256) splitkv_combine_kernel(const FwdArgs a) {
  constexpr int kPer = D / 32;
  constexpr int kRows = 4;
  const int S = a.num_splits;
  const long long rows = (long long)a.B * a.H * a.N;
  const int lane = threadIdx.x & 31;
  const long long warp0 = (blockIdx.x * (long long)blockDim.x + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * blockDim.x) >> 5;
  const long long o_lim = extent4(a.B, a.H, a.N, D, a.o_sb, a.o_sh, a.o_sn);
  (void)o_lim;
  int G = 32;
  while (G > 1 && (long long)G * nwarps > rows) G >>= 1;
  for (long long r0 = warp0 * G; r0 < rows; r0 += nwarps * G) {
    const long long rl = r0 + lane;
    float mx = -INFINITY, inv = 0.f;
    if (lane < G && rl < rows) {
      for (int s = 0; s < S; ++s) mx = fmaxf(mx, a.part_lse[(long long)s * rows + rl]);
      float lse = -INFINITY;
      if (mx != -INFINITY) {
        float wsum = 0.f;
        for (int s = 0; s < S; ++s) {
          const float ls = a.part_lse[(long long)s * rows + rl];
          wsum += ls == -INFINITY ? 0.f : __expf(ls - mx);
        }
        inv = 1.f / wsum;
        lse = mx + logf(wsum);
      }
      a.lse[rl] = lse;
    }
    const int nr = rows - r0 < G ? (int)(rows - r0) : G;
    for (int j0 = 0; j0 < nr; j0 += kRows) {
      float mxj[kRows], invj[kRows], acc[kRows][kPer];
#pragma unroll
      for (int j = 0; j < kRows; ++j) {
        mxj[j] = __shfl_sync(0xffffffffu, mx, (j0 + j) & 31);
        invj[j] = __shfl_sync(0xffffffffu, inv, (j0 + j) & 31);
#pragma unroll
        for (int e = 0; e < kPer; ++e) acc[j][e] = 0.f;
      }
#pragma unroll 2
      for (int s = 0; s < S; ++s) {
#pragma unroll
        for (int j = 0; j < kRows; ++j) {
          const long long r = r0 + j0 + j;
          if (j0 + j < nr && FA_IN(kSiteCombine, (long long)s * rows + r, 1, (long long)S * rows, a.err)) {
            const float ls = a.part_lse[(long long)s * rows + r];
            const float w = ls == -INFINITY ? 0.f : __expf(ls - mxj[j]);
            const float* src = a.part_o + ((long long)s * rows + r) * D + lane * kPer;
            if constexpr (kPer == 4) {
              const float4 v = *reinterpret_cast<const float4*>(src);
              acc[j][0] += w * v.x, acc[j][1] += w * v.y, acc[j][2] += w * v.z, acc[j][3] += w * v.w;
            } else {
              const float2 v = *reinterpret_cast<const float2*>(src);
              acc[j][0] += w * v.x, acc[j][1] += w * v.y;
            }
          }
        }
      }
#pragma unroll
      for (int j = 0; j < kRows; ++j) {
        if (j0 + j >= nr) continue;
        const long long r = r0 + j0 + j;
        const int bh = (int)(r / a.N), i = (int)(r - (long long)bh * a.N);
        const int b_ = bh / a.H, h_ = bh - b_ * a.H;
        const long long ooff = b_ * a.o_sb + h_ * a.o_sh + (long long)i * a.o_sn;
        if (!FA_IN(kSiteCombine, ooff, D, o_lim, a.err)) continue;
        __nv_bfloat16* orow = a.o + ooff + lane * kPer;
        if constexpr (kPer == 4)
          *reinterpret_cast<uint2*>(orow) = make_uint2(pack_bf16x2(acc[j][0] * invj[j], acc[j][1] * invj[j]),
                                                       pack_bf16x2(acc[j][2] * invj[j], acc[j][3] * invj[j]));
        else
          *reinterpret_cast<uint32_t*>(orow) = pack_bf16x2(acc[j][0] * invj[j], acc[j][1] * invj[j]);
      }
    }
  }
}

}  // namespace fa
