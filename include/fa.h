/*
 * fa.h -- C ABI of the sm_100a fused exact-attention library (libfa_sm100.so).
 *
 * Exact scaled-dot-product attention
 *     O = softmax(scale * Q K^T [+ causal mask]) V
 * ("FlashAttention for Efficient Training", section 1, attention equation),
 * computed by one fused, tiled forward kernel with an online softmax that
 * saves the per-row logsumexp ("How FlashAttention Optimizes GPU Memory for
 * Fast AI Training": Tiling, Online Softmax, Kernel Fusion; "FlashAttention
 * for Efficient Training" section 3.2, log_softmax / logsumexp), and a fused
 * backward that recomputes S and P tile by tile from Q, K, V and the saved
 * logsumexp ("How FlashAttention Optimizes GPU Memory for Fast AI Training",
 * Recomputation in the Backward Pass; "FlashAttention for Efficient
 * Training" section 3.2, dV = P^T dO, and the chain rule for dQ, dK).
 *
 * Conventions shared by every entry point
 *  - Tensors are dense, contiguous, row-major [B, H, N, d] arrays of bf16
 *    (IEEE bfloat16 bit patterns) in device memory, 16-byte aligned.
 *    lse and the backward's D are fp32 [B, H, N] in device memory.
 *  - d (head dimension) is 64 or 128.  N >= 1 is any length; B, H >= 1.
 *    B = 0, H = 0 or N = 0 is an empty problem: the call returns FA_OK and
 *    launches nothing (pointers are then not inspected).
 *  - scale > 0 and finite (1/sqrt(d) is the usual choice).  causal is 0 or 1:
 *    query i sees keys j <= i.  dropout_p in [0, 1): element (i, j) of head
 *    (b, h) is kept iff the 16-bit half h16(i, j) of the 32-bit mix
 *    hash32(seed, b, h, i, j >> 1) -- the low half for even j, the high half
 *    for odd j -- is >= ceil(dropout_p * 2^16) (both are defined in
 *    io_aware_exact_25_b200/csrc/dropout_hash.cuh);
 *    kept probabilities are scaled by 1/(1-p).
 *    Dropout is applied after the softmax, so lse is that of the undropped
 *    scores.  The backward with the same (seed, dropout_p) regenerates the
 *    same mask.
 *  - The caller owns every buffer.  The library allocates no device or host
 *    memory; it keeps one device-resident error word per device.
 *  - stream is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Calls are asynchronous on that stream; nothing synchronises.
 *  - On any error nothing is launched and a negative fa_status is returned.
 *    Calls are thread-safe.
 */
#ifndef FA_SM100_H_
#define FA_SM100_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum fa_status {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = -1, /* null pointer, negative size, bad scale/causal/p */
  FA_ERR_UNSUPPORTED = -2, /* head dimension other than 64 or 128 */
  FA_ERR_ALIGNMENT = -3,   /* a tensor not 16-byte aligned (lse/D: 4-byte) */
  FA_ERR_WORKSPACE = -4,   /* workspace null or smaller than required */
  FA_ERR_CUDA = -5,        /* a CUDA runtime/driver call or launch failed */
  FA_ERR_DEVICE = -6,      /* a kernel reported an error (fa_get_device_error) */
  FA_ERR_TOO_LARGE = -7    /* sizes overflow the library's index range */
} fa_status;

/*
 * Forward ("FlashAttention for Efficient Training" section 3, Workflow
 * Breakdown steps 1-3: block loading, local attention with the online
 * softmax, incremental output accumulation; fused scaling, masking and
 * dropout per section 3, Fused Kernel Design).  Reads q, k, v [B,H,N,d]
 * bf16; writes o [B,H,N,d] bf16 and lse [B,H,N] fp32 (natural-log logsumexp
 * of scale * q_i . k_j over the visible keys j).  o and lse must not alias
 * the inputs.  Errors: FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED,
 * FA_ERR_ALIGNMENT, FA_ERR_TOO_LARGE (nothing launched) or FA_ERR_CUDA.
 */
int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
           float scale, int causal, float dropout_p, uint64_t seed, void* stream);

/*
 * Element strides of one logical [B, H, N, d] bf16 tensor whose last (d)
 * dimension is contiguous: element (b, h, n, c) is at base[b*b_ + h*h_ +
 * n*n_ + c] with b_ = .b, h_ = .h, n_ = .n.  Every stride times 2 bytes must be
 * a multiple of 16.  Dense [B,H,N,d] is {H*N*d, N*d, d}; the pages' API layout
 * (batch, seq_len, num_heads, head_dim) ("FlashAttention for Efficient
 * Training", Integration with Frameworks) is {N*H*d, d, H*d}.
 */
typedef struct fa_strides {
  int64_t b, h, n;
} fa_strides;

/*
 * fa_fwd on strided tensors: strides[4] for q, k, v, o in that order (lse
 * stays a dense fp32 [B,H,N]).  Errors as fa_fwd; FA_ERR_ALIGNMENT for a
 * stride that breaks 16-byte row alignment.
 */
int fa_fwd_strided(const void* q, const void* k, const void* v, void* o, float* lse, const fa_strides* strides,
                   int B, int H, int N, int d, float scale, int causal, float dropout_p, uint64_t seed,
                   void* stream);

/*
 * Split-KV forward for problems with few query tiles (small B*H*N leaves
 * SMs idle: "FlashAttention for Efficient Training" section 6.1, Limited
 * Parallelism for Small Batch Sizes).  Each query tile's key range is cut
 * into num_splits consecutive pieces processed by separate CTAs; each piece
 * writes its normalised partial output O_s (fp32) and logsumexp lse_s, and a
 * combine pass forms lse = ln sum_s exp(lse_s) and O = sum_s exp(lse_s - lse)
 * O_s -- the exact merge of softmax pieces over disjoint key sets.  Output,
 * arguments and errors are those of fa_fwd, plus num_splits in [1, 64]
 * (1 = the plain kernel) and a caller-owned workspace of at least
 * fa_fwd_splitkv_workspace_size bytes (16-byte aligned; FA_ERR_WORKSPACE
 * if too small).  Two launches on `stream`.
 */
int fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                   float scale, int causal, float dropout_p, uint64_t seed, int num_splits, void* workspace,
                   size_t workspace_bytes, void* stream);

/* Workspace bytes for fa_fwd_splitkv (0 when num_splits == 1 or invalid). */
size_t fa_fwd_splitkv_workspace_size(int B, int H, int N, int d, int num_splits);

/* A split count for this shape: 1 when the plain grid fills at least half of
 * the SMs, else as many pieces as fill one wave (at most 16). */
int fa_splitkv_suggest(int B, int H, int N, int d);

/*
 * Bytes of device workspace fa_bwd needs for this shape: an fp32 dQ
 * accumulator [B,H,N,d] plus two fp32 row vectors (scaled lse and
 * D_i = dO_i . O_i) padded to a multiple of 128 rows.  Returns 0 for an empty
 * problem or invalid sizes.
 */
size_t fa_bwd_workspace_size(int B, int H, int N, int d);

/*
 * Backward with recomputation ("FlashAttention for Efficient Training"
 * section 3.2, Integration with Autograd Engines: dV = P^T dO, dQ and dK by
 * the chain rule; "How FlashAttention Optimizes GPU Memory for Fast AI
 * Training", Recomputation in the Backward Pass).  Three launches on
 * `stream`: a row pass (D_i = dO_i . O_i, scaled lse, zeroed dQ accumulator),
 * the fused recompute kernel, and the dQ conversion.  Reads q, k, v, o, dout [B,H,N,d] bf16 and lse [B,H,N] fp32
 * from fa_fwd with the same scale/causal/dropout_p/seed; writes dq, dk, dv
 * [B,H,N,d] bf16.  workspace (16-byte aligned, at least
 * fa_bwd_workspace_size bytes) is scratch owned by the caller; its contents
 * on entry do not matter.  dq/dk/dv must not alias any input.
 * Errors: as fa_fwd, plus FA_ERR_WORKSPACE.  dQ: each key tile's partial
 * dQ_i = dS K_j is staged in shared memory and added into an fp32 workspace
 * accumulator with bulk reductions (cp.reduce.async.bulk .add.f32); the order
 * of those additions varies, so dq bits may differ from run to run by
 * rounding; dk and dv are deterministic.
 */
int fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
           void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale, int causal, float dropout_p,
           uint64_t seed, void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_bwd on strided tensors: strides[8] for q, k, v, o, dout, dq, dk, dv in
 * that order (lse dense).  Errors as fa_bwd.
 */
int fa_bwd_strided(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                   void* dq, void* dk, void* dv, const fa_strides* strides, int B, int H, int N, int d, float scale,
                   int causal, float dropout_p, uint64_t seed, void* workspace, size_t workspace_bytes,
                   void* stream);

/*
 * The three stages fa_bwd runs, callable one by one on the same stream (for
 * overlap with other work or per-stage timing).  Same arguments and checks as
 * fa_bwd; running them in order is exactly fa_bwd.
 *   fa_bwd_prepare:   D_i = dO_i . O_i ("FlashAttention for Efficient
 *                     Training" section 3.2: the chain rule through the
 *                     row-wise softmax needs this row dot), lse in base 2,
 *                     and a zeroed fp32 dQ accumulator, all in workspace.
 *   fa_bwd_recompute: the fused recompute kernel; writes dk, dv and adds
 *                     the dQ partials into the workspace accumulator.
 *   fa_bwd_finalize:  dq = scale * accumulator, rounded to bf16.
 */
int fa_bwd_prepare(const void* o, const void* dout, const float* lse, int B, int H, int N, int d,
                   void* workspace, size_t workspace_bytes, void* stream);
int fa_bwd_recompute(const void* q, const void* k, const void* v, const void* dout, void* dk, void* dv, int B,
                     int H, int N, int d, float scale, int causal, float dropout_p, uint64_t seed,
                     void* workspace, size_t workspace_bytes, void* stream);
int fa_bwd_finalize(void* dq, int B, int H, int N, int d, float scale, void* workspace, size_t workspace_bytes,
                    void* stream);

/*
 * fa_bwd without a caller-provided workspace.  The paper has no counterpart:
 * this entry point exists for callers that cannot allocate device memory,
 * such as plugin or custom-op interfaces that pass a kernel only its input
 * and output tensors, or code that must not allocate at that point.
 * Arguments, outputs and errors are those of fa_bwd; the scratch fa_bwd
 * would take from `workspace` comes instead from a static device array of
 * FA_NOALLOC_SCRATCH_BYTES inside the library, which every GPU that loads
 * the library holds until the process exits.  Nothing is allocated.
 *  - Shapes whose fa_bwd_workspace_size exceeds FA_NOALLOC_SCRATCH_BYTES are
 *    rejected with FA_ERR_TOO_LARGE before anything is launched.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.
 *  - All calls on a device share the one array, which keeps whatever the
 *    last call left in it (the backward clears what must start at zero).
 *    Calls that overlap on the GPU, e.g. on two streams, race on it and
 *    produce wrong results; serialise them.
 */
#define FA_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                   void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale, int causal,
                   float dropout_p, uint64_t seed, void* stream);

/*
 * Block-sparse attention ("FlashAttention for Efficient Training" section
 * 3.2, Block-Sparse Attention Support: only the non-zero blocks of the
 * attention matrix are computed).  block_mask is a device array of bytes
 * [mask_heads][nt][nt], nt = ceil(N / 128), row-major; mask_heads is 1 (one
 * mask for every head) or H (head h uses slice h).  A nonzero byte at
 * [h][a][c] lets queries 128a..128a+127 see keys 128c..128c+127; a zero hides
 * that whole block (its scores count as -inf).  The causal mask, if set,
 * applies on top.  A query row that sees no key at all gets o = 0 and
 * lse = -inf (the pages do not define this case; it is the zero-weight limit),
 * and contributes nothing to dq, dk, dv; a key no query sees gets dk = dv = 0.
 * Work and memory traffic scale with the number of visible blocks.
 *  - strides: as fa_fwd_strided (4 entries: q, k, v, o) and fa_bwd_strided
 *    (8 entries); NULL means dense [B,H,N,d] tensors.
 *  - N is at most 4096 * 128 = 524288 (FA_ERR_TOO_LARGE beyond); a null
 *    block_mask or mask_heads other than 1 or H is FA_ERR_INVALID_ARG.
 *  - The backward must get the mask the forward used; the mask is read, not
 *    retained, and must stay unchanged while the calls run on the stream.
 *  - Other arguments, outputs, workspace and errors are those of
 *    fa_fwd_strided and fa_bwd_strided.
 */
int fa_fwd_blocksparse(const void* q, const void* k, const void* v, void* o, float* lse, const fa_strides* strides,
                       int B, int H, int N, int d, float scale, int causal, float dropout_p, uint64_t seed,
                       const uint8_t* block_mask, int mask_heads, void* stream);
int fa_bwd_blocksparse(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                       void* dq, void* dk, void* dv, const fa_strides* strides, int B, int H, int N, int d,
                       float scale, int causal, float dropout_p, uint64_t seed, const uint8_t* block_mask,
                       int mask_heads, void* workspace, size_t workspace_bytes, void* stream);
/* The recompute stage of fa_bwd_blocksparse on dense tensors, for the staged
 * backward: fa_bwd_prepare, this, fa_bwd_finalize in order is exactly
 * fa_bwd_blocksparse with strides == NULL.  Arguments as fa_bwd_recompute
 * plus the block mask. */
int fa_bwd_recompute_blocksparse(const void* q, const void* k, const void* v, const void* dout, void* dk, void* dv,
                                 int B, int H, int N, int d, float scale, int causal, float dropout_p, uint64_t seed,
                                 const uint8_t* block_mask, int mask_heads, void* workspace, size_t workspace_bytes,
                                 void* stream);

/*
 * Variable-length batches ("FlashAttention for Efficient Training" section
 * 5.2, Handling Variable Sequence Lengths: a score is -inf unless its key lies
 * within the sequence, j <= L_i, and no work is spent on padded tokens).
 *  - Layout: the B sequences are stored token-major, the pages'
 *    (batch, seq_len, num_heads, head_dim) layout with batch and sequence
 *    folded into one token dimension of total_tokens rows: element (token t,
 *    head h, c) of q, k, v, o (and dout, dq, dk, dv) is at
 *    base[t * s.n + h * s.h + c], s = strides[i] (.b is ignored; .n and .h
 *    times 2 bytes must be multiples of 16).  lse is fp32 [H, total_tokens].
 *  - cu_seqlens: device int32 [B + 1], non-decreasing, 0 <= cu_seqlens[b] and
 *    cu_seqlens[B] <= total_tokens; sequence b owns the slot of tokens
 *    [cu_seqlens[b], cu_seqlens[b + 1]).  seqused: device int32 [B] or NULL;
 *    if given, only the first seqused[b] tokens of the slot are the sequence
 *    and the rest of the slot is padding (a padded [B, N, H, d] batch is
 *    cu_seqlens = {0, N, 2N, ...} with seqused = the lengths); if NULL the
 *    whole slot is the sequence.  max_seqlen (host) is at least the largest
 *    slot size; it sizes the grid.
 *  - Semantics per sequence b of length L_b: query i (position within the
 *    sequence) sees key j iff j < L_b (and j <= i when causal); other
 *    sequences are never seen.  Dropout uses hash32(seed, b, h, i, j) with
 *    the positions within the sequence.  Padding rows (slot positions at or
 *    beyond L_b) get o = 0 and lse = -inf, and dq = dk = dv = 0 in the
 *    backward.  Every row of k and v inside a slot must hold finite values:
 *    rows past L_b get zero weight, but the tensor cores multiply them by
 *    that zero.
 *  - Offsets are read on the device and not validated on the host; offsets
 *    or lengths out of range are clamped into [0, total_tokens] and the slot
 *    (so no access leaves the tensors) and reported as device error 3
 *    (fa_get_device_error).
 *  - Work, memory traffic and grid: CTAs of tiles past a sequence's length
 *    return at once; the work is that of the B separate problems.
 *  - The backward needs a workspace of fa_bwd_varlen_workspace_size bytes
 *    and the forward's lse; its other arguments are those of fa_bwd_strided.
 *  - Errors: as fa_fwd_strided / fa_bwd_strided; a null cu_seqlens is
 *    FA_ERR_INVALID_ARG.  total_tokens = 0 is an empty problem.
 */
int fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse, const fa_strides* strides,
                  const int32_t* cu_seqlens, const int32_t* seqused, int B, int H, int max_seqlen, int total_tokens,
                  int d, float scale, int causal, float dropout_p, uint64_t seed, void* stream);
size_t fa_bwd_varlen_workspace_size(int B, int H, int max_seqlen, int d);
int fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                  void* dq, void* dk, void* dv, const fa_strides* strides, const int32_t* cu_seqlens,
                  const int32_t* seqused, int B, int H, int max_seqlen, int total_tokens, int d, float scale,
                  int causal, float dropout_p, uint64_t seed, void* workspace, size_t workspace_bytes,
                  void* stream);

/*
 * Sequence parallelism over a split key range ("FlashAttention for Efficient
 * Training" section 5.3, Sequence Parallelism for Long Contexts: each GPU
 * holds a chunk of the sequence, and the output of a query chunk is formed
 * from the softmax pieces of every key chunk, merged exactly by their
 * logsumexp as in section 6.1's split-KV).  These entry points are the
 * per-GPU pieces; io_aware_exact_25_b200/seqpar.py exchanges them over NCCL.
 * A key window [kv_begin, kv_end) of the N keys has kv_begin a multiple of
 * 128 and kv_end a multiple of 128 or N (else FA_ERR_INVALID_ARG); k, v, dk,
 * dv of these calls are dense [B, H, kv_end - kv_begin, d] bf16 holding
 * those key rows; q, dout are the full dense [B, H, N, d].
 *
 * fa_fwd_partial: for every query row, the softmax piece over the window's
 *   keys: part_o fp32 [B, H, N, d] = O normalised over those keys and
 *   part_lse fp32 [B, H, N] their logsumexp (-inf and O = 0 for a row that
 *   sees none of them, e.g. causal rows before kv_begin).  Dropout uses the
 *   global positions, so the pieces of all windows form one mask.
 * fa_merge_partials: o bf16 [B, H, N, d] and lse [B, H, N] from num_parts
 *   pieces stacked as part_o [num_parts][B, H, N, d], part_lse
 *   [num_parts][B, H, N]: lse = ln sum_s e^lse_s, O = sum_s e^(lse_s - lse) O_s.
 *   A row whose pieces are all -inf gets O = 0 and lse = -inf.
 * fa_weight_partial: the exchange by summation.  part_o fp32 [B, H, N, d]
 *   is piece number `part` of num_parts (from fa_fwd_partial) and all_lse
 *   fp32 [num_parts][B, H, N] every piece's logsumexp (an all-gather of
 *   part_lse).  Rescales part_o in place to e^(lse_part - lse) O_part, with
 *   lse = ln sum_s e^lse_s written to `lse` (fp32 [B, H, N]; may be null);
 *   a row whose pieces are all -inf gets 0 and lse -inf.  The sum of the
 *   weighted pieces over the parts (an all-reduce) is O in fp32;
 *   fa_merge_partials with num_parts = 1 on that sum and lse converts it to
 *   bf16.  d in {64, 128} (FA_ERR_UNSUPPORTED); part_o 16-byte aligned,
 *   all_lse and lse 4-byte aligned (FA_ERR_ALIGNMENT); 1 <= num_parts <=
 *   4096 and 0 <= part < num_parts (FA_ERR_INVALID_ARG); B*H*N*num_parts
 *   above 2^40 gives FA_ERR_TOO_LARGE; an empty problem returns FA_OK and
 *   launches nothing.  Asynchronous on `stream`.  A failed launch returns
 *   FA_ERR_CUDA without updating fa_last_cuda_error (cudaGetLastError has
 *   the code).
 * fa_bwd_recompute_range: the recompute stage of fa_bwd for the window's
 *   keys: writes dk, dv of those keys (complete) and adds their part of dQ
 *   into the workspace's fp32 accumulator.  Run fa_bwd_prepare (on the full
 *   o, dout, lse), this, then -- after summing the first
 *   fa_bwd_dq_accumulator_bytes(B, H, N, d) bytes of the workspace (the
 *   accumulator, fp32) over the windows that make up the sequence --
 *   fa_bwd_finalize.  With one window covering every key this is fa_bwd.
 */
int fa_fwd_partial(const void* q, const void* k, const void* v, float* part_o, float* part_lse, int B, int H, int N,
                   int d, float scale, int causal, float dropout_p, uint64_t seed, int kv_begin, int kv_end,
                   void* stream);
int fa_merge_partials(const float* part_o, const float* part_lse, int num_parts, void* o, float* lse, int B, int H,
                      int N, int d, void* stream);
int fa_weight_partial(float* part_o, const float* all_lse, int num_parts, int part, float* lse, int B, int H, int N,
                      int d, void* stream);
size_t fa_bwd_dq_accumulator_bytes(int B, int H, int N, int d);
int fa_bwd_recompute_range(const void* q, const void* k, const void* v, const void* dout, void* dk, void* dv, int B,
                           int H, int N, int d, float scale, int causal, float dropout_p, uint64_t seed, int kv_begin,
                           int kv_end, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Debug export of the dropout mask: for each listed head bh = b*H + h
 * (heads[nheads]) and query row (rows[nrows]), writes the keep bit of every
 * key j < N to out[(hi * nrows + ri) * N + j] (1 = kept).  heads, rows and
 * out are device pointers.  Uses the same device hash the kernels inline.
 */
int fa_dropout_mask(int B, int H, int N, float dropout_p, uint64_t seed, const int32_t* heads, int nheads,
                    const int32_t* rows, int nrows, uint8_t* out, void* stream);

/*
 * Fault injection for tests (the paper has no counterpart): fa_fwd on dense
 * tensors with the producer warp issuing no K/V load, so the MMA warp's first
 * bounded wait runs out (after about 2 s).  The kernel then records code 1
 * (timeout) in the device error word, every warp leaves its loop, tensor
 * memory is freed and the kernel exits; o and lse are left unwritten.  The
 * call itself returns the launch status (FA_OK); fa_get_device_error reports
 * the timeout and clears it, and the context stays usable.  No fault, trap or
 * hang is involved.
 */
int fa_debug_fwd_timeout(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N,
                         int d, float scale, int causal, void* stream);

/*
 * Test hook for the polynomial exponential (the paper has no counterpart):
 * y[i] = 2^x[i] computed by the device function the backward kernel uses for
 * part of its recomputed probabilities (a Cody-Waite split and a cubic
 * minimax fit on the FMA pipe), so that tests can hold it to its stated
 * error bound against CUDA's exp2.  x and y are device pointers to n floats
 * (n >= 0; 4-byte aligned).  Returns FA_ERR_INVALID_ARG for n < 0 or null
 * pointers with n > 0; asynchronous on `stream`.
 */
int fa_debug_exp2_poly(const float* x, float* y, int n, void* stream);

/*
 * The bounds-checking build (the paper has no counterpart).  The library
 * also builds as libfa_sm100_debug.so, compiled with FA_DEBUG: there every
 * global-memory access the kernels derive from their work decomposition
 * (output rows, dQ accumulator tiles, row statistics, split-KV pieces, work
 * items, TMA tile rows) is checked against the extent its buffer has by the
 * call's shape and strides before it is made.  A failed check skips the
 * access (a tile load is still issued: out-of-range rows read as zero),
 * sets device error 4 and records the first failure.
 *
 * fa_debug_build returns 1 in that build and 0 in the release build.
 * fa_debug_bounds_record synchronises `stream`, copies the record into
 * out[0..5] = {failed checks, site, offset, limit, block, thread} (offsets in
 * elements; site numbers are listed in csrc/debug_check.cuh) and clears it;
 * the release build returns FA_ERR_UNSUPPORTED.  out is a host pointer to 6
 * long longs.
 */
int fa_debug_build(void);
int fa_debug_bounds_record(long long* out, void* stream);

/* Static description of a status code. */
const char* fa_strerror(int status);

/* The cudaError_t of the most recent FA_ERR_CUDA on this thread (0 if none). */
int fa_last_cuda_error(void);

/*
 * Synchronises `stream`, then reads and clears the calling device's error
 * word.  Returns 0 if no kernel reported an error since the last read, else
 * the kernel's code (1 = a bounded wait timed out, 2 = shared memory
 * misaligned, 3 = variable-length offsets or lengths out of range, 4 = a
 * bounds check failed, bounds-checking build only);
 * FA_ERR_CUDA if the synchronisation itself failed.
 */
int fa_get_device_error(void* stream);

/* Library version, as major * 10000 + minor * 100 + patch. */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_SM100_H_ */
