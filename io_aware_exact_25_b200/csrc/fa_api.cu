// fa_api.cu -- host side of the C ABI declared in include/fa.h: argument
// validation, TMA tensor-map construction, kernel selection and launch on
// the caller's stream.  Allocates nothing; the only state is one device
// error word per device (a __device__ variable in this module).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstddef>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/fa.h"
#include "bwd_sm100.cuh"
#include "dropout_hash.cuh"
#include "fwd_sm100.cuh"

namespace {

// The device error word the kernels record into (kDevTimeout, kDevMisaligned,
// kDevBadSeqlens, kDevBounds), followed by the bounds-checking build's record
// of its first failed check: {count, site, offset, limit, block, thread}.
struct DeviceStatus {
  int err;
  int pad;
  long long rec[8];
};
__device__ DeviceStatus g_device_status;

thread_local int t_last_cuda_error = 0;

// Key-window upper bound meaning "every key tile".
constexpr int kAllTiles = 1 << 30;

int cuda_fail(cudaError_t e) {
  t_last_cuda_error = static_cast<int>(e);
  return FA_ERR_CUDA;
}

// cuTensorMapEncodeTiled, fetched from the driver through the runtime so the
// library needs no link-time dependency on libcuda.
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Tensor map of a bf16 [B, H, N, d] tensor with element strides s (d
// contiguous), addressed as {d, n, h, b} and read in box_rows-row x 64-column
// boxes with the 128-byte swizzle; rows past N read as zero.
int make_tile_map(CUtensorMap* m, const void* base, int B, int H, int N, int d, const fa_strides& s,
                  int box_rows = 128) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return cuda_fail(cudaErrorNotSupported);
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)H, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)s.n * 2u, (cuuint64_t)s.h * 2u, (cuuint64_t)s.b * 2u};
  cuuint32_t box[4] = {64u, (cuuint32_t)box_rows, 1u, 1u};
  cuuint32_t estride[4] = {1u, 1u, 1u, 1u};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estride,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
  return FA_OK;
}

fa_strides contiguous_strides(int H, int N, int d) {
  fa_strides s;
  s.n = d;
  s.h = (int64_t)N * d;
  s.b = (int64_t)H * N * d;
  return s;
}

// Strides are usable if every row start stays 16-byte aligned.
bool strides_ok(const fa_strides& s) {
  return s.b >= 0 && s.h >= 0 && s.n >= 0 && (s.b * 2) % 16 == 0 && (s.h * 2) % 16 == 0 && (s.n * 2) % 16 == 0;
}

int* device_error_ptr() {
  int* p = nullptr;
  if (cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_device_status) != cudaSuccess) return nullptr;
  return p;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Shared argument checks.  Returns FA_OK, a negative status, or 1 for an
// empty problem (nothing to do).
int check_common(int B, int H, int N, int d, float scale, int causal, float dropout_p) {
  if (B < 0 || H < 0 || N < 0) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (!(dropout_p >= 0.f && dropout_p < 1.f)) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (B == 0 || H == 0 || N == 0) return 1;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  const long long bh = (long long)B * H;
  const long long elems = bh * (long long)N * d;
  // grid sizes and 32-bit row counters stay in range
  if (bh > (1ll << 24) || (long long)N > (1ll << 24) || elems > (1ll << 40)) return FA_ERR_TOO_LARGE;
  if (bh * (((long long)N + 127) / 128) > 0x7fffffffll) return FA_ERR_TOO_LARGE;
  return FA_OK;
}

// T = ceil(p * 2^16), compared with the 16-bit halves of the pair hash
uint32_t keep_threshold(float p) {
  const double t = std::ceil((double)p * 65536.0);
  if (t <= 0.0) return 0u;
  if (t >= 65536.0) return 65536u;
  return (uint32_t)t;
}

template <int D, bool CAUSAL, bool DROPOUT, int MODE>
int launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const fa::FwdArgs& a,
               cudaStream_t st) {
  using L = fa::FwdLayout<D, fa::fwd_bn<D, MODE>()>;
  constexpr bool SPLIT = MODE == fa::kFwdSplit;
  auto kern = fa::fwd_kernel<D, CAUSAL, DROPOUT, MODE>;
  const int smem = (int)(MODE == fa::kFwdSparse ? L::kSmemSparse : L::kSmem);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return cuda_fail(e);
  const long long grid = (long long)a.B * a.H * ((a.N + 255) / 256) * (SPLIT ? a.num_splits : 1);
  kern<<<(unsigned)grid, L::kThreads, smem, st>>>(mq, mk, mv, a);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  if (SPLIT && !a.partial_only) {
    fa::splitkv_combine_kernel<D><<<148 * 8, 256, 0, st>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return FA_OK;
}

template <int D, int MODE>
int dispatch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const fa::FwdArgs& a,
                 bool causal, bool dropout, cudaStream_t st) {
  if (causal)
    return dropout ? launch_fwd<D, true, true, MODE>(mq, mk, mv, a, st)
                   : launch_fwd<D, true, false, MODE>(mq, mk, mv, a, st);
  return dropout ? launch_fwd<D, false, true, MODE>(mq, mk, mv, a, st)
                 : launch_fwd<D, false, false, MODE>(mq, mk, mv, a, st);
}

// Block-mask checks shared by the block-sparse entry points.
int check_block_mask(const uint8_t* mask, int mask_heads, int H, int N) {
  if (!mask || (mask_heads != 1 && mask_heads != H)) return FA_ERR_INVALID_ARG;
  if ((N + 127) / 128 > fa::kMaxSparseTiles) return FA_ERR_TOO_LARGE;
  return FA_OK;
}

size_t splitkv_bytes(int B, int H, int N, int d, int splits) {
  const size_t rows = (size_t)B * H * N * (size_t)splits;
  return fa::round_up(rows * d * 4, 256) + fa::round_up(rows * 4, 256);
}

__global__ void dropout_mask_kernel(int H, int N, uint32_t threshold, uint64_t seed, const int32_t* heads,
                                    int nheads, const int32_t* rows, int nrows, uint8_t* out) {
  const long long total = (long long)nheads * nrows * N;
  for (long long u = blockIdx.x * (long long)blockDim.x + threadIdx.x; u < total;
       u += (long long)gridDim.x * blockDim.x) {
    const int j = (int)(u % N);
    const long long hr = u / N;
    const int ri = (int)(hr % nrows);
    const int hi = (int)(hr / nrows);
    const int bh = heads[hi];
    const uint32_t key = fa::dropout_row_key(seed, (uint32_t)(bh / H), (uint32_t)(bh % H), (uint32_t)rows[ri]);
    const uint32_t w = fa::dropout_hash(key, (uint32_t)j >> 1);
    out[u] = ((j & 1) ? fa::keep_hi(w, threshold) : fa::keep_lo(w, threshold)) ? 1 : 0;
  }
}

// Variable-length batches with padded slots (seqused given): the slot rows
// [L_b, slot) of sequence b are padding.  Writes zeros into those rows of up
// to three bf16 tensors (null entries are skipped) and -inf into lse rows of
// a forward (lse may be null).  One thread per (sequence, slot row, head).
__global__ void varlen_pad_kernel(int B, int H, int max_slot, int total, const int* cu, const int* used, int d,
                                  __nv_bfloat16* t0, fa_strides s0, __nv_bfloat16* t1, fa_strides s1,
                                  __nv_bfloat16* t2, fa_strides s2, float* lse) {
  const long long n = (long long)B * max_slot * H;
  for (long long u = blockIdx.x * (long long)blockDim.x + threadIdx.x; u < n; u += (long long)gridDim.x * blockDim.x) {
    const int h = (int)(u % H);
    const long long br = u / H;
    const int r = (int)(br % max_slot);
    const int b = (int)(br / max_slot);
    const fa::SeqSpan sp = fa::varlen_span(cu, used, b, total, max_slot, nullptr, false);
    if (r < sp.len || r >= sp.slot) continue;
    const long long row = sp.row0 + r;
    __nv_bfloat16* ts[3] = {t0, t1, t2};
    const fa_strides ss[3] = {s0, s1, s2};
    for (int k = 0; k < 3; ++k) {
      if (!ts[k]) continue;
      const long long off = h * ss[k].h + row * ss[k].n;
      if (!FA_IN(fa::kSiteVarlenPad, off, d, fa::extent4(1, H, total, d, 0, ss[k].h, ss[k].n), &g_device_status.err))
        continue;
      __nv_bfloat16* p = ts[k] + off;
      for (int c = 0; c < d; c += 8) *reinterpret_cast<uint4*>(p + c) = make_uint4(0u, 0u, 0u, 0u);
    }
    if (lse && FA_IN(fa::kSiteVarlenPad, (long long)h * total + row, 1, (long long)H * total, &g_device_status.err))
      lse[(long long)h * total + row] = -INFINITY;
  }
}

int launch_varlen_pad(int B, int H, int max_slot, int total, const int* cu, const int* used, int d,
                      __nv_bfloat16* t0, fa_strides s0, __nv_bfloat16* t1, fa_strides s1, __nv_bfloat16* t2,
                      fa_strides s2, float* lse, cudaStream_t st) {
  varlen_pad_kernel<<<148 * 4, 256, 0, st>>>(B, H, max_slot, total, cu, used, d, t0, s0, t1, s1, t2, s2, lse);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

// Token-major strides {.n = token, .h = head} of a variable-length tensor as
// the 4-D {d, T, H, 1} tensor maps and the kernels take them (.b unused).
fa_strides varlen_strides(const fa_strides& s, int total) {
  fa_strides r;
  r.n = s.n;
  r.h = s.h;
  r.b = s.n * (int64_t)total;
  return r;
}

// Checks shared by the variable-length entry points.  Returns FA_OK, a
// negative status, or 1 when there is nothing to do.
int check_varlen(int B, int H, int max_seqlen, int total, int d, float scale, int causal, float dropout_p,
                 const int* cu_seqlens, const fa_strides* strides, int nstrides) {
  int rc = check_common(B, H, max_seqlen, d, scale, causal, dropout_p);
  if (rc != FA_OK) return rc;
  if (total < 0) return FA_ERR_INVALID_ARG;
  if (total == 0) return 1;
  if ((long long)total * H * d > (1ll << 40)) return FA_ERR_TOO_LARGE;
  if (!cu_seqlens || !strides) return FA_ERR_INVALID_ARG;
  if (!aligned(cu_seqlens, 4)) return FA_ERR_ALIGNMENT;
  for (int t = 0; t < nstrides; ++t) {
    fa_strides s = strides[t];
    s.b = 0;
    if (!strides_ok(s)) return FA_ERR_ALIGNMENT;
  }
  return FA_OK;
}

}  // namespace

extern "C" {

int fa_version(void) { return 200; }

const char* fa_strerror(int status) {
  switch (status) {
    case FA_OK: return "success";
    case FA_ERR_INVALID_ARG: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported head dimension (64 or 128)";
    case FA_ERR_ALIGNMENT: return "tensor pointer misaligned (16 bytes; lse/D 4 bytes)";
    case FA_ERR_WORKSPACE: return "workspace missing or too small";
    case FA_ERR_CUDA: return "CUDA call failed (see fa_last_cuda_error)";
    case FA_ERR_DEVICE: return "a kernel reported an error";
    case FA_ERR_TOO_LARGE: return "problem too large for this library";
    default: return "unknown status";
  }
}

int fa_last_cuda_error(void) { return t_last_cuda_error; }

int fa_debug_bounds_record(long long* out, void* stream) {
  if (!out) return FA_ERR_INVALID_ARG;
#ifdef FA_DEBUG
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  long long rec[8];
  e = cudaMemcpyFromSymbol(rec, g_device_status, sizeof(rec), offsetof(DeviceStatus, rec));
  if (e != cudaSuccess) return cuda_fail(e);
  const long long zero[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  e = cudaMemcpyToSymbol(g_device_status, zero, sizeof(zero), offsetof(DeviceStatus, rec));
  if (e != cudaSuccess) return cuda_fail(e);
  for (int i = 0; i < 6; ++i) out[i] = rec[i];
  return FA_OK;
#else
  (void)stream;
  return FA_ERR_UNSUPPORTED;
#endif
}

int fa_debug_build(void) {
#ifdef FA_DEBUG
  return 1;
#else
  return 0;
#endif
}

int fa_get_device_error(void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e);
  int value = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&value, g_device_status, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e);
  e = cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e);
  return value;
}

namespace {

int fwd_impl(const void* q, const void* k, const void* v, void* o, float* lse, const fa_strides* strides, int B,
             int H, int N, int d, float scale, int causal, float dropout_p, uint64_t seed, int num_splits,
             void* workspace, size_t workspace_bytes, const uint8_t* bmask, int bmask_heads, void* stream,
             int debug_skip_kv = 0) {
  int rc = check_common(B, H, N, d, scale, causal, dropout_p);
  if (rc == 1) return FA_OK;
  if (rc != FA_OK) return rc;
  if (bmask && (rc = check_block_mask(bmask, bmask_heads, H, N)) != FA_OK) return rc;
  if (bmask && num_splits > 1) return FA_ERR_INVALID_ARG;
  if (!q || !k || !v || !o || !lse || !strides) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
    return FA_ERR_ALIGNMENT;
  for (int t = 0; t < 4; ++t)
    if (!strides_ok(strides[t])) return FA_ERR_ALIGNMENT;
  if (num_splits > 1) {
    if (!workspace || workspace_bytes < splitkv_bytes(B, H, N, d, num_splits)) return FA_ERR_WORKSPACE;
    if (!aligned(workspace, 16)) return FA_ERR_ALIGNMENT;
  }
  CUtensorMap mq, mk, mv;
  // K/V boxes follow the kernel's key tile (64 rows for the plain d = 64 forward)
  const int kv_rows = (!bmask && num_splits <= 1) ? (d == 64 ? fa::fwd_bn<64, fa::kFwdPlain>()
                                                             : fa::fwd_bn<128, fa::kFwdPlain>())
                                                  : 128;
  if ((rc = make_tile_map(&mq, q, B, H, N, d, strides[0])) != FA_OK) return rc;
  if ((rc = make_tile_map(&mk, k, B, H, N, d, strides[1], kv_rows)) != FA_OK) return rc;
  if ((rc = make_tile_map(&mv, v, B, H, N, d, strides[2], kv_rows)) != FA_OK) return rc;
  fa::FwdArgs a;
  std::memset(&a, 0, sizeof(a));
  a.kv_hi = kAllTiles;
  a.B = B;
  a.H = H;
  a.N = N;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.drop_threshold = keep_threshold(dropout_p);
  a.drop_scale = (float)(1.0 / (1.0 - (double)dropout_p));
  a.seed = seed;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.o_sb = strides[3].b;
  a.o_sh = strides[3].h;
  a.o_sn = strides[3].n;
  a.lse = lse;
  a.num_splits = num_splits;
  a.part_o = nullptr;
  a.part_lse = nullptr;
  a.bmask = bmask;
  a.bmask_heads = bmask_heads;
  a.debug_skip_kv = debug_skip_kv;
  if (num_splits > 1) {
    a.part_o = static_cast<float*>(workspace);
    a.part_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                          fa::round_up((size_t)B * H * N * (size_t)num_splits * d * 4, 256));
  }
  a.err = device_error_ptr();
  if (!a.err) return cuda_fail(cudaErrorInvalidSymbol);
  const bool dropout = dropout_p > 0.f;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (bmask)
    return d == 64 ? dispatch_fwd<64, fa::kFwdSparse>(mq, mk, mv, a, causal != 0, dropout, st)
                   : dispatch_fwd<128, fa::kFwdSparse>(mq, mk, mv, a, causal != 0, dropout, st);
  if (num_splits > 1)
    return d == 64 ? dispatch_fwd<64, fa::kFwdSplit>(mq, mk, mv, a, causal != 0, dropout, st)
                   : dispatch_fwd<128, fa::kFwdSplit>(mq, mk, mv, a, causal != 0, dropout, st);
  return d == 64 ? dispatch_fwd<64, fa::kFwdPlain>(mq, mk, mv, a, causal != 0, dropout, st)
                 : dispatch_fwd<128, fa::kFwdPlain>(mq, mk, mv, a, causal != 0, dropout, st);
}

}  // namespace

int fa_fwd_strided(const void* q, const void* k, const void* v, void* o, float* lse, const fa_strides* strides,
                   int B, int H, int N, int d, float scale, int causal, float dropout_p, uint64_t seed,
                   void* stream) {
  return fwd_impl(q, k, v, o, lse, strides, B, H, N, d, scale, causal, dropout_p, seed, 1, nullptr, 0, nullptr, 0,
                  stream);
}

int fa_splitkv_suggest(int B, int H, int N, int d) {
  if (check_common(B, H, N, d, 1.f, 0, 0.f) != FA_OK) return 1;
  // Split only when the plain grid leaves more than half of the 148 SMs idle,
  // and then into as many pieces as fill one wave (partials cost an extra
  // write, read and combine pass, and a second, ragged wave costs more).
  const long long ctas = (long long)B * H * ((N + 255) / 256);
  const int nkv = (N + 127) / 128;
  if (2 * ctas > 148) return 1;
  long long s = 148 / ctas;
  if (s > nkv / 2) s = nkv / 2;  // at least two key tiles per split
  if (s > 16) s = 16;
  return s < 1 ? 1 : (int)s;
}

size_t fa_fwd_splitkv_workspace_size(int B, int H, int N, int d, int num_splits) {
  if (check_common(B, H, N, d, 1.f, 0, 0.f) != FA_OK || num_splits < 1 || num_splits > 64) return 0;
  return num_splits > 1 ? splitkv_bytes(B, H, N, d, num_splits) : 0;
}

int fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                   float scale, int causal, float dropout_p, uint64_t seed, int num_splits, void* workspace,
                   size_t workspace_bytes, void* stream) {
  if (num_splits < 1 || num_splits > 64) return FA_ERR_INVALID_ARG;
  const fa_strides s = contiguous_strides(H, N, d);
  const fa_strides all[4] = {s, s, s, s};
  return fwd_impl(q, k, v, o, lse, all, B, H, N, d, scale, causal, dropout_p, seed, num_splits, workspace,
                  workspace_bytes, nullptr, 0, stream);
}

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
           float scale, int causal, float dropout_p, uint64_t seed, void* stream) {
  const fa_strides s = contiguous_strides(H, N, d);
  const fa_strides all[4] = {s, s, s, s};
  return fa_fwd_strided(q, k, v, o, lse, all, B, H, N, d, scale, causal, dropout_p, seed, stream);
}

int fa_debug_fwd_timeout(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N,
                         int d, float scale, int causal, void* stream) {
  const fa_strides s = contiguous_strides(H, N, d);
  const fa_strides all[4] = {s, s, s, s};
  return fwd_impl(q, k, v, o, lse, all, B, H, N, d, scale, causal, 0.f, 0, 1, nullptr, 0, nullptr, 0, stream, 1);
}

namespace {
__global__ void exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
  const int stride = 2 * gridDim.x * blockDim.x;
  for (int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x); i < n; i += stride) {
    const bool two = i + 1 < n;
    float r0, r1;
    fa::exp2_poly_x2(fa::f2_pack(x[i], two ? x[i + 1] : 0.f), r0, r1);
    y[i] = r0;
    if (two) y[i + 1] = r1;
  }
}
}  // namespace

int fa_debug_exp2_poly(const float* x, float* y, int n, void* stream) {
  if (n < 0 || (n > 0 && (!x || !y))) return FA_ERR_INVALID_ARG;
  if (n == 0) return FA_OK;
  if (!aligned(x, 4) || !aligned(y, 4)) return FA_ERR_ALIGNMENT;
  const int blocks = (int)std::min<long long>(148 * 8, ((long long)n + 511) / 512);
  exp2_poly_kernel<<<blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

int fa_dropout_mask(int B, int H, int N, float dropout_p, uint64_t seed, const int32_t* heads, int nheads,
                    const int32_t* rows, int nrows, uint8_t* out, void* stream) {
  if (B < 0 || H < 0 || N < 0 || nheads < 0 || nrows < 0) return FA_ERR_INVALID_ARG;
  if (!(dropout_p >= 0.f && dropout_p < 1.f)) return FA_ERR_INVALID_ARG;
  if (B == 0 || H == 0 || N == 0 || nheads == 0 || nrows == 0) return FA_OK;
  if (!heads || !rows || !out) return FA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  dropout_mask_kernel<<<1184, 256, 0, st>>>(H, N, keep_threshold(dropout_p), seed, heads, nheads, rows, nrows,
                                             out);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d) {
  if (check_common(B, H, N, d, 1.f, 0, 0.f) != FA_OK) return 0;
  return fa::bwd_workspace_bytes(B * H, N, d);
}

namespace {

// Checks shared by the backward entry points; fills the workspace pointers.
int bwd_setup(int B, int H, int N, int d, float scale, int causal, float dropout_p, uint64_t seed, void* workspace,
              size_t workspace_bytes, fa::BwdArgs* a) {
  int rc = check_common(B, H, N, d, scale, causal, dropout_p);
  if (rc != FA_OK) return rc;
  const size_t need = fa::bwd_workspace_bytes(B * H, N, d);
  if (!workspace || workspace_bytes < need) return FA_ERR_WORKSPACE;
  if (!aligned(workspace, 16)) return FA_ERR_ALIGNMENT;
  std::memset(a, 0, sizeof(*a));
  a->kv_hi = kAllTiles;
  a->B = B;
  a->H = H;
  a->N = N;
  a->scale = scale;
  a->scale_log2 = scale * 1.4426950408889634f;
  a->drop_threshold = keep_threshold(dropout_p);
  a->drop_scale = (float)(1.0 / (1.0 - (double)dropout_p));
  a->seed = seed;
  fa::bwd_workspace_split(workspace, B * H, N, d, &a->dq_acc, &a->lse2, &a->drow, &a->sched);
  a->err = device_error_ptr();
  if (!a->err) return cuda_fail(cudaErrorInvalidSymbol);
  return FA_OK;
}

}  // namespace

namespace {

// Strides of the 8 backward tensors, in the order q, k, v, o, dout, dq, dk, dv.
int bwd_prepare_impl(const void* o, const void* dout, const float* lse, const fa_strides* s, int B, int H, int N,
                     int d, void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_common(B, H, N, d, 1.f, 0, 0.f);
  if (rc == 1) return FA_OK;
  if (rc != FA_OK) return rc;
  if (!o || !dout || !lse) return FA_ERR_INVALID_ARG;
  if (!aligned(o, 16) || !aligned(dout, 16) || !aligned(lse, 4) || !strides_ok(s[3]) || !strides_ok(s[4]))
    return FA_ERR_ALIGNMENT;
  fa::BwdArgs a;
  if ((rc = bwd_setup(B, H, N, d, 1.f, 0, 0.f, 0, workspace, workspace_bytes, &a)) != FA_OK) return rc;
  a.o = static_cast<const __nv_bfloat16*>(o);
  a.o_sb = s[3].b;
  a.o_sh = s[3].h;
  a.o_sn = s[3].n;
  a.dout = static_cast<const __nv_bfloat16*>(dout);
  a.do_sb = s[4].b;
  a.do_sh = s[4].h;
  a.do_sn = s[4].n;
  a.lse = lse;
  cudaError_t e = fa::launch_bwd_prepare(a, d, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

int bwd_recompute_impl(const void* q, const void* k, const void* v, const void* dout, void* dk, void* dv,
                       const fa_strides* s, int B, int H, int N, int d, float scale, int causal, float dropout_p,
                       uint64_t seed, void* workspace, size_t workspace_bytes, const uint8_t* bmask,
                       int bmask_heads, void* stream) {
  int rc = check_common(B, H, N, d, scale, causal, dropout_p);
  if (rc == 1) return FA_OK;
  if (rc != FA_OK) return rc;
  if (bmask && (rc = check_block_mask(bmask, bmask_heads, H, N)) != FA_OK) return rc;
  if (!q || !k || !v || !dout || !dk || !dv) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(dout, 16) || !aligned(dk, 16) ||
      !aligned(dv, 16))
    return FA_ERR_ALIGNMENT;
  for (int t : {0, 1, 2, 4, 6, 7})
    if (!strides_ok(s[t])) return FA_ERR_ALIGNMENT;
  fa::BwdArgs a;
  if ((rc = bwd_setup(B, H, N, d, scale, causal, dropout_p, seed, workspace, workspace_bytes, &a)) != FA_OK)
    return rc;
  a.dk = static_cast<__nv_bfloat16*>(dk);
  a.dk_sb = s[6].b;
  a.dk_sh = s[6].h;
  a.dk_sn = s[6].n;
  a.dv = static_cast<__nv_bfloat16*>(dv);
  a.dv_sb = s[7].b;
  a.dv_sh = s[7].h;
  a.dv_sn = s[7].n;
  a.bmask = bmask;
  a.bmask_heads = bmask_heads;
  CUtensorMap mq, mk, mv, mdo;
  if ((rc = make_tile_map(&mq, q, B, H, N, d, s[0])) != FA_OK) return rc;
  if ((rc = make_tile_map(&mk, k, B, H, N, d, s[1])) != FA_OK) return rc;
  if ((rc = make_tile_map(&mv, v, B, H, N, d, s[2])) != FA_OK) return rc;
  if ((rc = make_tile_map(&mdo, dout, B, H, N, d, s[4])) != FA_OK) return rc;
  cudaError_t e = fa::launch_bwd_recompute(mq, mk, mv, mdo, a, d, causal != 0, dropout_p > 0.f,
                                           static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

int bwd_finalize_impl(void* dq, const fa_strides* s, int B, int H, int N, int d, float scale, void* workspace,
                      size_t workspace_bytes, void* stream) {
  int rc = check_common(B, H, N, d, scale, 0, 0.f);
  if (rc == 1) return FA_OK;
  if (rc != FA_OK) return rc;
  if (!dq) return FA_ERR_INVALID_ARG;
  if (!aligned(dq, 16) || !strides_ok(s[5])) return FA_ERR_ALIGNMENT;
  fa::BwdArgs a;
  if ((rc = bwd_setup(B, H, N, d, scale, 0, 0.f, 0, workspace, workspace_bytes, &a)) != FA_OK) return rc;
  a.dq = static_cast<__nv_bfloat16*>(dq);
  a.dq_sb = s[5].b;
  a.dq_sh = s[5].h;
  a.dq_sn = s[5].n;
  cudaError_t e = fa::launch_bwd_finalize(a, d, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

void contiguous8(int H, int N, int d, fa_strides* s) {
  const fa_strides c = contiguous_strides(H, N, d);
  for (int t = 0; t < 8; ++t) s[t] = c;
}

}  // namespace

int fa_bwd_prepare(const void* o, const void* dout, const float* lse, int B, int H, int N, int d, void* workspace,
                   size_t workspace_bytes, void* stream) {
  fa_strides s[8];
  contiguous8(H, N, d, s);
  return bwd_prepare_impl(o, dout, lse, s, B, H, N, d, workspace, workspace_bytes, stream);
}

int fa_bwd_recompute(const void* q, const void* k, const void* v, const void* dout, void* dk, void* dv, int B, int H,
                     int N, int d, float scale, int causal, float dropout_p, uint64_t seed, void* workspace,
                     size_t workspace_bytes, void* stream) {
  fa_strides s[8];
  contiguous8(H, N, d, s);
  return bwd_recompute_impl(q, k, v, dout, dk, dv, s, B, H, N, d, scale, causal, dropout_p, seed, workspace,
                            workspace_bytes, nullptr, 0, stream);
}

int fa_bwd_recompute_blocksparse(const void* q, const void* k, const void* v, const void* dout, void* dk, void* dv,
                                 int B, int H, int N, int d, float scale, int causal, float dropout_p, uint64_t seed,
                                 const uint8_t* block_mask, int mask_heads, void* workspace, size_t workspace_bytes,
                                 void* stream) {
  fa_strides s[8];
  contiguous8(H, N, d, s);
  if (!block_mask && B > 0 && H > 0 && N > 0) return FA_ERR_INVALID_ARG;
  return bwd_recompute_impl(q, k, v, dout, dk, dv, s, B, H, N, d, scale, causal, dropout_p, seed, workspace,
                            workspace_bytes, block_mask, mask_heads, stream);
}

int fa_bwd_finalize(void* dq, int B, int H, int N, int d, float scale, void* workspace, size_t workspace_bytes,
                    void* stream) {
  fa_strides s[8];
  contiguous8(H, N, d, s);
  return bwd_finalize_impl(dq, s, B, H, N, d, scale, workspace, workspace_bytes, stream);
}

namespace {

int bwd_all_impl(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                 void* dq, void* dk, void* dv, const fa_strides* strides, int B, int H, int N, int d, float scale,
                 int causal, float dropout_p, uint64_t seed, const uint8_t* bmask, int bmask_heads, void* workspace,
                 size_t workspace_bytes, void* stream) {
  int rc = check_common(B, H, N, d, scale, causal, dropout_p);
  if (rc == 1) return FA_OK;
  if (rc != FA_OK) return rc;
  if (bmask && (rc = check_block_mask(bmask, bmask_heads, H, N)) != FA_OK) return rc;
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv || !strides) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(dout, 16) ||
      !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(lse, 4))
    return FA_ERR_ALIGNMENT;
  for (int t = 0; t < 8; ++t)
    if (!strides_ok(strides[t])) return FA_ERR_ALIGNMENT;
  if (!workspace || workspace_bytes < fa::bwd_workspace_bytes(B * H, N, d)) return FA_ERR_WORKSPACE;
  if ((rc = bwd_prepare_impl(o, dout, lse, strides, B, H, N, d, workspace, workspace_bytes, stream)) != FA_OK)
    return rc;
  if ((rc = bwd_recompute_impl(q, k, v, dout, dk, dv, strides, B, H, N, d, scale, causal, dropout_p, seed, workspace,
                               workspace_bytes, bmask, bmask_heads, stream)) != FA_OK)
    return rc;
  return bwd_finalize_impl(dq, strides, B, H, N, d, scale, workspace, workspace_bytes, stream);
}

}  // namespace

int fa_bwd_strided(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                   void* dq, void* dk, void* dv, const fa_strides* strides, int B, int H, int N, int d, float scale,
                   int causal, float dropout_p, uint64_t seed, void* workspace, size_t workspace_bytes,
                   void* stream) {
  return bwd_all_impl(q, k, v, o, dout, lse, dq, dk, dv, strides, B, H, N, d, scale, causal, dropout_p, seed, nullptr,
                      0, workspace, workspace_bytes, stream);
}

int fa_fwd_blocksparse(const void* q, const void* k, const void* v, void* o, float* lse, const fa_strides* strides,
                       int B, int H, int N, int d, float scale, int causal, float dropout_p, uint64_t seed,
                       const uint8_t* block_mask, int mask_heads, void* stream) {
  fa_strides c[4];
  if (!strides) {
    for (int t = 0; t < 4; ++t) c[t] = contiguous_strides(H, N, d);
    strides = c;
  }
  if (!block_mask && B > 0 && H > 0 && N > 0) return FA_ERR_INVALID_ARG;
  return fwd_impl(q, k, v, o, lse, strides, B, H, N, d, scale, causal, dropout_p, seed, 1, nullptr, 0, block_mask,
                  mask_heads, stream);
}

int fa_bwd_blocksparse(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                       void* dq, void* dk, void* dv, const fa_strides* strides, int B, int H, int N, int d,
                       float scale, int causal, float dropout_p, uint64_t seed, const uint8_t* block_mask,
                       int mask_heads, void* workspace, size_t workspace_bytes, void* stream) {
  fa_strides c[8];
  if (!strides) {
    contiguous8(H, N, d, c);
    strides = c;
  }
  if (!block_mask && B > 0 && H > 0 && N > 0) return FA_ERR_INVALID_ARG;
  return bwd_all_impl(q, k, v, o, dout, lse, dq, dk, dv, strides, B, H, N, d, scale, causal, dropout_p, seed,
                      block_mask, mask_heads, workspace, workspace_bytes, stream);
}

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse, void* dq,
           void* dk, void* dv, int B, int H, int N, int d, float scale, int causal, float dropout_p, uint64_t seed,
           void* workspace, size_t workspace_bytes, void* stream) {
  fa_strides s[8];
  contiguous8(H, N, d, s);
  return fa_bwd_strided(q, k, v, o, dout, lse, dq, dk, dv, s, B, H, N, d, scale, causal, dropout_p, seed, workspace,
                        workspace_bytes, stream);
}

int fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse, const fa_strides* strides,
                  const int32_t* cu_seqlens, const int32_t* seqused, int B, int H, int max_seqlen, int total_tokens,
                  int d, float scale, int causal, float dropout_p, uint64_t seed, void* stream) {
  int rc = check_varlen(B, H, max_seqlen, total_tokens, d, scale, causal, dropout_p, cu_seqlens, strides, 4);
  if (rc == 1) return FA_OK;
  if (rc != FA_OK) return rc;
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4) ||
      (seqused && !aligned(seqused, 4)))
    return FA_ERR_ALIGNMENT;
  fa_strides s[4];
  for (int t = 0; t < 4; ++t) s[t] = varlen_strides(strides[t], total_tokens);
  CUtensorMap mq, mk, mv;
  if ((rc = make_tile_map(&mq, q, 1, H, total_tokens, d, s[0])) != FA_OK) return rc;
  if ((rc = make_tile_map(&mk, k, 1, H, total_tokens, d, s[1])) != FA_OK) return rc;
  if ((rc = make_tile_map(&mv, v, 1, H, total_tokens, d, s[2])) != FA_OK) return rc;
  fa::FwdArgs a;
  std::memset(&a, 0, sizeof(a));
  a.kv_hi = kAllTiles;
  a.B = B;
  a.H = H;
  a.N = max_seqlen;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.drop_threshold = keep_threshold(dropout_p);
  a.drop_scale = (float)(1.0 / (1.0 - (double)dropout_p));
  a.seed = seed;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.o_sb = 0;
  a.o_sh = s[3].h;
  a.o_sn = s[3].n;
  a.lse = lse;
  a.num_splits = 1;
  a.cu_seqlens = cu_seqlens;
  a.seqused = seqused;
  a.total_tokens = total_tokens;
  a.err = device_error_ptr();
  if (!a.err) return cuda_fail(cudaErrorInvalidSymbol);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool dropout = dropout_p > 0.f;
  rc = d == 64 ? dispatch_fwd<64, fa::kFwdVarlen>(mq, mk, mv, a, causal != 0, dropout, st)
               : dispatch_fwd<128, fa::kFwdVarlen>(mq, mk, mv, a, causal != 0, dropout, st);
  if (rc != FA_OK || !seqused) return rc;
  return launch_varlen_pad(B, H, max_seqlen, total_tokens, cu_seqlens, seqused, d, static_cast<__nv_bfloat16*>(o),
                           s[3], nullptr, s[3], nullptr, s[3], lse, st);
}

size_t fa_bwd_varlen_workspace_size(int B, int H, int max_seqlen, int d) {
  return fa_bwd_workspace_size(B, H, max_seqlen, d);
}

int fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const void* dout, const float* lse,
                  void* dq, void* dk, void* dv, const fa_strides* strides, const int32_t* cu_seqlens,
                  const int32_t* seqused, int B, int H, int max_seqlen, int total_tokens, int d, float scale,
                  int causal, float dropout_p, uint64_t seed, void* workspace, size_t workspace_bytes,
                  void* stream) {
  int rc = check_varlen(B, H, max_seqlen, total_tokens, d, scale, causal, dropout_p, cu_seqlens, strides, 8);
  if (rc == 1) return FA_OK;
  if (rc != FA_OK) return rc;
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(dout, 16) ||
      !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(lse, 4) ||
      (seqused && !aligned(seqused, 4)))
    return FA_ERR_ALIGNMENT;
  fa::BwdArgs a;
  if ((rc = bwd_setup(B, H, max_seqlen, d, scale, causal, dropout_p, seed, workspace, workspace_bytes, &a)) !=
      FA_OK)
    return rc;
  fa_strides s[8];
  for (int t = 0; t < 8; ++t) s[t] = varlen_strides(strides[t], total_tokens);
  a.cu_seqlens = cu_seqlens;
  a.seqused = seqused;
  a.total_tokens = total_tokens;
  a.o = static_cast<const __nv_bfloat16*>(o);
  a.o_sh = s[3].h;
  a.o_sn = s[3].n;
  a.dout = static_cast<const __nv_bfloat16*>(dout);
  a.do_sh = s[4].h;
  a.do_sn = s[4].n;
  a.lse = lse;
  a.dq = static_cast<__nv_bfloat16*>(dq);
  a.dq_sh = s[5].h;
  a.dq_sn = s[5].n;
  a.dk = static_cast<__nv_bfloat16*>(dk);
  a.dk_sh = s[6].h;
  a.dk_sn = s[6].n;
  a.dv = static_cast<__nv_bfloat16*>(dv);
  a.dv_sh = s[7].h;
  a.dv_sn = s[7].n;
  CUtensorMap mq, mk, mv, mdo;
  if ((rc = make_tile_map(&mq, q, 1, H, total_tokens, d, s[0])) != FA_OK) return rc;
  if ((rc = make_tile_map(&mk, k, 1, H, total_tokens, d, s[1])) != FA_OK) return rc;
  if ((rc = make_tile_map(&mv, v, 1, H, total_tokens, d, s[2])) != FA_OK) return rc;
  if ((rc = make_tile_map(&mdo, dout, 1, H, total_tokens, d, s[4])) != FA_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = fa::launch_bwd_prepare(a, d, st);
  if (e != cudaSuccess) return cuda_fail(e);
  e = fa::launch_bwd_recompute(mq, mk, mv, mdo, a, d, causal != 0, dropout_p > 0.f, st);
  if (e != cudaSuccess) return cuda_fail(e);
  e = fa::launch_bwd_finalize(a, d, st);
  if (e != cudaSuccess) return cuda_fail(e);
  if (!seqused) return FA_OK;
  return launch_varlen_pad(B, H, max_seqlen, total_tokens, cu_seqlens, seqused, d, static_cast<__nv_bfloat16*>(dq),
                           s[5], static_cast<__nv_bfloat16*>(dk), s[6], static_cast<__nv_bfloat16*>(dv), s[7],
                           nullptr, st);
}

namespace {

// A key window [kv_begin, kv_end) of an N-key sequence: kv_begin a multiple
// of the 128-key tile, kv_end a multiple of it or N.
bool key_window_ok(int N, int kv_begin, int kv_end) {
  return 0 <= kv_begin && kv_begin <= kv_end && kv_end <= N && kv_begin % 128 == 0 &&
         (kv_end == N || kv_end % 128 == 0);
}

}  // namespace

int fa_fwd_partial(const void* q, const void* k, const void* v, float* part_o, float* part_lse, int B, int H, int N,
                   int d, float scale, int causal, float dropout_p, uint64_t seed, int kv_begin, int kv_end,
                   void* stream) {
  int rc = check_common(B, H, N, d, scale, causal, dropout_p);
  if (rc == 1) return FA_OK;
  if (rc != FA_OK) return rc;
  if (!key_window_ok(N, kv_begin, kv_end)) return FA_ERR_INVALID_ARG;
  const int nk = kv_end - kv_begin;
  if (!q || !part_o || !part_lse || (nk > 0 && (!k || !v))) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(part_o, 16) || !aligned(part_lse, 4) ||
      (nk > 0 && (!aligned(k, 16) || !aligned(v, 16))))
    return FA_ERR_ALIGNMENT;
  CUtensorMap mq, mk, mv;
  if ((rc = make_tile_map(&mq, q, B, H, N, d, contiguous_strides(H, N, d))) != FA_OK) return rc;
  // an empty window reads no key: its maps only need to be valid
  const void* kb = nk > 0 ? k : q;
  const void* vb = nk > 0 ? v : q;
  const int nkm = nk > 0 ? nk : N;
  if ((rc = make_tile_map(&mk, kb, B, H, nkm, d, contiguous_strides(H, nkm, d))) != FA_OK) return rc;
  if ((rc = make_tile_map(&mv, vb, B, H, nkm, d, contiguous_strides(H, nkm, d))) != FA_OK) return rc;
  fa::FwdArgs a;
  std::memset(&a, 0, sizeof(a));
  a.B = B;
  a.H = H;
  a.N = N;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.drop_threshold = keep_threshold(dropout_p);
  a.drop_scale = (float)(1.0 / (1.0 - (double)dropout_p));
  a.seed = seed;
  a.num_splits = 1;
  a.part_o = part_o;
  a.part_lse = part_lse;
  a.kv_lo = kv_begin / 128;
  a.kv_hi = nk > 0 ? (kv_end + 127) / 128 : kv_begin / 128;
  a.kv_row_off = kv_begin;
  a.partial_only = 1;
  a.err = device_error_ptr();
  if (!a.err) return cuda_fail(cudaErrorInvalidSymbol);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool dropout = dropout_p > 0.f;
  return d == 64 ? dispatch_fwd<64, fa::kFwdSplit>(mq, mk, mv, a, causal != 0, dropout, st)
                 : dispatch_fwd<128, fa::kFwdSplit>(mq, mk, mv, a, causal != 0, dropout, st);
}

int fa_merge_partials(const float* part_o, const float* part_lse, int num_parts, void* o, float* lse, int B, int H,
                      int N, int d, void* stream) {
  int rc = check_common(B, H, N, d, 1.f, 0, 0.f);
  if (rc == 1) return FA_OK;
  if (rc != FA_OK) return rc;
  if (num_parts < 1 || num_parts > 4096) return FA_ERR_INVALID_ARG;
  if (!part_o || !part_lse || !o || !lse) return FA_ERR_INVALID_ARG;
  if (!aligned(part_o, 16) || !aligned(o, 16) || !aligned(part_lse, 4) || !aligned(lse, 4)) return FA_ERR_ALIGNMENT;
  fa::FwdArgs a;
  std::memset(&a, 0, sizeof(a));
  a.B = B;
  a.H = H;
  a.N = N;
  const fa_strides s = contiguous_strides(H, N, d);
  a.o = static_cast<__nv_bfloat16*>(o);
  a.o_sb = s.b;
  a.o_sh = s.h;
  a.o_sn = s.n;
  a.lse = lse;
  a.num_splits = num_parts;
  a.part_o = const_cast<float*>(part_o);
  a.part_lse = const_cast<float*>(part_lse);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (d == 64)
    fa::splitkv_combine_kernel<64><<<148 * 8, 256, 0, st>>>(a);
  else
    fa::splitkv_combine_kernel<128><<<148 * 8, 256, 0, st>>>(a);
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

size_t fa_bwd_dq_accumulator_bytes(int B, int H, int N, int d) {
  if (check_common(B, H, N, d, 1.f, 0, 0.f) != FA_OK) return 0;
  return fa::round_up((size_t)B * H * fa::round_up((size_t)N, 128) * d * 4, 256);
}

int fa_bwd_recompute_range(const void* q, const void* k, const void* v, const void* dout, void* dk, void* dv, int B,
                           int H, int N, int d, float scale, int causal, float dropout_p, uint64_t seed, int kv_begin,
                           int kv_end, void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_common(B, H, N, d, scale, causal, dropout_p);
  if (rc == 1) return FA_OK;
  if (rc != FA_OK) return rc;
  if (!key_window_ok(N, kv_begin, kv_end)) return FA_ERR_INVALID_ARG;
  const int nk = kv_end - kv_begin;
  if (nk == 0) return FA_OK;  // no key of this window: nothing to add
  if (!q || !k || !v || !dout || !dk || !dv) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(dout, 16) || !aligned(dk, 16) ||
      !aligned(dv, 16))
    return FA_ERR_ALIGNMENT;
  fa::BwdArgs a;
  if ((rc = bwd_setup(B, H, N, d, scale, causal, dropout_p, seed, workspace, workspace_bytes, &a)) != FA_OK)
    return rc;
  const fa_strides sk = contiguous_strides(H, nk, d);
  a.dk = static_cast<__nv_bfloat16*>(dk);
  a.dk_sb = sk.b;
  a.dk_sh = sk.h;
  a.dk_sn = sk.n;
  a.dv = static_cast<__nv_bfloat16*>(dv);
  a.dv_sb = sk.b;
  a.dv_sh = sk.h;
  a.dv_sn = sk.n;
  a.kv_lo = kv_begin / 128;
  a.kv_hi = (kv_end + 127) / 128;
  a.kv_row_off = kv_begin;
  CUtensorMap mq, mk, mv, mdo;
  const fa_strides sq = contiguous_strides(H, N, d);
  if ((rc = make_tile_map(&mq, q, B, H, N, d, sq)) != FA_OK) return rc;
  if ((rc = make_tile_map(&mk, k, B, H, nk, d, sk)) != FA_OK) return rc;
  if ((rc = make_tile_map(&mv, v, B, H, nk, d, sk)) != FA_OK) return rc;
  if ((rc = make_tile_map(&mdo, dout, B, H, N, d, sq)) != FA_OK) return rc;
  cudaError_t e = fa::launch_bwd_recompute(mq, mk, mv, mdo, a, d, causal != 0, dropout_p > 0.f,
                                           static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FA_OK : cuda_fail(e);
}

}  // extern "C"
