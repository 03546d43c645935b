// debug_check.cuh -- the bounds-checking build.
//
// Compiled with -DFA_DEBUG (libfa_sm100_debug.so), every global-memory
// access of the kernels whose address comes from the work decomposition --
// output rows, the dQ accumulator tiles, the row statistics, the split-KV
// pieces, the work items and the TMA tile coordinates -- is checked, before
// it is made, against the extent that the C-ABI arguments give its buffer
// (shape and element strides).  A failed check skips the access, records the
// first failure (site, offset, limit, block, thread) next to the device error
// word and sets device error 4; fa_debug_bounds_record reads the record.  The
// checks catch index bugs of the kernels themselves (a wrong decode of a work
// item, a row past a sequence, a tile past the accumulator), not buffers that
// are smaller than their arguments say.  The release build compiles every
// check to `true`.
#pragma once

#include "sm100.cuh"

namespace fa {

// where a check sits (the record's site field)
enum DbgSite : int {
  kSiteFwdO = 1,         // forward: O row store
  kSiteFwdLse = 2,       // forward: lse store
  kSiteFwdPart = 3,      // forward: split-KV piece store (O / l, lse)
  kSiteFwdTile = 4,      // forward: TMA tile row of Q, K or V
  kSiteCombine = 5,      // split-KV merge: piece read, O / lse store
  kSiteBwdPreRow = 10,   // row pass: O, dO row read
  kSiteBwdPreLse = 11,   // row pass: lse read
  kSiteBwdItem = 12,     // fused backward: work-item decode
  kSiteBwdTile = 13,     // fused backward: TMA tile row of Q, dO, K or V
  kSiteBwdRow = 14,      // fused backward: row-statistics bulk load
  kSiteBwdAcc = 15,      // fused backward: dQ accumulator tile
  kSiteBwdKV = 16,       // fused backward: dK, dV row store
  kSiteBwdPost = 17,     // dQ conversion: accumulator read, dQ row store
  kSiteVarlenPad = 20,   // variable-length padding fill
};

#ifdef FA_DEBUG
// The record sits right after the device error word: {count, site, offset,
// limit, block, thread}.
static __device__ __noinline__ void dbg_report(int site, long long off, long long lim, int* err) {
  if (!err) return;
  long long* rec = reinterpret_cast<long long*>(err + 2);
  if (atomicAdd(reinterpret_cast<unsigned long long*>(rec), 1ull) == 0ull) {
    rec[1] = site;
    rec[2] = off;
    rec[3] = lim;
    rec[4] = blockIdx.x;
    rec[5] = threadIdx.x;
  }
  atomicCAS(err, kDevOk, kDevBounds);
}

// [off, off + len) within [0, lim)?
__device__ __forceinline__ bool dbg_in(int site, long long off, long long len, long long lim, int* err) {
  if (off >= 0 && len >= 0 && off + len <= lim) return true;
  dbg_report(site, off, lim, err);
  return false;
}
#define FA_IN(site, off, len, lim, err) (::fa::dbg_in((site), (off), (len), (lim), (err)))
#else
#define FA_IN(site, off, len, lim, err) (true)
#endif

// Extent in elements of a [b, h, rows, d] tensor with element strides (b, h,
// row; d contiguous): one past its last element.
__host__ __device__ __forceinline__ long long extent4(long long b, long long h, long long rows, long long d,
                                                      long long sb, long long sh, long long sn) {
  if (b <= 0 || h <= 0 || rows <= 0) return 0;
  return (b - 1) * sb + (h - 1) * sh + (rows - 1) * sn + d;
}

}  // namespace fa
