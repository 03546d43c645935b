// sm100.cuh -- inline-PTX building blocks for the sm_100a attention kernels:
// mbarriers with bounded waits, TMA tile loads, tcgen05 (TMEM allocation,
// MMA issue/commit, TMEM loads/stores) and the shared-memory / instruction
// descriptors the MMAs take.  Written from the PTX ISA's descriptions of these
// instructions; the descriptor bit positions are listed next to each builder.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace fa {

// Error word values written by a kernel that gives up (device side).
enum : int {
  kDevOk = 0,
  kDevTimeout = 1,      // a bounded mbarrier wait ran out
  kDevMisaligned = 2,   // shared-memory tile base not 1024-byte aligned
  kDevBadSeqlens = 3,   // variable-length offsets or lengths out of range (clamped)
  kDevBounds = 4,       // a bounds check failed (bounds-checking build only)
};

// Upper bound on any single wait (ns).  Kernels here run for milliseconds;
// two seconds without progress means something is broken.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Shared abort state of one CTA: the first role whose wait runs out records
// the error in global memory and raises the flag; every other role's waits
// then return false promptly, so all roles leave their loops and meet at
// the kernel's final barrier instead of hanging.
struct Abort {
  volatile int* flag;  // in shared memory
  int* err;            // global error word (may be null)
};

// Wait until phase `parity` of `bar` has completed.  Returns false if the
// CTA is aborting or if this wait exceeded kWaitLimitNs (then it aborts).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const Abort& ab) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 0u) {
      if (*ab.flag) return false;
      if (global_timer_ns() - t0 > kWaitLimitNs) {
        *ab.flag = 1;
        if (ab.err) atomicCAS(ab.err, kDevOk, kDevTimeout);
        return false;
      }
    }
  }
}

// Bounded wait that ignores the abort flag: used only while draining work
// already in flight before TMEM is freed.
__device__ __forceinline__ void mbar_wait_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > kWaitLimitNs) return;
  }
}

// ------------------------------------------------------------------ TMA

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(m) : "memory");
}

// Named barrier over `count` threads (a multiple of 32) of this CTA.
__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// 4-D tiled load (x innermost): tensors addressed as {d, n, h, b}.
__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* m, int x, int y, int z, int w,
                                            uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4, %5, %6}], [%2], %7;" ::"r"(smem_u32(dst)),
      "l"(m), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z), "r"(w), "l"(policy)
      : "memory");
}

// Untiled bulk copy global -> shared (16-byte aligned addresses and size).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Bulk reduction shared -> global: dst[i] += src[i] (fp32), `bytes` a
// multiple of 16, both addresses 16-byte aligned.  Tracked by this thread's
// bulk async-groups.
__device__ __forceinline__ void bulk_reduce_add_f32(float* dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(dst), "r"(src),
               "r"(bytes)
               : "memory");
}

// dst[0..3] += {a, b, c, d} (fp32 bit patterns) as one vector reduction
// performed at L2; dst 16-byte aligned.
__device__ __forceinline__ void red_add_v4_f32(float* dst, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(__uint_as_float(a)),
               "f"(__uint_as_float(b)), "f"(__uint_as_float(c)), "f"(__uint_as_float(d))
               : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// Wait until at most N of this thread's bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Wait until all of this thread's bulk groups have completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (tensor-core operand reads).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// -------------------------------------------------------------- tcgen05

__device__ __forceinline__ void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// Warpgroup register reallocation: every thread of the warpgroup executes
// the same instruction; `inc` waits until enough registers are free.
template <uint32_t N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, both operands described by descriptors.
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T.
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on `bar` when every tcgen05.mma this thread issued so far has
// completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// 32 lanes x 32 columns of 32-bit data: thread t of the warp gets lane
// (base lane + t), columns col..col+31.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// tcgen05.ld writes its destination registers asynchronously; they are valid
// only after tcgen05.wait::ld.  This empty statement, placed after the wait,
// makes every later use of `r` depend on it, so the compiler cannot hoist
// arithmetic on `r` above the wait.
__device__ __forceinline__ void reg_fence(uint32_t (&r)[32]) {
  asm volatile(""
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                 "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                 "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]),
                 "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]),
                 "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
}

// Load 32 columns and wait for them (single-batch convenience).
__device__ __forceinline__ void tmem_ld32_sync(uint32_t taddr, uint32_t (&r)[32]) {
  tmem_ld32(taddr, r);
  tmem_ld_wait();
  reg_fence(r);
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------- descriptors
//
// Shared-memory matrix descriptor (64 bit):
//   [0,14)  start address >> 4      [16,30) leading-dimension byte offset >> 4
//   [32,46) stride-dimension byte offset >> 4
//   [46,48) version (1 on sm_100)   [49,52) base offset (0: tiles 1024-aligned)
//   [52]    LBO mode (0)            [61,64) layout: 2 = 128-byte swizzle
//
// All operand tiles here are stored the way a 128-byte-swizzled TMA box of
// 64 bf16 columns lands in shared memory: rows of 128 bytes, 16-byte chunks
// XOR-permuted by (row mod 8), 8-row groups 1024 bytes apart, a second
// 64-column half of the tile (if any) `half_stride` bytes further on.
//
// K-major use (reduction dimension along the 128-byte rows): SBO = 1024 is
// the step between 8-row groups; LBO is unused.  A K=16 slice starts
// 32 bytes further along the row; slices 4..7 sit in the second half.
//
// MN-major use (reduction dimension down the rows): SBO = 1024 is the step
// between groups of 8 reduction rows, LBO = half_stride the step between the
// 64-element halves of the M/N dimension.  A K=16 slice starts 16 rows
// (2048 bytes) further down.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}

// K-major operand: slice kk (16 bf16 along K) of a tile whose 64-column
// halves are `half_stride` bytes apart.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t tile, int kk, uint32_t half_stride) {
  const uint32_t addr = tile + (uint32_t)(kk >> 2) * half_stride + (uint32_t)(kk & 3) * 32u;
  return smem_desc(addr, 16u, 1024u);
}

// MN-major operand: slice kk (16 rows along K).
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t tile, int kk, uint32_t half_stride) {
  const uint32_t addr = tile + (uint32_t)kk * 2048u;
  return smem_desc(addr, half_stride, 1024u);
}

// Instruction descriptor for kind::f16 with bf16 inputs and fp32 accumulate
// (32 bit):
//   [4,6) D format (1 = f32)   [7,10) A format (1 = bf16)  [10,13) B format
//   [15] A major (0 K, 1 MN)   [16] B major                [17,23) N >> 3
//   [24,29) M >> 4
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ----------------------------------------------------------- arithmetic

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Two fp32 values in one 64-bit register for the packed f32x2 pipe ops.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}

__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

// (a * b + c) on both halves.
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.ftz.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.ftz.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.ftz.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// 2^x for two values at once on the FMA pipe, for x <= 126 (x = -inf or
// below -125 gives a value in [0, 2^-124] instead of 2^x: the
// exponent arithmetic leaves the normal range).  Cody-Waite split
// x = n + f with n = round(x) and f in [-1/2, 1/2]: n comes from adding
// 1.5 * 2^23 (the rounded integer lands in the low mantissa bits), 2^f from a
// cubic, and n is added to the exponent field with integer arithmetic.  The
// cubic is a relative-error minimax fit of 2^f on [-1/2, 1/2] computed for
// this library (fp64 Remez exchange, coefficients rounded to fp32): max
// relative error 7.5e-5, far below the bf16 resolution of the
// probabilities it produces.
__device__ __forceinline__ void exp2_poly_x2(uint64_t x2, float& r0, float& r1) {
  float x0, x1;
  f2_unpack(x2, x0, x1);
  x0 = fmaxf(x0, -126.f);
  x1 = fmaxf(x1, -126.f);
  const uint64_t xc = f2_pack(x0, x1);
  const uint64_t t = f2_add(xc, f2_pack(12582912.f, 12582912.f));    // 1.5 * 2^23 + round(x)
  const uint64_t n = f2_add(t, f2_pack(-12582912.f, -12582912.f));   // round(x), exact
  const uint64_t fr = f2_fma(n, f2_pack(-1.f, -1.f), xc);            // x - round(x), exact
  uint64_t p = f2_fma(fr, f2_pack(0.0551716685295105f, 0.0551716685295105f),
                      f2_pack(0.2426111251115799f, 0.2426111251115799f));
  p = f2_fma(p, fr, f2_pack(0.6932609677314758f, 0.6932609677314758f));
  p = f2_fma(p, fr, f2_pack(0.9999280571937561f, 0.9999280571937561f));
  float p0, p1, t0, t1;
  f2_unpack(p, p0, p1);
  f2_unpack(t, t0, t1);
  // low mantissa bits of t hold round(x); the high bits of t shifted by 23
  // vanish mod 2^32, so t << 23 == round(x) << 23
  r0 = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23));
  r1 = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ void st_global_v4(void* p, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.global.v4.b32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ float4 ld_shared_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr));
  return v;
}

// ------------------------------------------------ variable-length batches

// Where sequence b of a variable-length batch lives: its first token, its slot
// size and its real length.  Offsets are clamped into [0, T] and lengths into
// the slot and into max_slot, so every row index derived from them stays
// inside the caller's tensors even if the offsets are inconsistent; an
// inconsistency is also recorded in the device error word.
struct SeqSpan {
  int row0, slot, len;
};

__device__ __forceinline__ SeqSpan varlen_span(const int* cu, const int* used, int b, int total, int max_slot,
                                               int* err, bool report) {
  int s0 = __ldg(cu + b), s1 = __ldg(cu + b + 1);
  const bool bad = s0 < 0 || s1 < s0 || s1 > total || s1 - s0 > max_slot;
  s0 = min(max(s0, 0), total);
  s1 = min(max(s1, s0), total);
  SeqSpan r;
  r.row0 = s0;
  r.slot = min(s1 - s0, max_slot);
  int L = used ? __ldg(used + b) : r.slot;
  const bool bad_used = used && (L < 0 || L > r.slot);
  r.len = min(max(L, 0), r.slot);
  if (report && (bad || bad_used) && err) atomicCAS(err, kDevOk, kDevBadSeqlens);
  return r;
}

// ---------------------------------------------------- block-sparse tile sets

// Largest tile count block-sparse kernels handle (bit sets in shared
// memory): N <= 4096 * 128.
constexpr int kMaxSparseTiles = 4096;
constexpr int kSparseWords = kMaxSparseTiles / 32;

// Walks the set bits of (x | y) in ascending order; the caller never asks for
// more indices than there are set bits.  Nothing is read before the first
// next(), so kernels without bit sets may construct one.
struct BitWalk {
  const uint32_t* x;
  const uint32_t* y;
  int w, nwords;
  uint32_t cur;
  __device__ __forceinline__ BitWalk(const uint32_t* x_, const uint32_t* y_, int nwords_)
      : x(x_), y(y_), w(-1), nwords(nwords_), cur(0u) {}
  __device__ __forceinline__ int next() {
    while (cur == 0u && w + 1 < nwords) {
      ++w;
      cur = x[w] | y[w];
    }
    const int b = __ffs(cur) - 1;
    cur &= cur - 1u;
    return 32 * w + b;
  }
};

__device__ __forceinline__ bool bit_set(const uint32_t* bits, int j) { return (bits[j >> 5] >> (j & 31)) & 1u; }

// One warp: bit sets of the nonzero bytes row[j * stride], begin <= j < end,
// of up to two mask rows (row1 and bits1 may be null), written to bits0/bits1
// (nwords words each).  Returns the popcounts of the two sets and of their
// union.
__device__ __forceinline__ int3 build_bit_sets(const uint8_t* row0, int end0, const uint8_t* row1, int end1,
                                               int begin, long long stride, int nwords, uint32_t* bits0,
                                               uint32_t* bits1, int lane) {
  int c0 = 0, c1 = 0, cu = 0;
  for (int w0 = 0; w0 < nwords; w0 += 4) {
    uint8_t v0[4], v1[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int j = 32 * (w0 + k) + lane;
      v0[k] = (j >= begin && j < end0) ? __ldg(row0 + (long long)j * stride) : (uint8_t)0;
      v1[k] = (row1 && j >= begin && j < end1) ? __ldg(row1 + (long long)j * stride) : (uint8_t)0;
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t m0 = __ballot_sync(0xffffffffu, v0[k] != 0);
      const uint32_t m1 = __ballot_sync(0xffffffffu, v1[k] != 0);
      if (w0 + k < nwords) {
        if (lane == 0) {
          bits0[w0 + k] = m0;
          if (bits1) bits1[w0 + k] = m1;
        }
        c0 += __popc(m0);
        c1 += __popc(m1);
        cu += __popc(m0 | m1);
      }
    }
  }
  return make_int3(c0, c1, cu);
}

}  // namespace fa
