// Device-side helpers shared by the sm_100a kernels: bounded mbarrier waits,
// TMA tile loads, tcgen05 (TMEM / UMMA) wrappers and the per-CTA KV schedule.
//
// Every wait on an mbarrier is bounded in time (the GPU's %globaltimer, in
// nanoseconds).  When the limit runs out the waiting thread records
// AS_DEVERR_TIMEOUT in the device error word, raises a CTA-local abort flag and
// returns false; every other wait in the CTA sees the flag and returns as
// well, so the CTA drains and exits instead of hanging.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "as_kernels.h"

namespace asp {

// ---------------------------------------------------------------------------
// device error word (read and cleared by as_device_status on the host).  The
// library is built without relocatable device code, so each translation unit
// holds its own copy; only the kernels with bounded waits (attn_tc_bf16.cu)
// set it, and the host reads that unit's copy.
// ---------------------------------------------------------------------------
static __device__ unsigned int g_dev_error = 0;

__device__ __forceinline__ void raise_dev_error(unsigned int bits) {
  atomicOr(&g_dev_error, bits);
}

// This translation unit's error word, read and cleared (host; the caller has
// synchronised the work whose errors it wants).
static inline cudaError_t read_and_clear_local_dev_error(unsigned int* bits) {
  unsigned int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_dev_error, sizeof(v));
  if (e != cudaSuccess) return e;
  if (v != 0) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(g_dev_error, &zero, sizeof(zero));
    if (e != cudaSuccess) return e;
  }
  *bits = v;
  return cudaSuccess;
}

// ---------------------------------------------------------------------------
// checked build (ASP_DEBUG=1): ASP_CHECK(cond) is cond, and when cond is false
// it also records AS_DEVERR_BOUNDS in the device error word, so that the
// access it guards is skipped and the host learns of it (no trap).  In the
// normal build it is `true` and costs nothing.
// ---------------------------------------------------------------------------
#ifndef ASP_DEBUG
#define ASP_DEBUG 0
#endif
__device__ __forceinline__ bool check_or_flag(bool ok) {
  if (!ok) raise_dev_error(AS_DEVERR_BOUNDS);
  return ok;
}
#if ASP_DEBUG
#define ASP_CHECK(cond) (::asp::check_or_flag(static_cast<bool>(cond)))
#else
#define ASP_CHECK(cond) true
#endif

// ---------------------------------------------------------------------------
// shared-memory addresses and mbarriers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}"
               ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}"
               ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}

// non-blocking probe of the phase: much cheaper than try_wait when the phase
// has already completed
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}

#ifndef ASP_TEST_FIRST
#define ASP_TEST_FIRST 1
#endif

// low 32 bits of the GPU's %globaltimer (nanoseconds); differences of up to
// 4.29 s are exact in unsigned arithmetic
__device__ __forceinline__ uint32_t global_ns32() {
  uint32_t t;
  asm volatile("mov.u32 %0, %%globaltimer_lo;" : "=r"(t));
  return t;
}

// The bound of every wait in the kernels: 1 s of GPU time.
constexpr uint32_t KERNEL_WAIT_NS = 1000000000u;

// Waits until the phase with the given parity has completed.  Returns false
// (after flagging) when `limit_ns` nanoseconds have passed, when COUNT_POLLS
// and `polls` rounds of try_wait have come back empty, or when another thread
// of the CTA has already aborted.  The clock is read only once a try_wait has
// come back empty, so a wait that succeeds at once costs nothing extra.  The
// kernels wait without a poll count; the test hook counts polls as well.
template <bool COUNT_POLLS>
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                                  uint32_t polls, uint32_t limit_ns) {
  if (ASP_TEST_FIRST && mbar_test_wait(bar, parity)) return true;
  if (mbar_try_wait(bar, parity)) return true;
  const uint32_t t0 = global_ns32();
  for (uint32_t it = 1; !COUNT_POLLS || it < polls; ++it) {
    if (*abort_flag) return false;
    if (mbar_try_wait(bar, parity)) return true;
    if (global_ns32() - t0 > limit_ns) break;
  }
  raise_dev_error(AS_DEVERR_TIMEOUT);
  *abort_flag = 1;
  return false;
}

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  return mbar_wait_bounded<false>(bar, parity, abort_flag, 0u, KERNEL_WAIT_NS);
}

// ---------------------------------------------------------------------------
// TMA
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

// 3-D tiled load (x = innermost element index, y = row, z = head) into
// shared memory; completion is signalled on `bar` as transaction bytes.
__device__ __forceinline__ void tma_load_3d(void* smem_dst, const void* tmap, uint64_t* bar,
                                            int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];"
      ::"r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(tmap)), "r"(smem_u32(bar)),
        "r"(x), "r"(y), "r"(z)
      : "memory");
}

// generic-proxy shared-memory writes -> visible to the async proxy (UMMA reads)
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: TMEM allocation, MMA, commit, loads and stores
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* smem_slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
               ::"r"(smem_u32(smem_slot)), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (bf16 in, fp32 accumulate)
__device__ __forceinline__ void umma_bf16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T, kind::f16.  A (M x K, bf16) lives in TMEM:
// lane = row, each 32-bit column holds two consecutive K elements (low half
// first), so one K=16 step spans 8 columns.
__device__ __forceinline__ void umma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// arrive once on `bar` when every MMA issued so far by this thread has completed
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
      ::"r"(smem_u32(bar)) : "memory");
}

#define ASP_R32(a) \
  "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]), "=r"(a[4]), "=r"(a[5]), "=r"(a[6]), "=r"(a[7]), \
  "=r"(a[8]), "=r"(a[9]), "=r"(a[10]), "=r"(a[11]), "=r"(a[12]), "=r"(a[13]), "=r"(a[14]), "=r"(a[15]), \
  "=r"(a[16]), "=r"(a[17]), "=r"(a[18]), "=r"(a[19]), "=r"(a[20]), "=r"(a[21]), "=r"(a[22]), "=r"(a[23]), \
  "=r"(a[24]), "=r"(a[25]), "=r"(a[26]), "=r"(a[27]), "=r"(a[28]), "=r"(a[29]), "=r"(a[30]), "=r"(a[31])
#define ASP_W32(a) \
  "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(a[4]), "r"(a[5]), "r"(a[6]), "r"(a[7]), \
  "r"(a[8]), "r"(a[9]), "r"(a[10]), "r"(a[11]), "r"(a[12]), "r"(a[13]), "r"(a[14]), "r"(a[15]), \
  "r"(a[16]), "r"(a[17]), "r"(a[18]), "r"(a[19]), "r"(a[20]), "r"(a[21]), "r"(a[22]), "r"(a[23]), \
  "r"(a[24]), "r"(a[25]), "r"(a[26]), "r"(a[27]), "r"(a[28]), "r"(a[29]), "r"(a[30]), "r"(a[31])

// each thread of the warp reads 32 consecutive fp32 columns of its TMEM lane
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : ASP_R32(r) : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
      ::"r"(taddr), ASP_W32(r) : "memory");
}
// each thread of the warp reads 128 consecutive fp32 columns of its TMEM lane (one instruction)
__device__ __forceinline__ void tmem_ld128(uint32_t taddr, uint32_t (&r)[128]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x128.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63, %64, %65, %66, %67, %68, %69, %70, %71, %72, %73, %74, %75, %76, %77, %78, %79, %80, %81, %82, %83, %84, %85, %86, %87, %88, %89, %90, %91, %92, %93, %94, %95, %96, %97, %98, %99, %100, %101, %102, %103, %104, %105, %106, %107, %108, %109, %110, %111, %112, %113, %114, %115, %116, %117, %118, %119, %120, %121, %122, %123, %124, %125, %126, %127}, [%128];"
      : ASP_R32(r), ASP_R32((r + 32)), ASP_R32((r + 64)), ASP_R32((r + 96)) : "r"(taddr));
}
__device__ __forceinline__ void tmem_st64(uint32_t taddr, const uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x64.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32, %33, %34, %35, %36, %37, %38, %39, %40, %41, %42, %43, %44, %45, %46, %47, %48, %49, %50, %51, %52, %53, %54, %55, %56, %57, %58, %59, %60, %61, %62, %63, %64};"
      ::"r"(taddr), ASP_W32(r), ASP_W32((r + 32)) : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Per-warpgroup register budget.  The sum over all warpgroups must not exceed
// the registers the CTA was launched with (threads x registers per thread at
// launch); the launcher checks the kernel's register count before launching.
template <int N>
__device__ __forceinline__ void regs_dealloc() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void regs_alloc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// ---------------------------------------------------------------------------
// UMMA descriptors
// ---------------------------------------------------------------------------
// Shared-memory matrix descriptor, 128-byte swizzle (layout type 2), version 1.
// lbo/sbo in bytes.  K-major tiles: rows of 128 B, 8-row groups 1024 B apart
// (sbo = 1024; lbo unused).  MN-major tiles: lbo = distance between 64-element
// column chunks, sbo = distance between 8-row groups along K.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) |
         (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
         (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) |
         (1ull << 46) | (2ull << 61);
}

// Instruction descriptor for kind::f16 with bf16 A/B and fp32 D.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) |
         ((b_mn_major ? 1u : 0u) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// ---------------------------------------------------------------------------
// fast exp2 on the MUFU unit
// ---------------------------------------------------------------------------
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// exp2 on the FMA pipe, to relieve the MUFU unit (exp2_poly2 below).  2^x = 2^n * 2^f with
// n = round(x) (by adding and subtracting 1.5 * 2^23) and f = x - n in
// [-1/2, 1/2]; 2^f is a degree-4 minimax polynomial (relative error 2.7e-6,
// coefficients from gen_exp2_poly.py) and 2^n is added to its exponent bits.
// x is clamped below at -125 so the result stays a normal float (2^-125 is
// negligible against a row maximum of 1).
constexpr float EXP2_C0 = 9.999992847e-01f;
constexpr float EXP2_C1 = 6.931217909e-01f;
constexpr float EXP2_C2 = 2.402474433e-01f;
constexpr float EXP2_C3 = 5.591785908e-02f;
constexpr float EXP2_C4 = 9.570102207e-03f;
constexpr float ROUND_MAGIC = 12582912.0f;  // 1.5 * 2^23

// ---------------------------------------------------------------------------
// packed fp32 pairs (Blackwell f32x2 FMA-pipe instructions)
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t r, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(r));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// exp2_poly on a pair, with the rounding and the polynomial in f32x2 form
__device__ __forceinline__ uint64_t exp2_poly2(float x0, float x1) {
  const uint64_t x = f2_pack(fmaxf(x0, -125.0f), fmaxf(x1, -125.0f));
  const uint64_t t = f2_add(x, f2_pack(ROUND_MAGIC, ROUND_MAGIC));
  const uint64_t n = f2_add(t, f2_pack(-ROUND_MAGIC, -ROUND_MAGIC));
  const uint64_t f = f2_fma(n, f2_pack(-1.0f, -1.0f), x);
  uint64_t p = f2_fma(f2_pack(EXP2_C4, EXP2_C4), f, f2_pack(EXP2_C3, EXP2_C3));
  p = f2_fma(p, f, f2_pack(EXP2_C2, EXP2_C2));
  p = f2_fma(p, f, f2_pack(EXP2_C1, EXP2_C1));
  p = f2_fma(p, f, f2_pack(EXP2_C0, EXP2_C0));
  float p0, p1, t0, t1;
  f2_unpack(p, p0, p1);
  f2_unpack(t, t0, t1);
  return f2_pack(__int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23)),
                 __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23)));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// ---------------------------------------------------------------------------
// per-CTA KV schedule derived from one row of the kernel code matrix
// ---------------------------------------------------------------------------
// A query row block reads a list of KV token ranges grouped into accumulation
// groups.  Group 0 (when present) gathers every code-1 partition (adjacent
// partitions merged into one range) and is emitted as one composed state.
// Consecutive code-2 partitions with the same destination plane form one
// group, emitted as the composed state of its partitions (a cache group entry;
// with one destination per partition, each partition's own state).
struct KvSchedule {
  int n_ranges;
  int n_groups;
  int range_lo[2 * AS_MAX_P];
  int range_hi[2 * AS_MAX_P];
  int group_first[AS_MAX_P + 1];
  int group_count[AS_MAX_P + 1];
  int group_dest[AS_MAX_P + 1];  // -1: the composite output; >= 0: destination plane
};

// KV partition j covers K/V rows [kv_row0[j], kv_row0[j] + n); partitions whose
// rows are adjacent merge into one range.
__device__ __forceinline__ void build_schedule(const uint8_t* code_row, const int8_t* dest_of,
                                               const int* kv_row0, int P, int n, KvSchedule& s) {
  s.n_ranges = 0;
  s.n_groups = 0;
  for (int j = 0; j < P; ++j) {
    if (code_row[j] != AS_KCODE_COMPOSE) continue;
    if (s.n_ranges > 0 && s.range_hi[s.n_ranges - 1] == kv_row0[j]) {
      s.range_hi[s.n_ranges - 1] = kv_row0[j] + n;
    } else {
      s.range_lo[s.n_ranges] = kv_row0[j];
      s.range_hi[s.n_ranges] = kv_row0[j] + n;
      ++s.n_ranges;
    }
  }
  if (s.n_ranges > 0) {
    s.group_first[0] = 0;
    s.group_count[0] = s.n_ranges;
    s.group_dest[0] = -1;
    s.n_groups = 1;
  }
  for (int j = 0; j < P; ++j) {
    if (code_row[j] != AS_KCODE_EMIT) continue;
    const int dst = dest_of[j];
    if (s.n_groups > 0 && s.group_dest[s.n_groups - 1] == dst) {
      // same destination as the previous emitted partition: one group
      if (s.range_hi[s.n_ranges - 1] == kv_row0[j]) {
        s.range_hi[s.n_ranges - 1] = kv_row0[j] + n;
      } else {
        s.range_lo[s.n_ranges] = kv_row0[j];
        s.range_hi[s.n_ranges] = kv_row0[j] + n;
        ++s.n_ranges;
        ++s.group_count[s.n_groups - 1];
      }
      continue;
    }
    s.range_lo[s.n_ranges] = kv_row0[j];
    s.range_hi[s.n_ranges] = kv_row0[j] + n;
    s.group_first[s.n_groups] = s.n_ranges;
    s.group_count[s.n_groups] = 1;
    s.group_dest[s.n_groups] = dst;
    ++s.n_ranges;
    ++s.n_groups;
  }
}

}  // namespace asp
