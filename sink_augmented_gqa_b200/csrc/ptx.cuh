// Thin inline-PTX wrappers for sm_100a: mbarriers, TMA tensor loads, tcgen05
// (TMEM alloc, MMA, commit, ld/st), warp-level ldmatrix / mma.sync /
// movmatrix, and the bounded-wait + status-word machinery every kernel of
// the library uses.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace sa {

// ---------------------------------------------------------------------------
// Device status word and wait limit (one copy per device, this library only)
// ---------------------------------------------------------------------------
__device__ int g_status;                          // OR of SA_STATUS_* bits
__device__ long long g_wait_limit = 2000000000LL; // SM cycles (~1 s at 2 GHz)

constexpr int STATUS_TIMEOUT = 1;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait for the phase of `parity` to complete. Returns false (and
// records STATUS_TIMEOUT) when the limit runs out; never traps or spins
// forever.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try(bar, parity)) return true;
  const long long limit = *((volatile long long*)&g_wait_limit);
  const long long t0 = clock64();
  while (true) {
    if (mbar_try(bar, parity)) return true;
    if (clock64() - t0 > limit) {
      atomicOr(&g_status, STATUS_TIMEOUT);
      return false;
    }
  }
}

// Bounded wait with a fixed limit (~1 s) that ignores the tunable one: used
// only to drain work already in flight (TMA copies, queued MMAs) before a CTA
// that aborted releases its shared or tensor memory. Such work always
// completes on its own, so this wait never runs out in practice.
__device__ __forceinline__ bool mbar_wait_drain(uint32_t bar, uint32_t parity) {
  if (mbar_try(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try(bar, parity)) return true;
    if (clock64() - t0 > 2000000000LL) {
      atomicOr(&g_status, STATUS_TIMEOUT);
      return false;
    }
  }
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// Fetch-and-add with acquire-release semantics at GPU scope: the adding
// thread's prior writes (and those ordered before it by a CTA barrier) are
// visible to whoever reads the new value, and writes released before the
// values it reads are visible to this thread afterwards.
__device__ __forceinline__ int atom_add_acq_rel_gpu(int* p, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
// Orders this thread's generic-proxy view of global memory (including what
// it acquired from other threads) before its later async-proxy (bulk copy)
// reads of global memory.
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Named barrier over `nthreads` threads (multiple of 32).
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// Named barrier that also returns whether `pred` held for any of the
// participating threads (every thread gets the same answer).
__device__ __forceinline__ bool named_bar_or(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

// ---------------------------------------------------------------------------
// TMA: 4-D tiled tensor load into shared memory, completion on an mbarrier.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                            int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar)
      : "memory");
}
// TMA tile store shared -> global (rows past the tensor map's bounds are
// dropped), tracked by this thread's bulk group.
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, uint32_t src, int c0, int c1,
                                             int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.tile.bulk_group [%0, {%1, %2, %3, %4}], [%5];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(src)
      : "memory");
}
// Untiled bulk copy global -> shared (both 16-byte aligned, bytes a multiple
// of 16), completion counted on an mbarrier.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until every committed bulk store of this thread has read its shared
// memory source (the source may be overwritten afterwards).
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Wait until every committed bulk store of this thread has completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
// Prefetch the 128-byte line holding p into L2 (a hint: nothing reaches the SM).
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<uint64_t>(p)) : "memory");
}
// TMA: prefetch a 4-D tile into L2 (nothing reaches shared memory; parts of
// the box outside the tensor are skipped).
__device__ __forceinline__ void tma_prefetch_l2_4d(const CUtensorMap* map, int c0, int c1, int c2, int c3) {
  asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global.tile [%0, {%1, %2, %3, %4}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(c0), "r"(c1), "r"(c2), "r"(c3)
               : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory and the 5th-generation tensor core
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
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
// D[tmem] (+)= A[smem desc] * B[smem desc], kind::f16 (bf16 in, fp32 accum).
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem desc].
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on `bar` once every tcgen05 op this thread issued so far completes.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns per warp (lane = TMEM row).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
      : "memory");
}
// One 32-bit column per lane (lane = TMEM row).
__device__ __forceinline__ void tmem_st1(uint32_t taddr, uint32_t r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(r) : "memory");
}
__device__ __forceinline__ uint32_t tmem_ld1(uint32_t taddr) {
  uint32_t r;
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r) : "r"(taddr));
  return r;
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor for tcgen05.mma (sm_100 format):
// start>>4 in [0,14), LBO>>4 in [16,30), SBO>>4 in [32,46), version 1 in
// [46,48), layout type in [61,64) (2 = 128-byte swizzle, 4 = 64-byte).
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)(layout & 7) << 61;
  return d;
}

// Instruction descriptor, kind::f16: bf16 A/B, fp32 D, M x N, operand majors.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn_major, int b_mn_major) {
  return (1u << 4)                        // D format: f32
         | (1u << 7)                      // A format: bf16
         | (1u << 10)                     // B format: bf16
         | ((uint32_t)a_mn_major << 15)   // A major (0 = K-major)
         | ((uint32_t)b_mn_major << 16)   // B major
         | ((uint32_t)(N >> 3) << 17)     // N / 8
         | ((uint32_t)(M >> 4) << 24);    // M / 16
}

// ---------------------------------------------------------------------------
// Warp-level tensor-core helpers (decode path)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                            uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                                  uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// C[16x8] += A[16x16] * B[16x8], bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// ---------------------------------------------------------------------------
// Register reallocation between warpgroups (all threads of a warpgroup).
// ---------------------------------------------------------------------------
template <int N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// ---------------------------------------------------------------------------
// Scalar helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// (d0, d1) = (a0 * b0 + c0, a1 * b1 + c1), one packed instruction.
__device__ __forceinline__ void fma2(float& d0, float& d1, float a0, float a1, float b0, float b1,
                                     float c0, float c1) {
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
// (d0, d1) = (a0 + b0, a1 + b1), one packed instruction.
__device__ __forceinline__ void addto2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// Two values of 2^x on the FMA pipe instead of the MUFU unit, for
// x in [-120, 8] (smaller x is clamped to -120: 2^-120 stands in for the
// vanishing weight). Range reduction: t = x + 1.5*2^23 rounds x to the
// nearest integer j (held in t's low mantissa bits), f = x - j in
// [-1/2, 1/2] exactly; then 2^x = 2^j * p(f), the 2^j applied as an integer
// add of j << 23 to p's bit pattern. p is the degree-3 fit of 2^f on
// [-1/2, 1/2] with constant term 1 (so integer x give exact powers of two)
// produced by fit_exp2_poly.py: relative error < 1.1e-4 in fp32 Horner form,
// well below the 2^-9 of the bf16 P it feeds.
constexpr float EXP2_C0 = 1.0f, EXP2_C1 = 0.693282962f, EXP2_C2 = 0.242210969f,
                EXP2_C3 = 0.0550089031f;
__device__ __forceinline__ void exp2_fma2(float& a, float& b) {
  constexpr float MAGIC = 12582912.0f;  // 1.5 * 2^23
  a = fmaxf(a, -120.0f);
  b = fmaxf(b, -120.0f);
  float ta, tb, ja, jb, fa, fb;
  addto2(ta, tb, a, b, MAGIC, MAGIC);
  addto2(ja, jb, ta, tb, -MAGIC, -MAGIC);
  addto2(fa, fb, a, b, -ja, -jb);
  float pa = EXP2_C3, pb = EXP2_C3;
  fma2(pa, pb, pa, pb, fa, fb, EXP2_C2, EXP2_C2);
  fma2(pa, pb, pa, pb, fa, fb, EXP2_C1, EXP2_C1);
  fma2(pa, pb, pa, pb, fa, fb, EXP2_C0, EXP2_C0);
  a = __int_as_float(__float_as_int(pa) + (__float_as_int(ta) << 23));
  b = __int_as_float(__float_as_int(pb) + (__float_as_int(tb) << 23));
}

// (a0, a1) += (b0, b1), one packed instruction.
__device__ __forceinline__ void add2(float& a0, float& a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%0, %1};\n\tmov.b64 rb, {%2, %3};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(b0), "f"(b1));
}
// (a0, a1) *= (b0, b1), one packed instruction.
__device__ __forceinline__ void mul2(float& a0, float& a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%0, %1};\n\tmov.b64 rb, {%2, %3};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(b0), "f"(b1));
}
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// Pack two floats into bf16x2 (round to nearest even); `lo` in the low half.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// fp64 -> bf16, round to nearest even, with a single rounding: round to odd
// into fp32 first (24 bits >= 8 + 2, so the second rounding cannot create a
// false tie), then round to nearest even.
__device__ __forceinline__ uint32_t bf16_bits_from_f64(double x) {
  float f = __double2float_rz(x);
  if ((double)f != x) f = __uint_as_float(__float_as_uint(f) | 1u);
  return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// One RoPE pair: (x1, x2) -> (x1 c - x2 s, x2 c + x1 s), each result the
// bf16 round-to-nearest-even of the exact value. The bf16 x fp32 products are
// exact in fp64, so an fp64 evaluation carries one fp64 rounding and is then
// rounded once more to bf16 (rope_pair_f64). The fast path evaluates in fp32
// and keeps the result only where the fp32 error bound proves that the exact
// value lies in the same bf16 rounding cell (rope_fast_ok); elsewhere (about
// one element in 2^14, and zeros) it falls back to fp64.
__device__ __forceinline__ void rope_pair_f64(float x1, float x2, float c, float s, uint32_t& y1,
                                              uint32_t& y2) {
  const double a = (double)x1, b = (double)x2, cd = (double)c, sd = (double)s;
  y1 = bf16_bits_from_f64(a * cd - b * sd);
  y2 = bf16_bits_from_f64(b * cd + a * sd);
}

// v = RN32(x c -+ t) with t = RN32(y s) differs from the exact x c -+ y s by at
// most 2^-24 (|v| + |t|)(1 + 2^-22) (one relative rounding in each of the two
// operations; |v| >= 2^-100 keeps both away from the subnormal range, where
// the bound is absolute and below 2^-149). e below is twice that bound. The
// bf16 rounding of a value changes only at the midpoints between adjacent
// bf16 numbers; the midpoint inside v's bf16 interval is v's bit pattern with
// the low 16 bits set to 0x8000 (same sign and binade, so v - mid is exact),
// and every other midpoint is at least |v| 2^-10 away. With both distances
// above e, v and the exact value round to the same bf16. The three tests
// are folded into one compare: min(|v - mid|, |v| 2^-10) > max(e, 2^-110)
// implies both distances exceed e and |v| > 2^-100.
__device__ __forceinline__ bool rope_fast_ok(float v, float t) {
  const float av = fabsf(v);
  const float e = (av + fabsf(t)) * 0x1p-23f;
  const float mid = __uint_as_float((__float_as_uint(v) & 0xFFFF0000u) | 0x8000u);
  return fminf(fabsf(v - mid), av * 0x1p-10f) > fmaxf(e, 0x1p-110f);
}

__device__ __forceinline__ void rope_pair(float x1, float x2, float c, float s, uint32_t& y1,
                                          uint32_t& y2) {
  const float t1 = __fmul_rn(x2, s), t2 = __fmul_rn(x1, s);
  const float v1 = __fmaf_rn(x1, c, -t1), v2 = __fmaf_rn(x2, c, t2);
  if (rope_fast_ok(v1, t1) & rope_fast_ok(v2, t2)) {
    y1 = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v1));
    y2 = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v2));
  } else {
    rope_pair_f64(x1, x2, c, s, y1, y2);
  }
}

// Two adjacent pairs packed as bf16x2 words (low half = lower index).
__device__ __forceinline__ void rope_pair2(uint32_t& w1, uint32_t& w2, float c0, float c1, float s0,
                                           float s1) {
  const float a0 = bf16_lo(w1), a1 = bf16_hi(w1), b0 = bf16_lo(w2), b1 = bf16_hi(w2);
  const float t0 = __fmul_rn(b0, s0), t1 = __fmul_rn(b1, s1);
  const float u0 = __fmul_rn(a0, s0), u1 = __fmul_rn(a1, s1);
  const float v0 = __fmaf_rn(a0, c0, -t0), v1 = __fmaf_rn(a1, c1, -t1);
  const float z0 = __fmaf_rn(b0, c0, u0), z1 = __fmaf_rn(b1, c1, u1);
  if (rope_fast_ok(v0, t0) & rope_fast_ok(v1, t1) & rope_fast_ok(z0, u0) & rope_fast_ok(z1, u1)) {
    w1 = pack_bf16(v0, v1);
    w2 = pack_bf16(z0, z1);
  } else {
    uint32_t p0, p1, q0, q1;
    rope_pair_f64(a0, b0, c0, s0, p0, q0);
    rope_pair_f64(a1, b1, c1, s1, p1, q1);
    w1 = p0 | (p1 << 16);
    w2 = q0 | (q1 << 16);
  }
}

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start while the kernel before it in the stream is still
// running; griddep_wait() returns once that kernel has completed and its
// memory operations are visible (at once when the launch had no such
// predecessor), so nothing before it may read memory another kernel writes.
// griddep_launch_dependents() lets the next such kernel be scheduled before
// this one has finished.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Byte offset of element (row, col) in a tile stored as column blocks of
// `CB` bf16 elements, each block [rows][CB] with the hardware swizzle
// (bits [4, 4+b) of the address XOR bits [7, 7+b); b = 3 for 128-byte rows,
// 2 for 64-byte rows). `block_bytes` must be a multiple of 1024 and the tile
// base 1024-byte aligned.
template <int CB>
__device__ __forceinline__ uint32_t swz_off(int row, int col, uint32_t block_bytes) {
  constexpr uint32_t SWZ = CB * 2;
  constexpr uint32_t MASK = SWZ / 16 - 1;
  const uint32_t off = (uint32_t)(col / CB) * block_bytes + (uint32_t)row * SWZ +
                       (uint32_t)(col % CB) * 2u;
  return off ^ (((off >> 7) & MASK) << 4);
}

}  // namespace sa
