// Thin inline-PTX wrappers for the sm_100a features the window-attention kernel uses:
// mbarriers with time-bounded waits, TMA tensor loads, the tcgen05 tensor-core MMA with
// TMEM accumulators, TMEM allocation and TMEM -> register loads, packed fp32x2 arithmetic.
#pragma once
#include <cstdint>

namespace s3w {
namespace sm100 {

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait that may suspend the thread in hardware (not spinning, so it takes no issue
// slots from the warps sharing its scheduler) until the phase completes or about
// `hint_ns` nanoseconds have passed.
__device__ __forceinline__ bool mbar_try_wait_hint(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Slow path of mbar_wait_bounded, kept out of line so that the many wait sites of the
// kernels stay small in the instruction cache (internal linkage: one copy per kernel file).
static __device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait_hint(bar, parity, 20000u)) return true;
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
}

// Wait for phase `parity` of an mbarrier, giving up after `limit_ns` nanoseconds.
// Returns false on timeout (the caller records the error and unwinds).
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, limit_ns);
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// 5-D tiled TMA load global -> shared (no multicast); completes `bytes` on the mbarrier.
__device__ __forceinline__ void tma_load_5d(uint32_t dst, const void* tmap, int c0, int c1, int c2, int c3, int c4,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4, %5, "
      "%6}], [%7];" ::"r"(dst),
      "l"(tmap), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void prefetch_tmap(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(tmap) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Make generic-proxy shared-memory writes visible to the async proxy (tensor core).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---- TMEM ------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 lanes x 32 bits, 16 consecutive columns: thread t of the warp gets lane (base + t).
// The registers are only valid after tmem_wait_ld() followed by reg_fence16() on them.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7]),
        "=f"(v[8]), "=f"(v[9]), "=f"(v[10]), "=f"(v[11]), "=f"(v[12]), "=f"(v[13]), "=f"(v[14]), "=f"(v[15])
      : "r"(taddr));
}
// 32 lanes x 32 bits, 8 consecutive columns (start column a multiple of 8).
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float* v) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7])
               : "r"(taddr));
}
__device__ __forceinline__ void reg_fence8(float* v) {
  asm volatile("" : "+f"(v[0]), "+f"(v[1]), "+f"(v[2]), "+f"(v[3]), "+f"(v[4]), "+f"(v[5]), "+f"(v[6]),
               "+f"(v[7]));
}
// 32 lanes x 32 bits, one column: thread t gets lane base + t.
__device__ __forceinline__ void tmem_ld1(uint32_t taddr, float* v) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=f"(v[0]) : "r"(taddr));
}
__device__ __forceinline__ void reg_fence1(float* v) { asm volatile("" : "+f"(v[0])); }
// 16 lanes x 32 bits, twice, one column each: threads 0..15 get lanes base + t, column c;
// threads 16..31 get lanes base + t - 16, column c + 1.
__device__ __forceinline__ void tmem_ld_16x32bx2_x1(uint32_t taddr, float* v) {
  asm volatile("tcgen05.ld.sync.aligned.16x32bx2.x1.b32 {%0}, [%1], 1;" : "=f"(v[0]) : "r"(taddr));
}
// 16 lanes x 32 bits, twice: threads 0..15 get lanes base + t, columns [c, c + 8); threads
// 16..31 get lanes base + t - 16, columns [c + 8, c + 16).
__device__ __forceinline__ void tmem_ld_16x32bx2_x8(uint32_t taddr, float* v) {
  asm volatile("tcgen05.ld.sync.aligned.16x32bx2.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8], 8;"
               : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7])
               : "r"(taddr));
}
// The same with 16 columns per half: threads 16..31 get columns [c + 16, c + 32).
__device__ __forceinline__ void tmem_ld_16x32bx2_x16(uint32_t taddr, float* v) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16], 16;"
      : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7]),
        "=f"(v[8]), "=f"(v[9]), "=f"(v[10]), "=f"(v[11]), "=f"(v[12]), "=f"(v[13]), "=f"(v[14]), "=f"(v[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// Emits nothing; ties 16 registers to a point after the preceding volatile asm (the
// tcgen05.wait::ld), so no use of them can be scheduled before the load has landed.
__device__ __forceinline__ void reg_fence16(float* v) {
  asm volatile("" : "+f"(v[0]), "+f"(v[1]), "+f"(v[2]), "+f"(v[3]), "+f"(v[4]), "+f"(v[5]), "+f"(v[6]),
               "+f"(v[7]), "+f"(v[8]), "+f"(v[9]), "+f"(v[10]), "+f"(v[11]), "+f"(v[12]), "+f"(v[13]),
               "+f"(v[14]), "+f"(v[15]));
}

// The same, executed by a whole warp with only the `leader` lane issuing: the warp stays
// converged, so the descriptor arithmetic around it can stay warp-uniform.
__device__ __forceinline__ void umma_bf16_ss_leader(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                                    uint32_t idesc, uint32_t accumulate, uint32_t leader) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.b32 p, %4, 0;\n\tsetp.ne.b32 q, %5, 0;\n\t"
      "@q tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(leader)
      : "memory");
}
// Whole MMA chains in one asm block, so the descriptor steps are plain 64-bit adds between
// the MMAs (each tcgen05.mma otherwise costs a block of operand moves).  Executed by the
// whole warp; only `leader` issues.  The first MMA of a chain overwrites D, the rest
// accumulate.
#define S3W_MMA_(A, B, P) "@q tcgen05.mma.cta_group::1.kind::f16 [%0], " A ", " B ", %3, " P ";\n\t"
// S = Q K^T over head_dim / 16 K steps of 32 bytes (K-major, 128B swizzle)
template <int KSTEPS>
__device__ __forceinline__ void umma_chain_qk(uint32_t d_tmem, uint64_t a0, uint64_t b0, uint32_t idesc,
                                              uint32_t leader) {
  static_assert(KSTEPS == 2 || KSTEPS == 4, "head_dim 32 or 64");
  if constexpr (KSTEPS == 4) {
    asm volatile(
        "{\n\t.reg .pred q, f, t;\n\t.reg .b64 a, b;\n\t"
        "setp.ne.b32 q, %4, 0;\n\tsetp.ne.b32 f, %4, %4;\n\tsetp.eq.b32 t, %4, %4;\n\t"
        "mov.b64 a, %1;\n\tmov.b64 b, %2;\n\t" S3W_MMA_("a", "b", "f")
        "add.s64 a, a, 2;\n\tadd.s64 b, b, 2;\n\t" S3W_MMA_("a", "b", "t")
        "add.s64 a, a, 2;\n\tadd.s64 b, b, 2;\n\t" S3W_MMA_("a", "b", "t")
        "add.s64 a, a, 2;\n\tadd.s64 b, b, 2;\n\t" S3W_MMA_("a", "b", "t") "}" ::"r"(d_tmem),
        "l"(a0), "l"(b0), "r"(idesc), "r"(leader)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred q, f, t;\n\t.reg .b64 a, b;\n\t"
        "setp.ne.b32 q, %4, 0;\n\tsetp.ne.b32 f, %4, %4;\n\tsetp.eq.b32 t, %4, %4;\n\t"
        "mov.b64 a, %1;\n\tmov.b64 b, %2;\n\t" S3W_MMA_("a", "b", "f")
        "add.s64 a, a, 2;\n\tadd.s64 b, b, 2;\n\t" S3W_MMA_("a", "b", "t") "}" ::"r"(d_tmem),
        "l"(a0), "l"(b0), "r"(idesc), "r"(leader)
        : "memory");
  }
}
// O = P V over 144 keys in 9 K steps of 16 keys.  P: steps of 32 bytes inside a 64-key
// block, `block_step` (descriptor units) to the next block after every fourth step, and the
// last 16 keys from `p_last` (a separately swizzled block).  V: each step moves the address
// field by 2048 / 16 and the leading byte offset (the ones block behind it) by the opposite.
__device__ __forceinline__ void umma_chain_pv(uint32_t d_tmem, uint64_t p0, uint64_t v0, uint32_t idesc,
                                              uint32_t leader, uint64_t p_last, uint64_t block_step) {
  asm volatile(
      "{\n\t.reg .pred q, f, t;\n\t.reg .b64 a, b;\n\t"
      "setp.ne.b32 q, %4, 0;\n\tsetp.ne.b32 f, %4, %4;\n\tsetp.eq.b32 t, %4, %4;\n\t"
      "mov.b64 a, %1;\n\tmov.b64 b, %2;\n\t" S3W_MMA_("a", "b", "f")
      "add.s64 a, a, 2;\n\tadd.s64 b, b, -8388480;\n\t" S3W_MMA_("a", "b", "t")
      "add.s64 a, a, 2;\n\tadd.s64 b, b, -8388480;\n\t" S3W_MMA_("a", "b", "t")
      "add.s64 a, a, 2;\n\tadd.s64 b, b, -8388480;\n\t" S3W_MMA_("a", "b", "t")
      "add.s64 a, a, %6;\n\tadd.s64 b, b, -8388480;\n\t" S3W_MMA_("a", "b", "t")
      "add.s64 a, a, 2;\n\tadd.s64 b, b, -8388480;\n\t" S3W_MMA_("a", "b", "t")
      "add.s64 a, a, 2;\n\tadd.s64 b, b, -8388480;\n\t" S3W_MMA_("a", "b", "t")
      "add.s64 a, a, 2;\n\tadd.s64 b, b, -8388480;\n\t" S3W_MMA_("a", "b", "t")
      "add.s64 b, b, -8388480;\n\t" S3W_MMA_("%5", "b", "t") "}" ::"r"(d_tmem),
      "l"(p0), "l"(v0), "r"(idesc), "r"(leader), "l"(p_last), "l"(block_step)
      : "memory");
}
#undef S3W_MMA_

__device__ __forceinline__ void umma_commit_leader(uint32_t bar, uint32_t leader) {
  asm volatile(
      "{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %1, 0;\n\t"
      "@q tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(bar),
      "r"(leader)
      : "memory");
}

// Arrive (once) on an mbarrier when every tcgen05 operation issued so far by this thread
// has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// Shared-memory matrix descriptor (sm_100 format): start address, leading and stride byte
// offsets (all >> 4), descriptor version 1, base offset 0, swizzle mode in bits 61..63.
enum : uint32_t { kSwizzleNone = 0, kSwizzle128B = 2, kSwizzle64B = 4, kSwizzle32B = 6 };
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                                              uint32_t swizzle) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;  // version
  d |= static_cast<uint64_t>(swizzle & 7u) << 61;
  return d;
}

// Instruction descriptor for kind::f16: bf16 A and B, fp32 accumulator, dense.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4)                                   // D format: f32
         | (1u << 7)                                 // A format: bf16
         | (1u << 10)                                // B format: bf16
         | (static_cast<uint32_t>(a_mn_major) << 15)  // A major-ness
         | (static_cast<uint32_t>(b_mn_major) << 16)  // B major-ness
         | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}

// Packed two-lane fp32 arithmetic (one instruction for two values).
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  uint64_t d;
  asm("{\n\t.reg .b64 a, b, c;\n\tmov.b64 a, {%1,%2};\n\tmov.b64 b, {%3,%4};\n\tmov.b64 c, {%5,%6};\n\t"
      "fma.rn.f32x2 %0, a, b, c;\n\t}"
      : "=l"(d) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  float2 r;
  asm("mov.b64 {%0,%1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(d));
  return r;
}
// max of three fp32 values in one instruction.
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Two finite fp32 values -> packed bf16x2, rounded to nearest with ties away from zero,
// on the integer pipe (add half an ulp of bf16 to the bit pattern, keep the upper halves).
// Differs from round-to-nearest-even only on exact ties.
__device__ __forceinline__ uint32_t pack_bf16x2_int(float lo, float hi) {
  const uint32_t a = __float_as_uint(lo) + 0x8000u;
  const uint32_t b = __float_as_uint(hi) + 0x8000u;
  return __byte_perm(a, b, 0x7632);
}

__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  uint64_t d;
  asm("{\n\t.reg .b64 a, b;\n\tmov.b64 a, {%1,%2};\n\tmov.b64 b, {%3,%4};\n\tmul.rn.f32x2 %0, a, b;\n\t}"
      : "=l"(d) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  float2 r;
  asm("mov.b64 {%0,%1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(d));
  return r;
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  uint64_t d;
  asm("{\n\t.reg .b64 a, b;\n\tmov.b64 a, {%1,%2};\n\tmov.b64 b, {%3,%4};\n\tadd.rn.f32x2 %0, a, b;\n\t}"
      : "=l"(d) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  float2 r;
  asm("mov.b64 {%0,%1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(d));
  return r;
}

// 32-byte global loads (one full sector per thread): plain, and evict-first for data read
// once.
__device__ __forceinline__ void ld_global_v8(const void* p, uint32_t (&v)[8]) {
  asm volatile("ld.global.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
               : "l"(p)
               : "memory");
}
__device__ __forceinline__ void ld_global_cs_v8(const void* p, uint32_t (&v)[8]) {
  asm volatile("ld.global.cs.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
               : "l"(p)
               : "memory");
}
// 32-byte evict-first global store (output written once).
__device__ __forceinline__ void st_global_cs_v8(void* p, const uint32_t (&v)[8]) {
  asm volatile("st.global.cs.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(v[0]), "r"(v[1]), "r"(v[2]),
               "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

// 32-byte global store (one full sector per thread).
__device__ __forceinline__ void st_global_v8(void* p, const uint32_t (&v)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(v[0]), "r"(v[1]), "r"(v[2]),
               "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

}  // namespace sm100
}  // namespace s3w
