// ptx.cuh -- thin inline-PTX wrappers for the sm_100a features the kernels use:
// mbarriers, bulk async copies, tcgen05 (TMEM alloc, block-scaled MMA, commit,
// smem->TMEM copy, TMEM loads/stores, fences) and the E2M1 conversions.
#pragma once
#include <cuda_fp16.h>

#include <cstdint>

namespace mxattn {

// ------------------------------------------------------------------------------------------------
// Addresses
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }

// Named barrier among `count` threads (a multiple of 32) of the CTA.
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Named barrier that also returns the OR of `pred` over the participating threads, so that a
// decision taken after it (such as leaving a loop) is the same in every participant.
__device__ __forceinline__ bool named_bar_or(uint32_t id, uint32_t count, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.or.pred po, %2, %3, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(count)
      : "memory");
  return r != 0;
}

// ------------------------------------------------------------------------------------------------
// mbarriers
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

// try_wait: the thread may sleep until the phase completes or a time limit passes, so waiting
// warps do not take issue slots from working ones.  MXATTN_WAIT_HINT_NS > 0 passes that limit
// (nanoseconds) as a suspend-time hint; 0 (the default, measured fastest here) leaves it to the
// hardware; < 0 selects the non-blocking test_wait, for experiments.
#ifndef MXATTN_WAIT_HINT_NS
#define MXATTN_WAIT_HINT_NS 0
#endif
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
#if MXATTN_WAIT_HINT_NS > 0
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"((uint32_t)MXATTN_WAIT_HINT_NS)
      : "memory");
#elif MXATTN_WAIT_HINT_NS == 0
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
#else  // negative: non-blocking test, the caller spins
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
#endif
  return ok != 0;
}

// Non-blocking test of a phase: true once it has completed (with the same acquire semantics as
// a successful try_wait).  Its result is only needed when the caller branches on it, so a test
// issued early overlaps its latency with other work.
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait with a suspend-time hint (nanoseconds): the thread sleeps until the phase completes
// or the hint expires, issuing nothing meanwhile.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Bounded wait for warps whose work has slack (the producer and the MMA issuers): each try
// may sleep up to `hint_ns`, so a waiting warp takes almost no issue slots from the warps that
// share its SM sub-partition.  Gives up as mbar_wait does.
__device__ __forceinline__ bool mbar_wait_sleep(uint32_t bar, uint32_t parity, const volatile int* abort,
                                                long long budget, uint32_t hint_ns) {
  if (mbar_try_wait_sleep(bar, parity, hint_ns)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait_sleep(bar, parity, hint_ns)) return true;
    if (*abort) return false;
    if (clock64() - t0 > budget) return false;
  }
}

// Bounded wait.  Gives up (returns false) after `budget` SM clock cycles, or as
// soon as *abort becomes non-zero (another warp gave up first).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, const volatile int* abort,
                                          long long budget) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (clock64() - t0 > budget) return false;
  }
}

// ------------------------------------------------------------------------------------------------
// Bulk async copy global -> shared, completion counted on an mbarrier (bytes).
// dst and src 16-byte aligned, bytes a multiple of 16.
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Make this thread's generic-proxy shared-memory writes visible to the async proxy
// (tensor-core operand reads).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------------------------------------
// tcgen05: tensor memory
// ------------------------------------------------------------------------------------------------
// Whole warp: allocate `ncols` TMEM columns, base address written to smem[dst].
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

// Shared-memory matrix descriptor for tcgen05 operands (K-major).
//   start address >> 4 in bits [0,14), leading byte offset >> 4 in [16,30),
//   stride byte offset >> 4 in [32,46), descriptor version 1 in [46,48),
//   layout (swizzle) type in [61,64): 0 none, 4 = 64-byte, 6 = 32-byte swizzle.
enum : uint32_t { kLayoutNone = 0, kLayoutSW64 = 4, kLayoutSW32 = 6 };

__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                                              uint32_t layout) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)(layout & 7u) << 61;
  return d;
}

// Instruction descriptor of tcgen05.mma kind::mxf4 (block-scaled E2M1 x E2M1 -> f32,
// UE8M0 scales, both operands K-major, dense, K = 64 per instruction):
//   b_sf_id [4,6), a_format [7,10) = 1 (E2M1), b_format [10,13) = 1, N>>3 in [17,23),
//   scale format bit 23 = 1 (UE8M0), M>>4 in [24,29), a_sf_id [29,31).
__host__ __device__ constexpr uint32_t mxf4_idesc(uint32_t M, uint32_t N, uint32_t a_sf_id,
                                                  uint32_t b_sf_id) {
  return ((b_sf_id & 3u) << 4) | (1u << 7) | (1u << 10) | ((N >> 3) << 17) | (1u << 23) |
         ((M >> 4) << 24) | ((a_sf_id & 3u) << 29);
}

// The same for kind::mxf4nvf4 with 16-element blocks and UE4M3 scales (the NVFP4 comparison
// format): scale format bit 23 = 0; a K = 64 instruction takes all four scale bytes of a
// row's 32-bit TMEM word, so both scale-factor ids are 0.
__host__ __device__ constexpr uint32_t nvf4_idesc(uint32_t M, uint32_t N) {
  return (1u << 7) | (1u << 10) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

__device__ __forceinline__ void mma_nvf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T with per-32-element scales from TMEM.  One thread issues.
__device__ __forceinline__ void mma_mxf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// Arrive on an mbarrier once all previously issued tcgen05 operations of this thread complete.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// Copy a 512-byte scale-factor atom (32 rows x 16 bytes, K-major, no swizzle) from shared
// memory to 4 TMEM columns, replicated into the 4 lane quadrants.  One thread issues.
__device__ __forceinline__ void tmem_cp_sf_atom(uint32_t taddr, uint32_t smem_atom) {
  const uint64_t desc = smem_desc(smem_atom, 0, 128, kLayoutNone);
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(desc) : "memory");
}

// 16-byte asynchronous copy global -> shared (cp.async, L2 only): src_bytes 16 copies, 0 fills
// the 16 bytes with zeros (src is not read).  Both addresses 16-byte aligned.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
// every cp.async of this thread has landed (visible to the thread; a barrier publishes them)
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// close the thread's current group of cp.async copies
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// wait until at most N of the thread's committed groups are still in flight
template <int N>
__device__ __forceinline__ void cp_async_wait_group() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Warp-collective TMEM loads / stores: lane i of warp w (w = warp index mod 4) touches TMEM lane
// 32*w + i; 32 consecutive 32-bit columns starting at taddr's column.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_ld1(uint32_t taddr, uint32_t& r) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r) : "r"(taddr) : "memory");
}
__device__ __forceinline__ void tmem_st1(uint32_t taddr, uint32_t r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(r) : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Registers filled by tcgen05.ld hold their values only after tcgen05.wait::ld.  These empty
// volatile asm statements, placed after the wait, make every later use of the registers depend
// on a point after it, so the compiler cannot move a use above the wait.
__device__ __forceinline__ void pin1(uint32_t& r) { asm volatile("" : "+r"(r)); }
// Two 32-column loads and the wait for both in one statement: the 64 outputs are defined only
// after the wait, so no use can be scheduled above it.
__device__ __forceinline__ void tmem_ld64_wait(uint32_t taddr0, uint32_t taddr1, uint32_t (&a)[32],
                                               uint32_t (&b)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%64];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%65];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3]), "=r"(a[4]), "=r"(a[5]), "=r"(a[6]), "=r"(a[7]),
        "=r"(a[8]), "=r"(a[9]), "=r"(a[10]), "=r"(a[11]), "=r"(a[12]), "=r"(a[13]), "=r"(a[14]),
        "=r"(a[15]), "=r"(a[16]), "=r"(a[17]), "=r"(a[18]), "=r"(a[19]), "=r"(a[20]), "=r"(a[21]),
        "=r"(a[22]), "=r"(a[23]), "=r"(a[24]), "=r"(a[25]), "=r"(a[26]), "=r"(a[27]), "=r"(a[28]),
        "=r"(a[29]), "=r"(a[30]), "=r"(a[31]),
        "=r"(b[0]), "=r"(b[1]), "=r"(b[2]), "=r"(b[3]), "=r"(b[4]), "=r"(b[5]), "=r"(b[6]), "=r"(b[7]),
        "=r"(b[8]), "=r"(b[9]), "=r"(b[10]), "=r"(b[11]), "=r"(b[12]), "=r"(b[13]), "=r"(b[14]),
        "=r"(b[15]), "=r"(b[16]), "=r"(b[17]), "=r"(b[18]), "=r"(b[19]), "=r"(b[20]), "=r"(b[21]),
        "=r"(b[22]), "=r"(b[23]), "=r"(b[24]), "=r"(b[25]), "=r"(b[26]), "=r"(b[27]), "=r"(b[28]),
        "=r"(b[29]), "=r"(b[30]), "=r"(b[31])
      : "r"(taddr0), "r"(taddr1)
      : "memory");
}

// 128 consecutive 32-bit columns in one load, waited for in the same statement (the outputs exist
// only after the wait, so no use can be scheduled above it).
__device__ __forceinline__ void tmem_ld128_wait(uint32_t taddr, uint32_t (&r)[128]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x128.b32 {"
      "%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,"
      "%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,"
      "%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,%64,%65,%66,%67,%68,%69,%70,%71,%72,%73,%74,%75,%76,%77,%78,%79,"
      "%80,%81,%82,%83,%84,%85,%86,%87,%88,%89,%90,%91,%92,%93,%94,%95,%96,%97,%98,%99,%100,%101,%102,%103,%104,"
      "%105,%106,%107,%108,%109,%110,%111,%112,%113,%114,%115,%116,%117,%118,%119,%120,%121,%122,%123,%124,%125,"
      "%126,%127}, [%128];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
        "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
        "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
        "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
        "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63]),
        "=r"(r[64]), "=r"(r[65]), "=r"(r[66]), "=r"(r[67]), "=r"(r[68]), "=r"(r[69]), "=r"(r[70]), "=r"(r[71]),
        "=r"(r[72]), "=r"(r[73]), "=r"(r[74]), "=r"(r[75]), "=r"(r[76]), "=r"(r[77]), "=r"(r[78]), "=r"(r[79]),
        "=r"(r[80]), "=r"(r[81]), "=r"(r[82]), "=r"(r[83]), "=r"(r[84]), "=r"(r[85]), "=r"(r[86]), "=r"(r[87]),
        "=r"(r[88]), "=r"(r[89]), "=r"(r[90]), "=r"(r[91]), "=r"(r[92]), "=r"(r[93]), "=r"(r[94]), "=r"(r[95]),
        "=r"(r[96]), "=r"(r[97]), "=r"(r[98]), "=r"(r[99]), "=r"(r[100]), "=r"(r[101]), "=r"(r[102]),
        "=r"(r[103]), "=r"(r[104]), "=r"(r[105]), "=r"(r[106]), "=r"(r[107]), "=r"(r[108]), "=r"(r[109]),
        "=r"(r[110]), "=r"(r[111]), "=r"(r[112]), "=r"(r[113]), "=r"(r[114]), "=r"(r[115]), "=r"(r[116]),
        "=r"(r[117]), "=r"(r[118]), "=r"(r[119]), "=r"(r[120]), "=r"(r[121]), "=r"(r[122]), "=r"(r[123]),
        "=r"(r[124]), "=r"(r[125]), "=r"(r[126]), "=r"(r[127])
      : "r"(taddr)
      : "memory");
}

// The same load without the wait: the registers hold the columns only after tmem_wait_ld(), and
// every use must be pinned below that wait (pin1 on each register).
__device__ __forceinline__ void tmem_ld128_nowait(uint32_t taddr, uint32_t (&r)[128]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x128.b32 {"
      "%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,"
      "%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,"
      "%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,%64,%65,%66,%67,%68,%69,%70,%71,%72,%73,%74,%75,%76,%77,%78,%79,"
      "%80,%81,%82,%83,%84,%85,%86,%87,%88,%89,%90,%91,%92,%93,%94,%95,%96,%97,%98,%99,%100,%101,%102,%103,%104,"
      "%105,%106,%107,%108,%109,%110,%111,%112,%113,%114,%115,%116,%117,%118,%119,%120,%121,%122,%123,%124,%125,"
      "%126,%127}, [%128];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
        "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
        "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
        "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
        "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63]),
        "=r"(r[64]), "=r"(r[65]), "=r"(r[66]), "=r"(r[67]), "=r"(r[68]), "=r"(r[69]), "=r"(r[70]), "=r"(r[71]),
        "=r"(r[72]), "=r"(r[73]), "=r"(r[74]), "=r"(r[75]), "=r"(r[76]), "=r"(r[77]), "=r"(r[78]), "=r"(r[79]),
        "=r"(r[80]), "=r"(r[81]), "=r"(r[82]), "=r"(r[83]), "=r"(r[84]), "=r"(r[85]), "=r"(r[86]), "=r"(r[87]),
        "=r"(r[88]), "=r"(r[89]), "=r"(r[90]), "=r"(r[91]), "=r"(r[92]), "=r"(r[93]), "=r"(r[94]), "=r"(r[95]),
        "=r"(r[96]), "=r"(r[97]), "=r"(r[98]), "=r"(r[99]), "=r"(r[100]), "=r"(r[101]), "=r"(r[102]),
        "=r"(r[103]), "=r"(r[104]), "=r"(r[105]), "=r"(r[106]), "=r"(r[107]), "=r"(r[108]), "=r"(r[109]),
        "=r"(r[110]), "=r"(r[111]), "=r"(r[112]), "=r"(r[113]), "=r"(r[114]), "=r"(r[115]), "=r"(r[116]),
        "=r"(r[117]), "=r"(r[118]), "=r"(r[119]), "=r"(r[120]), "=r"(r[121]), "=r"(r[122]), "=r"(r[123]),
        "=r"(r[124]), "=r"(r[125]), "=r"(r[126]), "=r"(r[127])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void pin32(uint32_t (&r)[32]) {
#pragma unroll
  for (int i = 0; i < 32; i++) pin1(r[i]);
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ------------------------------------------------------------------------------------------------
// E2M1 conversions and fast exp2
// ------------------------------------------------------------------------------------------------
// Four pairs of fp32 -> four bytes of packed E2M1 codes (round to nearest even, saturating).
// Byte i holds (lo = a[2i], hi = a[2i+1]); element 2i lands in the low nibble.
__device__ __forceinline__ uint32_t cvt_e2m1x8(float a0, float a1, float a2, float a3, float a4, float a5,
                                               float a6, float a7) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(a0), "f"(a1), "f"(a2), "f"(a3), "f"(a4), "f"(a5), "f"(a6), "f"(a7));
  return out;
}

// Sum of 32 non-negative E2M1 codes (four packed words), in units of 0.5, exact.
// Each nibble (magnitude index 0..7, sign bit clear) selects its value in half-units
// {0, 1, 2, 3, 4, 6, 8, 12} from an 8-byte table with one byte permute per 4 codes, and
// dp4a adds the four bytes into an integer accumulator.
__device__ __forceinline__ uint32_t e2m1x32_sum_halves(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3) {
  constexpr uint32_t kLo = 0x03020100u;  // half-units of codes 0..3
  constexpr uint32_t kHi = 0x0C080604u;  // half-units of codes 4..7
  const uint32_t w[4] = {w0, w1, w2, w3};
  uint32_t acc = 0;
#pragma unroll
  for (int i = 0; i < 4; i++) {
    acc = __dp4a(__byte_perm(kLo, kHi, w[i]), 0x01010101u, acc);
    acc = __dp4a(__byte_perm(kLo, kHi, w[i] >> 16), 0x01010101u, acc);
  }
  return acc;
}

// E4M3 (FP8, bias 7, subnormals, largest finite 448) conversions for the NVFP4 block scales:
// two fp32 -> two E4M3 bytes, round to nearest even, saturating (lo -> byte 0, hi -> byte 1).
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
  uint16_t out;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(out) : "f"(lo), "f"(hi));
  return out;
}

// Two E4M3 bytes (byte 0 -> .x) -> their exact fp32 values (through f16, which holds every E4M3).
__device__ __forceinline__ float2 e4m3x2_to_float2(uint32_t bytes) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"((uint16_t)bytes));
  return make_float2(__half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu))),
                     __half2float(__ushort_as_half((unsigned short)(h2 >> 16))));
}

// max of three fp32 values (one instruction on sm_100)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^x for a pair of fp32 values on the FMA pipe (no MUFU): Cody-Waite style range reduction
// x = n + f, n = round(x) via the 1.5 * 2^23 rounding constant, f in [-0.5, 0.5]; 2^f by a
// degree-5 polynomial with constant term exactly 1 (our own fit of 2^f on [-0.5, 0.5] by
// reweighted least squares toward minimax relative error, 1.9e-7 with fp32 Horner evaluation),
// so that integer x gives 2^x exactly; 2^n added to the exponent field.  Inputs are clamped below
// at -64 (2^-64 is far below every rounding threshold that matters here); inputs are at most a
// few units above 0 in the attention kernel.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  x.x = fmaxf(x.x, -64.f);
  x.y = fmaxf(x.y, -64.f);
  const float2 t = __fadd2_rn(x, make_float2(kRound, kRound));                         // kRound + n
  const float2 nn = __ffma2_rn(t, make_float2(-1.f, -1.f), make_float2(kRound, kRound));  // -n
  const float2 f = __fadd2_rn(x, nn);                                                  // x - n
  float2 p = __ffma2_rn(make_float2(1.3264724e-3f, 1.3264724e-3f), f, make_float2(9.6715130e-3f, 9.6715130e-3f));
  p = __ffma2_rn(p, f, make_float2(5.5507336e-2f, 5.5507336e-2f));
  p = __ffma2_rn(p, f, make_float2(2.4022242e-1f, 2.4022242e-1f));
  p = __ffma2_rn(p, f, make_float2(6.9314700e-1f, 6.9314700e-1f));
  p = __ffma2_rn(p, f, make_float2(1.f, 1.f));
  // the low bits of t hold n; (bits(t) << 23) adds n to the exponent (the constant's own bits
  // shift out entirely)
  return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// fma with the result clamped to [0, 1] (one instruction)
__device__ __forceinline__ float fma_sat(float a, float b, float c) {
  float d;
  asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// A stand-in for 2^u that gives the same E2M1 code as 2^u under cvt.rn.satfinite.e2m1x2 (round to
// nearest even, saturating at 6), for a pair of arguments given as w = clamp((u + 2.5) / 8, 0, 1),
// computed on the FMA pipe alone with six packed FMAs.
//
// The E2M1 code of a positive value depends only on where it lies against the grid midpoints
// 0.25, 0.75, 1.25, 1.75, 2.5, 3.5 and 5, i.e. on where u lies against their base-2 logarithms.
// So any function P of w that is increasing on [0, 1] and takes the midpoint values at those seven
// arguments gives every u its code (P(0) = 0.19 < 0.25: code 0 below the range; P(1) = 43 > 5:
// code 7 above it).  P is the degree-6 polynomial through the seven points (monotone on [0, 1],
// checked on a dense grid), with one change: at u = -2 it takes 0.25 (1 - 2^-20) instead of 0.25,
// so that u = -2 exactly (a score equal to the running max in a group of scale 2^2, whose
// exponential is exactly the tie 0.25 and rounds to 0) stays below the tie whatever the rounding
// of the evaluation; only u within 1.4e-6 above -2 is given code 0 instead of 1 by this.  Every
// other integer u lands on a grid value, far from any midpoint.  The result is a code-exact
// stand-in, not an accurate exponential: use it only in front of the E2M1 conversion.
constexpr float kStandInLo = -2.5f;   // w = (u - kStandInLo) / 8
constexpr float kStandInC0 = 0.19134787f, kStandInC1 = 0.54114223f, kStandInC2 = 7.1855769f,
                kStandInC3 = -17.132305f, kStandInC4 = 66.555229f, kStandInC5 = -78.487640f,
                kStandInC6 = 64.299675f;

__device__ __forceinline__ float2 e2m1_exp2_stand_in(float2 w) {
  float2 p = __ffma2_rn(w, make_float2(kStandInC6, kStandInC6), make_float2(kStandInC5, kStandInC5));
  p = __ffma2_rn(p, w, make_float2(kStandInC4, kStandInC4));
  p = __ffma2_rn(p, w, make_float2(kStandInC3, kStandInC3));
  p = __ffma2_rn(p, w, make_float2(kStandInC2, kStandInC2));
  p = __ffma2_rn(p, w, make_float2(kStandInC1, kStandInC1));
  return __ffma2_rn(p, w, make_float2(kStandInC0, kStandInC0));
}

__device__ __forceinline__ float lg2_approx(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ------------------------------------------------------------------------------------------------
// Shared-scale exponent: the smallest e with amax <= q * 2^e for q = mq * 2^eq (mq in [1,2)),
// i.e. e = E(amax) - eq + [mant(amax) > mant(q)]; the OCP floor rule passes mant_q = 0xFFFFFFFF.
// Exact integer arithmetic on the fp32 bit pattern; clamped to [-127, 127]; amax = 0 -> -127.
// ------------------------------------------------------------------------------------------------
struct ScaleRule {
  int eq;          // binary exponent of the boundary q
  uint32_t mq;     // its 23 mantissa bits (0xFFFFFFFF: never step up -> floor rule)
  float log2q;     // fl32(log2 q) for the ceiling rules (unused by the floor rule)
};

// shared_exponent for amax = 2^t given in the log2 domain: ceil(t - log2 q) for the ceiling
// rules, floor(t) - 2 for the OCP floor rule, clamped to [-127, 127] (exact at t = 0, the group
// holding the running max).  Computed on the FMA pipe alone and returned as an exact float,
// with its E8M0 byte (e + 127).  Adding x to M = 1.5 * 2^23 + 127 with rounding toward +inf
// (ceiling rules) or -inf (floor rule) lands on the integer M + ceil(x) or M + floor(x), in a
// binade whose ulp is 1, so the sum's low mantissa bits are 127 + e.  Clamping x to
// [-127, 127] first (an integer range) clamps e the same way; t = -inf gives -127.
template <bool FLOOR>  // FLOOR: the OCP floor rule; else a ceiling rule with boundary 2^log2q
__device__ __forceinline__ float shared_exponent_log2f_rule(float t, float log2q, uint32_t& byte) {
  constexpr float M = 12582912.f + 127.f;
  float y;
  if (FLOOR) {  // floor(t) - 2: floor t itself (t - 2 could round), M - 2 adds the -2
    y = __fadd_rd(fminf(fmaxf(t, -125.f), 129.f), M - 2.f);
  } else {
    y = __fadd_ru(fminf(fmaxf(t - log2q, -127.f), 127.f), M);
  }
  byte = __float_as_uint(y) & 0xFFu;
  return y - M;
}

__device__ __forceinline__ float shared_exponent_log2f(float t, ScaleRule r, uint32_t& byte) {
  return r.mq == 0xFFFFFFFFu ? shared_exponent_log2f_rule<true>(t, r.log2q, byte)
                             : shared_exponent_log2f_rule<false>(t, r.log2q, byte);
}

__device__ __forceinline__ int shared_exponent(float amax, ScaleRule r) {
  uint32_t b = __float_as_uint(amax) & 0x7FFFFFFFu;
  if (b == 0) return -127;
  int E;
  uint32_t m;
  if (b >= 0x00800000u) {
    E = (int)(b >> 23) - 127;
    m = b & 0x007FFFFFu;
  } else {  // subnormal: value = b * 2^-149
    const int p = 31 - __clz(b);
    E = p - 149;
    m = (b << (23 - p)) & 0x007FFFFFu;
  }
  int e = E - r.eq + (m > r.mq ? 1 : 0);
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

// 2^-e as an fp32 for e in [-127, 126] (a normal number).
__device__ __forceinline__ float pow2_neg(int e) { return __uint_as_float((uint32_t)(127 - e) << 23); }

}  // namespace mxattn
