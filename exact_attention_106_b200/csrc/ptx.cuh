// Thin inline-PTX layer for sm_100a: mbarriers with time-bounded waits, TMA
// tile loads, and the tcgen05 tensor-core / tensor-memory instructions.
//
// Every wait in this library goes through mbar_wait(): it polls the barrier,
// and after `timeout_ns` of %globaltimer it records EXATTN_STATUS_TIMEOUT in
// the device status word, raises the CTA-wide abort flag and returns false, so
// that every role leaves its loop and the kernel ends.  Nothing spins forever.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

namespace exattn {

// Device status word (read and cleared by attn_get_device_status()).
__device__ unsigned int g_status_word;
// Diagnostic: which wait site timed out first (0 = none).
__device__ unsigned int g_status_site;

enum : unsigned int {
  kDevStatusTimeout = 1u,
  kDevStatusBadSmemAlign = 2u,
};

// Fault injection (see attn_debug_inject_stall): the producer skips its first
// K/V load, so a consumer waits on a barrier that nothing will complete.
enum : unsigned int { kDebugSkipFirstKV = 1u };

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void record_status(unsigned int bits, unsigned int site) {
  atomicOr(&g_status_word, bits);
  atomicCAS(&g_status_site, 0u, site);
}

// ----------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

// One poll.  The suspend-time hint (in ns) lets the hardware park the thread
// until the phase completes instead of returning at once: waiting threads then
// neither spin on shared memory nor take issue slots from the working warps.
constexpr uint32_t kSuspendHintNs = 20000;
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar_addr, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar_addr), "r"(parity), "r"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}

// Wait until the phase with parity `parity` of `bar` has completed.
// Returns false (after recording a timeout) if it did not within timeout_ns,
// or if another role of this CTA has already given up (abort flag set).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          uint64_t timeout_ns, unsigned int site) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  // try_wait itself may suspend the thread for a while, so the clock and the
  // abort flag are checked after every poll.
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    if (mbar_try_wait(a, parity)) return true;
    if (*abort_flag) return false;
    if (global_timer_ns() - t0 > timeout_ns) {
      record_status(kDevStatusTimeout, site);
      *abort_flag = 1;
      return false;
    }
  }
}

// Bounded wait (0.2 s) for the error path: lets copies or MMAs already in
// flight finish before the CTA exits; ignores the abort flag.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, unsigned int site) {
  int dummy = 0;
  mbar_wait(bar, parity, &dummy, 200000000ull, site);
}

// --------------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int x,
                                            int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// Plain (untiled) bulk copy global -> shared; both addresses 16-byte aligned,
// bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Element-wise add of a shared-memory tile into global memory through a
// tensor map (fp32 add done by the TMA engine at L2); completion is tracked
// with bulk groups: commit, then wait until the source may be reused (.read)
// or until the writes are done.
__device__ __forceinline__ void tma_reduce_add_2d(const void* smem_src, const CUtensorMap* map, int x, int y) {
  asm volatile(
      "cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(smem_src)), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_group_read0() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_group0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (tcgen05.mma operand reads, TMA stores).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ----------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive (count 1) on `bar` once all tcgen05 async ops issued so far by this
// thread have completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// The MMAs below carry no "memory" clobber: they touch no memory the compiler
// tracks, and keeping the issuing thread's values in registers between them
// matters (one thread issues every MMA of the CTA).  They stay ordered with the
// other asm volatile statements (barrier waits, commits, fences).
// D(tmem) = A(smem) * B(smem) (+ D if accumulate)
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

// D(tmem) = A(tmem) * B(smem) (+ D if accumulate)
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate));
}

// The same two forms for kind::f8f6f4 (8-bit A and B, fp32 accumulate).
// The four zero words are the disable-output-lane mask (no lane disabled).
__device__ __forceinline__ void mma_ss_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0u));
}
__device__ __forceinline__ void mma_ts_f8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, {%5, %5, %5, %5}, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0u));
}

// Instruction descriptor with fp32 accumulate.  kind::f16: A/B format 0 =
// fp16, 1 = bf16 (both operands of one MMA have the same type); kind::f8f6f4:
// format 0 = e4m3.  a_mn / b_mn: 0 = K-major operand, 1 = MN-major operand
// (MN-major is allowed for the 16-bit and the 8-bit e4m3/e5m2 formats).
__host__ __device__ constexpr uint32_t idesc_16_f32(uint32_t ab_fmt, int M, int N, int a_mn, int b_mn) {
  return (1u << 4)                          // D format: f32
         | (ab_fmt << 7)                    // A format
         | (ab_fmt << 10)                   // B format
         | (uint32_t(a_mn) << 15)           // A major
         | (uint32_t(b_mn) << 16)           // B major
         | (uint32_t(N >> 3) << 17)         // N / 8
         | (uint32_t(M >> 4) << 24);        // M / 16
}

// Shared-memory matrix descriptor, 128-byte swizzle (layout type 2),
// descriptor version 1.  Addresses and offsets in bytes.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t smem_addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  return uint64_t((smem_addr >> 4) & 0x3FFFu) | (uint64_t((lbo_bytes >> 4) & 0x3FFFu) << 16) |
         (uint64_t((sbo_bytes >> 4) & 0x3FFFu) << 32) | (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

// A descriptor split in two words.  Only the 14-bit start address (low word)
// changes between the MMAs of a tile, so the issuing thread advances it with
// one 32-bit add per operand instead of rebuilding 64 bits: with one thread
// issuing every MMA, that per-instruction cost bounds the tensor-core rate.
struct SmemDesc {
  uint32_t lo, hi;
};
__device__ __forceinline__ SmemDesc make_desc_sw128(uint32_t smem_addr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  const uint64_t d = smem_desc_sw128(smem_addr, lbo_bytes, sbo_bytes);
  return SmemDesc{static_cast<uint32_t>(d), static_cast<uint32_t>(d >> 32)};
}
// The descriptor of the same layout starting `bytes` further (a multiple of
// 16; the address stays below 256 KB, so the 14-bit field cannot overflow).
__device__ __forceinline__ uint64_t desc_at(SmemDesc d, uint32_t bytes) {
  return (static_cast<uint64_t>(d.hi) << 32) | static_cast<uint64_t>(d.lo + (bytes >> 4));
}

// 32 lanes x 32 columns of 32-bit: thread i of the warp gets lane (base lane
// + i), columns [col, col+32).
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
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
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

// Register rebalancing between warpgroups (sm_90a+).  Every warp of a
// warpgroup executes the same instruction.  .inc draws only on registers that
// other warpgroups of the CTA released with .dec, so a split is safe only if
// the increases sum to no more than the decreases (checked on the host
// against the compiled register count before launch).
template <uint32_t R>
__device__ __forceinline__ void setmaxnreg_inc() {
  static_assert(R % 8 == 0 && R >= 24 && R <= 256, "setmaxnreg operand");
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(R));
}
template <uint32_t R>
__device__ __forceinline__ void setmaxnreg_dec() {
  static_assert(R % 8 == 0 && R >= 24 && R <= 256, "setmaxnreg operand");
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(R));
}

// 16-lane fragment shapes (the lane field of taddr selects the first of the 16
// lanes).  16x256b.x8: thread t holds, for column group g = 0..7, the four
// words r[4g..4g+3] = (lane t/4, col 8g+2(t%4)), (lane t/4, col 8g+2(t%4)+1),
// (lane t/4+8, col 8g+2(t%4)), (lane t/4+8, col 8g+2(t%4)+1).
__device__ __forceinline__ void tmem_ld16x256_x8(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x8.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

// 16x128b.x8: thread t writes, for column group g = 0..7, r[2g] to
// (lane t/4, col 4g + t%4) and r[2g+1] to (lane t/4+8, col 4g + t%4).
__device__ __forceinline__ void tmem_st16x128_x8(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x128b.x8.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// Two 8x8 b16 matrices to shared memory: lanes 0-7 give the row addresses of
// matrix 0, lanes 8-15 those of matrix 1; thread t supplies (row t/4, columns
// 2(t%4), 2(t%4)+1) of matrix 0 in r0 and of matrix 1 in r1.
__device__ __forceinline__ void stmatrix_x2(uint32_t saddr, uint32_t r0, uint32_t r1) {
  asm volatile("stmatrix.sync.aligned.m8n8.x2.shared.b16 [%0], {%1, %2};" ::"r"(saddr), "r"(r0), "r"(r1)
               : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// --------------------------------------------------------------- math bits
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ------------------------------------------------- packed fp32 pairs (sm_100)
// Two fp32 values in one 64-bit register pair; one instruction operates on
// both, halving the issue cost of the softmax's scale, sum and polynomial.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
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
__device__ __forceinline__ uint64_t f2_add_rm(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rm.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_sub(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^x on the FMA pipe instead of the special-function unit:
// 2^x = 2^n * p(f), n = floor(x), f = x - n in [0, 1), with p the degree-3
// minimax (relative error) polynomial for 2^f with p(0) = 1, p(1) = 2, fitted
// by csrc/gen_exp2_poly.py (max relative error 1.03e-4 in fp32).  floor(x)
// comes from adding 1.5 * 2^23 with round-down; the exponent is added to p's
// bits as an integer.  x is clamped to -127, where the result is exactly 0.
__device__ __forceinline__ float ex2_fma(float x) {
  x = fmaxf(x, -127.0f);
  const float r = __fadd_rd(x, 12582912.0f);  // 1.5 * 2^23 + floor(x), exactly
  const float f = x - (r - 12582912.0f);
  const float p = fmaf(fmaf(fmaf(0.07826796919107437f, f, 0.226307675242424f), f, 0.6954243183135986f), f, 1.0f);
  // low bits of r hold floor(x) (offset by 2^22, which shifts out)
  return __int_as_float(__float_as_int(p) + (__float_as_int(r) << 23));
}

// ex2_fma on a packed pair (same arithmetic, half the instructions).
__device__ __forceinline__ uint64_t ex2_fma2(uint64_t x) {
  float x0, x1;
  f2_unpack(x, x0, x1);
  x = f2_pack(fmaxf(x0, -127.0f), fmaxf(x1, -127.0f));
  const uint64_t magic = f2_pack(12582912.0f, 12582912.0f);
  const uint64_t r = f2_add_rm(x, magic);
  const uint64_t f = f2_sub(x, f2_sub(r, magic));
  uint64_t q = f2_fma(f2_pack(0.07826796919107437f, 0.07826796919107437f), f,
                      f2_pack(0.226307675242424f, 0.226307675242424f));
  q = f2_fma(q, f, f2_pack(0.6954243183135986f, 0.6954243183135986f));
  q = f2_fma(q, f, f2_pack(1.0f, 1.0f));
  float q0, q1, r0, r1;
  f2_unpack(q, q0, q1);
  f2_unpack(r, r0, r1);
  return f2_pack(__int_as_float(__float_as_int(q0) + (__float_as_int(r0) << 23)),
                 __int_as_float(__float_as_int(q1) + (__float_as_int(r1) << 23)));
}

// Maps a linear CTA index to (tile rank, head) so that the CTAs in flight
// cover only a few heads at a time (their K/V, Q/dO and dQ rows then stay in
// L2), and so that inside each group of `group` heads the heaviest tiles
// (rank 0) start first.
__device__ __forceinline__ void grouped_order(int bid, int ntile, int BH, int group, int& rank, int& bh) {
  const int full = BH / group;
  const int per_group = group * ntile;
  int g = bid / per_group;
  int gsz = group;
  int rem = bid - g * per_group;
  if (g >= full) {  // trailing group with fewer heads
    g = full;
    gsz = BH - full * group;
    rem = bid - full * per_group;
  }
  rank = rem / gsz;
  bh = g * group + rem % gsz;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // .x (low 16 bits) = lo
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);  // .x (low 16 bits) = lo
  return *reinterpret_cast<uint32_t*>(&h);
}

// The 16-bit input/output element types: bf16 (the default) and fp16.  The
// kernels are written once; this gives the tensor-core operand format, the
// round-to-nearest-even packing of two fp32 values, and the widening of a
// packed pair.
template <typename T>
struct Elem;
template <>
struct Elem<__nv_bfloat16> {
  using Out = __nv_bfloat16;  // output element type of a forward on this input type
  static constexpr bool kF8 = false;
  static constexpr uint32_t kMmaFmt = 1;
  __device__ static __forceinline__ uint32_t pack2(float lo, float hi) { return pack_bf16x2(lo, hi); }
  __device__ static __forceinline__ float2 unpack2(uint32_t w) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w));
  }
};
template <>
struct Elem<__half> {
  using Out = __half;
  static constexpr bool kF8 = false;
  static constexpr uint32_t kMmaFmt = 0;
  __device__ static __forceinline__ uint32_t pack2(float lo, float hi) { return pack_f16x2(lo, hi); }
  __device__ static __forceinline__ float2 unpack2(uint32_t w) {
    return __half22float2(*reinterpret_cast<const __half2*>(&w));
  }
};
// e4m3 inputs (a forward only): kind::f8f6f4 operands, bf16 outputs.  pack4
// rounds four fp32 values to nearest e4m3 (saturating at +-448), the first
// in the lowest byte: four consecutive keys in one 32-bit TMEM column.
template <>
struct Elem<__nv_fp8_e4m3> {
  using Out = __nv_bfloat16;
  static constexpr bool kF8 = true;
  static constexpr uint32_t kMmaFmt = 0;
  __device__ static __forceinline__ uint32_t pack4(float a, float b, float c, float d) {
    const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
    const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
    return lo | (hi << 16);
  }
};

}  // namespace exattn
