// Thin inline-PTX wrappers for the sm_100a features the attention kernels use:
// mbarriers with bounded waits, TMA tile copies (no multicast), and the
// tcgen05 tensor-core / tensor-memory instructions.
//
// Every wait in this library is bounded: after kWaitTimeoutNs of wall time a
// wait gives up, and the caller records an error and unwinds instead of
// spinning forever.
#pragma once

#include <cstdint>
#include <cuda.h>

namespace attn {

constexpr uint64_t kWaitTimeoutNs = 1500ull * 1000ull * 1000ull;  // 1.5 s
constexpr int kErrTimeout = 1;  // error word bit: a bounded wait ran out

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ----------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait with a suspend-time hint: the waiting warp sleeps in hardware until
// the phase completes (or the hint, in ns, runs out) instead of spinning, so
// it takes no issue slots from the warps that share its scheduler.
constexpr uint32_t kWaitHintNs = 1000000;  // 1 ms
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "n"(kWaitHintNs)
      : "memory");
  return ok != 0;
}

// Waits for the phase of parity `parity` to complete.  Returns false if it
// did not complete within kWaitTimeoutNs, or if another role of the CTA has
// already raised `abort_flag` (a shared-memory word).  Each sleeping try_wait
// lasts at most kWaitHintNs, so the flag and the clock are checked at
// least that often.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity,
                                          const volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait_sleep(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > kWaitTimeoutNs) return false;
  }
}

// A global load issued exactly where it is written (volatile: not sunk to its use).
__device__ __forceinline__ float ld_global_f32(const float* p) {
  float v;
  asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(v) : "l"(p));
  return v;
}

// ---------------------------------------------------------------------- TMA
__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// 3-D tiled load into this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_3d(const CUtensorMap* m, uint32_t dst, uint32_t bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// 4-D tile load (paged key/value pools: channel, position, kv head, block).
__device__ __forceinline__ void tma_load_4d(const CUtensorMap* m, uint32_t dst, uint32_t bar,
                                            int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

__device__ __forceinline__ void tma_store_3d(const CUtensorMap* m, uint32_t src, int c0, int c1,
                                             int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(m)),
      "r"(src), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// Contiguous global -> shared copy on the async proxy (untiled bulk copy; both
// addresses 16-byte aligned, size a multiple of 16), completing on `bar`.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst), "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Makes this thread's generic-proxy shared-memory writes visible to TMA.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ------------------------------------------------------------------ tcgen05
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
// Arrives once on `bar` when every tcgen05 operation this thread issued so far
// has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, 16-bit inputs, f32 accumulate.
__device__ __forceinline__ void mma_f16_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                           uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(accum)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]^T, 16-bit inputs, f32 accumulate.
__device__ __forceinline__ void mma_f16_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                           uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(accum)
      : "memory");
}
// D[tmem] (+)= A[smem] * B[smem]^T, signed 8-bit inputs, s32 accumulate.
__device__ __forceinline__ void mma_i8_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                          uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(accum)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]^T, 8-bit float inputs, f32 accumulate.
__device__ __forceinline__ void mma_f8_ts(uint32_t d, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                          uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(accum)
      : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T for MXFP4 operands (E2M1 elements, one E8M0
// scale per 32 along K), K = 64 per instruction; the two scales of a row are
// bytes `id`, id + 1 of its 32-bit cell at sfa / sfb (the id is carried in the
// top two bits of the tensor-memory address).
__device__ __forceinline__ void mma_mxf4_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                            uint32_t sfa, uint32_t sfb, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%4], "
      "[%5], p;\n\t}\n" ::"r"(d),
      "l"(a), "l"(b), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accum)
      : "memory");
}

// Copies 32 rows x 16 bytes from shared memory (descriptor `src`) into 4 columns of
// tensor memory at `taddr`, the same data into each of the four 32-lane quarters
// (the layout of block scale factors for a 128-row operand).
__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t src) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(src)
               : "memory");
}

// Instruction descriptor of the block-scaled kinds: A and B formats (E2M1 = 1 in
// kind::mxf4), N / 8 at bit 17, E8M0 scales (bit 23), M / 16 at bit 24.
__host__ __device__ constexpr uint32_t instr_desc_mx(uint32_t a_fmt, uint32_t b_fmt, uint32_t M,
                                                     uint32_t N) {
  return (a_fmt << 7) | (b_fmt << 10) | ((N >> 3) << 17) | (1u << 23) | ((M >> 4) << 24);
}

// Shared-memory matrix descriptor (Blackwell layout: version 1 in bits 46-47).
// layout: 0 = no swizzle, 2 = 128-byte swizzle, 4 = 64-byte swizzle.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(layout & 7u) << 61;
  return d;
}

// The same descriptor as two 32-bit words, so that per-MMA offsets are one add:
// lo = start address >> 4 | (LBO >> 4) << 16,  hi = SBO >> 4 | version 1 | layout.
__host__ __device__ constexpr uint32_t desc_lo(uint32_t saddr, uint32_t lbo) {
  return ((saddr >> 4) & 0x3FFFu) | (((lbo >> 4) & 0x3FFFu) << 16);
}
__host__ __device__ constexpr uint32_t desc_hi(uint32_t sbo, uint32_t layout) {
  return ((sbo >> 4) & 0x3FFFu) | (1u << 14) | ((layout & 7u) << 29);
}
__device__ __forceinline__ uint64_t desc_pack(uint32_t lo, uint32_t hi) {
  uint64_t d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "r"(lo), "r"(hi));
  return d;
}

// Instruction descriptor (dense).  c_fmt: 1 = f32, 2 = s32.  a/b_fmt: for
// kind::f16 0 = f16, 1 = bf16; for kind::i8 1 = signed; for kind::f8f6f4
// 0 = e4m3.  major: 0 = K-major, 1 = MN-major.
__host__ __device__ constexpr uint32_t instr_desc(uint32_t c_fmt, uint32_t a_fmt, uint32_t b_fmt,
                                                  uint32_t a_major, uint32_t b_major, uint32_t M,
                                                  uint32_t N) {
  return (c_fmt << 4) | (a_fmt << 7) | (b_fmt << 10) | (a_major << 15) | (b_major << 16) |
         ((N >> 3) << 17) | ((M >> 4) << 24);
}

// ---- tensor memory loads/stores: 32 lanes x 32-bit, 32 consecutive columns.
#define ATTN_R32(i) "=r"(r[i])
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : ATTN_R32(0), ATTN_R32(1), ATTN_R32(2), ATTN_R32(3), ATTN_R32(4), ATTN_R32(5), ATTN_R32(6),
        ATTN_R32(7), ATTN_R32(8), ATTN_R32(9), ATTN_R32(10), ATTN_R32(11), ATTN_R32(12),
        ATTN_R32(13), ATTN_R32(14), ATTN_R32(15), ATTN_R32(16), ATTN_R32(17), ATTN_R32(18),
        ATTN_R32(19), ATTN_R32(20), ATTN_R32(21), ATTN_R32(22), ATTN_R32(23), ATTN_R32(24),
        ATTN_R32(25), ATTN_R32(26), ATTN_R32(27), ATTN_R32(28), ATTN_R32(29), ATTN_R32(30),
        ATTN_R32(31)
      : "r"(taddr));
}
#undef ATTN_R32

// Waits for this thread's tensor-memory loads; the registers are passed
// through so that no use of them can be scheduled before the wait.
#define ATTN_RW(i) "+r"(r[i])
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : ATTN_RW(0), ATTN_RW(1), ATTN_RW(2), ATTN_RW(3), ATTN_RW(4), ATTN_RW(5), ATTN_RW(6),
                 ATTN_RW(7), ATTN_RW(8), ATTN_RW(9), ATTN_RW(10), ATTN_RW(11), ATTN_RW(12),
                 ATTN_RW(13), ATTN_RW(14), ATTN_RW(15), ATTN_RW(16), ATTN_RW(17), ATTN_RW(18),
                 ATTN_RW(19), ATTN_RW(20), ATTN_RW(21), ATTN_RW(22), ATTN_RW(23), ATTN_RW(24),
                 ATTN_RW(25), ATTN_RW(26), ATTN_RW(27), ATTN_RW(28), ATTN_RW(29), ATTN_RW(30),
                 ATTN_RW(31)
               :
               : "memory");
}
#undef ATTN_RW

#define ATTN_RI(i) "r"(r[i])
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      ATTN_RI(0), ATTN_RI(1), ATTN_RI(2), ATTN_RI(3), ATTN_RI(4), ATTN_RI(5), ATTN_RI(6),
      ATTN_RI(7), ATTN_RI(8), ATTN_RI(9), ATTN_RI(10), ATTN_RI(11), ATTN_RI(12), ATTN_RI(13),
      ATTN_RI(14), ATTN_RI(15), ATTN_RI(16), ATTN_RI(17), ATTN_RI(18), ATTN_RI(19), ATTN_RI(20),
      ATTN_RI(21), ATTN_RI(22), ATTN_RI(23), ATTN_RI(24), ATTN_RI(25), ATTN_RI(26), ATTN_RI(27),
      ATTN_RI(28), ATTN_RI(29), ATTN_RI(30), ATTN_RI(31)
      : "memory");
}
#undef ATTN_RI

#define ATTN_RI(i) "r"(r[i])
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      ATTN_RI(0), ATTN_RI(1), ATTN_RI(2), ATTN_RI(3), ATTN_RI(4), ATTN_RI(5), ATTN_RI(6),
      ATTN_RI(7), ATTN_RI(8), ATTN_RI(9), ATTN_RI(10), ATTN_RI(11), ATTN_RI(12), ATTN_RI(13),
      ATTN_RI(14), ATTN_RI(15)
      : "memory");
}
#undef ATTN_RI

#define ATTN_RI(i) "r"(r[i])
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
               ATTN_RI(0), ATTN_RI(1), ATTN_RI(2), ATTN_RI(3), ATTN_RI(4), ATTN_RI(5), ATTN_RI(6),
               ATTN_RI(7)
               : "memory");
}
#undef ATTN_RI

__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Per-warpgroup register budget changes (all warps of a warpgroup execute them).
template <int N>
__device__ __forceinline__ void regs_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <int N>
__device__ __forceinline__ void regs_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// ------------------------------------------------------------- arithmetic
// Hardware base-2 exponential (MUFU); flushes subnormal results to zero.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Packed float32 pairs (Blackwell f32x2 FMA / add: two lanes per instruction).
struct f32x2 {
  float x, y;
};
__device__ __forceinline__ f32x2 ffma2(f32x2 a, f32x2 b, f32x2 c) {
  uint64_t ra, rb, rc, rd;
  f32x2 d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(ra) : "f"(a.x), "f"(a.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(rb) : "f"(b.x), "f"(b.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(rc) : "f"(c.x), "f"(c.y));
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(rd) : "l"(ra), "l"(rb), "l"(rc));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(d.x), "=f"(d.y) : "l"(rd));
  return d;
}
__device__ __forceinline__ f32x2 fmul2(f32x2 a, f32x2 b) {
  uint64_t ra, rb, rd;
  f32x2 d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(ra) : "f"(a.x), "f"(a.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(rb) : "f"(b.x), "f"(b.y));
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(rd) : "l"(ra), "l"(rb));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(d.x), "=f"(d.y) : "l"(rd));
  return d;
}
__device__ __forceinline__ f32x2 fadd2(f32x2 a, f32x2 b) {
  uint64_t ra, rb, rd;
  f32x2 d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(ra) : "f"(a.x), "f"(a.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(rb) : "f"(b.x), "f"(b.y));
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(rd) : "l"(ra), "l"(rb));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(d.x), "=f"(d.y) : "l"(rd));
  return d;
}

__device__ __forceinline__ f32x2 fsub2(f32x2 a, f32x2 b) {
  uint64_t ra, rb, rd;
  f32x2 d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(ra) : "f"(a.x), "f"(a.y));
  asm("mov.b64 %0, {%1, %2};" : "=l"(rb) : "f"(b.x), "f"(b.y));
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(rd) : "l"(ra), "l"(rb));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(d.x), "=f"(d.y) : "l"(rd));
  return d;
}

// 2^x for a pair of arguments on the FMA pipe (keeps the MUFU free for the
// other exponentials).  Cody-Waite style range reduction x = n + f with
// n = round-to-nearest(x) through the 1.5*2^23 addition and f in [-1/2, 1/2];
// 2^f from a degree-3 polynomial fitted to minimise the maximum relative error
// on that interval (fit in float64, coefficients rounded to float32: max
// relative error 7.5e-5, about 13.7 bits, enough for the 16-bit and 8-bit P it
// feeds); 2^n is added to the exponent field.  Arguments are clamped to -125
// (so the result stays a normal float); callers only use this where no score
// is masked.  Packed float32 pairs: one instruction serves both lanes.
__device__ __forceinline__ f32x2 poly_ex2x2(f32x2 x) {
  x.x = fmaxf(x.x, -125.0f);
  x.y = fmaxf(x.y, -125.0f);
  const f32x2 big{12582912.0f, 12582912.0f};  // 1.5 * 2^23
  const f32x2 r = fadd2(x, big);              // x rounded to an integer in the low bits
  const f32x2 f = fsub2(x, fsub2(r, big));
  f32x2 p = ffma2(f32x2{0.05517113208770752f, 0.05517113208770752f}, f,
                  f32x2{0.24261008203029633f, 0.24261008203029633f});
  p = ffma2(p, f, f32x2{0.6932609677314758f, 0.6932609677314758f});
  p = ffma2(p, f, f32x2{0.9999281167984009f, 0.9999281167984009f});
  return f32x2{__int_as_float(__float_as_int(p.x) + (__float_as_int(r.x) << 23)),
               __int_as_float(__float_as_int(p.y) + (__float_as_int(r.y) << 23))};
}
__device__ __forceinline__ float poly_ex2(float x) { return poly_ex2x2(f32x2{x, x}).x; }

// acc_lo + (low 16-bit value of w), acc_hi + (high 16-bit value of w), for a
// pair of bf16 (or f16) values packed in one word: mixed-precision adds with a
// 16-bit operand and a float32 accumulator (exact widening, one rounding).
template <bool F16>
__device__ __forceinline__ void add_16x2(uint32_t w, float& acc_lo, float& acc_hi) {
  if constexpr (F16)
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
        "add.rn.f32.f16 %0, lo, %0;\n\tadd.rn.f32.f16 %1, hi, %1;\n\t}"
        : "+f"(acc_lo), "+f"(acc_hi) : "r"(w));
  else
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
        "add.rn.f32.bf16 %0, lo, %0;\n\tadd.rn.f32.bf16 %1, hi, %1;\n\t}"
        : "+f"(acc_lo), "+f"(acc_hi) : "r"(w));
}

// Two floats -> packed e4m3 pair, `lo` in the low byte (round to nearest even,
// saturating to +-448).
__device__ __forceinline__ uint16_t f32x2_to_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

}  // namespace attn
