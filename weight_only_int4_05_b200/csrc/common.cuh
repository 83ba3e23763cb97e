// common.cuh -- device helpers shared by the W4A16 kernels (sm_100a only).
//
// Thin inline-PTX wrappers for the Blackwell features the kernels use: mbarriers with bounded waits,
// TMA bulk and tensor copies, tcgen05 tensor-memory allocation / MMA / loads, programmatic dependent
// launch, and the int4 -> fp16 nibble trick.  Nothing here depends on torch.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "this library targets sm_100a (B200) only"
#endif

namespace awq {

// Status word values written by kernels (read back by awq_last_device_status).
enum : unsigned { kDevOk = 0u, kDevTimeout = 1u };

// Bounded waits give up after this many nanoseconds of %globaltimer.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- programmatic dependent launch
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait_prior_grids() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// Arrivals discard the returned barrier state (sink operand), so the thread does not wait for it.
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Non-blocking test of the phase with the given parity (for polling several barriers in turn).
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Waits for the phase with the given parity to complete.  Gives up after kWaitLimitNs, records a
// timeout in *status and returns false; the caller then abandons its work and exits cleanly.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, unsigned parity, unsigned* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  for (unsigned it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 63u && globaltimer_ns() - t0 > kWaitLimitNs) {
      atomicExch(status, kDevTimeout);
      return false;
    }
  }
}
// The same bounded wait with a short sleep between polls, for warps that share their scheduler with
// working warps (a poll that fails gives its issue slots back).
__device__ __forceinline__ bool mbar_wait_backoff(uint64_t* bar, unsigned parity, unsigned* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  for (unsigned it = 0;; ++it) {
    __nanosleep(64);
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 63u && globaltimer_ns() - t0 > kWaitLimitNs) {
      atomicExch(status, kDevTimeout);
      return false;
    }
  }
}

// ---------------------------------------------------------------- TMA (bulk and tensor copies)
// 1-D bulk copy global -> shared, completion counted on `bar` (bytes and addresses 16-B aligned).
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, unsigned bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
// 2-D tiled tensor copy global -> shared (coordinates: c0 innermost, in elements).
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}
// Fire-and-forget prefetch of `bytes` (multiple of 16, 16-B aligned) of global memory into L2.
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, unsigned bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
// 3-D tiled tensor copy global -> shared.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int c0, int c1, int c2, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}
// Generic-proxy shared-memory writes -> visible to the async proxy (TMA, tcgen05.mma).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- tcgen05 (tensor memory, UMMA)
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, unsigned ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, unsigned ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f16 (fp16 x fp16 -> fp32), one CTA.
__device__ __forceinline__ void umma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive (once) on `bar` when every tcgen05.mma issued so far by this thread has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
// 32 lanes x 32 bits, 16 consecutive columns per thread.
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor for a K-major operand stored in the 128-byte swizzle layout:
// rows of 128 bytes (64 fp16), 8-row atoms of 1024 bytes (stride byte offset), atoms 1024-B aligned.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr & 0x3FFFFu) >> 4);  // start address >> 4, bits 0..13
  d |= (uint64_t)(16u >> 4) << 16;               // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024u >> 4) << 32;             // stride byte offset: next 8-row atom
  d |= (uint64_t)1 << 46;                        // descriptor version for sm_100
  d |= (uint64_t)2 << 61;                        // layout: 128-byte swizzle
  return d;
}
// Instruction descriptor: kind::f16, A = B = fp16, D = fp32, both K-major, M x N tile.
__host__ __device__ constexpr uint32_t umma_idesc_f16(int M, int N) {
  return (1u << 4)                         // D format fp32
         | (0u << 7) | (0u << 10)          // A, B fp16
         | (0u << 15) | (0u << 16)         // A, B K-major
         | ((uint32_t)(N >> 3) << 17)      // N / 8
         | ((uint32_t)(M >> 4) << 24);     // M / 16
}

// Barrier over a subset of the CTA's warps (ids 1..15; `threads` a multiple of 32).
__device__ __forceinline__ void named_barrier_sync(unsigned id, unsigned threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// ---------------------------------------------------------------- warp-level MMA (register fragments)
// D = A . B + C for one 16 x 8 x 16 tile: A 16 x 16 fp16 (row major), B 16 x 8 fp16 (column major), C/D fp32.
// Thread (g = lane / 4, t = lane % 4) holds A rows g and g + 8 at columns {2t, 2t+1} (a0: row g, a1: row
// g + 8) and {2t+8, 2t+9} (a2: row g, a3: row g + 8); B column g at rows {2t, 2t+1} (b0) and {2t+8, 2t+9}
// (b1); C/D rows g (c[0], c[1]) and g + 8 (c[2], c[3]) at columns 2t and 2t + 1.  Products are exact in
// fp32 and accumulate in fp32.
__device__ __forceinline__ void mma_16816_f32(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------- shared-memory loads by 32-bit address
__device__ __forceinline__ uint32_t ld_shared_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint16_t ld_shared_u16(uint32_t addr) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
// Arrive (count 1) on an mbarrier given by its 32-bit shared address.
__device__ __forceinline__ void mbar_arrive_addr(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// ---------------------------------------------------------------- loads
__device__ __forceinline__ uint4 ldg_stream(const void* p) {  // read-once data: skip L1
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ uint4 ldg_cached(const void* p) {  // reused data (activations): keep in L1
  return *reinterpret_cast<const uint4*>(p);  // plain load: the compiler folds offsets into the address
}

// ---------------------------------------------------------------- int4 -> fp16 pairs
// (w & mask) | 0x64006400 puts fp16 1024 in both 16-bit halves with the nibble in the low mantissa
// bits: each half becomes exactly 1024 + code (mask 0x000F000F) or 1024 + 16 * code (mask 0x00F000F0)
// -- the bit trick for int4 -> fp16 described by Kim et al., "Who Says Elephants Can't Run", 2022.
// Written as plain C++ so that the compiler fuses the and/or into one logic op with immediates.
__device__ __forceinline__ __half2 u32_as_h2(uint32_t v) { return *reinterpret_cast<__half2*>(&v); }
__device__ __forceinline__ uint32_t h2_as_u32(__half2 v) { return *reinterpret_cast<uint32_t*>(&v); }

// (w & MASK) | magic in one logic instruction: the mask is an immediate, the magic a register.
template <uint32_t MASK>
__device__ __forceinline__ uint32_t and_or(uint32_t w, uint32_t magic) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(w), "n"(MASK), "r"(magic));
  return d;
}
// fp16 1024 in both halves, as an opaque register value (so the compiler keeps it in a register
// instead of rebuilding the constant for every use).
__device__ __forceinline__ uint32_t magic_1024x2() {
  uint32_t m;
  asm volatile("mov.b32 %0, 0x64006400;" : "=r"(m));
  return m;
}

// The four (code - zero) half2 pairs of one packed word, channel order (0,1) (2,3) (4,5) (6,7).
// z1024 = fp16 (1024 + z) and nz64 = fp16 -(64 + z), each in both halves; magic = magic_1024x2().
// All results are exact small integers.
__device__ __forceinline__ void word_minus_zero(uint32_t w, __half2 z1024, __half2 nz64, uint32_t magic,
                                                __half2 (&d)[4]) {
  const __half2 sixteenth = u32_as_h2(0x2C002C00u);  // fp16 0.0625 in both halves
  const uint32_t t = w >> 8;
  d[0] = __hsub2(u32_as_h2(and_or<0x000F000Fu>(w, magic)), z1024);
  d[1] = __hfma2(u32_as_h2(and_or<0x00F000F0u>(w, magic)), sixteenth, nz64);
  d[2] = __hsub2(u32_as_h2(and_or<0x000F000Fu>(t, magic)), z1024);
  d[3] = __hfma2(u32_as_h2(and_or<0x00F000F0u>(t, magic)), sixteenth, nz64);
}
// fp16 64 in both halves: with the nibble in mantissa bits 4..7 ((w & 0x00F000F0) | 0x54005400) each
// half is exactly 64 + code, since one unit in the last place of 64 is 1/16.
__device__ __forceinline__ uint32_t magic_64x2() {
  uint32_t m;
  asm volatile("mov.b32 %0, 0x54005400;" : "=r"(m));
  return m;
}
// fp16 (64 + z) in both halves, from a zero point 0..15.
__device__ __forceinline__ __half2 zero_64(uint32_t z) { return u32_as_h2((0x5400u | (z << 4)) * 0x00010001u); }

// fp16 (1024 + z) and -(64 + z), splatted into both halves, from a zero point 0..15.
__device__ __forceinline__ __half2 zero_1024(uint32_t z) { return u32_as_h2((0x6400u | z) * 0x00010001u); }
__device__ __forceinline__ __half2 neg_zero_64(uint32_t z) {
  return u32_as_h2((0xD400u | (z << 4)) * 0x00010001u);
}

}  // namespace awq
