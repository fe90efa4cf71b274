// Device helpers shared by the sm_100a kernels of the W4A16 MoE layer:
// bf16 bit tricks, mbarriers with bounded waits, TMA and cp.async copies,
// and thin wrappers over the tcgen05 (5th-generation tensor core) PTX.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define MOE_DEV __device__ __forceinline__

namespace moe {

// --------------------------------------------------------------------------
// status word shared with the host (lives in the caller's workspace)
// --------------------------------------------------------------------------
constexpr uint32_t kStatusTimeout = 1u;

// Bounded waits give up after this many nanoseconds of device time.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

MOE_DEV uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// --------------------------------------------------------------------------
// bf16 helpers
// --------------------------------------------------------------------------
MOE_DEV float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
MOE_DEV float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
MOE_DEV float bf16_to_f32(uint16_t v) { return __uint_as_float(uint32_t(v) << 16); }
MOE_DEV uint16_t f32_to_bf16_rn(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}
// two fp32 -> packed bf16x2 (lo = a), round to nearest even
MOE_DEV uint32_t pack_bf16x2(float a, float b) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
  return r;
}
MOE_DEV uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
  __nv_bfloat162 r = __hsub2(*reinterpret_cast<__nv_bfloat162*>(&a), *reinterpret_cast<__nv_bfloat162*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}
MOE_DEV uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  __nv_bfloat162 r = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&a), *reinterpret_cast<__nv_bfloat162*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}
MOE_DEV uint32_t lop3_and_or(uint32_t a, uint32_t mask, uint32_t magic) {
  // (a & mask) | magic in one instruction
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "r"(mask), "r"(magic));
  return r;
}
MOE_DEV uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

// INT4 offset-binary nibbles -> bf16 pairs.  For a 32-bit word holding 8
// nibbles u0..u7 (u0 lowest), int4_pairs(w, i) returns bf16x2 (u_i - 8,
// u_{i+4} - 8) for i in 0..3: OR-ing a nibble into the mantissa of bf16 128.0
// (0x4300) gives exactly 128 + u; subtracting 136 leaves u - 8 exactly.
MOE_DEV uint32_t int4_pair(uint32_t w, int i) {
  const uint32_t v = lop3_and_or(w >> (4 * i), 0x000F000Fu, 0x43004300u);
  return bf16x2_sub(v, 0x43084308u);
}

MOE_DEV uint32_t bf16x2_fma(uint32_t a, uint32_t b, uint32_t c) {
  __nv_bfloat162 r = __hfma2(*reinterpret_cast<__nv_bfloat162*>(&a), *reinterpret_cast<__nv_bfloat162*>(&b),
                             *reinterpret_cast<__nv_bfloat162*>(&c));
  return *reinterpret_cast<uint32_t*>(&r);
}

// E4M3 (fn) scale byte, sign bit ignored -> its fp32 value (exact): 4
// exponent bits with bias 7, 3 mantissa bits, subnormals m * 2^-9.
MOE_DEV float e4m3_to_f32(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  return e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : float(m) * 0.001953125f;
}

// NVFP4 block multiplier as bf16 bits: bf16_rne(fp32(e4m3(byte) * g)).
MOE_DEV uint32_t nv_mult_bits(uint32_t scale_byte, float g) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(e4m3_to_f32(scale_byte), g)));
}

// Multipliers of two adjacent NVFP4 blocks (scale bytes p[0], p[1]; p even)
// as bf16x2 pairs with both halves equal: the hardware E4M3 -> f16
// conversion is exact, f16 -> fp32 too, so this equals nv_mult_bits.
MOE_DEV void nv_mult_pair(const uint8_t* p, float g, uint32_t& m0, uint32_t& m1) {
  const uint16_t two = *reinterpret_cast<const uint16_t*>(p);
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(two));
  const float f0 = __half2float(__ushort_as_half(uint16_t(h2 & 0xFFFFu)));
  const float f1 = __half2float(__ushort_as_half(uint16_t(h2 >> 16)));
  const float v0 = __fmul_rn(f0, g), v1 = __fmul_rn(f1, g);
  asm("cvt.rn.bf16x2.f32 %0, %1, %1;" : "=r"(m0) : "f"(v0));
  asm("cvt.rn.bf16x2.f32 %0, %1, %1;" : "=r"(m1) : "f"(v1));
}

// E2M1 nibbles i and i+4 of `w` -> bf16x2 bit patterns of (value * 2^-126),
// exact: the magnitude code's three bits land on bf16 bits [8:6] (the two low
// exponent bits and the first mantissa bit, so code 1 = 0.5 becomes the
// subnormal 2^-127 and code (e, m) with e >= 1 the normal 2^(e-127) (1 + m/2)),
// the sign bit on bit 15.  One bf16 multiply by (multiplier * 2^126) then
// yields bf16(value * multiplier) with a single rounding.
MOE_DEV uint32_t e2m1_pair_scaled(uint32_t w, int i) {
  const uint32_t t = w >> (4 * i);
  return ((t << 6) & 0x01C001C0u) | ((t << 12) & 0x80008000u);
}
constexpr uint32_t kBf16x2Pow126 = 0x7E807E80u;  // 2^126 in both halves

// Like nv_mult_pair, but the multipliers come pre-scaled by 2^126 for
// e2m1_pair_scaled codes (two = 0) whenever that is exact: both fp32 products
// within [2^-126, 3.9), i.e. the bf16 rounding is in the normal range and the
// scaled value stays finite; otherwise the plain multipliers (two = 1, and
// the caller first multiplies the codes by 2^126).
MOE_DEV void nv_mult_pair_scaled_v(uint16_t pair, float g, uint32_t& m0, uint32_t& m1, uint32_t& two) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(pair));
  const float v0 = __fmul_rn(__half2float(__ushort_as_half(uint16_t(h2 & 0xFFFFu))), g);
  const float v1 = __fmul_rn(__half2float(__ushort_as_half(uint16_t(h2 >> 16))), g);
  const bool fold = v0 >= 0x1p-126f && v0 < 3.9f && v1 >= 0x1p-126f && v1 < 3.9f;
  const float sc = fold ? 0x1p126f : 1.0f;
  const float a = __fmul_rn(v0, sc), b = __fmul_rn(v1, sc);
  asm("cvt.rn.bf16x2.f32 %0, %1, %1;" : "=r"(m0) : "f"(a));
  asm("cvt.rn.bf16x2.f32 %0, %1, %1;" : "=r"(m1) : "f"(b));
  two = fold ? 0u : 1u;
}
MOE_DEV void nv_mult_pair_scaled(const uint8_t* p, float g, uint32_t& m0, uint32_t& m1, uint32_t& two) {
  nv_mult_pair_scaled_v(*reinterpret_cast<const uint16_t*>(p), g, m0, m1, two);
}

// --------------------------------------------------------------------------
// shared-memory addresses, fences
// --------------------------------------------------------------------------
MOE_DEV uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
MOE_DEV void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// --------------------------------------------------------------------------
// mbarriers
// --------------------------------------------------------------------------
MOE_DEV void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
MOE_DEV void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
MOE_DEV void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
MOE_DEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
MOE_DEV bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// try_wait with a suspend-time hint: a thread whose phase has not completed
// sleeps (issues nothing) until the phase completes or about `ns` pass, so a
// waiting warp leaves the issue slots to the warps doing work.
MOE_DEV bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t ns) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
      : "memory");
  return ok != 0;
}
constexpr uint32_t kSuspendNs = 20000;  // longest sleep per try: 20 us

// Wait for the phase of `bar` with the given parity.  Gives up (returns
// false) once `abort` is raised by another thread of the CTA or after
// kWaitLimitNs, in which case it raises `abort` and the global status word.
MOE_DEV bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort, uint32_t* gstatus) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity, kSuspendNs)) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      *abort = 1;
      if (gstatus) atomicOr(gstatus, kStatusTimeout);
      return false;
    }
  }
}

// mbar_wait for a thread off the critical path (a warp that waits for a whole
// tile, or a producer ahead of its consumers): between tries it sleeps about
// sleep_ns, so a long wait costs a few instructions per sleep instead of a
// stream of polls that would take issue slots from the warps doing work.
MOE_DEV bool mbar_wait_backoff(uint64_t* bar, uint32_t parity, volatile int* abort, uint32_t* gstatus,
                               uint32_t sleep_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    __nanosleep(sleep_ns);
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      *abort = 1;
      if (gstatus) atomicOr(gstatus, kStatusTimeout);
      return false;
    }
  }
}

// Wait for the phase of `bar` with the given parity, ignoring any abort flag;
// gives up (false) after limit_ns.  Used to drain copies still in flight.
MOE_DEV bool mbar_wait_drain(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait_sleep(bar, parity, kSuspendNs)) {
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
  return true;
}

// --------------------------------------------------------------------------
// device-wide counters (CTAs of one cooperative grid waiting on each other)
// --------------------------------------------------------------------------
MOE_DEV uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
MOE_DEV uint32_t ld_relaxed_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Spin until *ctr >= target (acquire).  Gives up (returns false) when `abort`
// is raised, when another CTA has already reported a timeout in the status
// word, or after kWaitLimitNs, in which case it raises both.
MOE_DEV bool spin_until_geq(const uint32_t* ctr, uint32_t target, volatile int* abort, uint32_t* gstatus) {
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (ld_acquire_gpu(ctr) >= target) return true;
    if (*abort) return false;
    if (ld_relaxed_gpu(gstatus) & kStatusTimeout) {
      *abort = 1;
      return false;
    }
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      *abort = 1;
      atomicOr(gstatus, kStatusTimeout);
      return false;
    }
    __nanosleep(32);
  }
}

// --------------------------------------------------------------------------
// TMA (tensor memory accelerator) and cp.async
// --------------------------------------------------------------------------
MOE_DEV void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
// 2-D tiled load of the box at (x, y) into shared memory; completion is
// signalled on `bar` as transaction bytes.  x must be 16-byte aligned in bytes.
MOE_DEV void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}
MOE_DEV void cp_async_16(uint32_t smem_dst, const void* gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_dst), "l"(gsrc) : "memory");
}
MOE_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Arrive on `bar` once every cp.async this thread issued so far has landed
// (the arrival is one of the barrier's expected arrivals: .noinc).
MOE_DEV void cp_async_mbar_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
template <int N>
MOE_DEV void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// 1-D bulk copy global -> shared (size and both addresses multiples of 16 B);
// completion is signalled on `bar` as transaction bytes.
MOE_DEV void bulk_g2s(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// L2 cache policy for data read once per launch (streamed expert weights):
// evicted first, so the stream does not push out kernel code, router weights
// and small activations that every launch reuses.
MOE_DEV uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// bulk_g2s with an L2 cache policy (see l2_policy_evict_first).
MOE_DEV void bulk_g2s_hint(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::
          "r"(smem_u32(smem_dst)),
      "l"(gsrc), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Prefetch `bytes` of global memory into L2 (address 16-byte aligned, bytes a
// multiple of 16): a later bulk copy of the range then reads L2, not HBM.
MOE_DEV void bulk_prefetch_l2(const void* gsrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(gsrc), "r"(bytes) : "memory");
}

// Element-wise fp32 add of `bytes` of shared memory into global memory
// (performed at L2; both addresses 16-byte aligned, bytes a multiple of 16),
// tracked by the issuing thread's bulk async-group.
MOE_DEV void bulk_reduce_add_f32(float* gdst, const void* ssrc, uint32_t bytes) {
  asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(gdst),
               "r"(smem_u32(ssrc)), "r"(bytes)
               : "memory");
}
// Copy `bytes` of shared memory to global memory (both addresses 16-byte
// aligned, bytes a multiple of 16), tracked by the thread's bulk async-group.
MOE_DEV void bulk_s2g(void* gdst, const void* ssrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(smem_u32(ssrc)),
               "r"(bytes)
               : "memory");
}
MOE_DEV void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until every bulk operation this thread committed has finished reading
// its shared-memory source.
MOE_DEV void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// Wait until every bulk operation this thread committed has completed.
MOE_DEV void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// --------------------------------------------------------------------------
// programmatic dependent launch: wait for the preceding kernel's results /
// allow the next kernel in the stream to start launching
// --------------------------------------------------------------------------
MOE_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Barrier among `count` threads of the CTA on hardware barrier `id` (1..15).
MOE_DEV void named_barrier_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
MOE_DEV void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// --------------------------------------------------------------------------
// tcgen05: tensor memory allocation, MMA, commit, loads
// --------------------------------------------------------------------------
MOE_DEV void tmem_alloc(uint32_t* smem_result, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_result)),
               "r"(ncols)
               : "memory");
}
MOE_DEV void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
MOE_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
MOE_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
MOE_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem] * B[smem]^T, both K-major, kind::f16 (bf16 in, fp32 acc)
MOE_DEV void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on `bar` once every previously issued tcgen05.mma of this thread completes.
MOE_DEV void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// Instruction descriptor of kind::f16: fp32 accumulator, bf16 A and B, both
// K-major, shape M x N (M = 128 here, N a multiple of 16 in [16, 256]).
MOE_DEV uint32_t umma_idesc_bf16(uint32_t M, uint32_t N) {
  return (1u << 4)            // D format: f32
         | (1u << 7)          // A format: bf16
         | (1u << 10)         // B format: bf16
         | ((N >> 3) << 17)   // N / 8
         | ((M >> 4) << 24);  // M / 16
}

// Shared-memory matrix descriptor for a K-major operand stored as rows of 128
// bytes (64 bf16) with the 128-byte swizzle, 8-row groups 1024 bytes apart.
// The tile base must be 1024-byte aligned; advancing K by 16 elements adds
// 32 bytes to the start address.
MOE_DEV uint64_t umma_desc_sw128(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= uint64_t((smem_addr >> 4) & 0x3FFFu);  // start address
  d |= uint64_t(1) << 16;                      // leading byte offset (unused for swizzled K-major)
  d |= uint64_t(1024 >> 4) << 32;              // stride byte offset: 8 rows x 128 B
  d |= uint64_t(1) << 46;                      // descriptor version for sm_100
  d |= uint64_t(2) << 61;                      // layout: 128-byte swizzle
  return d;
}

// Load 32 consecutive fp32 columns of this warp's 32 TMEM lanes.
MOE_DEV void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
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
MOE_DEV void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// --------------------------------------------------------------------------
// misc
// --------------------------------------------------------------------------
MOE_DEV float silu_mul(float g, float u) { return g / (1.0f + expf(-g)) * u; }

MOE_DEV void red_add_u32(uint32_t* addr, uint32_t v) {
  asm volatile("red.global.add.u32 [%0], %1;" ::"l"(addr), "r"(v) : "memory");
}

MOE_DEV void red_add_f32(float* addr, float v) {
  asm volatile("red.global.add.f32 [%0], %1;" ::"l"(addr), "f"(v) : "memory");
}

MOE_DEV uint4 ldg_nc_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

}  // namespace moe
