// Device helpers shared by the MXFP4 MoE kernels (sm_100a only).
//
// Hand-written inline PTX for mbarriers, TMA (cp.async.bulk / .tensor), tcgen05
// (TMEM alloc, MMA, ld/st, commit, fences), plus the MXFP4 -> bf16 converter.
// Every spin-wait here is bounded: on expiry the kernel records an error in the
// device error word and the caller unwinds.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "../../include/mxfp4_moe.h"

#define MOE_DEV __device__ __forceinline__

namespace moe {

// Debug build (-DMXFP4_MOE_DEBUG=1, libmxfp4_moe_debug.so): kernels also check the indices
// they read from the workspace and record MXFP4_MOE_ERR_DEVICE_BOUNDS with a tag instead of
// making the access.  The release build compiles those checks out.
#ifndef MXFP4_MOE_DEBUG
#define MXFP4_MOE_DEBUG 0
#endif

// ------------------------------------------------------------------ error word --------
// err[0]: first error code (MXFP4_MOE_ERR_*), err[1]: where (kernel-specific tag).
struct DevErr {
  int* word;
  MOE_DEV void set(int code, int where) const {
    if (word && atomicCAS(word, 0, code) == 0) word[1] = where;
  }
};

// Wall-clock bound on a single wait (nanoseconds).  Kernels here finish in
// milliseconds; a wait that lasts a second means a broken pipeline.
constexpr uint64_t kWaitLimitNs = 1000ull * 1000ull * 1000ull;

MOE_DEV uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

MOE_DEV uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------------ mbarrier ----------
MOE_DEV void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
MOE_DEV void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
MOE_DEV void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
MOE_DEV void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
               "r"(bytes)
               : "memory");
}
// Suspend bound handed to mbarrier.try_wait (ns): a waiting thread sleeps until the phase
// completes or this much time passes, so waiting warps do not take issue slots from the
// warps that compute.
constexpr uint32_t kSuspendHintNs = 200000;

MOE_DEV bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}
// Bounded wait for the phase with the given parity to complete.  Returns false
// (and records `where`) if it did not complete within kWaitLimitNs, or if
// another role already aborted the CTA (*abort != 0).
MOE_DEV bool mbar_wait(uint32_t bar, uint32_t parity, const DevErr& err, int where,
                       volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return true;
    if (abort && *abort) return false;
    if (globaltimer() - t0 > kWaitLimitNs) {
      err.set(MXFP4_MOE_ERR_DEVICE_TIMEOUT, where);
      if (abort) *abort = 1;
      return false;
    }
  }
}

// Bounded wait that yields the issue slot between probes (for waits off the critical path).
MOE_DEV bool mbar_wait_sleep(uint32_t bar, uint32_t parity, const DevErr& err, int where,
                             volatile int* abort, uint32_t ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (;;) {
    __nanosleep(ns);
    if (mbar_try_wait(bar, parity)) return true;
    if (abort && *abort) return false;
    if (globaltimer() - t0 > kWaitLimitNs) {
      err.set(MXFP4_MOE_ERR_DEVICE_TIMEOUT, where);
      if (abort) *abort = 1;
      return false;
    }
  }
}

// ------------------------------------------------------------------ TMA ---------------
MOE_DEV void prefetch_tmap(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}
// 2-D tiled load into this CTA's shared memory; completion counted on `bar`.
MOE_DEV void tma_load_2d(uint32_t dst, const void* tmap, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}
// 1-D bulk copy (global -> shared), 16-byte aligned addresses, size multiple of 16.
MOE_DEV void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

// ------------------------------------------------------------------ tcgen05 -----------
MOE_DEV void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
MOE_DEV void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
MOE_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
MOE_DEV void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
MOE_DEV void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A[tmem] * B[smem desc]; kind::f16 (bf16 inputs, fp32 accumulate).
MOE_DEV void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on `bar` when every tcgen05.mma issued so far by this thread completes.
MOE_DEV void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
MOE_DEV void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
MOE_DEV void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 lanes x 32 consecutive 32-bit columns; thread i of the warp owns lane (quarter base + i).
MOE_DEV void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
      "%29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
MOE_DEV void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}
MOE_DEV void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
      : "memory");
}
MOE_DEV void tmem_st1(uint32_t taddr, uint32_t r) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(r) : "memory");
}
MOE_DEV void tmem_st4(uint32_t taddr, const uint32_t (&r)[4]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1, %2, %3, %4};" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3])
               : "memory");
}
MOE_DEV void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
      "%29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

// D[tmem] (+)= (A[tmem] x SFA) * (B[smem desc] x SFB); kind::mxf8f6f4 with one UE8M0 scale
// per 32 elements of K on each side (scale_vec::1X), fp32 accumulate.  sfa/sfb are the TMEM
// addresses of the scale-factor columns; which byte of them the MMA uses comes from the
// instruction descriptor's scale-factor ids.
MOE_DEV void mma_mxf8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                         uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale.scale_vec::1X [%0], [%1], %2, %3, "
      "[%4], [%5], p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
      : "memory");
}

// Shared-memory matrix descriptor for a K-major operand tile written by TMA with 64-byte
// swizzle: rows of 64 bytes (64 E4M3 values), 8-row core groups 512 bytes apart.
MOE_DEV uint64_t smem_desc_kmajor_sw64(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);  // start address
  d |= (uint64_t)1u << 16;                   // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(512u >> 4) << 32;           // stride byte offset: next 8-row group
  d |= (uint64_t)1u << 46;                   // descriptor version (sm_100)
  d |= (uint64_t)4u << 61;                   // 64-byte swizzle
  return d;
}
// Instruction descriptor of the block-scaled MMA: A = E2M1 (format 5, one code per byte in
// bits 5..2), B = E4M3 (format 0), UE8M0 scales, fp32 D, both K-major, M = 128, N = n; the
// scale-factor ids pick byte `sfid` of each scale column.
MOE_DEV uint32_t idesc_mxf4a_m128(int n, uint32_t sfid) {
  return (sfid << 4) | (5u << 7) | ((uint32_t)(n >> 3) << 17) | (1u << 23) | ((128u >> 4) << 24) |
         (sfid << 29);
}

// Shared-memory matrix descriptor for a K-major operand tile written by TMA with
// 128-byte swizzle: rows of 64 bf16 (128 B), 8-row core groups 1024 B apart.
MOE_DEV uint64_t smem_desc_kmajor_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);  // start address
  d |= (uint64_t)1u << 16;                   // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024u >> 4) << 32;          // stride byte offset: next 8-row group
  d |= (uint64_t)1u << 46;                   // descriptor version (sm_100)
  d |= (uint64_t)2u << 61;                   // 128-byte swizzle
  return d;
}
// Instruction descriptor: kind::f16, A = B = bf16, D = fp32, both K-major, M = 128.
MOE_DEV uint32_t idesc_bf16_m128(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((128u >> 4) << 24);
}

// ------------------------------------------------------------------ small math --------
MOE_DEV uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
MOE_DEV uint32_t bmul2(uint32_t a, uint32_t b) {  // bf16x2 multiply, round to nearest even
  uint32_t d;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
MOE_DEV float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
MOE_DEV float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
MOE_DEV float bf16_to_f(uint16_t v) { return __uint_as_float((uint32_t)v << 16); }
MOE_DEV uint16_t f_to_bf16(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}
// sigmoid(z) = (1 + tanh(z/2)) / 2 with the single-instruction tanh approximation
// (relative error about 2^-11, below the bf16 rounding of every value it feeds).
MOE_DEV float fast_sigmoid(float z) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * z));
  return fmaf(0.5f, t, 0.5f);
}
// Two fp32 values in one 64-bit register for the paired fp32 arithmetic of sm_100
// (add / mul / fma .f32x2: one instruction for both lanes of the pair).
MOE_DEV uint64_t f2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
MOE_DEV float f2lo(uint64_t v) { return __uint_as_float((uint32_t)v); }
MOE_DEV float f2hi(uint64_t v) { return __uint_as_float((uint32_t)(v >> 32)); }
MOE_DEV uint64_t f2add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
MOE_DEV uint64_t f2mul(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
MOE_DEV uint64_t f2fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
MOE_DEV uint32_t pack_bf16x2(float lo, float hi) {
  return (uint32_t)f_to_bf16(lo) | ((uint32_t)f_to_bf16(hi) << 16);
}

// ------------------------------------------------------------------ MXFP4 decode ------
// Eight E2M1 codes (q: byte i holds element 2i in its low nibble, 2i+1 in its high
// nibble) -> four bf16x2 words whose value is (E2M1 value) * 2^-126, exactly.
//
// The three magnitude bits (e1 e0 m) land on bf16 bits 8..6, i.e. exponent field
// = e and top mantissa bit = m.  For e >= 1 that is 2^(e-127) * (1 + m/2), the
// E2M1 value times 2^-126; for e == 0 it is the bf16 subnormal m * 2^-127, again
// the E2M1 value (m/2) times 2^-126.  The sign goes to bit 15.  Each 16-bit half
// gets its nibble at bit 0 (zero bytes come from prmt's sign-replicate mode on a
// byte below 0x80); multiplying by 0x1040 adds copies shifted by 6 and 12 that do
// not overlap, and the mask keeps bits 15 and 8..6 of each half.
MOE_DEV void e2m1x8_to_bf16x2_pattern(uint32_t q, uint32_t (&p)[4]) {
  const uint32_t ev = q & 0x0F0F0F0Fu;         // elements 0, 2, 4, 6
  const uint32_t od = (q >> 4) & 0x0F0F0F0Fu;  // elements 1, 3, 5, 7
  p[0] = (prmt(ev, od, 0x8480u) * 0x1040u) & 0x81C081C0u;
  p[1] = (prmt(ev, od, 0x9591u) * 0x1040u) & 0x81C081C0u;
  p[2] = (prmt(ev, od, 0xA6A2u) * 0x1040u) & 0x81C081C0u;
  p[3] = (prmt(ev, od, 0xB7B3u) * 0x1040u) & 0x81C081C0u;
}

// Eight packed E2M1 codes (byte i of q: element 2i in the low nibble, 2i+1 in the high one)
// -> eight bytes in element order, each code in bits 5..2 of its byte: the 8-bit container
// the block-scaled MMA reads E2M1 A operands from in tensor memory.  The codes are not
// decoded; the MMA applies the E2M1 values and the UE8M0 scales itself.
MOE_DEV void e2m1x8_to_containers(uint32_t q, uint32_t& lo4, uint32_t& hi4) {
  const uint32_t ev = (q << 2) & 0x3C3C3C3Cu;  // elements 0, 2, 4, 6
  const uint32_t od = (q >> 2) & 0x3C3C3C3Cu;  // elements 1, 3, 5, 7
  lo4 = prmt(ev, od, 0x5140u);                 // elements 0, 1, 2, 3
  hi4 = prmt(ev, od, 0x7362u);                 // elements 4, 5, 6, 7
}

// UE8M0 scale s -> two bf16 factors f1, f2 with pattern * f1 * f2 = value * 2^(s-127)
// exactly (or +-inf on overflow, NaN for s == 255), each as a bf16 bit pattern.
// s <= 128: f1 = 2^(s-1), f2 = 1.  s in [129, 254]: f1 = 2^127, f2 = 2^(s-128).
MOE_DEV uint32_t ue8m0_f1(uint32_t s) { return s <= 128u ? (s + 126u) << 7 : 0x7F00u; }
MOE_DEV uint32_t ue8m0_f2(uint32_t s) {
  return s <= 128u ? 0x3F80u : (s == 255u ? 0x7FC0u : (s - 1u) << 7);
}
MOE_DEV uint32_t dup16(uint32_t v) { return v | (v << 16); }

}  // namespace moe
