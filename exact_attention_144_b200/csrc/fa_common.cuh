// fa_common.cuh -- sm_100a building blocks shared by the attention kernels:
// mbarriers with bounded waits, TMA tile loads, tcgen05 MMA / TMEM access and
// the shared-memory matrix descriptors they read.
//
// Everything here is written against the PTX ISA (tcgen05, cp.async.bulk.tensor,
// mbarrier); descriptor bit positions follow the sm_100 UMMA descriptor
// definitions (shared-memory descriptor: start address, leading and stride
// byte offsets in 16-byte units, version 1 at bit 46, swizzle mode at bits
// 61-63; instruction descriptor: formats at bits 4/7/10, operand majors at
// bits 15/16, N>>3 at bit 17, M>>4 at bit 24).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace fa {

// ------------------------------------------------------------------ status
// Device-side status word (one per device, owned by fa_api.cu, passed to the
// kernels by address): 0 while every bounded wait has succeeded.  A wait that
// gives up stores  kind | site << 8 | blockIdx.x << 32  (first writer wins)
// and the kernel returns early.
enum : unsigned long long { kStatusWaitTimeout = 0x5A };

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void report_timeout(unsigned long long* status, int site) {
  unsigned long long code = kStatusWaitTimeout | ((unsigned long long)(site & 0xFF) << 8) |
                            ((unsigned long long)blockIdx.x << 32);
  if (status) atomicCAS(status, 0ull, code);
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// Issue helpers below take `issue`: the control warps run their loops with
// all 32 lanes (so loop state and descriptors stay warp-uniform) and only the
// lane with issue = true executes the predicated instruction.
__device__ __forceinline__ void mbar_expect_tx(bool issue, uint32_t bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %2, 0;\n\t"
      "@p mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;\n\t}" ::"r"(bar),
      "r"(bytes), "r"((uint32_t)issue)
      : "memory");
}
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
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

// Waits until the phase with the given parity has completed.  Gives up when
// another role of the block has already given up (abort flag set) or after
// `limit_ns` of wall time; then records the site and sets the abort flag.
struct WaitCtl {
  volatile int* abort;
  uint64_t limit_ns;
  unsigned long long* status;
};

static __device__ __forceinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, WaitCtl w, int site) {
  const uint64_t t0 = global_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_test(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (*w.abort) return false;
      if (global_ns() - t0 > w.limit_ns) {
        report_timeout(w.status, site);
        *w.abort = 1;
        return false;
      }
    }
  }
}

__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, WaitCtl w, int site) {
  if (mbar_test(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, w, site);
}

// mbar_wait by every lane of a warp, with one warp-uniform result.
__device__ __forceinline__ bool mbar_wait_warp(uint32_t bar, uint32_t parity, WaitCtl w, int site) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, w, site));
}

// Wait used while draining at exit: ignores the abort flag, bounded by time.
static __device__ __forceinline__ bool mbar_drain(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = global_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_test(bar, parity)) return true;
    if ((it & 63u) == 0 && global_ns() - t0 > limit_ns) return false;
  }
}

// --------------------------------------------------------------------- TMA
// 4-d tiled load (coordinates innermost first) completing on an mbarrier.
__device__ __forceinline__ void tma_load_4d(bool issue, uint32_t dst, const CUtensorMap* map,
                                            uint32_t bar, int c0, int c1, int c2, int c3) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %7, 0;\n\t"
      "@p cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];\n\t}" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(bar),
      "r"((uint32_t)issue)
      : "memory");
}
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ----------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t dst_slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_slot),
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

// D[tmem] (+)= A[smem] * B[smem]
__device__ __forceinline__ void umma_ss(bool issue, uint32_t d_tmem, uint64_t adesc,
                                        uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.ne.b32 q, %5, 0;\n\t"
      "@q tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"((uint32_t)issue)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]
__device__ __forceinline__ void umma_ts(bool issue, uint32_t d_tmem, uint32_t a_tmem,
                                        uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.ne.b32 q, %5, 0;\n\t"
      "@q tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"((uint32_t)issue)
      : "memory");
}
// The same two products for 8-bit operands (kind::f8f6f4; K = 32 elements
// per instruction, the same 32 bytes of each operand row as kind::f16).
__device__ __forceinline__ void umma_ss_f8(bool issue, uint32_t d_tmem, uint64_t adesc,
                                           uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.ne.b32 q, %5, 0;\n\t"
      "@q tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"((uint32_t)issue)
      : "memory");
}
__device__ __forceinline__ void umma_ts_f8(bool issue, uint32_t d_tmem, uint32_t a_tmem,
                                           uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "setp.ne.b32 q, %5, 0;\n\t"
      "@q tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"((uint32_t)issue)
      : "memory");
}
// Arrive (once) on `bar` when every MMA issued so far by this thread is done.
__device__ __forceinline__ void umma_commit(bool issue, uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %1, 0;\n\t"
      "@p tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
          bar),
      "r"((uint32_t)issue)
      : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread t of the warp receives
// lane (quadrant base + t), columns [col, col+32).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
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
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
// Registers filled by tcgen05.ld are only valid after wait::ld; this empty asm
// makes every later use depend on a point after the wait.
__device__ __forceinline__ void reg_fence(uint32_t (&r)[32]) {
#pragma unroll
  for (int i = 0; i < 32; ++i) asm volatile("" : "+r"(r[i]));
}

// -------------------------------------------------------------- descriptors
// Shared-memory matrix descriptor for a 128-byte-swizzled operand whose
// swizzle atoms (8 rows x 128 bytes) start on 1024-byte boundaries.
//   K-major:  rows of the M/N dimension are 128 bytes apart, 8-row groups are
//             `sbo` bytes apart; `lbo` is unused (16).
//   MN-major: 64-element runs of the M/N dimension are `lbo` bytes apart,
//             8-row groups of the K dimension are `sbo` bytes apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;  // descriptor version (sm_100)
  d |= 2ull << 61;  // 128-byte swizzle
  return d;
}

// The descriptor of the same layout starting `bytes` further on (bytes is a
// multiple of 16; the start field cannot carry out: shared addresses fit it).
__device__ __forceinline__ uint64_t desc_advance(uint64_t desc, uint32_t bytes) {
  return desc + (uint64_t)(bytes >> 4);
}

// Instruction descriptor for kind::f16 with fp32 accumulation.
// fmt: 0 = fp16, 1 = bf16 (same for A and B).  b_mn: B operand is MN-major.
// kind::f8f6f4 reads the same fields; there format 0 is E4M3 (the MN-major
// B operand is allowed for E4M3).
__host__ __device__ constexpr uint32_t f16_idesc(uint32_t fmt, int M, int N, bool b_mn) {
  return (1u << 4) | (fmt << 7) | (fmt << 10) | ((b_mn ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// ------------------------------------------------------------ element types
template <class T>
struct Elem;
// kFmt: instruction-descriptor format; kBytes: bytes an element; kF8: 8-bit
// operands (kind::f8f6f4); Out: the type O is stored in; kMapFmt: tensor-map
// element type (0 fp16, 1 bf16, 2 one byte).  pack(lo, hi) rounds two values
// to the element type, lo in the low bits (16-bit types: one 32-bit word;
// E4M3: the low 16 bits).
template <>
struct Elem<__nv_bfloat16> {
  static constexpr uint32_t kFmt = 1;
  static constexpr int kBytes = 2, kMapFmt = 1;
  static constexpr bool kF8 = false;
  using Out = __nv_bfloat16;
  __device__ __forceinline__ static uint32_t pack(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
  __device__ __forceinline__ static float2 unpack(uint32_t u) {
    __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162*>(&u);
    return __bfloat1622float2(v);
  }
};
template <>
struct Elem<__half> {
  static constexpr uint32_t kFmt = 0;
  static constexpr int kBytes = 2, kMapFmt = 0;
  static constexpr bool kF8 = false;
  using Out = __half;
  __device__ __forceinline__ static uint32_t pack(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  }
  __device__ __forceinline__ static float2 unpack(uint32_t u) {
    __half2 v = *reinterpret_cast<__half2*>(&u);
    return __half22float2(v);
  }
};

template <>
struct Elem<__nv_fp8_e4m3> {
  static constexpr uint32_t kFmt = 0;  // E4M3 in kind::f8f6f4
  static constexpr int kBytes = 1, kMapFmt = 2;
  static constexpr bool kF8 = true;
  using Out = __nv_bfloat16;
  // round to nearest even, saturating at +-448 (no value here reaches it)
  __device__ __forceinline__ static uint32_t pack(float lo, float hi) {
    return (uint32_t)__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3);
  }
};

// D (+)= A B for the element type T (kind::f16 or kind::f8f6f4).
template <class T>
__device__ __forceinline__ void mma_ss(bool issue, uint32_t d_tmem, uint64_t adesc,
                                       uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  if constexpr (Elem<T>::kF8)
    umma_ss_f8(issue, d_tmem, adesc, bdesc, idesc, accumulate);
  else
    umma_ss(issue, d_tmem, adesc, bdesc, idesc, accumulate);
}
template <class T>
__device__ __forceinline__ void mma_ts(bool issue, uint32_t d_tmem, uint32_t a_tmem,
                                       uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  if constexpr (Elem<T>::kF8)
    umma_ts_f8(issue, d_tmem, a_tmem, bdesc, idesc, accumulate);
  else
    umma_ts(issue, d_tmem, a_tmem, bdesc, idesc, accumulate);
}

// ------------------------------------------------------ register rebalance
// Per-warpgroup register limits for the 384-thread kernels: launched with 168
// registers a thread (64,512 in all), the two compute warpgroups grow to 208
// and the producer/MMA warpgroup shrinks to 88 (2*128*208 + 128*88 = 64,512).
// Executed by all four warps of a warpgroup.
constexpr int kLaunchRegs = 168, kComputeRegs = 208, kControlRegs = 88;
static_assert(2 * 128 * kComputeRegs + 128 * kControlRegs <= 384 * kLaunchRegs,
              "register split exceeds the launch allocation");
__device__ __forceinline__ void regs_grow() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kComputeRegs) : "memory");
}
__device__ __forceinline__ void regs_shrink() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kControlRegs) : "memory");
}

// --------------------------------------------------------------- fast math
// Hardware base-2 exponential and logarithm (PTX ex2.approx / lg2.approx).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Three-input max / min (one instruction for two new values of a running
// reduction).
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float min3f(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Packed fp32x2 arithmetic (one instruction for two lanes of work, each lane
// rounded exactly as the scalar operation).  A pair (lo, hi) travels as one
// 64-bit operand; f32x2(v, v) broadcasts.
__device__ __forceinline__ uint64_t f32x2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
// (x0, x1) = (s0 * c.lo + n.lo, s1 * c.hi + n.hi)
__device__ __forceinline__ void fma2(float& x0, float& x1, float s0, float s1, uint64_t c,
                                     uint64_t n) {
  asm("{\n\t.reg .b64 a, r;\n\tmov.b64 a, {%2, %3};\n\tfma.rn.f32x2 r, a, %4, %5;\n\t"
      "mov.b64 {%0, %1}, r;\n\t}"
      : "=f"(x0), "=f"(x1)
      : "f"(s0), "f"(s1), "l"(c), "l"(n));
}
// (a0, a1) += (b0, b1)
__device__ __forceinline__ void add2(float& a0, float& a1, float b0, float b1) {
  asm("{\n\t.reg .b64 a, b, r;\n\tmov.b64 a, {%0, %1};\n\tmov.b64 b, {%2, %3};\n\t"
      "add.rn.f32x2 r, a, b;\n\tmov.b64 {%0, %1}, r;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(b0), "f"(b1));
}

// (r0, r1) = ((a0 - b0) * m0, (a1 - b1) * m1): packed subtract, then multiply
__device__ __forceinline__ void sub_mul2(float& r0, float& r1, float a0, float a1, float b0,
                                         float b1, float m0, float m1) {
  asm("{\n\t.reg .b64 a, b, m, t;\n\tmov.b64 a, {%2, %3};\n\tmov.b64 b, {%4, %5};\n\t"
      "mov.b64 m, {%6, %7};\n\tsub.rn.f32x2 t, a, b;\n\tmul.rn.f32x2 t, t, m;\n\t"
      "mov.b64 {%0, %1}, t;\n\t}"
      : "=f"(r0), "=f"(r1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(m0), "f"(m1));
}

// 2^x0, 2^x1 on the FMA pipe instead of MUFU, for offloading part of the
// softmax exponentials.  Method: round-to-nearest range reduction x = n + f,
// |f| <= 1/2, by adding 1.5 * 2^23 (the integer n lands in the low mantissa
// bits of the sum); a degree-3 polynomial for 2^f whose coefficients were
// fitted here by least squares on the relative error at Chebyshev nodes of
// [-1/2, 1/2] (max relative error 7.5e-5 evaluated in fp32, far below the
// 16-bit rounding of P); n is then added to the exponent field.  x is clamped
// at -125 so that the result stays a normal number (2^-125 is far below every
// p that matters: the row maximum gives p >= 2^-8).  Valid for x <= 127.
__device__ __forceinline__ void ex2_poly2(float& y0, float& y1, float x0, float x1) {
  const uint64_t magic = f32x2(12582912.f, 12582912.f);
  const uint64_t c3 = f32x2(0.0551716648f, 0.0551716648f), c2 = f32x2(0.242611125f, 0.242611125f),
                 c1 = f32x2(0.693260968f, 0.693260968f), c0 = f32x2(0.999928057f, 0.999928057f);
  const uint64_t x = f32x2(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  uint64_t t, pv;
  asm("{\n\t.reg .b64 n, f;\n\t"
      "add.rn.f32x2 %0, %2, %3;\n\t"      // t = x + 1.5 * 2^23
      "sub.rn.f32x2 n, %0, %3;\n\t"       // n = round(x)
      "sub.rn.f32x2 f, %2, n;\n\t"        // f = x - n
      "fma.rn.f32x2 %1, %4, f, %5;\n\t"
      "fma.rn.f32x2 %1, %1, f, %6;\n\t"
      "fma.rn.f32x2 %1, %1, f, %7;\n\t}"
      : "=&l"(t), "=&l"(pv)
      : "l"(x), "l"(magic), "l"(c3), "l"(c2), "l"(c1), "l"(c0));
  const uint32_t tl = (uint32_t)t, th = (uint32_t)(t >> 32);
  const uint32_t pl = (uint32_t)pv, ph = (uint32_t)(pv >> 32);
  y0 = __uint_as_float(pl + (tl << 23));
  y1 = __uint_as_float(ph + (th << 23));
}

// Where sequence b lies on the token axis.  Fixed length (cu null): batch
// entry b, tokens [0, N).  Varlen: tokens [cu[b], cu[b+1]) of the one packed
// batch entry, clamped into [0, total) and to at most N (max_seqlen) tokens,
// so that no contents of cu can send an access out of bounds.
__host__ __device__ __forceinline__ void seq_bounds(const int* cu, int b, int N, int total,
                                                   int& tb, int& tok0, int& len) {
  if (cu == nullptr) {
    tb = b;
    tok0 = 0;
    len = N;
    return;
  }
  int st = cu[b], en = cu[b + 1];
  st = st < 0 ? 0 : (st > total ? total : st);
  const int lim = (st + N < total) ? st + N : total;
  en = en < st ? st : (en > lim ? lim : en);
  tb = 0;
  tok0 = st;
  len = en - st;
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

}  // namespace fa
