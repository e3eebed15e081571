// Device helpers shared by the Hiera kernels: bf16 packing, the device status word,
// bounded mbarrier waits, TMA loads and the tcgen05 (5th-gen tensor core) primitives.
// Every wait on an mbarrier is bounded by wall-clock time read from %globaltimer; on
// expiry it records HIERA_ERR_TIMEOUT in the device status word and reports failure
// to the caller, which then winds its kernel down instead of hanging the GPU.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "hiera.h"

namespace hiera {

typedef __nv_bfloat16 bf16;

// Record `code` in the device status word (first error wins). The word lives in the
// library's api translation unit; kernels receive its address as a parameter.
__device__ __forceinline__ void record_status(unsigned int* status, unsigned int code) {
  if (status != nullptr) atomicCAS(status, 0u, code);
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait until the phase with the given parity has completed, for at most limit_ns.
// Returns false (and records HIERA_ERR_TIMEOUT in *status) if the limit ran out. If
// `abort` is given and becomes non-zero (another role of the CTA gave up), returns
// false at once.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns,
                                          unsigned int* status,
                                          const volatile int* abort = nullptr) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  uint32_t spins = 0;
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((++spins & 255u) == 0u) {
      if (abort != nullptr && *abort != 0) return false;
      if (global_ns() - t0 > limit_ns) {
        record_status(status, HIERA_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

// Programmatic dependent launch: wait until the grids this one depends on have completed
// and their memory is visible (a no-op when the launch had no such dependency), and let
// the next grid of the stream start its launch and set-up.
__device__ __forceinline__ void griddep_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Orders this thread's prior generic-proxy shared-memory accesses before later
// async-proxy (TMA / tensor-core) accesses of the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------ TMA
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void tma_load_4d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2),
      "r"(c3)
      : "memory");
}

// ------------------------------------------------------------------ tcgen05
__device__ __forceinline__ void tc_alloc(uint32_t* smem_result, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(smem_result)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tc_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Arrive on an mbarrier once every tcgen05 op issued so far by this thread has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tc_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i gets lane (base lane + i).
__device__ __forceinline__ void tc_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tc_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tc_ld_32x32b_x8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7])
      : "r"(taddr));
}

// 32 lanes x 32 consecutive 32-bit columns from registers into TMEM.
__device__ __forceinline__ void tc_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
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

__device__ __forceinline__ void tc_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tma_load_3d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// 2^x on the MUFU unit (approximate, flush-to-zero), for softmax weights.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Named barrier among `count` threads (a multiple of 32) of the CTA.
__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// Shared-memory matrix descriptor for a K-major operand tile stored with the 128-byte
// swizzle: rows of 64 bf16 (128 B), 8-row core groups 1024 B apart. Fields: start
// address >> 4 in bits 0-13, leading-dimension byte offset >> 4 in bits 16-29 (unused
// for this layout, set to 1), stride-dimension byte offset >> 4 in bits 32-45,
// descriptor version 1 in bits 46-47, layout type 2 (128-byte swizzle) in bits 61-63.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;
  d |= (uint64_t)(1024u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}

// The same for an MN-major operand tile 64 elements (one 128-byte swizzle atom) wide: rows of
// K, 8-row groups 1024 B apart. The stride to a next atom along MN is never used at this
// width; both offset fields hold 1024 B.
__device__ __forceinline__ uint64_t smem_desc_sw128_mn64(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)(1024u >> 4) << 16;
  d |= (uint64_t)(1024u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}

// A descriptor with its start address advanced by `bytes` (a multiple of 16, staying inside
// shared memory, so the 14-bit address field cannot carry into the next field): only the
// low word changes, one 32-bit add instead of rebuilding the descriptor.
__device__ __forceinline__ uint64_t desc_advance(uint64_t desc, uint32_t bytes) {
  return desc + (uint64_t)(bytes >> 4);
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (bf16 in, fp32 accumulate), one CTA, with the
// accumulate flag fixed at compile time.
template <bool ACC>
__device__ __forceinline__ void tc_mma_bf16_k(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                              uint32_t idesc) {
  if constexpr (ACC) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.eq.u32 p, 1, 1;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.eq.u32 p, 1, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc)
        : "memory");
  }
}

// The same with the A operand in tensor memory: M = 128 rows in the 128 lanes, K along the
// columns, two 16-bit elements per 32-bit column (one K = 16 step spans 8 columns).
template <bool ACC>
__device__ __forceinline__ void tc_mma_bf16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                               uint32_t idesc) {
  if constexpr (ACC) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.eq.u32 p, 1, 1;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.eq.u32 p, 1, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc)
        : "memory");
  }
}

// Instruction descriptor for kind::f16 with bf16 A/B, fp32 accumulator, both operands
// K-major: D format bits 4-5 = 1 (f32), A format bits 7-9 = 1 (bf16), B format bits
// 10-12 = 1 (bf16), N >> 3 in bits 17-22, M >> 4 in bits 24-28.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// Instruction-descriptor bit 16: the B operand is MN-major (its N elements contiguous in
// shared memory, K along the 128-byte-swizzled rows) instead of K-major. With N = 64 bf16
// (one 128-byte swizzle atom wide) the shared-memory descriptor is the same as for a K-major
// tile: 8-row groups 1024 bytes apart.
constexpr uint32_t IDESC_B_MN_MAJOR = 1u << 16;

// ------------------------------------------------------------------ small numeric helpers
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ float gelu_erf(float x) {
  return 0.5f * x * (1.0f + erff(x * 0.70710678118654752440f));
}

// GELU(x) = x Phi(x) = x sigmoid(g(x)) with g = logit(Phi). g is odd; it is approximated by
// x (c0 + c1 x^2 + c2 x^4), a minimax fit (made for this library, weighted by dGELU/dg) of
// c0 = 1.5950153, c1 = 0.074011831, c2 = -7.0316069e-4, with x^2 clamped at 36: past
// |x| = 6 the sigmoid is 0 or 1 to fp32 precision and the clamp keeps the polynomial
// positive. The sigmoid is taken as (1 + tanh(g / 2)) / 2, so GELU(x) = h + h tanh(g(x) / 2)
// with h = x / 2: one MUFU operation (tanh.approx.f32, within 7.9e-6 of tanh over [-12, 12]
// as measured on sm_100a, and exactly +-1 far out) and six FP32 operations per element.
// Max |GELU error| about 3e-5 over the real line (fit 2.6e-5 plus |x| / 2 times the tanh
// error), far below bf16 resolution of the stored result. The constants below are c_k / 2.
// Used by the bf16 tensor-core path.
__device__ __forceinline__ float gelu_fast(float x) {
  const float x2 = fminf(x * x, 36.0f);
  float p = fmaf(-3.51580345e-04f, x2, 3.70059155e-02f);
  p = fmaf(p, x2, 7.97507650e-01f);
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(x * p));
  const float h = 0.5f * x;
  return fmaf(h, t, h);
}

// Two fp32 values in one 64-bit register pair for sm_100's packed fp32 instructions
// (fma.rn.f32x2, mul.rn.f32x2): each half is the IEEE operation on its own value, the same
// bits as the scalar instruction, in half the issue slots. The epilogues whose arithmetic is
// bound by instruction issue (the GELU of fc1 and of the fused MLP) work on pairs.
typedef unsigned long long f32x2;
__device__ __forceinline__ f32x2 f2_pack(float lo, float hi) {
  f32x2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(f32x2 v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ f32x2 f2_fma(f32x2 a, f32x2 b, f32x2 c) {
  f32x2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ f32x2 f2_add(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f32x2 f2_mul(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// gelu_fast of two values with the packed instructions: the same operations in the same
// order on each value, so the same bits as two gelu_fast calls.
__device__ __forceinline__ f32x2 gelu_fast2(f32x2 x) {
  const f32x2 sq = f2_mul(x, x);
  float s0, s1;
  f2_unpack(sq, s0, s1);
  const f32x2 x2 = f2_pack(fminf(s0, 36.0f), fminf(s1, 36.0f));
  f32x2 p = f2_fma(f2_pack(-3.51580345e-04f, -3.51580345e-04f), x2,
                   f2_pack(3.70059155e-02f, 3.70059155e-02f));
  p = f2_fma(p, x2, f2_pack(7.97507650e-01f, 7.97507650e-01f));
  float u0, u1;
  f2_unpack(f2_mul(x, p), u0, u1);
  float t0, t1;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t0) : "f"(u0));
  asm("tanh.approx.f32 %0, %1;" : "=f"(t1) : "f"(u1));
  const f32x2 h = f2_mul(f2_pack(0.5f, 0.5f), x);
  return f2_fma(h, f2_pack(t0, t1), h);
}

// (mean, M2) of the N values of a row piece in column order, as four interleaved partial
// sums (values i = q mod 4 in accumulator q) combined as (a0 + a1) + (a2 + a3): chains a
// quarter as long as one running sum. Every kernel that writes LayerNorm partials of such a
// piece uses this order (stats_piece on fp32 values, stats_piece_bf16 on packed bf16 rows), so
// the fused and unfused paths produce the same bits.
template <int N>
__device__ __forceinline__ void stats_piece(const float (&v)[N], float& mean, float& m2) {
  static_assert(N % 4 == 0, "four accumulators");
  float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < N; ++i) s4[i & 3] += v[i];
  mean = ((s4[0] + s4[1]) + (s4[2] + s4[3])) * (1.f / (float)N);
  float q4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < N; ++i) q4[i & 3] = fmaf(v[i] - mean, v[i] - mean, q4[i & 3]);
  m2 = (q4[0] + q4[1]) + (q4[2] + q4[3]);
}
// the same on NG * 8 values held as packed bf16 (value 8 g + 2 e + h is word e's half h)
template <int NG>
__device__ __forceinline__ void stats_piece_bf16(const uint4 (&w)[NG], float& mean, float& m2) {
  float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int g = 0; g < NG; ++g) {
    const uint32_t w4[4] = {w[g].x, w[g].y, w[g].z, w[g].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      s4[(2 * e) & 3] += __uint_as_float(w4[e] << 16);
      s4[(2 * e + 1) & 3] += __uint_as_float(w4[e] & 0xFFFF0000u);
    }
  }
  mean = ((s4[0] + s4[1]) + (s4[2] + s4[3])) * (1.f / (float)(NG * 8));
  float q4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int g = 0; g < NG; ++g) {
    const uint32_t w4[4] = {w[g].x, w[g].y, w[g].z, w[g].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float lo = __uint_as_float(w4[e] << 16) - mean;
      const float hi = __uint_as_float(w4[e] & 0xFFFF0000u) - mean;
      q4[(2 * e) & 3] = fmaf(lo, lo, q4[(2 * e) & 3]);
      q4[(2 * e + 1) & 3] = fmaf(hi, hi, q4[(2 * e + 1) & 3]);
    }
  }
  m2 = (q4[0] + q4[1]) + (q4[2] + q4[3]);
}

// ------------------------------------------------------------------ tcgen05 epilogue helpers
// Every lane observes the barrier phase itself (so each has acquired the producer's
// writes), then the warp agrees on the outcome so that it stays converged for the
// .sync.aligned tcgen05 instructions that follow.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, uint64_t limit,
                                          unsigned int* status, volatile int* abort_flag) {
  int ok = mbar_wait(bar, parity, limit, status, abort_flag) ? 1 : 0;
  ok = __all_sync(0xffffffffu, ok);
  if (!ok) *abort_flag = 1;
  return ok != 0;
}

// CH consecutive accumulator columns of this thread's TMEM lane, one wait.
template <int CH>
__device__ __forceinline__ void tmem_load(uint32_t taddr, uint32_t (&r)[CH]) {
  if constexpr (CH == 56) {
    tc_ld_32x32b_x32(taddr, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
    tc_ld_32x32b_x16(taddr + 32, *reinterpret_cast<uint32_t(*)[16]>(&r[32]));
    tc_ld_32x32b_x8(taddr + 48, *reinterpret_cast<uint32_t(*)[8]>(&r[48]));
  } else if constexpr (CH == 32) {
    tc_ld_32x32b_x32(taddr, r);
  } else if constexpr (CH == 16) {
    tc_ld_32x32b_x16(taddr, r);
  } else {
    static_assert(CH == 8, "chunk");
    tc_ld_32x32b_x8(taddr, r);
  }
  tc_wait_ld();
  // tcgen05.ld fills its registers asynchronously; only after tcgen05.wait::ld are they
  // valid. Re-define each one after the wait so no use can be scheduled above it.
#pragma unroll
  for (int i = 0; i < CH; ++i) asm volatile("" : "+r"(r[i]));
}

__device__ __forceinline__ uint4 pack8(const float* v) {
  uint4 pk;
  pk.x = pack_bf16x2(v[0], v[1]);
  pk.y = pack_bf16x2(v[2], v[3]);
  pk.z = pack_bf16x2(v[4], v[5]);
  pk.w = pack_bf16x2(v[6], v[7]);
  return pk;
}

// LayerNorm of a row of K values from P partial (mean, M2) pairs over K / P values each
// (Chan et al. merge with equal counts): LN(x) W^T + b = fa (x W'^T) + fb s + c with
// fa = rstd, fb = -mean rstd (s, c the packed column constants of the folded weight).
// Constants of the LayerNorm of a row of K values kept as P partials (P a power of two, so
// 1 / P is exact): computed once per kernel, so that merging a row's partials needs no
// division on the epilogue's critical path.
struct LnConsts {
  float inv_p, k_over_p, inv_k;
};
__device__ __forceinline__ LnConsts ln_consts(int P, int K) {
  return {1.0f / (float)P, (float)(K / P), 1.0f / (float)K};
}

__device__ __forceinline__ void ln_merge_parts(const float2 (&part)[8], int P, const LnConsts& c,
                                               float eps, float& fa, float& fb) {
  float mean = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) mean += part[j].x;
  mean *= c.inv_p;
  float m2 = 0.f, dev2 = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j < P) {
      const float dlt = part[j].x - mean;
      m2 += part[j].y;
      dev2 = fmaf(dlt, dlt, dev2);
    }
  }
  m2 = fmaf(c.k_over_p, dev2, m2);
  fa = rsqrtf(fmaf(m2, c.inv_k, eps));
  fb = -mean * fa;
}

__device__ __forceinline__ void ln_fold_coeffs(const float2* __restrict__ sp, int P,
                                               const LnConsts& c, float eps, float& fa,
                                               float& fb) {
  float2 part[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) part[j] = j < P ? __ldg(sp + j) : make_float2(0.f, 0.f);
  ln_merge_parts(part, P, c, eps, fa, fb);
}

// ------------------------------------------------------------------ Unroll map
// Unrolled index of spatial (y, x) on a GxG grid with L levels (mask-unit side 2^L):
// u = (sum_{k=1..L} (2 a_k + b_k) 4^(L-k)) * M^2 + my*M + mx.
__device__ __forceinline__ int unrolled_of_spatial(int y, int x, int L, int M) {
  int off = 0;
  for (int k = 1; k <= L; ++k) {
    const int a = (y >> (k - 1)) & 1, b = (x >> (k - 1)) & 1;
    off = off * 4 + (2 * a + b);
  }
  return off * M * M + (y >> L) * M + (x >> L);
}

// Inverse: raster index y*G + x of unrolled token u.
__device__ __forceinline__ int spatial_of_unrolled(int u, int L, int M, int G) {
  const int MM = M * M;
  int off = u / MM, mu = u - (u / MM) * MM;
  int y = (mu / M) << L, x = (mu % M) << L;
  // off = sum_k c_k 4^(L-k): the last digit is c_L (coarsest offset).
  for (int k = L; k >= 1; --k) {
    const int c = off & 3;
    off >>= 2;
    y += (c >> 1) << (k - 1);
    x += (c & 1) << (k - 1);
  }
  return y * G + x;
}

}  // namespace hiera
