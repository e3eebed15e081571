// Pieces shared by the two tcgen05 GEMM kernels of the Hiera block's Linear layers (the
// one-CTA kernel and the CTA-pair kernel): the kernel parameters, the TMA-store helpers of
// the row-major epilogues, and the host-side tensor-map encoders.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace hiera {

constexpr int BM = 128;  // accumulator rows per CTA (TMEM lanes)
constexpr int BK = 64;   // K per pipeline stage (one 128-byte swizzle row of bf16)

struct KParams {
  int M, N, K;
  const float* colsum;
  const float* colconst;
  const bf16* bias16;
  float ln_eps;
  bf16* out;
  const bf16* residual;
  int ldo;
  bf16* q;
  bf16* k;
  bf16* v;
  bf16* r;
  int tokens, nW, heads, d_out, Tq, Tkv;
  uint64_t limit_ns;
  unsigned int* status;
  const float2* stats_in;  // FOLD: [M][stats_parts] partial (mean, M2) of A's rows
  int stats_parts;
  float2* stats_out;       // STORE: [M][stats_out_parts] partials of the output, or nullptr
  int stats_out_parts;
  int w_static;            // W may be read before the wait for the previous kernel
  int qkv_tma;             // q / k / v rows leave through TMA tensor stores (global attention)
};

constexpr int cmin(int a, int b) { return a < b ? a : b; }

// Chan et al. merge of a chunk's (mean_b, M2_b) over nb values into the running (mean, M2)
// over na values. Every rounding is explicit (no contraction left to the compiler), so the
// one-CTA kernel's running merge and the CTA-pair kernel's merge of two column quarters
// give the same bits.
__device__ __forceinline__ void chan_merge(float& mean, float& m2, float mean_b, float m2_b,
                                           float na, float nb) {
  const float nt = na + nb;
  const float dlt = __fsub_rn(mean_b, mean);
  mean = fmaf(dlt, nb / nt, mean);
  m2 = __fadd_rn(__fadd_rn(m2, m2_b), __fmul_rn(__fmul_rn(dlt, dlt), na * nb / nt));
}

// Plain row-major outputs (EPI_STORE, EPI_GELU) leave through TMA tensor stores: each
// epilogue warp stages its 32 rows x CH columns densely in shared memory and one lane stores
// the block (rows past M are clipped by the tensor map).
template <int EPI>
struct TmaOut {
  static constexpr bool value = EPI != EPI_QKV;
};

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* smem_src, int c0,
                                             int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(smem_src)), "r"(c0), "r"(c1)
      : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// the bulk stores this thread committed have finished reading shared memory
__device__ __forceinline__ void tma_store_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// ... and have completed
__device__ __forceinline__ void tma_store_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// 2-D bf16 tensor map without swizzle (the dense staging blocks of the TMA-store epilogue)
bool encode_bf16_plain(CUtensorMap* map, const void* base, cuuint64_t cols, cuuint64_t rows,
                       cuuint64_t row_bytes, cuuint32_t box_cols, cuuint32_t box_rows);

// The sixteen-epilogue-warp GEMMs for the non-pooled 224-column variants: one CTA per
// 128 x 224 tile (PAIR false) or a CTA pair per 256 x 224 tile (cta_group::2, PAIR true).
template <int EPI, bool FOLD, bool PAIR>
hiera_status run_wide(const TcGemmArgs& a, cudaStream_t stream);

}  // namespace hiera
