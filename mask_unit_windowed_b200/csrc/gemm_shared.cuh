// Pieces shared by the two tcgen05 GEMM kernels of the Hiera block's Linear layers (the
// one-CTA kernel and the CTA-pair kernel): the kernel parameters, the TMA-store helpers of
// the row-major epilogues, and the host-side tensor-map encoders.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace hiera {

constexpr int BM = 128;  // accumulator rows per CTA (TMEM lanes)
constexpr int BK = 64;   // K per pipeline stage (one 128-byte swizzle row of bf16)

// Division by a divisor fixed at launch as a multiply-high, an add and two shifts (Granlund
// and Montgomery, "Division by invariant integers using multiplication", 1994: the variant
// for any divisor d >= 1 with an m' of 32 bits, exact for every 32-bit unsigned dividend).
// The per-tile row bookkeeping of the epilogue divides by the token count, the pooled token
// count, the window count and the tile count; done with the hardware-less integer divide
// sequence each costs a long dependent chain on the epilogue warps' critical path.
struct FastDiv {
  uint32_t d, mul, sh1, sh2;
  __device__ __forceinline__ uint32_t div(uint32_t n) const {
    const uint32_t t = __umulhi(mul, n);
    return (t + ((n - t) >> sh1)) >> sh2;
  }
};

inline FastDiv make_fastdiv(uint32_t d) {
  FastDiv f{};
  f.d = d < 1 ? 1 : d;
  uint32_t l = 0;  // ceil(log2 d)
  while ((1ull << l) < f.d) ++l;
  f.mul = (uint32_t)(((1ull << 32) * ((1ull << l) - f.d)) / f.d + 1);
  f.sh1 = l < 1 ? l : 1;
  f.sh2 = l > 1 ? l - 1 : 0;
  return f;
}

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
  int qkv_tma;             // q / k / v rows leave through TMA tensor stores: QKV_TMA_*
  FastDiv fd_ntiles;       // N / BN column tiles
  FastDiv fd_tokens;       // tokens per image
  FastDiv fd_per;          // pooled tokens per image (tokens / 4)
  FastDiv fd_nw;           // windows per image
  FastDiv fd_dout;         // d_out (which of q / k / v / r a column tile holds)
};

// How the q / k / v head rows of the qkv GEMM leave (KParams::qkv_tma). A warp's 32 staged
// rows (one head, 128 bytes each, in the 128-byte swizzle) are one TMA box when
//   QKV_TMA_GLOBAL : one window: 32 consecutive tokens are 32 consecutive rows of the head's
//                    [T][64] block (map [64][B * heads * T], box 64 x 32);
//   QKV_TMA_WINDOWS: mask-unit windows, no pooling, 32 | nW: tokens j nW + w, w = w0..w0+31,
//                    are row j of 32 consecutive windows (map [64][T][heads][B nW], box
//                    64 x 1 x 1 x 32);
//   QKV_TMA_POOLED : the pooled tiles of a transition (8 pooled positions x 4 candidates per
//                    warp), k and v only, 8 | nW and nW | tokens / 4: candidate c of pooled
//                    position np is token c tokens / 4 + np, i.e. in-window index
//                    c (tokens / 4 nW) + np / nW of window np mod nW (map
//                    [64][tokens / 4 nW][4][heads][B nW], box 64 x 1 x 4 x 1 x 8).
// Otherwise (QKV_TMA_NONE) the lanes copy the staged rows out.
constexpr int QKV_TMA_NONE = 0, QKV_TMA_GLOBAL = 1, QKV_TMA_WINDOWS = 2, QKV_TMA_POOLED = 3;

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
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, const void* smem_src, int c0,
                                             int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(smem_src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void tma_store_5d(const CUtensorMap* map, const void* smem_src, int c0,
                                             int c1, int c2, int c3, int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5, %6}], [%1];" ::
          "l"(reinterpret_cast<uint64_t>(map)),
      "r"(smem_u32(smem_src)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
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
