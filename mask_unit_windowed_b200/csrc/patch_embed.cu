// PatchEmbed + pos_embed + Unroll in one pass ("Phase 4: Hiera Backbone MLX Port",
// Architecture Summary: PatchEmbed is Conv2d(4 -> 112, 7x7, stride 4) reshaped to
// [B, N, C]; a learned pos_embed (1, N, 112) is added; Unroll permutes the tokens).
// Padding 3, so an img x img image gives a (img/4) x (img/4) token grid.
//
// bf16: an implicit GEMM on the tensor cores (mma.sync m16n8k16, fp32 accumulation): a CTA
// holds the weight as bf16 [112][208] in shared memory and, per output row, the 7 input rows
// its 128 output columns need (3-pixel halo, zero outside the image); each warp computes 16
// output pixels x 112 channels over K = 196 (padded to 208) with A fragments gathered
// straight from the staged input (the (ky, kx, c) ordering keeps every fragment pair in one
// 4-byte word). The epilogue adds bias and pos_embed[raster token] (loaded before the MMA
// loop) to the accumulator fragments, rounds once to bf16 and stages the rows per warp in
// the input buffer, which the MMA no longer needs; a lane per (pixel, 56-channel half) then
// stores the half row at its unrolled position (3 unroll levels) and, when asked, the
// LayerNorm partial (mean, M2) of the half for block 0's norm1. 79 KB of shared memory
// per CTA: two CTAs per SM overlap one's loads with the other's MMA.
// fp32: the same computation in fp32 SIMT (weights fp32 [196][112] in shared memory, 56
// accumulators per thread).
#include "common.cuh"
#include "internal.h"

namespace hiera {
namespace {

constexpr int COUT = 112, KSZ = 7, CIN = 4, KTOT = KSZ * KSZ * CIN;  // 196
constexpr int SEG = 128;                                            // outputs per CTA row
constexpr int XSPAN = 4 * (SEG - 1) + KSZ;                          // 515 input columns
constexpr int XPITCH = 516;
constexpr int ROWS = 4;
constexpr int SMEM_W = KTOT * COUT * 4;                   // 87808
constexpr int SMEM_IN = KSZ * CIN * XPITCH * 4;           // 57792
constexpr int SMEM_TOTAL = SMEM_W + SMEM_IN;

__global__ void __launch_bounds__(256, 1) patch_embed_kernel(const float* __restrict__ img,
                                                             const float* __restrict__ wt,
                                                             const float* __restrict__ bias,
                                                             const float* __restrict__ pos,
                                                             float* __restrict__ out,
                                                             int img_side) {
  extern __shared__ __align__(16) float smem_f[];
  float* sW = smem_f;                 // [196][112]
  float* sIn = smem_f + KTOT * COUT;  // [7][4][XPITCH]
  const int G = img_side / 4;
  const int M = G / 8;
  const int N = G * G;
  const int b = blockIdx.z;
  const int ox0 = blockIdx.x * SEG;
  const int tid = threadIdx.x;
  const int px = tid & (SEG - 1), half = tid >> 7;

  for (int i = tid; i < KTOT * COUT / 4; i += 256)
    reinterpret_cast<float4*>(sW)[i] = __ldg(reinterpret_cast<const float4*>(wt) + i);

  for (int r = 0; r < ROWS; ++r) {
    const int oy = blockIdx.y * ROWS + r;
    if (oy >= G) break;
    __syncthreads();  // previous row's readers are done with sIn
    for (int i = tid; i < KSZ * XSPAN; i += 256) {
      const int ky = i / XSPAN, xi = i - ky * XSPAN;
      const int iy = 4 * oy - 3 + ky, ix = 4 * ox0 - 3 + xi;
      float v[CIN] = {0.f, 0.f, 0.f, 0.f};
      if (iy >= 0 && iy < img_side && ix >= 0 && ix < img_side) {
        const float* src = img + (((long long)b * img_side + iy) * img_side + ix) * CIN;
#pragma unroll
        for (int c = 0; c < CIN; ++c) v[c] = src[c];
      }
#pragma unroll
      for (int c = 0; c < CIN; ++c) sIn[(ky * CIN + c) * XPITCH + xi] = v[c];
    }
    __syncthreads();

    const int ox = ox0 + px;
    float acc[56];
#pragma unroll
    for (int j = 0; j < 56; ++j) acc[j] = 0.f;
    const float* wbase = sW + half * 56;
#pragma unroll 1
    for (int ky = 0; ky < KSZ; ++ky) {
#pragma unroll 1
      for (int kx = 0; kx < KSZ; ++kx) {
#pragma unroll
        for (int c = 0; c < CIN; ++c) {
          const float xv = sIn[(ky * CIN + c) * XPITCH + 4 * px + kx];
          const float4* wr = reinterpret_cast<const float4*>(wbase + ((ky * KSZ + kx) * CIN + c) * COUT);
#pragma unroll
          for (int j = 0; j < 14; ++j) {
            const float4 w4 = wr[j];
            acc[4 * j + 0] = fmaf(xv, w4.x, acc[4 * j + 0]);
            acc[4 * j + 1] = fmaf(xv, w4.y, acc[4 * j + 1]);
            acc[4 * j + 2] = fmaf(xv, w4.z, acc[4 * j + 2]);
            acc[4 * j + 3] = fmaf(xv, w4.w, acc[4 * j + 3]);
          }
        }
      }
    }
    if (ox < G) {
      const int t = oy * G + ox;
      const int u = unrolled_of_spatial(oy, ox, 3, M);
      const float* pr = pos + (long long)t * COUT + half * 56;
      float* dst = out + ((long long)b * N + u) * COUT + half * 56;
#pragma unroll
      for (int j = 0; j < 56; ++j) dst[j] = acc[j] + __ldg(bias + half * 56 + j) + pr[j];
    }
  }
}

// ---------------------------------------------------------------- bf16 tensor-core path
constexpr int KP = 208;                 // K padded to 13 k-steps of 16
constexpr int WPITCH = 216;             // bf16 per weight row in smem (conflict-free fragments)
constexpr int IN_PITCH = 516;           // pixels per staged input row
constexpr int SPITCH = 120;             // bf16 per staged output pixel (240 B: 16-byte rows)
constexpr int MMA_ROWS = 4;             // output rows per CTA (weights loaded once)
constexpr int IN_BYTES = KSZ * IN_PITCH * CIN * 2;
constexpr int STG_BYTES = 8 * 16 * SPITCH * 2;  // 8 warps x 16 pixels, aliases the input rows
constexpr int BUF_BYTES = IN_BYTES > STG_BYTES ? IN_BYTES : STG_BYTES;
constexpr int MMA_SMEM = PATCH_CO * WPITCH * 2 + BUF_BYTES;  // 79 KB: two CTAs per SM

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// element offset of (k, local pixel px) in the staged input [ky][x][c]; k even
__device__ __forceinline__ int in_off(int k, int px) {
  const int ky = k / 28, rem = k - 28 * ky;
  return (ky * IN_PITCH + 4 * px + (rem >> 2)) * CIN + (rem & 3);
}

__global__ void __launch_bounds__(256, 2) patch_embed_mma_kernel(
    const bf16* __restrict__ img, const bf16* __restrict__ w16, const float* __restrict__ bias,
    const bf16* __restrict__ pos, bf16* __restrict__ out, float2* __restrict__ stats_out,
    int img_side) {
  griddep_wait();  // everything below reads or writes data of earlier kernels
  griddep_launch_dependents();
  extern __shared__ __align__(16) uint8_t smem_pe[];
  bf16* sW = reinterpret_cast<bf16*>(smem_pe);  // [112][WPITCH]
  bf16* sIn = sW + PATCH_CO * WPITCH;           // [7][IN_PITCH][4] during the MMA
  const int G = img_side / 4;
  const int M = G / 8;
  const int N = G * G;
  const int b = blockIdx.z;
  const int ox0 = blockIdx.x * SEG;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t4 = lane & 3;
  // after the MMA the input rows are dead: each warp stages its 16 pixels x 112 channels
  // there, rounded to bf16 ([16][SPITCH])
  bf16* so = sIn + warp * 16 * SPITCH;

  for (int i = tid; i < PATCH_CO * (KP / 8); i += 256) {
    const int co = i / (KP / 8), c8 = i - co * (KP / 8);
    *reinterpret_cast<uint4*>(sW + co * WPITCH + c8 * 8) =
        __ldg(reinterpret_cast<const uint4*>(w16 + co * KP) + c8);
  }
  for (int rr = 0; rr < MMA_ROWS; ++rr) {
    const int oy = blockIdx.y * MMA_ROWS + rr;
    if (oy >= G) break;
    __syncthreads();  // the previous row's staged outputs have been copied out
    for (int i = tid; i < KSZ * XSPAN; i += 256) {
      const int ky = i / XSPAN, xi = i - ky * XSPAN;
      const int iy = 4 * oy - 3 + ky, ix = 4 * ox0 - 3 + xi;
      uint2 v = make_uint2(0u, 0u);
      if (iy >= 0 && iy < img_side && ix >= 0 && ix < img_side)
        v = __ldg(reinterpret_cast<const uint2*>(img + (((long long)b * img_side + iy) * img_side + ix) * CIN));
      *reinterpret_cast<uint2*>(sIn + (ky * IN_PITCH + xi) * CIN) = v;
    }
    // pos_embed of this lane's two pixels (rows g, g + 8 of the warp's 16) and 28 channels
    // (8 nt + 2 t4, +1), in flight while the MMA runs
    uint32_t pw[2][14];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int ox = ox0 + warp * 16 + g + 8 * h;
      const bf16* pr = pos + (long long)(oy * G + (ox < G ? ox : 0)) * PATCH_CO + 2 * t4;
#pragma unroll
      for (int nt = 0; nt < 14; ++nt)
        pw[h][nt] = __ldg(reinterpret_cast<const unsigned int*>(pr + nt * 8));
    }
    __syncthreads();
    const int px = warp * 16 + g;  // fragment rows g and g + 8
    float acc[14][4];
#pragma unroll
    for (int nt = 0; nt < 14; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll 1
    for (int ks = 0; ks < KP / 16; ++ks) {
      const int kA = 16 * ks + 2 * t4, kB = kA + 8;
      uint32_t a0 = 0, a1 = 0, a2 = 0, a3 = 0;
      if (kA < PATCH_K) {
        a0 = *reinterpret_cast<const uint32_t*>(sIn + in_off(kA, px));
        a1 = *reinterpret_cast<const uint32_t*>(sIn + in_off(kA, px + 8));
      }
      if (kB < PATCH_K) {
        a2 = *reinterpret_cast<const uint32_t*>(sIn + in_off(kB, px));
        a3 = *reinterpret_cast<const uint32_t*>(sIn + in_off(kB, px + 8));
      }
#pragma unroll
      for (int nt = 0; nt < 14; ++nt) {
        const bf16* wr = sW + (nt * 8 + g) * WPITCH;
        const uint32_t b0 = *reinterpret_cast<const uint32_t*>(wr + kA);
        const uint32_t b1 = *reinterpret_cast<const uint32_t*>(wr + kB);
        mma_bf16_16816(acc[nt], a0, a1, a2, a3, b0, b1);
      }
    }
    __syncthreads();  // every warp is done reading the input rows
    // (acc + bias) + pos_embed, rounded once to bf16, staged per pixel row
#pragma unroll
    for (int nt = 0; nt < 14; ++nt) {
      const int co = nt * 8 + 2 * t4;
      const float b0 = __ldg(bias + co), b1 = __ldg(bias + co + 1);
      *reinterpret_cast<uint32_t*>(so + g * SPITCH + co) =
          pack_bf16x2((acc[nt][0] + b0) + bf16_lo(pw[0][nt]), (acc[nt][1] + b1) + bf16_hi(pw[0][nt]));
      *reinterpret_cast<uint32_t*>(so + (g + 8) * SPITCH + co) =
          pack_bf16x2((acc[nt][2] + b0) + bf16_lo(pw[1][nt]), (acc[nt][3] + b1) + bf16_hi(pw[1][nt]));
    }
    __syncwarp();
    // lane = (pixel, half): the half row to its unrolled position, LayerNorm partial
    {
      const int lp = lane & 15, half = lane >> 4;
      const int ox = ox0 + warp * 16 + lp;
      if (ox < G) {
        const int u = unrolled_of_spatial(oy, ox, 3, M);
        const uint4* src = reinterpret_cast<const uint4*>(so + lp * SPITCH + half * 56);
        uint4* dst = reinterpret_cast<uint4*>(out + ((long long)b * N + u) * PATCH_CO + half * 56);
        float vals[56];
#pragma unroll
        for (int c8 = 0; c8 < 7; ++c8) {
          const uint4 pk = src[c8];
          dst[c8] = pk;
          vals[8 * c8 + 0] = bf16_lo(pk.x);
          vals[8 * c8 + 1] = bf16_hi(pk.x);
          vals[8 * c8 + 2] = bf16_lo(pk.y);
          vals[8 * c8 + 3] = bf16_hi(pk.y);
          vals[8 * c8 + 4] = bf16_lo(pk.z);
          vals[8 * c8 + 5] = bf16_hi(pk.z);
          vals[8 * c8 + 6] = bf16_lo(pk.w);
          vals[8 * c8 + 7] = bf16_hi(pk.w);
        }
        if (stats_out != nullptr) {
          float s = 0.f;
#pragma unroll
          for (int j = 0; j < 56; ++j) s += vals[j];
          const float mean = s * (1.f / 56.f);
          float m2 = 0.f;
#pragma unroll
          for (int j = 0; j < 56; ++j) m2 = fmaf(vals[j] - mean, vals[j] - mean, m2);
          stats_out[((long long)b * N + u) * 2 + half] = make_float2(mean, m2);
        }
      }
    }
  }
}

}  // namespace

hiera_status launch_patch_embed(const void* img, const void* packed, const void* pos, void* out,
                                float2* stats_out, int B, int img_side, int dtype_bf16,
                                cudaStream_t stream) {
  const int G = img_side / 4;
  const uint8_t* pk = static_cast<const uint8_t*>(packed);
  const float* wt = reinterpret_cast<const float*>(pk);
  const float* bias = reinterpret_cast<const float*>(pk + PATCH_OFF_BIAS);
  const bf16* w16 = reinterpret_cast<const bf16*>(pk + PATCH_OFF_W16);
  profile_mark(K_PATCH_EMBED, stream);
  if (dtype_bf16) {
    dim3 grid((G + SEG - 1) / SEG, (G + MMA_ROWS - 1) / MMA_ROWS, B);
    if (grid.y > 65535 || grid.z > 65535) return HIERA_ERR_SHAPE;
    if (!ensure_smem_attr(reinterpret_cast<const void*>(patch_embed_mma_kernel), MMA_SMEM))
      return HIERA_ERR_CUDA;
    launch_k(patch_embed_mma_kernel, grid, dim3(256), MMA_SMEM, stream,
             static_cast<const bf16*>(img), w16, bias, static_cast<const bf16*>(pos),
             static_cast<bf16*>(out), stats_out, img_side);
  } else {
    dim3 grid((G + SEG - 1) / SEG, (G + ROWS - 1) / ROWS, B);
    if (grid.y > 65535 || grid.z > 65535) return HIERA_ERR_SHAPE;
    if (!ensure_smem_attr(reinterpret_cast<const void*>(patch_embed_kernel), SMEM_TOTAL))
      return HIERA_ERR_CUDA;
    patch_embed_kernel<<<grid, 256, SMEM_TOTAL, stream>>>(
        static_cast<const float*>(img), wt, bias, static_cast<const float*>(pos),
        static_cast<float*>(out), img_side);
  }
  return cudaGetLastError() == cudaSuccess ? HIERA_OK : HIERA_ERR_CUDA;
}

}  // namespace hiera
