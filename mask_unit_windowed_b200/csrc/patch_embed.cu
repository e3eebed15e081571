// PatchEmbed + pos_embed + Unroll in one pass ("Phase 4: Hiera Backbone MLX Port",
// Architecture Summary: PatchEmbed is Conv2d(4 -> 112, 7x7, stride 4) reshaped to
// [B, N, C]; a learned pos_embed (1, N, 112) is added; Unroll permutes the tokens).
// Padding 3, so an img x img image gives a (img/4) x (img/4) token grid.
//
// A CTA computes ROWS output rows x 128 output columns of one image. Per output row the
// 7 input rows it needs (x range of the 128 outputs plus the 3-pixel halo) are staged in
// shared memory as fp32 channel planes; the kernel weights live in shared memory as fp32
// [196][112] (k = (ky*7 + kx)*4 + c). Thread = (output pixel, half of the 112 channels):
// 56 fp32 accumulators, weights read as warp-wide broadcasts. The epilogue adds bias and
// pos_embed[raster token] and stores the row at its unrolled position (3 unroll levels).
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

template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) {
  return v;
}
template <>
__device__ __forceinline__ float to_f<bf16>(bf16 v) {
  return __bfloat162float(v);
}

template <typename T>
__global__ void __launch_bounds__(256, 1) patch_embed_kernel(const T* __restrict__ img,
                                                             const float* __restrict__ wt,
                                                             const float* __restrict__ bias,
                                                             const T* __restrict__ pos,
                                                             T* __restrict__ out,
                                                             float2* __restrict__ stats_out,
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
        const T* src = img + (((long long)b * img_side + iy) * img_side + ix) * CIN;
#pragma unroll
        for (int c = 0; c < CIN; ++c) v[c] = to_f(src[c]);
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
      const T* pr = pos + (long long)t * COUT + half * 56;
      T* dst = out + ((long long)b * N + u) * COUT + half * 56;
#pragma unroll
      for (int j = 0; j < 56; ++j) {
        const float v = acc[j] + __ldg(bias + half * 56 + j) + to_f(pr[j]);
        if constexpr (sizeof(T) == 2) {
          const bf16 rv = __float2bfloat16_rn(v);
          dst[j] = rv;
          acc[j] = __bfloat162float(rv);  // the value as stored, for the statistics below
        } else {
          dst[j] = v;
        }
      }
      if (stats_out != nullptr) {
        // partial (mean, M2) of this half of the token, for the first block's norm1
        float s = 0.f;
#pragma unroll
        for (int j = 0; j < 56; ++j) s += acc[j];
        const float mean = s * (1.f / 56.f);
        float m2 = 0.f;
#pragma unroll
        for (int j = 0; j < 56; ++j) m2 = fmaf(acc[j] - mean, acc[j] - mean, m2);
        stats_out[((long long)b * N + u) * 2 + half] = make_float2(mean, m2);
      }
    }
  }
}

}  // namespace

hiera_status launch_patch_embed(const void* img, const void* w, const float* b, const void* pos,
                                void* out, float2* stats_out, int B, int img_side,
                                int dtype_bf16, cudaStream_t stream) {
  const int G = img_side / 4;
  dim3 grid((G + SEG - 1) / SEG, (G + ROWS - 1) / ROWS, B);
  if (grid.y > 65535 || grid.z > 65535) return HIERA_ERR_SHAPE;
  static bool attr_done[2][64] = {{false}};
  int dev = 0;
  cudaGetDevice(&dev);
  profile_mark(K_PATCH_EMBED, stream);
  if (dtype_bf16) {
    if (dev < 64 && !attr_done[1][dev]) {
      if (cudaFuncSetAttribute(patch_embed_kernel<bf16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               SMEM_TOTAL) != cudaSuccess)
        return HIERA_ERR_CUDA;
      attr_done[1][dev] = true;
    }
    patch_embed_kernel<bf16><<<grid, 256, SMEM_TOTAL, stream>>>(
        static_cast<const bf16*>(img), static_cast<const float*>(w), b,
        static_cast<const bf16*>(pos), static_cast<bf16*>(out), stats_out, img_side);
  } else {
    if (dev < 64 && !attr_done[0][dev]) {
      if (cudaFuncSetAttribute(patch_embed_kernel<float>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               SMEM_TOTAL) != cudaSuccess)
        return HIERA_ERR_CUDA;
      attr_done[0][dev] = true;
    }
    patch_embed_kernel<float><<<grid, 256, SMEM_TOTAL, stream>>>(
        static_cast<const float*>(img), static_cast<const float*>(w), b,
        static_cast<const float*>(pos), static_cast<float*>(out), nullptr, img_side);
  }
  return cudaGetLastError() == cudaSuccess ? HIERA_OK : HIERA_ERR_CUDA;
}

}  // namespace hiera
