// Per-row LayerNorm statistics of a bf16 [M, K] matrix as (mean, M2) partials, for block
// inputs that no kernel of this library produced (the first LayerNorm of a standalone
// block call). One warp per row, 16-byte loads, exact two-pass mean and sum of squared
// deviations in fp32 (plan, Sub-phase 4a item 7: HieraBlock starts with norm1).
#include "common.cuh"
#include "internal.h"

namespace hiera {
namespace {

__global__ void __launch_bounds__(256) row_partials_bf16_kernel(const bf16* __restrict__ x, int M,
                                                                int K, float2* __restrict__ out) {
  griddep_wait();  // everything below reads or writes data of earlier kernels
  griddep_launch_dependents();
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= M) return;
  const uint4* r = reinterpret_cast<const uint4*>(x + (long long)row * K);
  const int nv = K / 8;
  float s = 0.f;
  for (int i = lane; i < nv; i += 32) {
    const uint4 v = __ldg(r + i);
    s += bf16_lo(v.x) + bf16_hi(v.x) + bf16_lo(v.y) + bf16_hi(v.y) + bf16_lo(v.z) +
         bf16_hi(v.z) + bf16_lo(v.w) + bf16_hi(v.w);
  }
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float mean = s / (float)K;
  float q = 0.f;
  for (int i = lane; i < nv; i += 32) {
    const uint4 v = __ldg(r + i);
    const float e[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                        bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
#pragma unroll
    for (int j = 0; j < 8; ++j) q = fmaf(e[j] - mean, e[j] - mean, q);
  }
  for (int o = 16; o; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
  if (lane == 0) out[row] = make_float2(mean, q);
}

}  // namespace

hiera_status launch_row_partials_bf16(const void* x, int M, int K, float2* out,
                                      cudaStream_t stream) {
  if (M <= 0) return HIERA_OK;
  if (K % 8 != 0) return HIERA_ERR_SHAPE;
  const long long threads = (long long)M * 32;
  profile_mark(K_ROW_STATS, stream);
  const cudaError_t e =
      launch_k(row_partials_bf16_kernel, dim3((unsigned)((threads + 255) / 256)), dim3(256), 0,
               stream, static_cast<const bf16*>(x), M, K, out);
  return e == cudaSuccess ? HIERA_OK : HIERA_ERR_CUDA;
}

}  // namespace hiera
