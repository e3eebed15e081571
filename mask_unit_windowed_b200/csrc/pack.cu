// Weight packing, run once per set of weights.
//
// LayerNorm fold: a LayerNorm (gamma, beta) followed by a Linear (W [N, K], b) equals
//   LN(x) W^T + b = rstd * (x W'^T - mean * s) + c,
//   W'_nk = W_nk * gamma_k,  s_n = sum_k W'_nk,  c_n = b_n + sum_k beta_k W_nk,
// with mean / rstd the row statistics of x. s is summed over the W' values exactly as
// stored (after rounding to the operand dtype) so that x W'^T - mean * s is the GEMM of
// the centred row up to accumulation rounding.
#include "common.cuh"
#include "internal.h"

namespace hiera {
namespace {

template <typename T>
__device__ __forceinline__ float ld(const T* p, long long i);
template <>
__device__ __forceinline__ float ld<float>(const float* p, long long i) {
  return p[i];
}
template <>
__device__ __forceinline__ float ld<bf16>(const bf16* p, long long i) {
  return __bfloat162float(p[i]);
}

__device__ __forceinline__ float round_to(float v, float*) { return v; }
__device__ __forceinline__ float round_to(float v, bf16*) {
  return __bfloat162float(__float2bfloat16_rn(v));
}
__device__ __forceinline__ void st(float* p, long long i, float v) { p[i] = v; }
__device__ __forceinline__ void st(bf16* p, long long i, float v) { p[i] = __float2bfloat16_rn(v); }

// one warp per output row n
template <typename T>
__global__ void __launch_bounds__(256) fold_pack_kernel(const T* __restrict__ w,
                                                        const T* __restrict__ gamma,
                                                        const T* __restrict__ beta,
                                                        const T* __restrict__ bias, int N, int K,
                                                        T* __restrict__ w_out,
                                                        float* __restrict__ colsum,
                                                        float* __restrict__ colconst) {
  const int n = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (n >= N) return;
  float s = 0.f, c = 0.f;
  for (int k = lane; k < K; k += 32) {
    const float wv = ld(w, (long long)n * K + k);
    const float g = gamma != nullptr ? ld(gamma, k) : 1.f;
    const float folded = round_to(wv * g, (T*)nullptr);
    st(w_out, (long long)n * K + k, folded);
    s += folded;
    if (beta != nullptr) c = fmaf(ld(beta, k), wv, c);
  }
  for (int o = 16; o; o >>= 1) {
    s += __shfl_xor_sync(0xffffffffu, s, o);
    c += __shfl_xor_sync(0xffffffffu, c, o);
  }
  if (lane == 0) {
    colsum[n] = s;
    colconst[n] = c + (bias != nullptr ? ld(bias, n) : 0.f);
  }
}

template <typename T>
__global__ void __launch_bounds__(256) copy_pack_kernel(const T* __restrict__ w,
                                                        const T* __restrict__ bias, long long NK,
                                                        int N, T* __restrict__ w_out,
                                                        float* __restrict__ bias_out) {
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < NK; i += stride)
    w_out[i] = w[i];
  if (bias_out == nullptr) return;  // plain copy (no bias vector to convert)
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < N; i += stride)
    bias_out[i] = bias != nullptr ? ld(bias, i) : 0.f;
}

// OHWI [112][7][7][4] kernel -> fp32 [196][112] (k = (ky*7 + kx)*4 + c), bias -> fp32, and
// a bf16 [112][208] copy (k fastest, zero-padded) for the tensor-core patch embedding
template <typename T>
__global__ void __launch_bounds__(256) patch_pack_kernel(const T* __restrict__ w,
                                                         const T* __restrict__ bias,
                                                         float* __restrict__ wt,
                                                         float* __restrict__ bias_out,
                                                         bf16* __restrict__ w16) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < PATCH_CO * PATCH_K) {
    const int k = i / PATCH_CO, co = i - (i / PATCH_CO) * PATCH_CO;
    wt[i] = ld(w, (long long)co * PATCH_K + k);
  }
  if (i < PATCH_CO * PATCH_KP) {
    const int co = i / PATCH_KP, k = i - (i / PATCH_KP) * PATCH_KP;
    w16[i] = __float2bfloat16_rn(k < PATCH_K ? ld(w, (long long)co * PATCH_K + k) : 0.f);
  }
  if (i < PATCH_CO) bias_out[i] = bias != nullptr ? ld(bias, i) : 0.f;
}

}  // namespace

hiera_status launch_patch_pack(const void* w, const void* bias, int dtype_bf16, void* packed,
                               cudaStream_t stream) {
  uint8_t* pk = static_cast<uint8_t*>(packed);
  float* wt = reinterpret_cast<float*>(pk);
  float* bias_out = reinterpret_cast<float*>(pk + PATCH_OFF_BIAS);
  bf16* w16 = reinterpret_cast<bf16*>(pk + PATCH_OFF_W16);
  const unsigned blocks = (PATCH_CO * PATCH_KP + 255) / 256;
  profile_mark(K_PACK, stream);
  if (dtype_bf16)
    patch_pack_kernel<bf16><<<blocks, 256, 0, stream>>>(static_cast<const bf16*>(w),
                                                        static_cast<const bf16*>(bias), wt,
                                                        bias_out, w16);
  else
    patch_pack_kernel<float><<<blocks, 256, 0, stream>>>(static_cast<const float*>(w),
                                                         static_cast<const float*>(bias), wt,
                                                         bias_out, w16);
  return cudaGetLastError() == cudaSuccess ? HIERA_OK : HIERA_ERR_CUDA;
}

hiera_status launch_fold_pack(const void* w, const void* gamma, const void* beta,
                              const void* bias, int N, int K, int dtype_bf16, void* w_out,
                              float* colsum, float* colconst, cudaStream_t stream) {
  if (N <= 0 || K <= 0) return HIERA_OK;
  const unsigned blocks = (unsigned)(((long long)N * 32 + 255) / 256);
  profile_mark(K_PACK, stream);
  if (dtype_bf16)
    fold_pack_kernel<bf16><<<blocks, 256, 0, stream>>>(
        static_cast<const bf16*>(w), static_cast<const bf16*>(gamma),
        static_cast<const bf16*>(beta), static_cast<const bf16*>(bias), N, K,
        static_cast<bf16*>(w_out), colsum, colconst);
  else
    fold_pack_kernel<float><<<blocks, 256, 0, stream>>>(
        static_cast<const float*>(w), static_cast<const float*>(gamma),
        static_cast<const float*>(beta), static_cast<const float*>(bias), N, K,
        static_cast<float*>(w_out), colsum, colconst);
  return cudaGetLastError() == cudaSuccess ? HIERA_OK : HIERA_ERR_CUDA;
}

hiera_status launch_copy_pack(const void* w, const void* bias, int N, int K, int dtype_bf16,
                              void* w_out, float* bias_out, cudaStream_t stream) {
  const long long NK = (long long)N * K;
  if (NK <= 0) return HIERA_OK;
  long long blocks = (NK + 255) / 256;
  if (blocks > 4096) blocks = 4096;
  profile_mark(K_PACK, stream);
  if (dtype_bf16)
    copy_pack_kernel<bf16><<<(unsigned)blocks, 256, 0, stream>>>(
        static_cast<const bf16*>(w), static_cast<const bf16*>(bias), NK, N,
        static_cast<bf16*>(w_out), bias_out);
  else
    copy_pack_kernel<float><<<(unsigned)blocks, 256, 0, stream>>>(
        static_cast<const float*>(w), static_cast<const float*>(bias), NK, N,
        static_cast<float*>(w_out), bias_out);
  return cudaGetLastError() == cudaSuccess ? HIERA_OK : HIERA_ERR_CUDA;
}

}  // namespace hiera
