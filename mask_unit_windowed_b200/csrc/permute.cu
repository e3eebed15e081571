// Unroll / Reroll token permutations ("Phase 4: Hiera Backbone MLX Port", Architecture
// Summary: Unroll permutes tokens for mask-unit windowed attention, Reroll undoes it to
// spatial [B, H, W, C]). Pure copies, one 16-byte vector per thread step, iterated over
// the DESTINATION so stores are fully coalesced; each source row (C * elem bytes) is read
// contiguously by consecutive threads.
#include "common.cuh"
#include "internal.h"

namespace hiera {

template <bool kUnroll>
__global__ void __launch_bounds__(256) permute_kernel(const uint4* __restrict__ src,
                                                      uint4* __restrict__ dst, int B, int G,
                                                      int L, int chunks_per_row,
                                                      long long total) {
  griddep_wait();  // everything below reads or writes data of earlier kernels
  griddep_launch_dependents();
  const int M = G >> L;
  const int N = G * G;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
    const long long row = i / chunks_per_row;
    const int ch = (int)(i - row * chunks_per_row);
    const int b = (int)(row / N);
    const int t = (int)(row - (long long)b * N);
    int s;
    if (kUnroll) {
      s = spatial_of_unrolled(t, L, M, G);          // dst t is unrolled, src raster
    } else {
      s = unrolled_of_spatial(t / G, t % G, L, M);  // dst t is raster, src unrolled
    }
    const uint4 v = __ldg(src + ((long long)b * N + s) * chunks_per_row + ch);
    __stcs(dst + i, v);
  }
}

// Same copy with 32-bit index arithmetic (tensors of fewer than 2^31 vectors), four
// independent vectors in flight per thread; source reads and destination writes bypass
// persistence in L1/L2 (each byte is touched once).
template <bool kUnroll>
__global__ void __launch_bounds__(256) permute32_kernel(const uint4* __restrict__ src,
                                                        uint4* __restrict__ dst, int G, int L,
                                                        int chunks_per_row, int total) {
  griddep_wait();  // everything below reads or writes data of earlier kernels
  griddep_launch_dependents();
  const int M = G >> L;
  const int N = G * G;
  const int stride = gridDim.x * blockDim.x;
  auto src_index = [&](int i) {
    const int row = i / chunks_per_row;
    const int ch = i - row * chunks_per_row;
    const int b = row / N;
    const int t = row - b * N;
    const int sp = kUnroll ? spatial_of_unrolled(t, L, M, G) : unrolled_of_spatial(t / G, t % G, L, M);
    return (b * N + sp) * chunks_per_row + ch;
  };
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  for (; i + 3 * stride < total; i += 4 * stride) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) v[u] = __ldcs(src + src_index(i + u * stride));
#pragma unroll
    for (int u = 0; u < 4; ++u) __stcs(dst + i + u * stride, v[u]);
  }
  for (; i < total; i += stride) __stcs(dst + i, __ldcs(src + src_index(i)));
}

cudaError_t launch_permute(bool unroll, const void* x, void* y, int B, int G, int C, int L,
                           int elem_bytes, cudaStream_t stream) {
  const int chunks = C * elem_bytes / 16;
  const long long total = (long long)B * G * G * chunks;
  if (total == 0) return cudaSuccess;
  long long blocks = (total + 255) / 256;
  const long long cap = (long long)g_num_sms() * 16;
  if (blocks > cap) blocks = cap;
  profile_mark(K_PERMUTE, stream);
  const uint4* src = static_cast<const uint4*>(x);
  uint4* dst = static_cast<uint4*>(y);
  if (total < (1ll << 31)) {
    const int t32 = (int)total;
    long long blocks32 = (total + 4 * 256 - 1) / (4 * 256);
    const long long cap32 = (long long)g_num_sms() * 8;
    if (blocks32 > cap32) blocks32 = cap32;
    if (unroll)
      return launch_k(permute32_kernel<true>, dim3((unsigned)blocks32), dim3(256), 0, stream,
                      src, dst, G, L, chunks, t32);
    return launch_k(permute32_kernel<false>, dim3((unsigned)blocks32), dim3(256), 0, stream,
                    src, dst, G, L, chunks, t32);
  }
  if (unroll)
    return launch_k(permute_kernel<true>, dim3((unsigned)blocks), dim3(256), 0, stream, src,
                    dst, B, G, L, chunks, total);
  return launch_k(permute_kernel<false>, dim3((unsigned)blocks), dim3(256), 0, stream, src, dst,
                  B, G, L, chunks, total);
}

}  // namespace hiera
