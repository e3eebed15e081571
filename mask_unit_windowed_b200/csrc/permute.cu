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
  if (unroll)
    return launch_k(permute_kernel<true>, dim3((unsigned)blocks), dim3(256), 0, stream, src,
                    dst, B, G, L, chunks, total);
  return launch_k(permute_kernel<false>, dim3((unsigned)blocks), dim3(256), 0, stream, src, dst,
                  B, G, L, chunks, total);
}

}  // namespace hiera
