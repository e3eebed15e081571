// fp32 variant of the Hiera block's kernels (true fp32 SIMT arithmetic, no TF32), the
// dtype used where the block must agree with an fp64 evaluation to ~1e-4 absolute.
// Same block as the bf16 path ("Phase 4: Hiera Backbone MLX Port", Architecture
// Summary: HieraBlock, MaskUnitAttention, MLP), organised as plainer steps:
//   row statistics  ->  LayerNorm-folded Linear (q|k|v|proj, token-major, unpooled)
//   -> attention with the q max-pool in its prologue -> proj Linear + residual (the
//   transition residual max-pooled on the fly) -> statistics -> fc1 + GELU -> fc2 + residual.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace hiera {
namespace {

// one warp per row: exact two-pass mean / population variance
__global__ void __launch_bounds__(256) row_stats_kernel(const float* __restrict__ x, int M, int K,
                                                        float eps, float2* __restrict__ stats) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= M) return;
  const float* r = x + (long long)warp * K;
  float s = 0.f;
  for (int k = lane; k < K; k += 32) s += r[k];
  for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float mean = s / (float)K;
  float q = 0.f;
  for (int k = lane; k < K; k += 32) {
    const float d = r[k] - mean;
    q += d * d;
  }
  for (int o = 16; o; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
  if (lane == 0) stats[warp] = make_float2(mean, 1.0f / sqrtf(q / (float)K + eps));
}

constexpr int TB = 64, TK = 16;

// C = A W^T with a 64x64 tile per CTA, 256 threads each owning 4x4 outputs.
__global__ void __launch_bounds__(256) gemm_f32_kernel(const F32GemmArgs p) {
  __shared__ float sA[TK][TB + 4];
  __shared__ float sW[TK][TB + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.y * TB, n0 = blockIdx.x * TB;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < p.K; k0 += TK) {
    for (int i = threadIdx.x; i < TB * TK; i += 256) {
      const int r = i / TK, c = i % TK;
      const int gm = m0 + r, gn = n0 + r, gk = k0 + c;
      sA[c][r] = (gm < p.M && gk < p.K) ? p.A[(long long)gm * p.lda + gk] : 0.f;
      sW[c][r] = (gn < p.N && gk < p.K) ? p.W[(long long)gn * p.K + gk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float a[4], w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = sA[kk][ty * 4 + i];
        w[i] = sW[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], w[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= p.M) continue;
    float2 st = make_float2(0.f, 1.f);
    if (p.stats != nullptr) st = p.stats[m];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= p.N) continue;
      float v = acc[i][j];
      const float cc = p.colconst != nullptr ? p.colconst[n] : 0.f;
      v = (p.stats != nullptr) ? st.y * (v - st.x * p.colsum[n]) + cc : v + cc;
      if (p.gelu) v = gelu_erf(v);
      if (p.residual != nullptr) {
        if (p.resid_pool_tokens > 0) {
          const int per = p.resid_pool_tokens / 4;
          const int b = m / per, np = m - (m / per) * per;
          float r = -INFINITY;
          for (int c = 0; c < 4; ++c)
            r = fmaxf(r, p.residual[((long long)b * p.resid_pool_tokens + c * per + np) * p.ldr + n]);
          v += r;
        } else {
          v += p.residual[(long long)m * p.ldr + n];
        }
      }
      p.out[(long long)m * p.ldo + n] = v;
    }
  }
}

constexpr int QPB = 32;   // queries per CTA
constexpr int KT = 64;    // keys per tile
constexpr int HD = 56;

// grid (units = B*nW*heads, ceil(Tq/32)); 8 warps x 4 queries
__global__ void __launch_bounds__(256) attention_f32_kernel(const F32AttnArgs p) {
  __shared__ float sq[QPB][HD + 1];
  __shared__ float sk[KT][HD + 1];
  __shared__ float sv[KT][HD + 1];
  const int unit = blockIdx.x;
  const int h = unit % p.heads;
  const int w = (unit / p.heads) % p.nW;
  const int b = unit / (p.heads * p.nW);
  const int Tkv = p.tokens / p.nW;
  const int Tq = Tkv / p.q_stride;
  const int q0 = blockIdx.y * QPB;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float scale = 1.0f / sqrtf((float)HD);
  const float* Tb = p.T + (long long)b * p.tokens * p.ldT;

  // prologue: queries, max-pooled over the q_stride outermost chunks of the window
  for (int i = threadIdx.x; i < QPB * HD; i += 256) {
    const int qi = i / HD, e = i % HD;
    const int jq = q0 + qi;
    float v = 0.f;
    if (jq < Tq) {
      v = -INFINITY;
      for (int c = 0; c < p.q_stride; ++c) {
        const int j = c * Tq + jq;
        v = fmaxf(v, Tb[(long long)(j * p.nW + w) * p.ldT + p.q_off + h * HD + e]);
      }
    }
    sq[qi][e] = v;
  }
  float m[4], l[4], o0[4], o1[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    m[i] = -INFINITY;
    l[i] = 0.f;
    o0[i] = 0.f;
    o1[i] = 0.f;
  }
  for (int t0 = 0; t0 < Tkv; t0 += KT) {
    __syncthreads();
    for (int i = threadIdx.x; i < KT * HD; i += 256) {
      const int kk = i / HD, e = i % HD;
      const int j = t0 + kk;
      float kv = 0.f, vv = 0.f;
      if (j < Tkv) {
        const long long row = (long long)(j * p.nW + w) * p.ldT;
        kv = Tb[row + p.k_off + h * HD + e];
        vv = Tb[row + p.v_off + h * HD + e];
      }
      sk[kk][e] = kv;
      sv[kk][e] = vv;
    }
    __syncthreads();
#pragma unroll
    for (int qi = 0; qi < 4; ++qi) {
      const int ql = warp * 4 + qi;
      float s0 = 0.f, s1 = 0.f;
      for (int e = 0; e < HD; ++e) {
        const float qv = sq[ql][e];
        s0 = fmaf(qv, sk[lane][e], s0);
        s1 = fmaf(qv, sk[lane + 32][e], s1);
      }
      s0 = (t0 + lane < Tkv) ? s0 * scale : -INFINITY;
      s1 = (t0 + lane + 32 < Tkv) ? s1 * scale : -INFINITY;
      float mx = fmaxf(s0, s1);
      for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float mn = fmaxf(m[qi], mx);
      const float alpha = expf(m[qi] - mn);
      const float p0 = expf(s0 - mn), p1 = expf(s1 - mn);
      float ps = p0 + p1;
      for (int o = 16; o; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
      l[qi] = l[qi] * alpha + ps;
      m[qi] = mn;
      float a0 = o0[qi] * alpha, a1 = o1[qi] * alpha;
      for (int kk = 0; kk < KT; ++kk) {
        const float pk = __shfl_sync(0xffffffffu, kk < 32 ? p0 : p1, kk & 31);
        a0 = fmaf(pk, sv[kk][lane], a0);
        if (lane + 32 < HD) a1 = fmaf(pk, sv[kk][lane + 32], a1);
      }
      o0[qi] = a0;
      o1[qi] = a1;
    }
  }
  const int Nq = Tq * p.nW;
#pragma unroll
  for (int qi = 0; qi < 4; ++qi) {
    const int jq = q0 + warp * 4 + qi;
    if (jq >= Tq) continue;
    float* dst = p.o + ((long long)b * Nq + (long long)jq * p.nW + w) * p.d_out + h * HD;
    dst[lane] = o0[qi] / l[qi];
    if (lane + 32 < HD) dst[lane + 32] = o1[qi] / l[qi];
  }
}

}  // namespace

hiera_status launch_row_stats_f32(const float* x, int M, int K, float eps, float2* stats,
                                  cudaStream_t stream) {
  if (M <= 0) return HIERA_OK;
  const long long threads = (long long)M * 32;
  profile_mark(K_F32_STATS, stream);
  row_stats_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, stream>>>(x, M, K, eps, stats);
  return cudaGetLastError() == cudaSuccess ? HIERA_OK : HIERA_ERR_CUDA;
}

hiera_status launch_gemm_f32(const F32GemmArgs& a, cudaStream_t stream) {
  if (a.M <= 0 || a.N <= 0) return HIERA_OK;
  dim3 grid((a.N + TB - 1) / TB, (a.M + TB - 1) / TB);
  if (grid.y > 65535) return HIERA_ERR_SHAPE;
  profile_mark(K_F32_GEMM, stream);
  gemm_f32_kernel<<<grid, 256, 0, stream>>>(a);
  return cudaGetLastError() == cudaSuccess ? HIERA_OK : HIERA_ERR_CUDA;
}

hiera_status launch_attention_f32(const F32AttnArgs& a, cudaStream_t stream) {
  const int units = a.B * a.nW * a.heads;
  const int Tq = a.tokens / a.nW / a.q_stride;
  if (units <= 0 || Tq <= 0) return HIERA_OK;
  dim3 grid(units, (Tq + QPB - 1) / QPB);
  if (grid.y > 65535) return HIERA_ERR_SHAPE;
  profile_mark(K_F32_ATTN, stream);
  attention_f32_kernel<<<grid, 256, 0, stream>>>(a);
  return cudaGetLastError() == cudaSuccess ? HIERA_OK : HIERA_ERR_CUDA;
}

}  // namespace hiera
