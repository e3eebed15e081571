// PatchEmbed + pos_embed + Unroll in one pass ("Phase 4: Hiera Backbone MLX Port",
// Architecture Summary: PatchEmbed is Conv2d(4 -> 112, 7x7, stride 4) reshaped to
// [B, N, C]; a learned pos_embed (1, N, 112) is added; Unroll permutes the tokens).
// Padding 3, so an img x img image gives a (img/4) x (img/4) token grid.
//
// bf16: an implicit GEMM on the tcgen05 tensor cores with fp32 accumulation in TMEM (see
// patch_embed_tc_kernel below): im2col tiles built in shared memory from the NHWC image,
// the weight TMA-loaded once per CTA, bias and pos_embed added in the epilogue with one
// rounding to bf16, the rows stored at their unrolled positions (3 unroll levels) together
// with the LayerNorm partials (mean, M2 per 56-channel half) for block 0's norm1.
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
// Implicit GEMM on the 5th-generation tensor cores. A tile is 128 consecutive output
// pixels of one output row (oy, ox0 .. ox0 + 127) of one image:
//   A [128 pixels][K = 208]   im2col rows, k = (ky * 7 + kx) * 4 + c for k < 196, zero for
//                             196 <= k < 208; built in shared memory by four warps, one
//                             pixel row per thread, in the 128-byte-swizzled K-major layout
//                             (four 64-column blocks); double-buffered
//   W [112][208]              the packed bf16 weight, TMA-loaded once per CTA
//   D [128][112] fp32         13 tcgen05.mma (M = 128, N = 112, K = 16) into one of two TMEM
//                             accumulators
// The epilogue warps (TMEM lane = pixel) add the bias and pos_embed[raster token] in fp32,
// round once to bf16, store the two 56-channel halves at the pixel's unrolled position
// (3 unroll levels) and, when asked, the LayerNorm partial (mean, M2) of each half for
// block 0's norm1.
// Roles (320 threads, persistent CTAs, tiles strided over the grid): warp 0 weight TMA,
// warp 1 TMEM owner and MMA issuer, warps 2-5 im2col, warps 6-9 epilogue.
constexpr int KP = 208;                       // K padded to 13 steps of 16
constexpr int PE_KB = 4;                      // 64-column k-blocks of A and W
constexpr int PE_A_BYTES = PE_KB * 128 * 128; // one A buffer (64 KB)
constexpr int PE_W_BYTES = PE_KB * PATCH_CO * 128;  // 4 x 14 KB
constexpr int PE_OFF_A = 0;
constexpr int PE_OFF_W = 2 * PE_A_BYTES;
constexpr int PE_OFF_BIAS = PE_OFF_W + PE_W_BYTES;
constexpr int PE_OFF_BAR = PE_OFF_BIAS + PATCH_CO * 4;
constexpr int PE_SMEM = PE_OFF_BAR + 128 + 1024;
static_assert((PATCH_CO * 128) % 1024 == 0, "W k-blocks keep 1024-byte alignment");

struct PeParams {
  const bf16* img;
  const float* bias;
  const bf16* pos;
  bf16* out;
  float2* stats_out;
  int img_side, G, M, segs, tiles;
  uint64_t limit_ns;
  unsigned int* status;
};

__global__ void __launch_bounds__(320, 1)
    patch_embed_tc_kernel(const __grid_constant__ CUtensorMap tmW, const PeParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + PE_OFF_BAR);
  uint64_t* w_full = bars;
  uint64_t* a_full = bars + 1;     // [2] count 128: the im2col warps wrote buffer b
  uint64_t* a_empty = a_full + 2;  // [2] the MMAs reading buffer b completed
  uint64_t* acc_full = a_empty + 2;
  uint64_t* acc_empty = acc_full + 2;  // [2] count 128: the epilogue read accumulator a
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* s_bias = reinterpret_cast<float*>(smem + PE_OFF_BIAS);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_local = (int)blockIdx.x < p.tiles
                          ? (p.tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

  if (threadIdx.x == 0) {
    mbar_init(w_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&a_full[i], 128);
      mbar_init(&a_empty[i], 1);
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmW);
  }
  if (warp == 1) {
    tc_alloc(tmem_slot, 256);
    tc_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();  // everything below reads or writes data of earlier kernels
  griddep_launch_dependents();

  // the tile's image, output row and first output column
  auto tile_pos = [&](int tile, int& b, int& oy, int& ox0) {
    const int seg = tile % p.segs, row = tile / p.segs;
    b = row / p.G;
    oy = row - b * p.G;
    ox0 = seg * 128;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ weights (once)
    if (lane == 0 && n_local > 0) {
      mbar_arrive_expect_tx(w_full, PE_W_BYTES);
      for (int kb = 0; kb < PE_KB; ++kb)
        tma_load_2d(smem + PE_OFF_W + kb * PATCH_CO * 128, &tmW, w_full, kb * 64, 0);
      mbar_wait(w_full, 0, p.limit_ns, p.status);  // landed before the CTA can exit
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_local > 0) {
      constexpr uint32_t IDESC = idesc_bf16_f32(128, PATCH_CO);
      bool ok = mbar_wait(w_full, 0, p.limit_ns, p.status, abort_flag);
      const uint64_t adesc0 = smem_desc_sw128(smem_u32(smem + PE_OFF_A));
      const uint64_t wdesc0 = smem_desc_sw128(smem_u32(smem + PE_OFF_W));
      for (int t = 0; ok && t < n_local; ++t) {
        const int b = t & 1;
        if (!mbar_wait(&a_full[b], (uint32_t)((t >> 1) & 1), p.limit_ns, p.status, abort_flag) ||
            !mbar_wait(&acc_empty[b], (uint32_t)(((t >> 1) & 1) ^ 1), p.limit_ns, p.status,
                       abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(128 * b);
#pragma unroll
        for (int st = 0; st < KP / 16; ++st) {
          const int kb = st >> 2, kk = st & 3;
          const uint64_t ad = desc_advance(adesc0, (uint32_t)(b * PE_A_BYTES + kb * 16384 + 32 * kk));
          const uint64_t wd = desc_advance(wdesc0, (uint32_t)(kb * PATCH_CO * 128 + 32 * kk));
          if (st == 0)
            tc_mma_bf16_k<false>(d, ad, wd, IDESC);
          else
            tc_mma_bf16_k<true>(d, ad, wd, IDESC);
        }
        tc_commit(&a_empty[b]);
        tc_commit(&acc_full[b]);
      }
      if (!ok) *abort_flag = 1;
      tc_commit(drain);
      mbar_wait(drain, 0, p.limit_ns, p.status);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ im2col (one pixel per thread)
    const int px = (warp - 2) * 32 + lane;  // pixel of the tile = row of A
    const uint32_t sw = (uint32_t)(px & 7);
    // the padding columns 196..207 (k-block 3, 16-byte chunks 0..1 after the first 4
    // elements) stay zero: the weight is zero there too, but stale shared memory could hold
    // a NaN pattern, and 0 * NaN would not vanish
    for (int b = 0; b < 2; ++b) {
      uint8_t* row = smem + PE_OFF_A + b * PE_A_BYTES + 3 * 16384 + px * 128;
      *reinterpret_cast<uint2*>(row + ((0u ^ sw) << 4) + 8) = make_uint2(0u, 0u);
      *reinterpret_cast<uint4*>(row + ((1u ^ sw) << 4)) = make_uint4(0u, 0u, 0u, 0u);
    }
    for (int t = 0; t < n_local; ++t) {
      const int tile = (int)blockIdx.x + t * (int)gridDim.x;
      const int b = t & 1;
      if (!warp_wait(&a_empty[b], (uint32_t)(((t >> 1) & 1) ^ 1), p.limit_ns, p.status,
                     abort_flag))
        break;
      int bi, oy, ox0;
      tile_pos(tile, bi, oy, ox0);
      const int ix0 = 4 * (ox0 + px) - 3;  // first image column of this pixel's window
      uint8_t* arow = smem + PE_OFF_A + b * PE_A_BYTES + px * 128;
      const bf16* ib = p.img + (long long)bi * p.img_side * p.img_side * CIN;
      // all 49 pixel loads of the window first (one round trip to L2 per tile rather than
      // one per kernel row), then the 49 shared-memory stores
      uint2 v[KSZ * KSZ];
#pragma unroll
      for (int ky = 0; ky < KSZ; ++ky) {
        const int iy = 4 * oy - 3 + ky;
        const bool row_in = iy >= 0 && iy < p.img_side;
        const bf16* irow = ib + (long long)(row_in ? iy : 0) * p.img_side * CIN;
#pragma unroll
        for (int kx = 0; kx < KSZ; ++kx) {
          const int ix = ix0 + kx;
          v[ky * KSZ + kx] = make_uint2(0u, 0u);
          if (row_in && ix >= 0 && ix < p.img_side)
            v[ky * KSZ + kx] = __ldg(reinterpret_cast<const uint2*>(irow + (long long)ix * CIN));
        }
      }
#pragma unroll
      for (int i = 0; i < KSZ * KSZ; ++i) {
        const int k = i * CIN;  // (ky * 7 + kx) * 4, compile-time after unrolling
        const int kb = k >> 6, kc = k & 63;
        *reinterpret_cast<uint2*>(arow + kb * 16384 + ((((uint32_t)(kc >> 3)) ^ sw) << 4) +
                                  (kc & 7) * 2) = v[i];
      }
      fence_proxy_async_smem();  // generic-proxy writes before the tensor core reads them
      mbar_arrive(&a_full[b]);
    }
  } else {
    // ------------------------------------------------------------ epilogue (pixel per thread)
    const int quarter = warp & 3;
    const int px = quarter * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    for (int i = threadIdx.x - 192; i < PATCH_CO; i += 128) s_bias[i] = __ldg(p.bias + i);
    named_bar_sync(1, 128);
    const int N = p.G * p.G;
    for (int t = 0; t < n_local; ++t) {
      const int tile = (int)blockIdx.x + t * (int)gridDim.x;
      const int b = t & 1;
      int bi, oy, ox0;
      tile_pos(tile, bi, oy, ox0);
      const int ox = ox0 + px;
      const bool valid = ox < p.G;
      // pos_embed of this pixel (raster token), in flight while the MMA runs
      uint4 pos4[14];
      const uint4* pr = reinterpret_cast<const uint4*>(
          p.pos + (long long)(oy * p.G + (valid ? ox : 0)) * PATCH_CO);
#pragma unroll
      for (int i = 0; i < 14; ++i) pos4[i] = __ldg(pr + i);
      if (!warp_wait(&acc_full[b], (uint32_t)((t >> 1) & 1), p.limit_ns, p.status, abort_flag))
        break;
      tc_fence_after();
      const int u = unrolled_of_spatial(oy, valid ? ox : 0, 3, p.M);
      bf16* dst = p.out + ((long long)bi * N + u) * PATCH_CO;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t r[56];
        tmem_load<56>(lane_base + (uint32_t)(128 * b + 56 * half), r);
        if (half == 1) {
          tc_fence_before();
          mbar_arrive(&acc_empty[b]);  // accumulator b may take tile t + 2
        }
        float vals[56];
        uint4 pk[7];
#pragma unroll
        for (int c8 = 0; c8 < 7; ++c8) {
          const uint4 pp = pos4[half * 7 + c8];
          const uint32_t pw[4] = {pp.x, pp.y, pp.z, pp.w};
          float f[8];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int c = half * 56 + c8 * 8 + 2 * e;
            f[2 * e] = (__uint_as_float(r[c8 * 8 + 2 * e]) + s_bias[c]) + bf16_lo(pw[e]);
            f[2 * e + 1] = (__uint_as_float(r[c8 * 8 + 2 * e + 1]) + s_bias[c + 1]) + bf16_hi(pw[e]);
          }
          pk[c8] = pack8(f);
          vals[8 * c8 + 0] = bf16_lo(pk[c8].x);
          vals[8 * c8 + 1] = bf16_hi(pk[c8].x);
          vals[8 * c8 + 2] = bf16_lo(pk[c8].y);
          vals[8 * c8 + 3] = bf16_hi(pk[c8].y);
          vals[8 * c8 + 4] = bf16_lo(pk[c8].z);
          vals[8 * c8 + 5] = bf16_hi(pk[c8].z);
          vals[8 * c8 + 6] = bf16_lo(pk[c8].w);
          vals[8 * c8 + 7] = bf16_hi(pk[c8].w);
        }
        if (valid) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + half * 56);
#pragma unroll
          for (int c8 = 0; c8 < 7; ++c8) d4[c8] = pk[c8];
          if (p.stats_out != nullptr) {
            float sm = 0.f;
#pragma unroll
            for (int j = 0; j < 56; ++j) sm += vals[j];
            const float mean = sm * (1.f / 56.f);
            float m2 = 0.f;
#pragma unroll
            for (int j = 0; j < 56; ++j) m2 = fmaf(vals[j] - mean, vals[j] - mean, m2);
            p.stats_out[((long long)bi * N + u) * 2 + half] = make_float2(mean, m2);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tc_dealloc(tmem, 256);
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
    CUtensorMap tmW;
    {
      cuuint64_t dims[2] = {(cuuint64_t)PATCH_KP, (cuuint64_t)PATCH_CO};
      cuuint64_t str[1] = {(cuuint64_t)PATCH_KP * 2};
      cuuint32_t box[2] = {64, (cuuint32_t)PATCH_CO};
      if (!encode_tmap_bf16_sw128(&tmW, w16, 2, dims, str, box)) return HIERA_ERR_CUDA;
    }
    PeParams pp;
    pp.img = static_cast<const bf16*>(img);
    pp.bias = bias;
    pp.pos = static_cast<const bf16*>(pos);
    pp.out = static_cast<bf16*>(out);
    pp.stats_out = stats_out;
    pp.img_side = img_side;
    pp.G = G;
    pp.M = G / 8;
    pp.segs = (G + 127) / 128;
    const long long tiles = (long long)B * G * pp.segs;
    if (tiles > (1ll << 30)) return HIERA_ERR_SHAPE;
    pp.tiles = (int)tiles;
    pp.limit_ns = g_wait_limit_ns();
    pp.status = g_status_ptr();
    if (!ensure_smem_attr(reinterpret_cast<const void*>(patch_embed_tc_kernel), PE_SMEM))
      return HIERA_ERR_CUDA;
    const int grid = (int)(tiles < g_num_sms() ? tiles : g_num_sms());
    launch_k(patch_embed_tc_kernel, dim3(grid), dim3(320), PE_SMEM, stream, tmW, pp);
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
