// Fused Hiera MLP for the narrow stages ("Phase 4: Hiera Backbone MLX Port",
// Architecture Summary: the block's MLP is fc1 -> GELU -> fc2 with hidden width 4 dim,
// applied to norm2 of the attention residual and added back to it):
//
//   y = x + GELU(LN2(x) W1^T + b1) W2^T + b2     per 128-row tile of x, dim D in {112, 224}
//
// The hidden activation never leaves the SM. It is produced in 64-column chunks:
//   fc1 chunk j   x tile (smem, resident for the tile) x W1 rows [64 j, 64 j + 64)
//                 -> one of NB fp32 accumulators of 64 TMEM columns
//   epilogue      tcgen05.ld, LayerNorm fold (as in the stand-alone GEMM), GELU, bf16,
//                 written to a shared-memory chunk buffer in the tensor-core operand layout
//   fc2 chunk j   hidden chunk (128 x 64) x W2 columns [64 j, 64 j + 64)
//                 -> the D-column fp32 output accumulator in TMEM, accumulated over j
// fc2 of chunk j is issued after fc1 of chunk j + LAG, so the tensor pipe computes the next
// fc1 chunks while the epilogue warps turn chunk j into bf16. After the last chunk the
// epilogue adds b2 and the residual, rounds to bf16, stores the tile and emits the
// LayerNorm partials (mean, M2 per row half) of what it stored for the next block's norm1.
//
// The order of the tensor-core K steps for every output element is the same as in the
// stand-alone fc1 (K = D in steps of 16) and fc2 (K = 4 D in steps of 16) GEMMs, and the
// fold / GELU / rounding code is shared, so the result is the same as the unfused pair's.
//
// Roles (320 threads, one CTA per SM, row tiles strided over the grid):
//   warp 0      TMA producer: x tile, W1 chunk and W2 chunk rings (128-byte swizzle)
//   warp 1      TMEM owner (all 512 columns) and single-thread tcgen05.mma issuer
//   warps 2-9   epilogue, two warps per TMEM lane quarter, each half of the columns
// TMEM: output accumulator at column 0 (D columns), fc1 chunk accumulators from ACC1_COL.
#include "common.cuh"
#include "internal.h"

namespace hiera {
namespace {

constexpr int BM = 128;
constexpr int HC = 64;  // hidden chunk width
constexpr int EPI_WARPS = 8;
constexpr int EPI_THREADS = EPI_WARPS * 32;

template <int D>
struct MlpCfg {
  static constexpr int HID = 4 * D;
  static constexpr int NC = HID / HC;           // hidden chunks per tile
  static constexpr int KB1 = (D + 63) / 64;     // 64-column k-blocks of x and W1
  static constexpr int K1_STEPS = D / 16;       // fc1 K = 16 steps
  static constexpr int NX = D <= 128 ? 2 : 1;   // x tile buffers
  static constexpr int NB = 4;                  // fc1 accumulators in TMEM
  static constexpr int NH = 2;                  // hidden chunk buffers in shared memory
  static constexpr int S1 = D <= 128 ? 4 : 2;   // W1 chunk ring
  static constexpr int S2 = D <= 128 ? 4 : 2;   // W2 chunk ring
  static constexpr int LAG = D <= 128 ? 2 : 1;  // fc2(j) is issued after fc1(j + LAG)
  static constexpr int X_BYTES = KB1 * BM * 128;
  static constexpr int H_BYTES = BM * 128;
  static constexpr int W1_BYTES = KB1 * HC * 128;
  static constexpr int W2_BYTES = D * 128;
  static constexpr int X_OFF = 0;
  static constexpr int H_OFF = X_OFF + NX * X_BYTES;
  static constexpr int W1_OFF = H_OFF + NH * H_BYTES;
  static constexpr int W2_OFF = W1_OFF + S1 * W1_BYTES;
  static constexpr int CONST_OFF = W2_OFF + S2 * W2_BYTES;   // colsum1, colconst1 [HID], b2 [D]
  static constexpr int BAR_OFF = CONST_OFF + (2 * HID + D) * 4;
  static constexpr int SMEM_BYTES = BAR_OFF + 512 + 1024;    // + alignment slack
  static constexpr int ACC1_COL = D <= 128 ? 128 : 256;
  static constexpr int TMEM_COLS = 512;
  static constexpr int HALF = D / 2;                         // output columns per thread
  static_assert(D % 56 == 0 && D % 16 == 0, "D is a multiple of 112");
  static_assert(ACC1_COL >= D && ACC1_COL + NB * HC <= TMEM_COLS, "TMEM plan");
  static_assert(LAG < S2 && LAG < NB, "issue lag within the rings");
  static_assert(W2_BYTES % 1024 == 0 && X_BYTES % 1024 == 0, "operand alignment");
  static_assert(NH * H_BYTES >= EPI_WARPS * 4096, "output staging aliases the hidden buffers");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
  static_assert(NC > LAG, "chunks");
};

struct MlpParams {
  int M;
  const float2* stats_in;  // [M][stats_parts] partial (mean, M2) of x's rows
  int stats_parts;
  float ln_eps;
  const float* colsum1;    // [HID] folded fc1 column sums
  const float* colconst1;  // [HID] folded fc1 constants (beta W1^T + b1)
  const float* bias2;      // [D]
  const bf16* x;           // [M][D] residual (the fc1 input)
  bf16* out;               // [M][D]
  float2* stats_out;       // [M][2] partials of out, or nullptr
  uint64_t limit_ns;
  unsigned int* status;
};

template <int D>
__global__ void __launch_bounds__(320, 1)
    mlp_fused_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW1,
                     const __grid_constant__ CUtensorMap tmW2, const MlpParams p) {
  using C = MlpCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  uint8_t* sX = smem + C::X_OFF;
  uint8_t* sH = smem + C::H_OFF;
  uint8_t* sW1 = smem + C::W1_OFF;
  uint8_t* sW2 = smem + C::W2_OFF;
  float* c_sum = reinterpret_cast<float*>(smem + C::CONST_OFF);
  float* c_const = c_sum + C::HID;
  float* c_bias2 = c_const + C::HID;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* x_full = bars;                  // [NX]
  uint64_t* x_empty = x_full + C::NX;       // [NX]
  uint64_t* w1_full = x_empty + C::NX;      // [S1]
  uint64_t* w1_empty = w1_full + C::S1;     // [S1]
  uint64_t* w2_full = w1_empty + C::S1;     // [S2]
  uint64_t* w2_empty = w2_full + C::S2;     // [S2]
  uint64_t* a1_full = w2_empty + C::S2;     // [NB]
  uint64_t* a1_empty = a1_full + C::NB;     // [NB]
  uint64_t* h_full = a1_empty + C::NB;      // [NH]
  uint64_t* h_empty = h_full + C::NH;       // [NH]
  uint64_t* a2_full = h_empty + C::NH;
  uint64_t* a2_empty = a2_full + 1;
  uint64_t* drain = a2_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_tiles = (p.M + BM - 1) / BM;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NX; ++i) {
      mbar_init(&x_full[i], 1);
      mbar_init(&x_empty[i], 1);
    }
    for (int i = 0; i < C::S1; ++i) {
      mbar_init(&w1_full[i], 1);
      mbar_init(&w1_empty[i], 1);
    }
    for (int i = 0; i < C::S2; ++i) {
      mbar_init(&w2_full[i], 1);
      mbar_init(&w2_empty[i], 1);
    }
    for (int i = 0; i < C::NB; ++i) {
      mbar_init(&a1_full[i], 1);
      mbar_init(&a1_empty[i], EPI_THREADS);
    }
    for (int i = 0; i < C::NH; ++i) {
      mbar_init(&h_full[i], EPI_THREADS);
      mbar_init(&h_empty[i], 1);
    }
    mbar_init(a2_full, 1);
    mbar_init(a2_empty, EPI_THREADS);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW1);
    tma_prefetch_desc(&tmW2);
  }
  if (warp == 1) {
    tc_alloc(tmem_slot, C::TMEM_COLS);
    tc_relinquish();
  }
  for (int i = threadIdx.x; i < C::HID; i += blockDim.x) {
    c_sum[i] = __ldg(p.colsum1 + i);
    c_const[i] = __ldg(p.colconst1 + i);
  }
  for (int i = threadIdx.x; i < D; i += blockDim.x) c_bias2[i] = __ldg(p.bias2 + i);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int xs = 0, s1 = 0, s2 = 0;
      uint32_t xph = 0, ph1 = 0, ph2 = 0;
      long long nx = 0, n1 = 0, n2 = 0;  // loads issued per ring
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        if (!mbar_wait(&x_empty[xs], xph ^ 1u, p.limit_ns, p.status, abort_flag)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&x_full[xs], C::X_BYTES);
#pragma unroll
        for (int kb = 0; kb < C::KB1; ++kb)
          tma_load_2d(sX + xs * C::X_BYTES + kb * BM * 128, &tmX, &x_full[xs], kb * 64, tile * BM);
        ++nx;
        if (++xs == C::NX) {
          xs = 0;
          xph ^= 1u;
        }
        for (int j = 0; j < C::NC + C::LAG && ok; ++j) {
          if (j < C::NC) {
            if (!mbar_wait(&w1_empty[s1], ph1 ^ 1u, p.limit_ns, p.status, abort_flag)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&w1_full[s1], C::W1_BYTES);
#pragma unroll
            for (int kb = 0; kb < C::KB1; ++kb)
              tma_load_2d(sW1 + s1 * C::W1_BYTES + kb * HC * 128, &tmW1, &w1_full[s1], kb * 64,
                          j * HC);
            ++n1;
            if (++s1 == C::S1) {
              s1 = 0;
              ph1 ^= 1u;
            }
          }
          if (j >= C::LAG) {
            if (!mbar_wait(&w2_empty[s2], ph2 ^ 1u, p.limit_ns, p.status, abort_flag)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&w2_full[s2], C::W2_BYTES);
            tma_load_2d(sW2 + s2 * C::W2_BYTES, &tmW2, &w2_full[s2], (j - C::LAG) * HC, 0);
            ++n2;
            if (++s2 == C::S2) {
              s2 = 0;
              ph2 ^= 1u;
            }
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        // let copies already in flight land before the CTA's shared memory goes away
        for (long long i = nx > C::NX ? nx - C::NX : 0; i < nx; ++i)
          mbar_wait(&x_full[i % C::NX], (uint32_t)((i / C::NX) & 1), p.limit_ns, p.status);
        for (long long i = n1 > C::S1 ? n1 - C::S1 : 0; i < n1; ++i)
          mbar_wait(&w1_full[i % C::S1], (uint32_t)((i / C::S1) & 1), p.limit_ns, p.status);
        for (long long i = n2 > C::S2 ? n2 - C::S2 : 0; i < n2; ++i)
          mbar_wait(&w2_full[i % C::S2], (uint32_t)((i / C::S2) & 1), p.limit_ns, p.status);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC1 = idesc_bf16_f32(BM, HC);
      constexpr uint32_t IDESC2 = idesc_bf16_f32(BM, D);
      int xs = 0, s1 = 0, s2 = 0;
      uint32_t xph = 0, ph1 = 0, ph2 = 0;
      long long a1 = 0, hc = 0, t = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++t) {
        if (!mbar_wait(&x_full[xs], xph, p.limit_ns, p.status, abort_flag)) {
          ok = false;
          break;
        }
        const uint32_t xa = smem_u32(sX + xs * C::X_BYTES);
        for (int j = 0; j < C::NC + C::LAG && ok; ++j) {
          if (j < C::NC) {
            const int b = (int)(a1 % C::NB);
            const uint32_t bph = (uint32_t)((a1 / C::NB) & 1);
            if (!mbar_wait(&a1_empty[b], bph ^ 1u, p.limit_ns, p.status, abort_flag) ||
                !mbar_wait(&w1_full[s1], ph1, p.limit_ns, p.status, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t wa = smem_u32(sW1 + s1 * C::W1_BYTES);
            const uint32_t d1 = tmem + (uint32_t)(C::ACC1_COL + b * HC);
#pragma unroll
            for (int ks = 0; ks < C::K1_STEPS; ++ks) {
              const int kb = ks >> 2, kk = ks & 3;
              tc_mma_bf16(d1, smem_desc_sw128(xa + kb * BM * 128) + (uint64_t)(2 * kk),
                          smem_desc_sw128(wa + kb * HC * 128) + (uint64_t)(2 * kk), IDESC1,
                          ks != 0 ? 1u : 0u);
            }
            tc_commit(&w1_empty[s1]);
            tc_commit(&a1_full[b]);
            ++a1;
            if (++s1 == C::S1) {
              s1 = 0;
              ph1 ^= 1u;
            }
            if (j == C::NC - 1) {
              tc_commit(&x_empty[xs]);
              if (++xs == C::NX) {
                xs = 0;
                xph ^= 1u;
              }
            }
          }
          if (j >= C::LAG) {
            const int i = j - C::LAG;
            const int hb = (int)(hc % C::NH);
            const uint32_t hph = (uint32_t)((hc / C::NH) & 1);
            // the output accumulator is free once the previous tile's epilogue read it
            if ((i == 0 && !mbar_wait(a2_empty, (uint32_t)(t & 1) ^ 1u, p.limit_ns, p.status,
                                      abort_flag)) ||
                !mbar_wait(&h_full[hb], hph, p.limit_ns, p.status, abort_flag) ||
                !mbar_wait(&w2_full[s2], ph2, p.limit_ns, p.status, abort_flag)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t ha = smem_u32(sH + hb * C::H_BYTES);
            const uint32_t w2a = smem_u32(sW2 + s2 * C::W2_BYTES);
#pragma unroll
            for (int kk = 0; kk < HC / 16; ++kk)
              tc_mma_bf16(tmem, smem_desc_sw128(ha) + (uint64_t)(2 * kk),
                          smem_desc_sw128(w2a) + (uint64_t)(2 * kk), IDESC2,
                          (i | kk) != 0 ? 1u : 0u);
            tc_commit(&w2_empty[s2]);
            tc_commit(&h_empty[hb]);
            ++hc;
            if (++s2 == C::S2) {
              s2 = 0;
              ph2 ^= 1u;
            }
          }
        }
        if (ok) tc_commit(a2_full);
      }
      if (!ok) *abort_flag = 1;
      // no MMA may still be writing TMEM when it is released
      tc_commit(drain);
      mbar_wait(drain, 0, p.limit_ns, p.status);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 2;
    const int quarter = warp & 3;  // TMEM lanes 32 quarter .. + 31
    const int half = ew >> 2;      // which half of the columns
    const int rt = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    long long a1 = 0, hc = 0, t = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++t) {
      const long long m = (long long)tile * BM + rt;
      const bool row_ok = m < p.M;
      float fa = 1.f, fb = 0.f;
      if (ok && row_ok)
        ln_fold_coeffs(p.stats_in + m * p.stats_parts, p.stats_parts, D, p.ln_eps, fa, fb);
      // ---- hidden chunks: fc1 accumulator -> LayerNorm fold -> GELU -> bf16 operand
      for (int j = 0; j < C::NC && ok; ++j) {
        const int b = (int)(a1 % C::NB);
        if (!warp_wait(&a1_full[b], (uint32_t)((a1 / C::NB) & 1), p.limit_ns, p.status,
                       abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t r[32];
        tmem_load<32>(tmem + lane_base + (uint32_t)(C::ACC1_COL + b * HC + half * 32), r);
        tc_fence_before();
        mbar_arrive(&a1_empty[b]);
        ++a1;
        const float* cs = c_sum + j * HC + half * 32;
        const float* cc = c_const + j * HC + half * 32;
        uint4 pk[4];
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          float v[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int i = 8 * g + e;
            v[e] = gelu_fast(fmaf(fa, __uint_as_float(r[i]), fmaf(fb, cs[i], cc[i])));
          }
          pk[g] = pack8(v);
        }
        const int hb = (int)(hc % C::NH);
        if (!warp_wait(&h_empty[hb], (uint32_t)((hc / C::NH) & 1) ^ 1u, p.limit_ns, p.status,
                       abort_flag)) {
          ok = false;
          break;
        }
        uint8_t* hrow = sH + hb * C::H_BYTES + rt * 128;
#pragma unroll
        for (int g = 0; g < 4; ++g)
          *reinterpret_cast<uint4*>(hrow + (((half * 4 + g) ^ (rt & 7)) << 4)) = pk[g];
        fence_proxy_async_smem();
        mbar_arrive(&h_full[hb]);
        ++hc;
      }
      // ---- output: + b2 + residual, bf16, LayerNorm partials, coalesced store
      if (ok) {
        constexpr int NV = C::HALF / 8;
        uint4 res[NV];
        const bf16* xrow = p.x + m * D + half * C::HALF;
#pragma unroll
        for (int i = 0; i < NV; ++i)
          res[i] = row_ok ? __ldg(reinterpret_cast<const uint4*>(xrow) + i) : make_uint4(0u, 0u, 0u, 0u);
        if (!warp_wait(a2_full, (uint32_t)(t & 1), p.limit_ns, p.status, abort_flag)) ok = false;
        if (ok) {
          tc_fence_after();
          uint8_t* stg = sH + (ew << 12);  // the hidden buffers are idle until the next tile
          float st_mean = 0.f, st_m2 = 0.f;
#pragma unroll
          for (int c = 0; c < C::HALF; c += 56) {
            uint32_t r[56];
            tmem_load<56>(tmem + lane_base + (uint32_t)(half * C::HALF + c), r);
            if (c + 56 == C::HALF) {
              tc_fence_before();
              mbar_arrive(a2_empty);
            }
            float v[56];
#pragma unroll
            for (int g = 0; g < 7; ++g) {
              const uint4 rr = res[c / 8 + g];
              const float* bb = c_bias2 + half * C::HALF + c + 8 * g;
              v[8 * g + 0] = __uint_as_float(r[8 * g + 0]) + bb[0] + bf16_lo(rr.x);
              v[8 * g + 1] = __uint_as_float(r[8 * g + 1]) + bb[1] + bf16_hi(rr.x);
              v[8 * g + 2] = __uint_as_float(r[8 * g + 2]) + bb[2] + bf16_lo(rr.y);
              v[8 * g + 3] = __uint_as_float(r[8 * g + 3]) + bb[3] + bf16_hi(rr.y);
              v[8 * g + 4] = __uint_as_float(r[8 * g + 4]) + bb[4] + bf16_lo(rr.z);
              v[8 * g + 5] = __uint_as_float(r[8 * g + 5]) + bb[5] + bf16_hi(rr.z);
              v[8 * g + 6] = __uint_as_float(r[8 * g + 6]) + bb[6] + bf16_lo(rr.w);
              v[8 * g + 7] = __uint_as_float(r[8 * g + 7]) + bb[7] + bf16_hi(rr.w);
            }
#pragma unroll
            for (int g = 0; g < 7; ++g) {
              const uint4 pkv = pack8(&v[8 * g]);
              *reinterpret_cast<uint4*>(stg + (lane << 7) + ((g ^ (lane & 7)) << 4)) = pkv;
              v[8 * g + 0] = bf16_lo(pkv.x);
              v[8 * g + 1] = bf16_hi(pkv.x);
              v[8 * g + 2] = bf16_lo(pkv.y);
              v[8 * g + 3] = bf16_hi(pkv.y);
              v[8 * g + 4] = bf16_lo(pkv.z);
              v[8 * g + 5] = bf16_hi(pkv.z);
              v[8 * g + 6] = bf16_lo(pkv.w);
              v[8 * g + 7] = bf16_hi(pkv.w);
            }
            if (p.stats_out != nullptr) {
              float s = 0.f;
#pragma unroll
              for (int i = 0; i < 56; ++i) s += v[i];
              const float cmean = s * (1.f / 56.f);
              float cm2 = 0.f;
#pragma unroll
              for (int i = 0; i < 56; ++i) cm2 = fmaf(v[i] - cmean, v[i] - cmean, cm2);
              const float na = (float)c, nb = 56.f, ntot = na + nb;
              const float dlt = cmean - st_mean;
              st_mean = fmaf(dlt, nb / ntot, st_mean);
              st_m2 = st_m2 + cm2 + dlt * dlt * (na * nb / ntot);
            }
            __syncwarp();
            // copy out: 8 lanes per row, 4 rows per instruction
            const unsigned long long my_dst =
                reinterpret_cast<unsigned long long>(p.out + m * D + half * C::HALF + c);
#pragma unroll
            for (int it = 0; it < 8; ++it) {
              const int row = it * 4 + (lane >> 3), ch = lane & 7;
              const unsigned long long dst = __shfl_sync(0xffffffffu, my_dst, row);
              const int wr = __shfl_sync(0xffffffffu, row_ok ? 1 : 0, row);
              if (wr && ch < 7) {
                const uint4 val =
                    *reinterpret_cast<const uint4*>(stg + (row << 7) + ((ch ^ (row & 7)) << 4));
                *reinterpret_cast<uint4*>(reinterpret_cast<bf16*>(dst) + ch * 8) = val;
              }
            }
            __syncwarp();
          }
          if (p.stats_out != nullptr && row_ok)
            p.stats_out[m * 2 + half] = make_float2(st_mean, st_m2);
        }
      }
      // every epilogue warp is done with the staging area (it aliases the hidden buffers)
      // before any warp writes the next tile's hidden chunk; taken on every path, so the
      // warps stay matched even after a timeout
      named_bar_sync(1, EPI_THREADS);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tc_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int D>
hiera_status run_mlp(const MlpArgs& a, cudaStream_t stream) {
  using C = MlpCfg<D>;
  CUtensorMap tmX, tmW1, tmW2;
  {
    cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)a.M};
    cuuint64_t str[1] = {(cuuint64_t)D * 2};
    cuuint32_t box[2] = {64, BM};
    if (!encode_tmap_bf16_sw128(&tmX, a.x, 2, dims, str, box)) return HIERA_ERR_CUDA;
  }
  {
    cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)C::HID};
    cuuint64_t str[1] = {(cuuint64_t)D * 2};
    cuuint32_t box[2] = {64, HC};
    if (!encode_tmap_bf16_sw128(&tmW1, a.w1, 2, dims, str, box)) return HIERA_ERR_CUDA;
  }
  {
    cuuint64_t dims[2] = {(cuuint64_t)C::HID, (cuuint64_t)D};
    cuuint64_t str[1] = {(cuuint64_t)C::HID * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)D};
    if (!encode_tmap_bf16_sw128(&tmW2, a.w2, 2, dims, str, box)) return HIERA_ERR_CUDA;
  }
  MlpParams p;
  p.M = a.M;
  p.stats_in = static_cast<const float2*>(a.stats_in);
  p.stats_parts = a.stats_parts;
  p.ln_eps = a.ln_eps;
  p.colsum1 = a.colsum1;
  p.colconst1 = a.colconst1;
  p.bias2 = a.bias2;
  p.x = static_cast<const bf16*>(a.x);
  p.out = static_cast<bf16*>(a.out);
  p.stats_out = static_cast<float2*>(a.stats_out);
  p.limit_ns = g_wait_limit_ns();
  p.status = g_status_ptr();
  auto kern = mlp_fused_kernel<D>;
  static bool attr_done[64] = {false};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !attr_done[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) !=
        cudaSuccess)
      return HIERA_ERR_CUDA;
    attr_done[dev] = true;
  }
  const int tiles = (a.M + BM - 1) / BM;
  int grid = g_num_sms();
  if (grid > tiles) grid = tiles;
  profile_mark(K_MLP_FUSED, stream);
  kern<<<grid, 320, C::SMEM_BYTES, stream>>>(tmX, tmW1, tmW2, p);
  return cudaGetLastError() == cudaSuccess ? HIERA_OK : HIERA_ERR_CUDA;
}

}  // namespace

bool mlp_fused_supported(int d) { return d == 112 || d == 224; }

hiera_status launch_mlp_fused(const MlpArgs& a, cudaStream_t stream) {
  if (a.M <= 0) return HIERA_OK;
  if (a.stats_in == nullptr || a.stats_parts < 1 || a.stats_parts > 8 ||
      a.D % a.stats_parts != 0 || a.x == nullptr || a.out == nullptr || a.w1 == nullptr ||
      a.w2 == nullptr || a.colsum1 == nullptr || a.colconst1 == nullptr || a.bias2 == nullptr)
    return HIERA_ERR_INVALID_ARG;
  switch (a.D) {
    case 112: return run_mlp<112>(a, stream);
    case 224: return run_mlp<224>(a, stream);
    default: return HIERA_ERR_SHAPE;
  }
}

}  // namespace hiera
