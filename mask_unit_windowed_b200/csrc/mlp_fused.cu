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
// fc1 runs up to NB chunks ahead of the epilogue, so the tensor pipe computes the next fc1
// chunks while the epilogue warps turn chunk j into bf16; the producer loads the W2 chunk
// LAG chunks behind the W1 chunk, in the order the two issuers consume them. After the
// last chunk the epilogue adds b2 and the residual, rounds to bf16, stores the tile and
// emits the LayerNorm partials (mean, M2 per row half) of what it stored for the next
// block's norm1.
//
// The order of the tensor-core K steps for every output element is the same as in the
// stand-alone fc1 (K = D in steps of 16) and fc2 (K = 4 D in steps of 16) GEMMs, and the
// fold / GELU / rounding code is shared, so the result is the same as the unfused pair's.
//
// Roles (608 threads, one CTA per SM, row tiles strided over the grid):
//   warp 0      TMA producer: x tile, W1 chunk and W2 chunk rings (128-byte swizzle)
//   warp 1      TMEM owner (all 512 columns), fc1 tcgen05.mma issuer (one thread)
//   warp 2      fc2 tcgen05.mma issuer (one thread)
//   warps 3-18  epilogue, four warps per TMEM lane quarter (a warp reaches only the lanes
//               32 (warp % 4) .. + 31).
//               D = 224: all sixteen take 16 columns of every hidden chunk and one 56-column
//               piece of the output each; the per-row LayerNorm partial of each 112-column
//               half is merged from its two pieces in shared memory, in the order the
//               stand-alone GEMM's epilogue merges them.
//               D = 112: two roles. Eight hidden warps take 32 columns of every hidden
//               chunk; eight output warps take one 56-column piece of the output, from a
//               double-buffered output accumulator, so a tile's output epilogue (bias,
//               residual, rounding, partials, store) runs while the next tile's hidden
//               chunks are produced.
// TMEM: output accumulator(s) at column 0 (D = 112: 0 and 128), fc1 chunk accumulators from
// ACC1_COL.
#include "common.cuh"
#include "internal.h"

namespace hiera {
namespace {

constexpr int BM = 128;
constexpr int HC = 64;  // hidden chunk width
constexpr int EPI_WARPS = 16;
constexpr int EPI_THREADS = EPI_WARPS * 32;
constexpr int THREADS = 96 + EPI_THREADS;

template <int D>
struct MlpCfg {
  static constexpr int HID = 4 * D;
  static constexpr int NC = HID / HC;           // hidden chunks per tile
  static constexpr int KB1 = (D + 63) / 64;     // 64-column k-blocks of x and W1
  static constexpr int K1_STEPS = D / 16;       // fc1 K = 16 steps
  static constexpr int NX = D <= 128 ? 2 : 1;   // x tile buffers
  static constexpr int NB = 4;                  // fc1 accumulators in TMEM
  static constexpr int NH = 2;                  // hidden chunk buffers in shared memory
  // D = 112: the epilogue warps split into eight hidden warps (32 columns of every hidden
  // chunk each) and eight output warps (one 56-column piece each) with a double-buffered
  // output accumulator, so a tile's output epilogue overlaps the next tile's hidden chunks
  static constexpr bool SPLIT = D <= 128;
  static constexpr int S1 = D <= 128 ? 3 : 2;   // W1 chunk ring
  static constexpr int S2 = D <= 128 ? 4 : 2;   // W2 chunk ring
  static constexpr int LAG = D <= 128 ? 2 : 1;  // W2 chunk j is loaded after W1 chunk j + LAG
  static constexpr int X_BYTES = KB1 * BM * 128;
  static constexpr int H_BYTES = BM * 128;
  static constexpr int W1_BYTES = KB1 * HC * 128;
  static constexpr int W2_BYTES = D * 128;
  static constexpr int X_OFF = 0;
  static constexpr int H_OFF = X_OFF + NX * X_BYTES;
  static constexpr int W1_OFF = H_OFF + NH * H_BYTES;
  static constexpr int W2_OFF = W1_OFF + S1 * W1_BYTES;
  static constexpr int STG_OFF = W2_OFF + S2 * W2_BYTES;     // SPLIT: output staging
  static constexpr int STG_BYTES = SPLIT ? 8 * 2048 : 0;     // (8 warps x 16 rows x 128 B)
  static constexpr int CONST_OFF = STG_OFF + STG_BYTES;      // colsum1, colconst1 [HID]
  static constexpr int BAR_OFF = CONST_OFF + 2 * HID * 4;
  static constexpr int SMEM_BYTES = BAR_OFF + 512 + 2 * BM * 8 + 1024;  // + alignment slack
  static constexpr int ACC1_COL = D <= 128 ? 256 : 256;  // (SPLIT: outputs at 0 and 128)
  static constexpr int HID_THREADS = SPLIT ? EPI_THREADS / 2 : EPI_THREADS;  // hidden chunks
  static constexpr int TMEM_COLS = 512;
  static constexpr int PIECES = D / 56;                      // 56-column output pieces per row
  static constexpr int FIN_THREADS = PIECES * 4 * 32;        // threads that read the output
  static constexpr int XCH_OFF = BAR_OFF + 512;              // float2 [2][128] partial exchange
  static_assert(D % 56 == 0 && D % 16 == 0, "D is a multiple of 112");
  static_assert(ACC1_COL >= (SPLIT ? 128 + D : D) && ACC1_COL + NB * HC <= TMEM_COLS,
                "TMEM plan");
  static_assert(!SPLIT || PIECES == 2, "split roles: two output pieces per row");
  static_assert(LAG < S2 && LAG < NB, "issue lag within the rings");
  static_assert(W2_BYTES % 1024 == 0 && X_BYTES % 1024 == 0, "operand alignment");
  static_assert(NH * H_BYTES >= EPI_WARPS * 2048, "output staging aliases the hidden buffers");
  static_assert(PIECES == 2 || PIECES == 4, "output pieces");
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

// Output groups G0 .. G0 + NG - 1 (8 columns each) of a 56-column piece: accumulator + b2 +
// residual (res[g], bf16), rounded; the packed result replaces res[g].
template <int G0, int NG, int NR>
__device__ __forceinline__ void out_groups(const uint32_t (&r)[NR], uint4 (&res)[7],
                                           const float4* b4) {
#pragma unroll
  for (int gg = 0; gg < NG; ++gg) {
    const int g = G0 + gg;
    const uint4 rr = res[g];
    const float4 q0 = __ldg(b4 + 2 * g), q1 = __ldg(b4 + 2 * g + 1);
    float v[8];
    v[0] = __uint_as_float(r[8 * gg + 0]) + q0.x + bf16_lo(rr.x);
    v[1] = __uint_as_float(r[8 * gg + 1]) + q0.y + bf16_hi(rr.x);
    v[2] = __uint_as_float(r[8 * gg + 2]) + q0.z + bf16_lo(rr.y);
    v[3] = __uint_as_float(r[8 * gg + 3]) + q0.w + bf16_hi(rr.y);
    v[4] = __uint_as_float(r[8 * gg + 4]) + q1.x + bf16_lo(rr.z);
    v[5] = __uint_as_float(r[8 * gg + 5]) + q1.y + bf16_hi(rr.z);
    v[6] = __uint_as_float(r[8 * gg + 6]) + q1.z + bf16_lo(rr.w);
    v[7] = __uint_as_float(r[8 * gg + 7]) + q1.w + bf16_hi(rr.w);
    res[g] = pack8(v);
  }
}

template <int D>
__global__ void __launch_bounds__(THREADS, 1)
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
  uint64_t* a2_full = h_empty + C::NH;      // [2] (one used unless SPLIT)
  uint64_t* a2_empty = a2_full + 2;         // [2]
  uint64_t* drain = a2_empty + 2;
  uint64_t* drain2 = drain + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain2 + 1);
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
      mbar_init(&a1_empty[i], C::HID_THREADS);
    }
    for (int i = 0; i < C::NH; ++i) {
      mbar_init(&h_full[i], C::HID_THREADS);
      mbar_init(&h_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&a2_full[i], 1);
      mbar_init(&a2_empty[i], C::FIN_THREADS);
    }
    mbar_init(drain, 1);
    mbar_init(drain2, 1);
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();  // everything below reads or writes data of earlier kernels
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // One thread's TMA loads complete one after another, so the boxes are issued by lanes
    // rotating over 8; every lane walks the same sequence and waits on the same barriers.
    int xs = 0, s1 = 0, s2 = 0, rr = 0;
    uint32_t xph = 0, ph1 = 0, ph2 = 0;
    uint32_t nx = 0, n1 = 0, n2 = 0;  // loads issued per ring
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      if (!warp_wait(&x_empty[xs], xph ^ 1u, p.limit_ns, p.status, abort_flag)) {
        ok = false;
        break;
      }
      if (lane == 0) mbar_arrive_expect_tx(&x_full[xs], C::X_BYTES);
      __syncwarp();
#pragma unroll
      for (int kb = 0; kb < C::KB1; ++kb)
        if (lane == ((rr + kb) & 7))
          tma_load_2d(sX + xs * C::X_BYTES + kb * BM * 128, &tmX, &x_full[xs], kb * 64, tile * BM);
      rr = (rr + C::KB1) & 7;
      ++nx;
      if (++xs == C::NX) {
        xs = 0;
        xph ^= 1u;
      }
      for (int j = 0; j < C::NC + C::LAG && ok; ++j) {
        if (j < C::NC) {
          if (!warp_wait(&w1_empty[s1], ph1 ^ 1u, p.limit_ns, p.status, abort_flag)) {
            ok = false;
            break;
          }
          if (lane == 0) mbar_arrive_expect_tx(&w1_full[s1], C::W1_BYTES);
          __syncwarp();
#pragma unroll
          for (int kb = 0; kb < C::KB1; ++kb)
            if (lane == ((rr + kb) & 7))
              tma_load_2d(sW1 + s1 * C::W1_BYTES + kb * HC * 128, &tmW1, &w1_full[s1], kb * 64,
                          j * HC);
          rr = (rr + C::KB1) & 7;
          ++n1;
          if (++s1 == C::S1) {
            s1 = 0;
            ph1 ^= 1u;
          }
        }
        if (j >= C::LAG) {
          if (!warp_wait(&w2_empty[s2], ph2 ^ 1u, p.limit_ns, p.status, abort_flag)) {
            ok = false;
            break;
          }
          if (lane == 0) mbar_arrive_expect_tx(&w2_full[s2], C::W2_BYTES);
          __syncwarp();
          if (lane == rr)
            tma_load_2d(sW2 + s2 * C::W2_BYTES, &tmW2, &w2_full[s2], (j - C::LAG) * HC, 0);
          rr = (rr + 1) & 7;
          ++n2;
          if (++s2 == C::S2) {
            s2 = 0;
            ph2 ^= 1u;
          }
        }
      }
    }
    if (!ok && lane == 0) {
      *abort_flag = 1;
      // let copies already in flight land before the CTA's shared memory goes away
      for (uint32_t i = nx > (uint32_t)C::NX ? nx - C::NX : 0; i < nx; ++i)
        mbar_wait(&x_full[i % C::NX], (uint32_t)((i / C::NX) & 1), p.limit_ns, p.status);
      for (uint32_t i = n1 > (uint32_t)C::S1 ? n1 - C::S1 : 0; i < n1; ++i)
        mbar_wait(&w1_full[i % C::S1], (uint32_t)((i / C::S1) & 1), p.limit_ns, p.status);
      for (uint32_t i = n2 > (uint32_t)C::S2 ? n2 - C::S2 : 0; i < n2; ++i)
        mbar_wait(&w2_full[i % C::S2], (uint32_t)((i / C::S2) & 1), p.limit_ns, p.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ fc1 issuer
    // Two issuing threads: the issue cost of tcgen05.mma / commit / barrier waits is paid
    // by one thread each for fc1 and fc2. Their MMAs touch disjoint TMEM columns and
    // shared memory, so they need no ordering between them; each commits its own.
    if (lane == 0) {
      constexpr uint32_t IDESC1 = idesc_bf16_f32(BM, HC);
      const uint64_t xdesc0 = smem_desc_sw128(smem_u32(sX));
      const uint64_t w1desc0 = smem_desc_sw128(smem_u32(sW1));
      int xs = 0, s1 = 0;
      uint32_t xph = 0, ph1 = 0, a1 = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        if (!mbar_wait(&x_full[xs], xph, p.limit_ns, p.status, abort_flag)) {
          ok = false;
          break;
        }
        const uint64_t xdesc = desc_advance(xdesc0, (uint32_t)(xs * C::X_BYTES));
        for (int j = 0; j < C::NC; ++j) {
          const int b = (int)(a1 % C::NB);
          if (!mbar_wait(&a1_empty[b], (uint32_t)((a1 / C::NB) & 1) ^ 1u, p.limit_ns, p.status,
                         abort_flag) ||
              !mbar_wait(&w1_full[s1], ph1, p.limit_ns, p.status, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t wdesc = desc_advance(w1desc0, (uint32_t)(s1 * C::W1_BYTES));
          const uint32_t d1 = tmem + (uint32_t)(C::ACC1_COL + b * HC);
          tc_mma_bf16_k<false>(d1, xdesc, wdesc, IDESC1);
#pragma unroll
          for (int ks = 1; ks < C::K1_STEPS; ++ks) {
            const int kb = ks >> 2, kk = ks & 3;
            tc_mma_bf16_k<true>(d1, desc_advance(xdesc, (uint32_t)(kb * BM * 128 + 32 * kk)),
                                desc_advance(wdesc, (uint32_t)(kb * HC * 128 + 32 * kk)), IDESC1);
          }
          tc_commit(&w1_empty[s1]);
          tc_commit(&a1_full[b]);
          ++a1;
          if (++s1 == C::S1) {
            s1 = 0;
            ph1 ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(&x_empty[xs]);
        if (++xs == C::NX) {
          xs = 0;
          xph ^= 1u;
        }
      }
      if (!ok) *abort_flag = 1;
      // no MMA of this thread may still be writing TMEM when it is released
      tc_commit(drain);
      mbar_wait(drain, 0, p.limit_ns, p.status);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ fc2 issuer
    if (lane == 0) {
      constexpr uint32_t IDESC2 = idesc_bf16_f32(BM, D);
      const uint64_t hdesc0 = smem_desc_sw128(smem_u32(sH));
      const uint64_t w2desc0 = smem_desc_sw128(smem_u32(sW2));
      int s2 = 0;
      uint32_t ph2 = 0, hc = 0, t = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++t) {
        for (int i = 0; i < C::NC; ++i) {
          const int hb = (int)(hc % C::NH);
          // the output accumulator is free once the epilogue read it (SPLIT: the one of tile
          // t - 2; otherwise of tile t - 1)
          const int ob = C::SPLIT ? (int)(t & 1u) : 0;
          const uint32_t oph = C::SPLIT ? ((t >> 1) & 1u) : (t & 1u);
          if ((i == 0 && !mbar_wait(&a2_empty[ob], oph ^ 1u, p.limit_ns, p.status, abort_flag)) ||
              !mbar_wait(&h_full[hb], (uint32_t)((hc / C::NH) & 1), p.limit_ns, p.status,
                         abort_flag) ||
              !mbar_wait(&w2_full[s2], ph2, p.limit_ns, p.status, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t hdesc = desc_advance(hdesc0, (uint32_t)(hb * C::H_BYTES));
          const uint64_t w2desc = desc_advance(w2desc0, (uint32_t)(s2 * C::W2_BYTES));
          const uint32_t dout = tmem + (uint32_t)(ob * 128);
          if (i == 0)
            tc_mma_bf16_k<false>(dout, hdesc, w2desc, IDESC2);
          else
            tc_mma_bf16_k<true>(dout, hdesc, w2desc, IDESC2);
#pragma unroll
          for (int kk = 1; kk < HC / 16; ++kk)
            tc_mma_bf16_k<true>(dout, desc_advance(hdesc, 32u * kk), desc_advance(w2desc, 32u * kk),
                                IDESC2);
          tc_commit(&w2_empty[s2]);
          tc_commit(&h_empty[hb]);
          ++hc;
          if (++s2 == C::S2) {
            s2 = 0;
            ph2 ^= 1u;
          }
        }
        if (ok) tc_commit(&a2_full[C::SPLIT ? (int)(t & 1u) : 0]);
      }
      if (!ok) *abort_flag = 1;
      tc_commit(drain2);
      mbar_wait(drain2, 0, p.limit_ns, p.status);
    }
  } else if constexpr (C::SPLIT) {
    // ------------------------------------------------------------ epilogue, split roles
    const int ew = warp - 3;
    const int quarter = warp & 3;  // TMEM lanes 32 quarter .. + 31
    const int cg = ew >> 2;        // 0, 1: output piece cg; 2, 3: hidden column half cg - 2
    const int rt = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    bool ok = true;
    if (cg >= 2) {
      // ---- hidden chunks: fc1 accumulator -> LayerNorm fold -> GELU -> bf16 operand,
      //      32 columns of every chunk per warp
      const int hh = cg - 2;
      uint32_t a1 = 0, hc = 0;
      // the norm2 partials of this thread's row are loaded a tile ahead
      float2 part[8];
      auto load_parts = [&](int tile) {
        const long long m = (long long)tile * BM + rt;
        const float2* sp = p.stats_in + (m < p.M ? m : 0) * p.stats_parts;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          part[j] = j < p.stats_parts ? __ldg(sp + j) : make_float2(0.f, 0.f);
      };
      const LnConsts lnc = ln_consts(p.stats_parts, D);
      if ((int)blockIdx.x < num_tiles) load_parts(blockIdx.x);
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const long long m = (long long)tile * BM + rt;
        float fa = 1.f, fb = 0.f;
        if (m < p.M) ln_merge_parts(part, p.stats_parts, lnc, p.ln_eps, fa, fb);
        if (tile + (int)gridDim.x < num_tiles) load_parts(tile + gridDim.x);
        for (int j = 0; j < C::NC; ++j) {
          const int b = (int)(a1 % C::NB);
          if (!warp_wait(&a1_full[b], (uint32_t)((a1 / C::NB) & 1), p.limit_ns, p.status,
                         abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          uint32_t r[32];
          tmem_load<32>(tmem + lane_base + (uint32_t)(C::ACC1_COL + b * HC + hh * 32), r);
          tc_fence_before();
          mbar_arrive(&a1_empty[b]);
          ++a1;
          const float4* cs4 = reinterpret_cast<const float4*>(c_sum + j * HC + hh * 32);
          const float4* cc4 = reinterpret_cast<const float4*>(c_const + j * HC + hh * 32);
          uint4 pk[4];
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const float4 s0 = cs4[2 * g], s1 = cs4[2 * g + 1];
            const float4 k0 = cc4[2 * g], k1 = cc4[2 * g + 1];
            const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
            const float kv[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
            float v[8];
            const f32x2 fa2 = f2_pack(fa, fa), fb2 = f2_pack(fb, fb);
#pragma unroll
            for (int e = 0; e < 8; e += 2) {  // fold + GELU on pairs (packed fp32)
              const f32x2 x = f2_fma(fa2, f2_pack(__uint_as_float(r[8 * g + e]),
                                                  __uint_as_float(r[8 * g + e + 1])),
                                     f2_fma(fb2, f2_pack(sv[e], sv[e + 1]), f2_pack(kv[e], kv[e + 1])));
              f2_unpack(gelu_fast2(x), v[e], v[e + 1]);
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
            *reinterpret_cast<uint4*>(hrow + (((hh * 4 + g) ^ (rt & 7)) << 4)) = pk[g];
          fence_proxy_async_smem();
          mbar_arrive(&h_full[hb]);
          ++hc;
        }
      }
    } else {
      // ---- output piece [56 cg, 56 cg + 56) of every tile: + b2 + residual, bf16, the
      //      LayerNorm partial of this 56-column half, coalesced store; the accumulator of
      //      tile t is buffer t & 1, so the next tile's fc2 runs meanwhile
      const int c0 = cg * 56;
      uint8_t* stg = smem + C::STG_OFF + (ew << 11);  // 16 rows x 128 B, this warp's own
      uint32_t t = 0;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++t) {
        const long long m = (long long)tile * BM + rt;
        const bool row_ok = m < p.M;
        uint4 res[7];
        const bf16* xrow = p.x + m * D + c0;
#pragma unroll
        for (int i = 0; i < 7; ++i)
          res[i] = row_ok ? __ldg(reinterpret_cast<const uint4*>(xrow) + i) : make_uint4(0u, 0u, 0u, 0u);
        const int ob = (int)(t & 1u);
        if (!warp_wait(&a2_full[ob], (uint32_t)((t >> 1) & 1u), p.limit_ns, p.status,
                       abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float4* b4 = reinterpret_cast<const float4*>(p.bias2 + c0);
        const uint32_t obase = tmem + lane_base + (uint32_t)(ob * 128 + c0);
        {
          uint32_t r[32];
          tmem_load<32>(obase, r);
          out_groups<0, 4>(r, res, b4);
        }
        {
          uint32_t r[24];
          tc_ld_32x32b_x16(obase + 32, *reinterpret_cast<uint32_t(*)[16]>(&r[0]));
          tc_ld_32x32b_x8(obase + 48, *reinterpret_cast<uint32_t(*)[8]>(&r[16]));
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 24; ++i) asm volatile("" : "+r"(r[i]));
          tc_fence_before();
          mbar_arrive(&a2_empty[ob]);
          out_groups<4, 3>(r, res, b4);
        }
        if (p.stats_out != nullptr && row_ok) {
          // statistics of the values as stored (the order every partial's producer uses)
          float st_mean, st_m2;
          stats_piece_bf16<7>(res, st_mean, st_m2);
          p.stats_out[m * 2 + cg] = make_float2(st_mean, st_m2);
        }
        // staging: 16 rows at a time, then 8 lanes per row, 4 rows per store instruction
        const unsigned long long my_dst = reinterpret_cast<unsigned long long>(p.out + m * D + c0);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          if ((lane >> 4) == hh) {
            const int sr = lane & 15;
#pragma unroll
            for (int g = 0; g < 7; ++g)
              *reinterpret_cast<uint4*>(stg + (sr << 7) + ((g ^ (sr & 7)) << 4)) = res[g];
          }
          __syncwarp();
#pragma unroll
          for (int it = 0; it < 4; ++it) {
            const int sr = it * 4 + (lane >> 3), ch = lane & 7;
            const int row = hh * 16 + sr;
            const unsigned long long dst = __shfl_sync(0xffffffffu, my_dst, row);
            const int wr = __shfl_sync(0xffffffffu, row_ok ? 1 : 0, row);
            if (wr && ch < 7) {
              const uint4 val =
                  *reinterpret_cast<const uint4*>(stg + (sr << 7) + ((ch ^ (sr & 7)) << 4));
              *reinterpret_cast<uint4*>(reinterpret_cast<bf16*>(dst) + ch * 8) = val;
            }
          }
          __syncwarp();
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int ew = warp - 3;
    const int quarter = warp & 3;  // TMEM lanes 32 quarter .. + 31
    const int cg = ew >> 2;        // column group: 16 hidden columns / one 56-column piece
    const int rt = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    float2* xch = reinterpret_cast<float2*>(smem + C::XCH_OFF);
    uint32_t a1 = 0, hc = 0, t = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++t) {
      const long long m = (long long)tile * BM + rt;
      const bool row_ok = m < p.M;
      float fa = 1.f, fb = 0.f;
      // (the constants are formed here rather than kept live across the loop: registers)
      if (ok && row_ok)
        ln_fold_coeffs(p.stats_in + m * p.stats_parts, p.stats_parts,
                       ln_consts(p.stats_parts, D), p.ln_eps, fa, fb);
      // ---- hidden chunks: fc1 accumulator -> LayerNorm fold -> GELU -> bf16 operand
      for (int j = 0; j < C::NC && ok; ++j) {
        const int b = (int)(a1 % C::NB);
        if (!warp_wait(&a1_full[b], (uint32_t)((a1 / C::NB) & 1), p.limit_ns, p.status,
                       abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t r[16];
        tmem_load<16>(tmem + lane_base + (uint32_t)(C::ACC1_COL + b * HC + cg * 16), r);
        tc_fence_before();
        mbar_arrive(&a1_empty[b]);
        ++a1;
        const float4* cs4 = reinterpret_cast<const float4*>(c_sum + j * HC + cg * 16);
        const float4* cc4 = reinterpret_cast<const float4*>(c_const + j * HC + cg * 16);
        uint4 pk[2];
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          const float4 s0 = cs4[2 * g], s1 = cs4[2 * g + 1];
          const float4 k0 = cc4[2 * g], k1 = cc4[2 * g + 1];
          const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
          const float kv[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
          float v[8];
          const f32x2 fa2 = f2_pack(fa, fa), fb2 = f2_pack(fb, fb);
#pragma unroll
          for (int e = 0; e < 8; e += 2) {  // fold + GELU on pairs (packed fp32)
            const f32x2 x = f2_fma(fa2, f2_pack(__uint_as_float(r[8 * g + e]),
                                                __uint_as_float(r[8 * g + e + 1])),
                                   f2_fma(fb2, f2_pack(sv[e], sv[e + 1]), f2_pack(kv[e], kv[e + 1])));
            f2_unpack(gelu_fast2(x), v[e], v[e + 1]);
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
        for (int g = 0; g < 2; ++g)
          *reinterpret_cast<uint4*>(hrow + (((cg * 2 + g) ^ (rt & 7)) << 4)) = pk[g];
        fence_proxy_async_smem();
        mbar_arrive(&h_full[hb]);
        ++hc;
      }
      // ---- output piece [56 cg, 56 cg + 56): + b2 + residual, bf16, LayerNorm partial,
      //      coalesced store
      const bool fin = cg < C::PIECES;
      float st_mean = 0.f, st_m2 = 0.f;
      if (fin && ok) {
        const int c0 = cg * 56;
        uint4 res[7];
        const bf16* xrow = p.x + m * D + c0;
#pragma unroll
        for (int i = 0; i < 7; ++i)
          res[i] = row_ok ? __ldg(reinterpret_cast<const uint4*>(xrow) + i) : make_uint4(0u, 0u, 0u, 0u);
        if (!warp_wait(a2_full, (uint32_t)(t & 1), p.limit_ns, p.status, abort_flag)) ok = false;
        if (ok) {
          tc_fence_after();
          const float4* b4 = reinterpret_cast<const float4*>(p.bias2 + c0);
          // columns 0..31 then 32..55 of the piece (fewer live registers); the packed
          // bf16 results replace the residual words in res[]
          {
            uint32_t r[32];
            tmem_load<32>(tmem + lane_base + (uint32_t)c0, r);
            out_groups<0, 4>(r, res, b4);
          }
          {
            uint32_t r[24];
            tc_ld_32x32b_x16(tmem + lane_base + (uint32_t)(c0 + 32),
                             *reinterpret_cast<uint32_t(*)[16]>(&r[0]));
            tc_ld_32x32b_x8(tmem + lane_base + (uint32_t)(c0 + 48),
                            *reinterpret_cast<uint32_t(*)[8]>(&r[16]));
            tc_wait_ld();
#pragma unroll
            for (int i = 0; i < 24; ++i) asm volatile("" : "+r"(r[i]));
            tc_fence_before();
            mbar_arrive(a2_empty);
            out_groups<4, 3>(r, res, b4);
          }
          if (p.stats_out != nullptr) {
            // statistics of the values as stored (the order every partial's producer uses)
            stats_piece_bf16<7>(res, st_mean, st_m2);
          }
          // staging (2 KB per warp, aliasing the idle hidden buffers): 16 rows at a time,
          // then 8 lanes per row, 4 rows per store instruction
          uint8_t* stg = sH + (ew << 11);
          const unsigned long long my_dst =
              reinterpret_cast<unsigned long long>(p.out + m * D + c0);
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            if ((lane >> 4) == hh) {
              const int sr = lane & 15;
#pragma unroll
              for (int g = 0; g < 7; ++g)
                *reinterpret_cast<uint4*>(stg + (sr << 7) + ((g ^ (sr & 7)) << 4)) = res[g];
            }
            __syncwarp();
#pragma unroll
            for (int it = 0; it < 4; ++it) {
              const int sr = it * 4 + (lane >> 3), ch = lane & 7;
              const int row = hh * 16 + sr;
              const unsigned long long dst = __shfl_sync(0xffffffffu, my_dst, row);
              const int wr = __shfl_sync(0xffffffffu, row_ok ? 1 : 0, row);
              if (wr && ch < 7) {
                const uint4 val =
                    *reinterpret_cast<const uint4*>(stg + (sr << 7) + ((ch ^ (sr & 7)) << 4));
                *reinterpret_cast<uint4*>(reinterpret_cast<bf16*>(dst) + ch * 8) = val;
              }
            }
            __syncwarp();
          }
          // LayerNorm partial per 112-column half: D = 112 pieces are halves already; for
          // D = 224 the odd piece hands its (mean, M2) to the even one
          if (p.stats_out != nullptr && C::PIECES == 4 && (cg & 1)) xch[(cg >> 1) * BM + rt] =
              make_float2(st_mean, st_m2);
        }
      }
      if (C::PIECES == 4) named_bar_sync(2, EPI_THREADS);
      if (fin && ok && p.stats_out != nullptr && row_ok) {
        if (C::PIECES == 2) {
          p.stats_out[m * 2 + cg] = make_float2(st_mean, st_m2);
        } else if ((cg & 1) == 0) {
          // Chan et al. merge of the second 56 columns into the first, as the GEMM's
          // epilogue merges its consecutive chunks
          const float2 o = xch[(cg >> 1) * BM + rt];
          const float na = 56.f, nb = 56.f, ntot = na + nb;
          const float dlt = o.x - st_mean;
          const float mean = fmaf(dlt, nb / ntot, st_mean);
          const float m2 = st_m2 + o.y + dlt * dlt * (na * nb / ntot);
          p.stats_out[m * 2 + (cg >> 1)] = make_float2(mean, m2);
        }
      }
      // every epilogue warp is done with the staging area (it aliases the hidden buffers)
      // and the exchange slots before any warp writes the next tile's hidden chunk; taken
      // on every path, so the warps stay matched even after a timeout
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
  if (!ensure_smem_attr(reinterpret_cast<const void*>(kern), C::SMEM_BYTES)) return HIERA_ERR_CUDA;
  const int tiles = (a.M + BM - 1) / BM;
  int grid = g_num_sms();
  if (grid > tiles) grid = tiles;
  profile_mark(K_MLP_FUSED, stream);
  launch_k(kern, dim3(grid), dim3(THREADS), C::SMEM_BYTES, stream, tmX, tmW1, tmW2, p);
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
