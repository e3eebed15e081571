// The attention half of a stage-0 Hiera block in one kernel ("Phase 4: Hiera Backbone MLX
// Port", Sub-phase 4a item 7, HieraBlock, and Architecture Summary, MaskUnitAttention):
//
//   x1 = x + proj(MaskUnitAttention(norm1(x)))      dim 112, 2 heads of 56, windows of 64
//
// for every token, plus the LayerNorm partials (mean, M2 per 56-channel half) of x1 that the
// fused MLP's norm2 consumes. q, k, v and the attention output never leave the SM: one tile
// is two mask-unit windows (128 tokens) of one image, and per tile
//   1. a 4-D TMA box over (channel, window, in-window index, image) brings the 128 token
//      rows (row r = 2 j + window, j the in-window index), and 13 + 7 tcgen05.mma compute
//      [q | k | v] = x W1'^T (norm1 folded into W1', as in the stand-alone qkv GEMM) into TMEM;
//   2. eight epilogue warps apply the LayerNorm fold (row statistics merged from the partials
//      the producer of x wrote), round to bf16 and write per-head q, k, v tiles into shared
//      memory in the tensor-core operand layouts (v with its ones channel 56);
//   3. S_h = q_h k_h^T over the tile's 128 keys; a row attends only to the keys of its own
//      window (the keys of the same parity), one exact softmax pass, the weights cut to bf16
//      and written over S; O_h = P_h V_h with V read as an MN-major operand, so O's column 56
//      holds the softmax denominator;
//   4. the normalised heads are merged in shared memory (the proj operand), proj = o Wo^T,
//      and the epilogue adds the bias and the residual x, rounds to bf16, stores x1 at the
//      tokens' positions and writes the norm2 partials.
// Every formula (K order of each product, fold, exponent, truncating pack, normalisation,
// epilogue rounding) is the one the separate qkv GEMM, windowed attention and proj GEMM
// use; only the summation order inside the P V product differs (the two windows' keys are
// interleaved), so the result agrees with the unfused path to rounding.
// Roles (320 threads, persistent CTAs, tiles strided over the grid): warp 0 TMA producer
// (the q, k, v and proj weights once per CTA, resident in shared memory; the x tile of each
// tile, whose buffer then holds q, so the next x loads as soon as the scores are computed),
// warp 1 TMEM owner and MMA issuer, warps 2-9 epilogue / softmax (two per TMEM lane quarter:
// head or column half 0 and 1). The merged heads are written over k, which the scores no
// longer need.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace hiera {
namespace {

constexpr int FD = 112;                        // dim
constexpr int FW_BYTES = 2 * FD * 128;          // one 112-row weight chunk, two 64-column blocks
constexpr int FX_BYTES = 2 * 128 * 128;         // [128 rows][two 64-column blocks]
constexpr int FH_BYTES = 128 * 128;             // one head's [128 rows][64] operand tile
constexpr int F_OFF_X = 0;                      // x, then q (per head)
constexpr int F_OFF_K = F_OFF_X + FX_BYTES;     // k (per head), then the merged heads
constexpr int F_OFF_V = F_OFF_K + 2 * FH_BYTES;
constexpr int F_OFF_W = F_OFF_V + 2 * FH_BYTES; // W_q, W_k, W_v, W_o, resident
constexpr int F_OFF_C = F_OFF_W + 4 * FW_BYTES;           // colsum1[336], colconst1[336], bo[112]
constexpr int F_OFF_BAR = F_OFF_C + (2 * 3 * FD + FD) * 4;
constexpr int F_SMEM = F_OFF_BAR + 256 + 1024;
// TMEM: q, k, v accumulators at 0, 128, 256; then S_h at 128 h and O_h at 256 + 64 h;
// proj at 384
constexpr uint32_t F_PROJ_COL = 384;
static_assert(F_OFF_W % 1024 == 0 && FW_BYTES % 1024 == 0, "operand alignment");

struct FParams {
  const bf16* x;
  const float2* stats_in;  // [B * N][stats_parts] partials of x's rows
  int stats_parts;
  const float* colsum1;    // [336]
  const float* colconst1;  // [336]
  const float* bias_o;     // [112]
  bf16* x1;                // [B, N, 112]
  float2* stats_out;       // [B * N][2]
  int N, nW, tiles;
  float ln_eps, sl2;
  uint64_t limit_ns;
  unsigned int* status;
};

__device__ __forceinline__ uint32_t pack_trunc2(float lo, float hi) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(d) : "r"(__float_as_uint(lo)), "r"(__float_as_uint(hi)));
  return d;
}

__global__ void __launch_bounds__(320, 1)
    attn_block_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW1,
                      const __grid_constant__ CUtensorMap tmWo, const FParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + F_OFF_BAR);
  uint64_t* x_full = bars;
  uint64_t* x_empty = x_full + 1;       // the scores have consumed q (written over x)
  uint64_t* w_full = x_empty + 1;
  uint64_t* qkv_done = w_full + 1;
  uint64_t* qkv_staged = qkv_done + 1;  // 256
  uint64_t* s_full = qkv_staged + 1;
  uint64_t* p_full = s_full + 1;        // 256
  uint64_t* o_full = p_full + 1;
  uint64_t* o_staged = o_full + 1;      // 256
  uint64_t* proj_full = o_staged + 1;
  uint64_t* proj_read = proj_full + 1;  // 256
  uint64_t* drain = proj_read + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* c_sum = reinterpret_cast<float*>(smem + F_OFF_C);
  float* c_const = c_sum + 3 * FD;
  float* c_bo = c_const + 3 * FD;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_local = (int)blockIdx.x < p.tiles
                          ? (p.tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  const int pairs = p.nW >> 1;  // window pairs (tiles) per image

  if (threadIdx.x == 0) {
    mbar_init(x_full, 1);
    mbar_init(x_empty, 1);
    mbar_init(w_full, 1);
    mbar_init(qkv_done, 1);
    mbar_init(qkv_staged, 256);
    mbar_init(s_full, 1);
    mbar_init(p_full, 256);
    mbar_init(o_full, 1);
    mbar_init(o_staged, 256);
    mbar_init(proj_full, 1);
    mbar_init(proj_read, 256);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW1);
    tma_prefetch_desc(&tmWo);
  }
  if (warp == 1) {
    tc_alloc(tmem_slot, 512);
    tc_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();  // everything below reads or writes data of earlier kernels
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && n_local > 0) {
      // the four weight chunks once: W_q, W_k, W_v (rows of the packed qkv weight), W_o
      mbar_arrive_expect_tx(w_full, 4 * FW_BYTES);
      for (int g = 0; g < 4; ++g) {
        uint8_t* dst = smem + F_OFF_W + g * FW_BYTES;
        const CUtensorMap* map = g < 3 ? &tmW1 : &tmWo;
        const int row0 = g < 3 ? g * FD : 0;
        tma_load_2d(dst, map, w_full, 0, row0);
        tma_load_2d(dst + FD * 128, map, w_full, 64, row0);
      }
      int issued = 0;
      for (int t = 0; t < n_local; ++t) {
        const int tile = (int)blockIdx.x + t * (int)gridDim.x;
        const int b = tile / pairs, w0 = 2 * (tile - b * pairs);
        if (!mbar_wait(x_empty, (uint32_t)((t & 1) ^ 1), p.limit_ns, p.status, abort_flag)) {
          *abort_flag = 1;
          break;
        }
        uint8_t* xd = smem + F_OFF_X;
        mbar_arrive_expect_tx(x_full, FX_BYTES);
        tma_load_4d(xd, &tmX, x_full, 0, w0, 0, b);
        tma_load_4d(xd + 128 * 128, &tmX, x_full, 64, w0, 0, b);
        ++issued;
      }
      // the copies in flight land before the CTA's shared memory goes away
      mbar_wait(w_full, 0, p.limit_ns, p.status);
      if (issued > 0) mbar_wait(x_full, (uint32_t)((issued - 1) & 1), p.limit_ns, p.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_112 = idesc_bf16_f32(128, FD);
      constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128);
      constexpr uint32_t IDESC_O = idesc_bf16_f32(128, 64) | IDESC_B_MN_MAJOR;
      const uint64_t desc0 = smem_desc_sw128(smem_u32(smem));
      bool ok = true;
      if (n_local > 0) ok = mbar_wait(w_full, 0, p.limit_ns, p.status, abort_flag);
      // D[tmem] = A[128 x 112] W_g[112 x 112]^T: 7 K steps over two 64-column blocks
      auto gemm112 = [&](uint32_t d, uint32_t a_off, int g) {
        const uint32_t w_off = (uint32_t)(F_OFF_W + g * FW_BYTES);
#pragma unroll
        for (int st = 0; st < FD / 16; ++st) {
          const uint32_t kb = (uint32_t)(st >> 2), kk = (uint32_t)(st & 3);
          const uint64_t ad = desc_advance(desc0, a_off + kb * 16384u + 32u * kk);
          const uint64_t wd = desc_advance(desc0, w_off + kb * (uint32_t)(FD * 128) + 32u * kk);
          if (st == 0)
            tc_mma_bf16_k<false>(d, ad, wd, IDESC_112);
          else
            tc_mma_bf16_k<true>(d, ad, wd, IDESC_112);
        }
      };
      for (int t = 0; ok && t < n_local; ++t) {
        const uint32_t ph = (uint32_t)(t & 1);
        const uint32_t x_off = (uint32_t)F_OFF_X;
        if (!mbar_wait(x_full, ph, p.limit_ns, p.status, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // (the previous tile's O was read before its merged heads were staged, which the
        // previous iteration waited for: TMEM columns 0..383 are free)
        for (int g = 0; g < 3; ++g) gemm112(tmem + (uint32_t)(128 * g), x_off, g);
        tc_commit(qkv_done);
        // S_h = q_h k_h^T
        if (!mbar_wait(qkv_staged, ph, p.limit_ns, p.status, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint64_t qd = desc_advance(desc0, x_off + (uint32_t)(h * FH_BYTES));
          const uint64_t kd = desc_advance(desc0, (uint32_t)(F_OFF_K + h * FH_BYTES));
          const uint32_t sd = tmem + (uint32_t)(128 * h);
          tc_mma_bf16_k<false>(sd, qd, kd, IDESC_S);
#pragma unroll
          for (int kk = 1; kk < 4; ++kk)
            tc_mma_bf16_k<true>(sd, desc_advance(qd, 32u * kk), desc_advance(kd, 32u * kk), IDESC_S);
        }
        tc_commit(x_empty);  // q consumed: the next x may overwrite it
        tc_commit(s_full);
        // O_h = P_h V_h (P over the S columns, 128 keys in 64 columns)
        if (!mbar_wait(p_full, ph, p.limit_ns, p.status, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint64_t vd = smem_desc_sw128_mn64(smem_u32(smem + F_OFF_V + h * FH_BYTES));
          const uint32_t pa = tmem + (uint32_t)(128 * h);
          const uint32_t od = tmem + 256u + (uint32_t)(64 * h);
          tc_mma_bf16_ta<false>(od, pa, vd, IDESC_O);
#pragma unroll
          for (int kk = 1; kk < 8; ++kk)
            tc_mma_bf16_ta<true>(od, pa + 8u * kk, desc_advance(vd, 2048u * kk), IDESC_O);
        }
        tc_commit(o_full);
        // proj = o Wo^T, once the merged heads are staged and the previous proj was read
        if (!mbar_wait(o_staged, ph, p.limit_ns, p.status, abort_flag) ||
            (t > 0 && !mbar_wait(proj_read, ph ^ 1u, p.limit_ns, p.status, abort_flag))) {
          ok = false;
          break;
        }
        tc_fence_after();
        gemm112(tmem + F_PROJ_COL, (uint32_t)F_OFF_K, 3);  // merged heads over k, W_o
        tc_commit(proj_full);
      }
      if (!ok) *abort_flag = 1;
      tc_commit(drain);
      mbar_wait(drain, 0, p.limit_ns, p.status);
    }
  } else {
    // ------------------------------------------------------------ epilogue / softmax warps
    const int quarter = warp & 3;
    const int hs = (warp - 2) >> 2;            // head (steps 2-3) or column half (step 4)
    const int r = quarter * 32 + lane;         // tile row = TMEM lane
    const int par = r & 1, jr = r >> 1;        // window within the pair, in-window index
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const float sl2 = p.sl2;
    for (int i = threadIdx.x - 64; i < 3 * FD; i += 256) {
      c_sum[i] = __ldg(p.colsum1 + i);
      c_const[i] = __ldg(p.colconst1 + i);
    }
    for (int i = threadIdx.x - 64; i < FD; i += 256) c_bo[i] = __ldg(p.bias_o + i);
    named_bar_sync(1, 256);
    // the norm1 partials of this thread's row are loaded a tile ahead
    auto tok_of = [&](int tt) -> long long {
      const int tile = (int)blockIdx.x + tt * (int)gridDim.x;
      const int b = tile / pairs, w0 = 2 * (tile - b * pairs);
      return (long long)b * p.N + (long long)jr * p.nW + w0 + par;
    };
    float2 part[8];
    auto load_parts = [&](int tt) {
      const float2* sp = p.stats_in + tok_of(tt) * p.stats_parts;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        part[j] = j < p.stats_parts ? __ldg(sp + j) : make_float2(0.f, 0.f);
    };
    const LnConsts lnc = ln_consts(p.stats_parts, FD);
    if (n_local > 0) load_parts(0);
    for (int t = 0; t < n_local; ++t) {
      const int tile = (int)blockIdx.x + t * (int)gridDim.x;
      const int b = tile / pairs, w0 = 2 * (tile - b * pairs);
      const long long tok = (long long)b * p.N + (long long)jr * p.nW + w0 + par;
      const uint32_t ph = (uint32_t)(t & 1);
      uint8_t* xq = smem + F_OFF_X;  // q (written over x)
      uint8_t* om = smem + F_OFF_K;  // the merged heads (written over k)
      float fa = 1.f, fb = 0.f;
      ln_merge_parts(part, p.stats_parts, lnc, p.ln_eps, fa, fb);
      if (t + 1 < n_local) load_parts(t + 1);
      // ---- 2. q, k, v of head hs: fold, bf16, operand tiles
      if (!warp_wait(qkv_done, ph, p.limit_ns, p.status, abort_flag)) break;
      tc_fence_after();
#pragma unroll 1
      for (int g = 0; g < 3; ++g) {
        uint32_t rr[56];
        tmem_load<56>(lane_base + (uint32_t)(128 * g + 56 * hs), rr);
        const float4* cs4 = reinterpret_cast<const float4*>(c_sum + g * FD + 56 * hs);
        const float4* cc4 = reinterpret_cast<const float4*>(c_const + g * FD + 56 * hs);
        uint8_t* row = (g == 0 ? xq : smem + (g == 1 ? F_OFF_K : F_OFF_V)) + hs * FH_BYTES + r * 128;
#pragma unroll
        for (int c8 = 0; c8 < 7; ++c8) {
          float v[8];
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const float4 s4 = cs4[2 * c8 + h2], k4 = cc4[2 * c8 + h2];
            const float sc[4] = {s4.x, s4.y, s4.z, s4.w};
            const float kc[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
            for (int e = 0; e < 4; e += 2)  // the fold on pairs (packed fp32, the scalar bits)
              f2_unpack(f2_fma(f2_pack(fa, fa),
                               f2_pack(__uint_as_float(rr[8 * c8 + 4 * h2 + e]),
                                       __uint_as_float(rr[8 * c8 + 4 * h2 + e + 1])),
                               f2_fma(f2_pack(fb, fb), f2_pack(sc[e], sc[e + 1]),
                                      f2_pack(kc[e], kc[e + 1]))),
                        v[4 * h2 + e], v[4 * h2 + e + 1]);
          }
          *reinterpret_cast<uint4*>(row + (((uint32_t)c8 ^ (uint32_t)(r & 7)) << 4)) = pack8(v);
        }
        // channels 56..63: zero padding for q and k, v's ones channel 56 (softmax denominator)
        *reinterpret_cast<uint4*>(row + ((7u ^ (uint32_t)(r & 7)) << 4)) =
            make_uint4(g == 2 ? 0x3F80u : 0u, 0u, 0u, 0u);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(qkv_staged);
      // ---- 3. softmax of head hs over the row's own window (keys of the same parity)
      if (!warp_wait(s_full, ph, p.limit_ns, p.status, abort_flag)) break;
      tc_fence_after();
      {
        const uint32_t sc = lane_base + (uint32_t)(128 * hs);
        float own[64];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t ld[32];
          tc_ld_32x32b_x32(sc + (uint32_t)(32 * c), ld);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            asm volatile("" : "+r"(ld[2 * i]), "+r"(ld[2 * i + 1]));
            own[16 * c + i] = __uint_as_float(par ? ld[2 * i + 1] : ld[2 * i]);
          }
        }
        float m = own[0];
#pragma unroll
        for (int i = 1; i < 64; ++i) m = fmaxf(m, own[i]);
        const float ms = m * sl2;
        // key 2u + par of the tile is in-window key u; the pair's other key gets weight 0
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t pw[32];
#pragma unroll
          for (int u = 0; u < 32; u += 2) {
            float x0, x1;  // two keys' exponents in one packed FMA
            f2_unpack(f2_fma(f2_pack(own[32 * hh + u], own[32 * hh + u + 1]), f2_pack(sl2, sl2),
                             f2_pack(-ms, -ms)), x0, x1);
            const float e0 = ex2_approx(x0), e1 = ex2_approx(x1);
            pw[u] = par ? pack_trunc2(0.f, e0) : pack_trunc2(e0, 0.f);
            pw[u + 1] = par ? pack_trunc2(0.f, e1) : pack_trunc2(e1, 0.f);
          }
          tc_st_32x32b_x32(sc + (uint32_t)(32 * hh), pw);
        }
        tc_wait_st();
      }
      tc_fence_before();
      mbar_arrive(p_full);
      // the residual of this row's column half, in flight while P V and the merge run
      uint4 res[7];
      const uint4* xr = reinterpret_cast<const uint4*>(p.x + tok * FD + 56 * hs);
#pragma unroll
      for (int i = 0; i < 7; ++i) res[i] = __ldg(xr + i);
      // ---- 4a. normalised head hs into the merged-heads operand (channels 56 hs ..)
      if (!warp_wait(o_full, ph, p.limit_ns, p.status, abort_flag)) break;
      tc_fence_after();
      {
        uint32_t ov[64];
        tc_ld_32x32b_x32(lane_base + 256u + (uint32_t)(64 * hs), *reinterpret_cast<uint32_t(*)[32]>(&ov[0]));
        tc_ld_32x32b_x32(lane_base + 256u + (uint32_t)(64 * hs + 32), *reinterpret_cast<uint32_t(*)[32]>(&ov[32]));
        tc_wait_ld();
#pragma unroll
        for (int i = 0; i < 64; ++i) asm volatile("" : "+r"(ov[i]));
        const float inv = 1.f / __uint_as_float(ov[56]);
#pragma unroll
        for (int c8 = 0; c8 < 7; ++c8) {
          float f[8];
#pragma unroll
          for (int e = 0; e < 8; e += 2)
            f2_unpack(f2_mul(f2_pack(__uint_as_float(ov[8 * c8 + e]), __uint_as_float(ov[8 * c8 + e + 1])),
                             f2_pack(inv, inv)), f[e], f[e + 1]);
          const int ch = 7 * hs + c8;  // 16-byte chunk of the 112-channel row
          *reinterpret_cast<uint4*>(om + (ch >> 3) * 16384 + r * 128 +
                                    ((((uint32_t)ch & 7u) ^ (uint32_t)(r & 7)) << 4)) = pack8(f);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(o_staged);
      // ---- 4b. proj + bias + residual, bf16, x1 and its norm2 partial (column half hs)
      if (!warp_wait(proj_full, ph, p.limit_ns, p.status, abort_flag)) break;
      tc_fence_after();
      {
        uint32_t rr[56];
        tmem_load<56>(lane_base + F_PROJ_COL + (uint32_t)(56 * hs), rr);
        tc_fence_before();
        mbar_arrive(proj_read);
        float v[56];
        // the proj bias of this column half, four per 16-byte shared-memory load (every lane
        // reads the same address: one broadcast per load; 56 hs floats is 16-byte aligned)
        const float4* bo4 = reinterpret_cast<const float4*>(c_bo + 56 * hs);
        // (proj + bias) + residual on pairs (packed fp32, the scalar bits)
#pragma unroll
        for (int g = 0; g < 14; ++g) {
          const float4 b4 = bo4[g];
          f2_unpack(f2_add(f2_pack(__uint_as_float(rr[4 * g + 0]), __uint_as_float(rr[4 * g + 1])),
                           f2_pack(b4.x, b4.y)), v[4 * g + 0], v[4 * g + 1]);
          f2_unpack(f2_add(f2_pack(__uint_as_float(rr[4 * g + 2]), __uint_as_float(rr[4 * g + 3])),
                           f2_pack(b4.z, b4.w)), v[4 * g + 2], v[4 * g + 3]);
        }
#pragma unroll
        for (int g = 0; g < 7; ++g) {
          const uint32_t rw[4] = {res[g].x, res[g].y, res[g].z, res[g].w};
#pragma unroll
          for (int q = 0; q < 4; ++q)
            f2_unpack(f2_add(f2_pack(v[8 * g + 2 * q], v[8 * g + 2 * q + 1]),
                             f2_pack(bf16_lo(rw[q]), bf16_hi(rw[q]))),
                      v[8 * g + 2 * q], v[8 * g + 2 * q + 1]);
        }
        uint4* dst = reinterpret_cast<uint4*>(p.x1 + tok * FD + 56 * hs);
#pragma unroll
        for (int g = 0; g < 7; ++g) {
          const uint4 pk = pack8(&v[8 * g]);
          dst[g] = pk;
          v[8 * g + 0] = bf16_lo(pk.x);
          v[8 * g + 1] = bf16_hi(pk.x);
          v[8 * g + 2] = bf16_lo(pk.y);
          v[8 * g + 3] = bf16_hi(pk.y);
          v[8 * g + 4] = bf16_lo(pk.z);
          v[8 * g + 5] = bf16_hi(pk.z);
          v[8 * g + 6] = bf16_lo(pk.w);
          v[8 * g + 7] = bf16_hi(pk.w);
        }
        if (p.stats_out != nullptr) {
          // (mean, M2) of the 56 stored values, four interleaved accumulators per sum so the
          // additions are not one serial chain
          float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int i = 0; i < 56; ++i) s4[i & 3] += v[i];
          const float mean = ((s4[0] + s4[1]) + (s4[2] + s4[3])) * (1.f / 56.f);
          float q4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int i = 0; i < 56; ++i) q4[i & 3] = fmaf(v[i] - mean, v[i] - mean, q4[i & 3]);
          const float m2 = (q4[0] + q4[1]) + (q4[2] + q4[3]);
          p.stats_out[tok * 2 + hs] = make_float2(mean, m2);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tc_dealloc(tmem, 512);
  }
}

}  // namespace

bool attention_block_supported(int B, int tokens, int d_in, int d_out, int heads, int q_stride,
                               int window_tokens, int mask_unit_attn) {
  if (!mask_unit_attn || d_in != FD || d_out != FD || heads != 2 || q_stride != 1 ||
      window_tokens != 64 || tokens % 64 != 0)
    return false;
  const int nW = tokens / 64;
  return B >= 1 && nW % 2 == 0;
}

hiera_status launch_attention_block(const AttnBlockArgs& a, cudaStream_t stream) {
  const int nW = a.tokens / 64;
  CUtensorMap tmX, tmW1, tmWo;
  {
    // x viewed as (channel, window, in-window index, image): token n = j * nW + w
    cuuint64_t dims[4] = {(cuuint64_t)FD, (cuuint64_t)nW, 64, (cuuint64_t)a.B};
    cuuint64_t str[3] = {(cuuint64_t)FD * 2, (cuuint64_t)nW * FD * 2, (cuuint64_t)a.tokens * FD * 2};
    cuuint32_t box[4] = {64, 2, 64, 1};
    if (!encode_tmap_bf16_sw128(&tmX, a.x, 4, dims, str, box)) return HIERA_ERR_CUDA;
  }
  {
    cuuint64_t dims[2] = {(cuuint64_t)FD, (cuuint64_t)(3 * FD)};
    cuuint64_t str[1] = {(cuuint64_t)FD * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)FD};
    if (!encode_tmap_bf16_sw128(&tmW1, a.w1, 2, dims, str, box)) return HIERA_ERR_CUDA;
  }
  {
    cuuint64_t dims[2] = {(cuuint64_t)FD, (cuuint64_t)FD};
    cuuint64_t str[1] = {(cuuint64_t)FD * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)FD};
    if (!encode_tmap_bf16_sw128(&tmWo, a.wo, 2, dims, str, box)) return HIERA_ERR_CUDA;
  }
  FParams p;
  p.x = static_cast<const bf16*>(a.x);
  p.stats_in = static_cast<const float2*>(a.stats_in);
  p.stats_parts = a.stats_parts;
  p.colsum1 = a.colsum1;
  p.colconst1 = a.colconst1;
  p.bias_o = a.bias_o;
  p.x1 = static_cast<bf16*>(a.x1);
  p.stats_out = static_cast<float2*>(a.stats_out);
  p.N = a.tokens;
  p.nW = nW;
  const long long tiles = (long long)a.B * (nW / 2);
  if (tiles > (1ll << 30)) return HIERA_ERR_SHAPE;
  p.tiles = (int)tiles;
  p.ln_eps = a.ln_eps;
  p.sl2 = (float)(1.4426950408889634 / sqrt(56.0));
  p.limit_ns = g_wait_limit_ns();
  p.status = g_status_ptr();
  if (!ensure_smem_attr(reinterpret_cast<const void*>(attn_block_kernel), F_SMEM))
    return HIERA_ERR_CUDA;
  const int grid = (int)(tiles < g_num_sms() ? tiles : g_num_sms());
  if (grid <= 0) return HIERA_OK;
  profile_mark(K_ATTN_BLOCK, stream);
  launch_k(attn_block_kernel, dim3(grid), dim3(320), F_SMEM, stream, tmX, tmW1, tmWo, p);
  return cudaGetLastError() == cudaSuccess ? HIERA_OK : HIERA_ERR_CUDA;
}

}  // namespace hiera
