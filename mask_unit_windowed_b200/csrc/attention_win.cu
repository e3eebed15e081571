// Tensor-core (tcgen05) attention for small mask-unit windows ("Phase 4: Hiera Backbone MLX
// Port", Architecture Summary, MaskUnitAttention: scaled dot-product attention inside each
// mask-unit window, q max-pooled at transitions, heads merged before proj).
//
// A window holds at most 64 keys (stage 0: 64 keys and 64 queries; the stage-1 transition:
// 64 keys, 16 pooled queries; stage 1: 16 and 16), so one 128-key tile holds the keys of
// U = 128 / TKV whole (image, window, head) units and the softmax is a single exact pass,
// with no running max. A tile stacks the U units' queries in U row slots (TQ rows each, or
// 32 rows of which TQ are used when TQ < 32 <= TKV, so that a warp never holds two units'
// keys) and their keys in 128 columns:
//   S = Q K^T     M = 128, N = 128, K = 64: unit i's rows meet every unit's keys, and only
//                 the diagonal block [i*TQ, +TQ) x [i*TKV, +TKV) is used;
//   P             per row, 2^(s*log2(e)/sqrt(56) - m) over its own unit's keys and exactly 0
//                 elsewhere, cut to bf16 pairs and stored into the S columns it came from;
//   O = P V       M = 128, N = 64, K = 128, P read from TMEM, V in its natural [keys][64]
//                 layout as an MN-major B operand. v's channel 56 holds 1, so O's column 56
//                 is each row's softmax denominator, summed from the very bf16 P values the
//                 tensor core used.
// Roles (persistent CTAs, tiles strided over the grid):
//   warp 0      TMA: Q (R rows), K and V (128 rows each) of a tile into a 4-stage ring;
//   warp 1      TMEM owner and MMA issuer; S of tile t+1 is issued before P V of tile t;
//   warps 2-5   softmax and output of even tiles (TMEM buffer 0), warps 6-9 of odd tiles
//               (buffer 1), one tile row per thread (TMEM lane = row).
// Units past the end of the tensors arrive as TMA zero fill and are not stored.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace hiera {
namespace {

constexpr int WIN_STAGES = 4;
constexpr int WQ_BYTES = 128 * 128;   // Q tile buffer (R <= 128 rows of 64 bf16)
constexpr int WK_BYTES = 128 * 128;   // 128 keys x 64 channels
constexpr int WSTAGE_BYTES = WQ_BYTES + 2 * WK_BYTES;
constexpr int WOFF_BAR = WIN_STAGES * WSTAGE_BYTES;
constexpr int WSMEM_BYTES = WOFF_BAR + 256 + 1024;
constexpr uint32_t WTMEM_COLS = 512;  // buffer b: S/P at 256 b, O at 256 b + 128

struct WParams {
  int units, nW, heads, d_out;
  float sl2;  // log2(e) / sqrt(56)
  bf16* o;
  uint64_t limit_ns;
  unsigned int* status;
};

__device__ __forceinline__ bool wwait(uint64_t* bar, uint32_t parity, const WParams& p,
                                      volatile int* abort_flag) {
  int ok = mbar_wait(bar, parity, p.limit_ns, p.status, abort_flag) ? 1 : 0;
  ok = __all_sync(0xffffffffu, ok);
  if (!ok) *abort_flag = 1;
  return ok != 0;
}

__device__ __forceinline__ void tc_st_32x32b_x16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

// Softmax weights in [0, 1] to a bf16 pair by truncation (high halves, lo first).
__device__ __forceinline__ uint32_t pack_trunc(float lo, float hi) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(d) : "r"(__float_as_uint(lo)), "r"(__float_as_uint(hi)));
  return d;
}

template <int TQ, int TKV>
struct WinCfg {
  static_assert(TKV >= 4 && TKV <= 64 && (TKV & (TKV - 1)) == 0, "window keys");
  static_assert(TQ == TKV || TQ * 4 == TKV, "q_stride 1 or 4");
  // Rows per unit: TQ, or a 32-row slot (one unit per warp, TQ rows used) when a unit has
  // fewer than 32 queries but 32 or more keys, so that no warp reads two units' keys.
  static constexpr bool SLOT = TQ < 32 && TKV >= 32;
  static constexpr int SR = SLOT ? 32 : TQ;
  static constexpr int U = (128 / SR < 128 / TKV) ? 128 / SR : 128 / TKV;  // units per tile
  static constexpr int R = U * SR;                            // tile rows in use
  static constexpr int CW = SR >= 32 ? TKV : TKV * 32 / TQ;   // S columns one warp reads
  static constexpr int Q_TX = U * TQ * 128;                   // Q bytes per tile
  static_assert(CW >= 32 && CW <= 128 && 128 % CW == 0, "warp column window");
  static_assert(U * TKV <= 128 && R <= 128, "tile");
};

template <int TQ, int TKV>
__global__ void __launch_bounds__(320, 1)
    attn_win_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const WParams p) {
  using C = WinCfg<TQ, TKV>;
  constexpr int U = C::U, R = C::R, CW = C::CW, SR = C::SR;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + WOFF_BAR);
  uint64_t* full = bars;                    // [WIN_STAGES]
  uint64_t* empty = full + WIN_STAGES;      // [WIN_STAGES]
  uint64_t* s_full = empty + WIN_STAGES;    // [2] per TMEM buffer
  uint64_t* p_full = s_full + 2;
  uint64_t* o_full = p_full + 2;
  uint64_t* t_free = o_full + 2;
  uint64_t* drain = t_free + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = (p.units + U - 1) / U;
  const int n_local = (int)blockIdx.x < n_tiles ? (n_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < WIN_STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 128);
      mbar_init(&o_full[b], 1);
      mbar_init(&t_free[b], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tc_alloc(tmem_slot, WTMEM_COLS);
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
    long long issued = 0;
    bool ok = true;
    for (int t = 0; t < n_local; ++t) {
      const int tile = (int)blockIdx.x + t * (int)gridDim.x;
      const int s = t % WIN_STAGES;
      if (!wwait(&empty[s], (uint32_t)(((t / WIN_STAGES) & 1) ^ 1), p, abort_flag)) {
        ok = false;
        break;
      }
      uint8_t* st = smem + s * WSTAGE_BYTES;
      if (lane == 0) mbar_arrive_expect_tx(&full[s], C::Q_TX + 2 * WK_BYTES);
      __syncwarp();
      if constexpr (C::SLOT) {
        // unit u's TQ query rows into its 32-row slot (4 KB apart: the swizzle pattern of
        // every slot starts on a 1024-byte boundary)
        if (lane >= 3 && lane < 3 + U)
          tma_load_2d(st + (lane - 3) * SR * 128, &tmQ, &full[s], 0, (tile * U + lane - 3) * TQ);
      } else {
        if (lane == 0) tma_load_2d(st, &tmQ, &full[s], 0, tile * R);
      }
      if (lane == 1) tma_load_2d(st + WQ_BYTES, &tmK, &full[s], 0, tile * 128);
      if (lane == 2) tma_load_2d(st + WQ_BYTES + WK_BYTES, &tmV, &full[s], 0, tile * 128);
      ++issued;
    }
    if (!ok && lane == 0) {
      // let the copies in flight land before the CTA's shared memory goes away
      for (long long i = issued > WIN_STAGES ? issued - WIN_STAGES : 0; i < issued; ++i)
        mbar_wait(&full[i % WIN_STAGES], (uint32_t)((i / WIN_STAGES) & 1), p.limit_ns, p.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16_f32(128, 128);
      constexpr uint32_t IDESC_O = idesc_bf16_f32(128, 64) | IDESC_B_MN_MAJOR;
      const uint64_t desc0 = smem_desc_sw128(smem_u32(smem));
      bool ok = true;
      for (int t = 0; ok && t <= n_local; ++t) {
        if (t < n_local) {
          const int s = t % WIN_STAGES, b = t & 1;
          if (!mbar_wait(&full[s], (uint32_t)((t / WIN_STAGES) & 1), p.limit_ns, p.status,
                         abort_flag)) {
            ok = false;
            break;
          }
          // buffer b is free once the softmax group has read the O of tile t-2
          if (t >= 2 && !mbar_wait(&t_free[b], (uint32_t)(((t >> 1) - 1) & 1), p.limit_ns,
                                   p.status, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t qd = desc_advance(desc0, (uint32_t)(s * WSTAGE_BYTES));
          const uint64_t kd = desc_advance(qd, (uint32_t)WQ_BYTES);
          const uint32_t sd = tmem + (uint32_t)(256 * b);
          tc_mma_bf16_k<false>(sd, qd, kd, IDESC_S);
#pragma unroll
          for (int kk = 1; kk < 4; ++kk)
            tc_mma_bf16_k<true>(sd, desc_advance(qd, 32u * kk), desc_advance(kd, 32u * kk), IDESC_S);
          tc_commit(&s_full[b]);
        }
        if (t >= 1) {
          const int tp = t - 1, sp = tp % WIN_STAGES, bp = tp & 1;
          if (!mbar_wait(&p_full[bp], (uint32_t)((tp >> 1) & 1), p.limit_ns, p.status,
                         abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t vd = smem_desc_sw128_mn64(
              smem_u32(smem + sp * WSTAGE_BYTES + WQ_BYTES + WK_BYTES));
          const uint32_t pa = tmem + (uint32_t)(256 * bp);        // P: 128 keys in 64 columns
          const uint32_t od = tmem + (uint32_t)(256 * bp + 128);
          tc_mma_bf16_ta<false>(od, pa, vd, IDESC_O);
#pragma unroll
          for (int kk = 1; kk < 8; ++kk)
            tc_mma_bf16_ta<true>(od, pa + 8u * kk, desc_advance(vd, 2048u * kk), IDESC_O);
          tc_commit(&o_full[bp]);
          tc_commit(&empty[sp]);
        }
      }
      if (!ok) *abort_flag = 1;
      tc_commit(drain);
      mbar_wait(drain, 0, p.limit_ns, p.status);
    }
  } else {
    // ------------------------------------------------------------ softmax + output
    const int g = (warp - 2) >> 2;           // TMEM buffer / tile parity of this group
    const int quarter = warp & 3;            // TMEM lanes 32*quarter .. +31
    const int r = quarter * 32 + lane;       // tile row
    const bool warp_rows = quarter * 32 < R; // warp-uniform: this warp holds rows of the tile
    const int c0 = ((quarter * 32) / SR) * TKV;  // first S column this warp reads
    const int my_chunk = ((r / SR) * TKV - c0) / TKV;  // this row's keys: chunk my_chunk of
                                                        // TKV columns of the warp's window
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t sb = lane_base + (uint32_t)(256 * g), ob = sb + 128u;
    const float sl2 = p.sl2;
    int k = 0;
    for (int t = g; t < n_local; t += 2, ++k) {
      const int tile = (int)blockIdx.x + t * (int)gridDim.x;
      if (!wwait(&s_full[g], (uint32_t)(k & 1), p, abort_flag)) break;
      tc_fence_after();
      if (warp_rows) {
        // This row's TKV scores. The warp reads its CW-column window in 32-column blocks;
        // column i of the window belongs to the warp's unit i / TKV, and each lane keeps the
        // columns of its own unit (a select with compile-time register indices).
        float mine[TKV];
#pragma unroll
        for (int kb = 0; kb < CW / 32; ++kb) {
          uint32_t ld[32];
          tc_ld_32x32b_x32(sb + (uint32_t)(c0 + 32 * kb), ld);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            asm volatile("" : "+r"(ld[i]));
            const int key = 32 * kb + i;
            if constexpr (CW == TKV)
              mine[key] = __uint_as_float(ld[i]);
            else if (key / TKV == my_chunk)
              mine[key % TKV] = __uint_as_float(ld[i]);
          }
        }
        float m = mine[0];
#pragma unroll
        for (int i = 1; i < TKV; ++i) m = fmaxf(m, mine[i]);
        const float ms = m * sl2;
        uint32_t pw[TKV / 2];
#pragma unroll
        for (int u = 0; u < TKV / 2; ++u) {
          float x0, x1;  // a pair of keys in one packed FMA
          f2_unpack(f2_fma(f2_pack(mine[2 * u], mine[2 * u + 1]), f2_pack(sl2, sl2),
                           f2_pack(-ms, -ms)), x0, x1);
          pw[u] = pack_trunc(ex2_approx(x0), ex2_approx(x1));
        }
        // P into the S columns it came from (the thread has read its scores): this lane's
        // weights in its own unit's columns, zero in every other column of the row
        uint32_t zero[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) zero[u] = 0u;
#pragma unroll
        for (int kb = 0; kb < 4; ++kb) {  // 32-key blocks of the tile's 128 keys
          const uint32_t col = sb + (uint32_t)(16 * kb);
          if (32 * kb < c0 || 32 * kb >= c0 + CW) tc_st_32x32b_x16(col, zero);
        }
#pragma unroll
        for (int kb = 0; kb < CW / 32; ++kb) {
          uint32_t val[16];
#pragma unroll
          for (int u = 0; u < 16; ++u) {
            const int key = 32 * kb + 2 * u;
            if constexpr (CW == TKV)
              val[u] = pw[key / 2];
            else
              val[u] = (key / TKV == my_chunk) ? pw[(key % TKV) / 2] : 0u;
          }
          tc_st_32x32b_x16(sb + (uint32_t)((c0 + 32 * kb) / 2), val);
        }
        tc_wait_st();
      }
      tc_fence_before();
      mbar_arrive(&p_full[g]);
      if (!wwait(&o_full[g], (uint32_t)(k & 1), p, abort_flag)) break;
      tc_fence_after();
      uint32_t ov[64];
      if (warp_rows) {
        tc_ld_32x32b_x32(ob, *reinterpret_cast<uint32_t(*)[32]>(&ov[0]));
        tc_ld_32x32b_x32(ob + 32u, *reinterpret_cast<uint32_t(*)[32]>(&ov[32]));
        tc_wait_ld();
#pragma unroll
        for (int i = 0; i < 64; ++i) asm volatile("" : "+r"(ov[i]));
      }
      tc_fence_before();
      mbar_arrive(&t_free[g]);  // buffer g may take the S of tile t+2
      const int unit = tile * U + r / SR;
      const int j = r % SR;
      if (warp_rows && r < R && j < TQ && unit < p.units) {
        const int h = unit % p.heads;
        const int w = (unit / p.heads) % p.nW;
        const int bimg = unit / (p.heads * p.nW);
        const float inv = 1.f / __uint_as_float(ov[56]);
        const long long Nq = (long long)TQ * p.nW;
        bf16* dst = p.o + ((long long)bimg * Nq + (long long)j * p.nW + w) * p.d_out + h * 56;
#pragma unroll
        for (int c = 0; c < 7; ++c) {
          float f[8];
#pragma unroll
          for (int e = 0; e < 8; e += 2)
            f2_unpack(f2_mul(f2_pack(__uint_as_float(ov[8 * c + e]), __uint_as_float(ov[8 * c + e + 1])),
                             f2_pack(inv, inv)), f[e], f[e + 1]);
          *reinterpret_cast<uint4*>(dst + 8 * c) = pack8(f);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tc_dealloc(tmem, WTMEM_COLS);
  }
}

template <int TQ, int TKV>
hiera_status run_win(const AttnArgs& a, cudaStream_t stream) {
  using C = WinCfg<TQ, TKV>;
  const long long units = (long long)a.B * a.nW * a.heads;
  CUtensorMap tmQ, tmK, tmV;
  {
    cuuint64_t dims[2] = {64, (cuuint64_t)(units * TQ)};
    cuuint64_t str[1] = {128};
    cuuint32_t box[2] = {64, (cuuint32_t)(C::SLOT ? TQ : C::R)};
    if (!encode_tmap_bf16_sw128(&tmQ, a.q, 2, dims, str, box)) return HIERA_ERR_CUDA;
  }
  {
    cuuint64_t dims[2] = {64, (cuuint64_t)(units * TKV)};
    cuuint64_t str[1] = {128};
    cuuint32_t box[2] = {64, 128};
    if (!encode_tmap_bf16_sw128(&tmK, a.k, 2, dims, str, box)) return HIERA_ERR_CUDA;
    if (!encode_tmap_bf16_sw128(&tmV, a.v, 2, dims, str, box)) return HIERA_ERR_CUDA;
  }
  WParams p;
  p.units = (int)units;
  p.nW = a.nW;
  p.heads = a.heads;
  p.d_out = a.d_out;
  p.sl2 = (float)(1.4426950408889634 / sqrt(56.0));
  p.o = static_cast<bf16*>(a.o);
  p.limit_ns = g_wait_limit_ns();
  p.status = g_status_ptr();
  auto kern = attn_win_kernel<TQ, TKV>;
  if (!ensure_smem_attr(reinterpret_cast<const void*>(kern), WSMEM_BYTES)) return HIERA_ERR_CUDA;
  const long long tiles = (units + C::U - 1) / C::U;
  const int grid = (int)(tiles < g_num_sms() ? tiles : g_num_sms());
  profile_mark(K_ATTN_WIN, stream);
  launch_k(kern, dim3(grid), dim3(320), WSMEM_BYTES, stream, tmQ, tmK, tmV, p);
  return cudaGetLastError() == cudaSuccess ? HIERA_OK : HIERA_ERR_CUDA;
}

}  // namespace

bool attention_win_supported(int Tq, int Tkv) {
  const bool pow2 = Tkv >= 4 && Tkv <= 64 && (Tkv & (Tkv - 1)) == 0;
  return pow2 && (Tq == Tkv || Tq * 4 == Tkv);
}

hiera_status launch_attention_win(const AttnArgs& a, cudaStream_t stream) {
  const long long units = (long long)a.B * a.nW * a.heads;
  if (units <= 0) return HIERA_OK;
  if (units * a.Tkv > (1ll << 31)) return HIERA_ERR_SHAPE;
  const bool pooled = a.Tq != a.Tkv;
  switch (a.Tkv) {
    case 4: return pooled ? run_win<1, 4>(a, stream) : run_win<4, 4>(a, stream);
    case 8: return pooled ? run_win<2, 8>(a, stream) : run_win<8, 8>(a, stream);
    case 16: return pooled ? run_win<4, 16>(a, stream) : run_win<16, 16>(a, stream);
    case 32: return pooled ? run_win<8, 32>(a, stream) : run_win<32, 32>(a, stream);
    case 64: return pooled ? run_win<16, 64>(a, stream) : run_win<64, 64>(a, stream);
    default: return HIERA_ERR_SHAPE;
  }
}

hiera_status launch_attention(const AttnArgs& a, cudaStream_t stream) {
  return attention_win_supported(a.Tq, a.Tkv) ? launch_attention_win(a, stream)
                                              : launch_attention_tc(a, stream);
}

}  // namespace hiera
