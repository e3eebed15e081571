// Persistent, warp-specialised tcgen05 GEMM for the Hiera block's Linear layers
// ("Phase 4: Hiera Backbone MLX Port", Architecture Summary: qkv = Linear(dim_in,
// 3 dim_out), proj = Linear(dim_out, dim_out), MLP fc1 -> GELU -> fc2, and the
// transition's proj Linear + max-pool).
//
//   C[M, N] = A[M, K] * W[N, K]^T      bf16 operands, fp32 accumulation in TMEM
//
// Roles (one CTA per SM, tiles strided over the grid):
//   warp 0      TMA producer: A tile 128 x 64 and W tile BN x 64 per stage, 128-byte
//               swizzle, STAGES-deep ring guarded by full/empty mbarriers.
//   warp 1      owns TMEM (2 accumulators of BN fp32 columns) and issues tcgen05.mma
//               (M = 128, N = BN, K = 16 per instruction) from one thread.
//   warps 2-9   epilogue, two warps per TMEM lane quarter (each half of the columns):
//               tcgen05.ld of the accumulator (TMEM lane = tile row), the LayerNorm fold /
//               bias / GELU / residual, and the store or the scatter into head-major
//               q/k/v with the q_stride max-pool.
//
// LayerNorm fold: with W' = W diag(gamma) (packed once), s_n = sum_k W'_nk and
// c_n = sum_k beta_k W_nk + b_n,  LN(x) W^T + b = rstd * (x W'^T - mean * s) + c.
// The row statistics arrive as P partial (mean, M2) pairs per row, each over K/P
// columns, written by whichever kernel produced x (the epilogue of the previous GEMM,
// the patch embedding, or a statistics pass); the epilogue merges them with Chan's
// formula, so LayerNorm costs no extra pass over x. A STORE epilogue can itself emit
// such partials of the values it writes (after rounding to bf16), one per (row, column
// half of its tile).
// Transition pooling: a 4-D tensor map loads, for 32 pooled tokens n, the four rows
// n + c*T/4 (c = 0..3) interleaved, so the four pooling candidates are adjacent TMEM
// lanes, hence adjacent rows of the epilogue's staging buffer; the copy-out takes their
// max on the packed bf16 values.
#include <mutex>

#include "common.cuh"
#include "gemm_shared.cuh"
#include "internal.h"

namespace hiera {
namespace {

constexpr int EPI_WARPS = 8;              // 2 per TMEM lane quarter, each half the columns
constexpr int EPI_THREADS = EPI_WARPS * 32;

// element-wise max of two groups of 8 bf16 (finite values)
__device__ __forceinline__ uint4 bf16x8_max(uint4 a, uint4 b) {
  uint4 d;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(d.x) : "r"(a.x), "r"(b.x));
  asm("max.bf16x2 %0, %1, %2;" : "=r"(d.y) : "r"(a.y), "r"(b.y));
  asm("max.bf16x2 %0, %1, %2;" : "=r"(d.z) : "r"(a.z), "r"(b.z));
  asm("max.bf16x2 %0, %1, %2;" : "=r"(d.w) : "r"(a.w), "r"(b.w));
  return d;
}

template <int BN>
struct Cfg {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STG_BYTES = 8 * 32 * 128;  // per epilogue warp: 32 rows x 128 B staging
  static constexpr int STAGES =
      cmin(8, (227 * 1024 - 1024 - 256 - EPI_WARPS * BN * 4 - 1024 - STG_BYTES) / STAGE_BYTES);
  static constexpr int ACC_STRIDE = BN <= 128 ? 128 : 256;
  static constexpr int TMEM_COLS = 2 * ACC_STRIDE;
  static constexpr int HALF = BN / 2;                    // columns per epilogue thread
  static constexpr int CH = (HALF % 56 == 0) ? 56 : cmin(HALF, 32);  // columns per chunk
  static constexpr int BAR_OFF = STAGES * STAGE_BYTES;
  // per epilogue warp: colsum and colconst (fp32) of its half of the tile's columns
  static constexpr int CONST_OFF = BAR_OFF + 256;
  static constexpr int CONST_BYTES = EPI_WARPS * 2 * (BN / 2) * 4;
  // (1024-byte aligned: a staged block of 128-byte swizzled rows is the layout of a
  // SWIZZLE_128B tensor store)
  static constexpr int STG_OFF = (CONST_OFF + CONST_BYTES + 1023) / 1024 * 1024;
  static constexpr int SMEM_BYTES = STG_OFF + STG_BYTES + 1024;
  static_assert(B_BYTES % 1024 == 0, "W tile must keep 1024-byte alignment");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "UMMA N for M=128");
  static_assert(HALF % CH == 0 && CH % 8 == 0, "epilogue chunking");
  static_assert(CONST_OFF % 16 == 0 && (HALF * 4) % 16 == 0, "16-byte constant loads");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
};

template <int BN, int EPI, bool FOLD, bool POOLED>
__global__ void __launch_bounds__(320, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmK2,
                   const __grid_constant__ CUtensorMap tmV2, const KParams p) {
  using C = Cfg<BN>;
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* acc_full = bars + 2 * STAGES;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint8_t* stg_all = smem + C::STG_OFF;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_tiles = POOLED ? ((p.M >> 2) + 31) / 32 : (p.M + BM - 1) / BM;
  const int n_tiles = p.N / BN;
  const int num_tiles = m_tiles * n_tiles;
  const int kblocks = (p.K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&acc_full[a], 1);
      mbar_init(&acc_empty[a], EPI_THREADS);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tc_alloc(tmem_slot, C::TMEM_COLS);
    tc_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Packed weights are written by no kernel this one can overlap: the producer requests the
  // first stages' W tiles before it waits for the previous kernel (whose output is A)
  const int npre = (p.w_static && (int)blockIdx.x < num_tiles) ? cmin(STAGES, kblocks) : 0;
  if (warp == 0 && npre > 0) {
    const int nt0 = (int)blockIdx.x - (int)p.fd_ntiles.div(blockIdx.x) * n_tiles;
    for (int i = 0; i < npre; ++i) {
      if (lane == 0) mbar_arrive_expect_tx(&full[i], C::STAGE_BYTES);
      __syncwarp();
      if (lane == ((2 * i + 1) & 7))
        tma_load_2d(smem + i * C::STAGE_BYTES + C::A_BYTES, &tmB, &full[i], i * BK, nt0 * BN);
    }
  }
  griddep_wait();  // everything below reads or writes data of earlier kernels
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // One thread's TMA loads complete one after another, so the loads of consecutive
    // stages are issued by different lanes (A and B of a stage by two lanes, rotating over
    // 8 lanes); every lane walks the same stage sequence and waits on the same barriers.
    // The first npre stages' B tiles (and their barriers' byte counts) are in flight already.
    int s = 0;
    uint32_t ph = 0;
    long long issued = 0;
    bool ok = true;
    int rr = 0;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      const int mt = (int)p.fd_ntiles.div((uint32_t)tile), nt = tile - mt * n_tiles;
      for (int kb = 0; kb < kblocks; ++kb) {
        const bool pre = issued < npre;  // (the first tile's first stages: ring not yet wrapped)
        if (!pre && !warp_wait(&empty[s], ph ^ 1u, p.limit_ns, p.status, abort_flag)) {
          ok = false;
          break;
        }
        uint8_t* sa = smem + s * C::STAGE_BYTES;
        if (lane == 0 && !pre) mbar_arrive_expect_tx(&full[s], C::STAGE_BYTES);
        __syncwarp();
        if (lane == rr) {
          if (POOLED) {
            const int per = p.tokens >> 2;
            if (per >= 32) {
              const int pm0 = mt * 32;
              const int bb = (int)p.fd_per.div((uint32_t)pm0);
              tma_load_4d(sa, &tmA, &full[s], kb * BK, 0, pm0 - bb * per, bb);
            } else {
              // 32 / per whole images per tile, one box of per x 4 rows each
              for (int i = 0; i < 32 / per; ++i)
                tma_load_4d(sa + i * per * 512, &tmA, &full[s], kb * BK, 0, 0,
                            mt * (32 / per) + i);
            }
          } else {
            tma_load_2d(sa, &tmA, &full[s], kb * BK, mt * BM);
          }
        }
        if (lane == rr + 1 && !pre)
          tma_load_2d(sa + C::A_BYTES, &tmB, &full[s], kb * BK, nt * BN);
        rr = (rr + 2) & 7;
        ++issued;
        if (++s == STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
    if (!ok && lane == 0) {
      // let copies already in flight land before the CTA's shared memory goes away
      for (long long i = issued > STAGES ? issued - STAGES : 0; i < issued; ++i)
        mbar_wait(&full[i % STAGES], (uint32_t)((i / STAGES) & 1), p.limit_ns, p.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN);
      const uint64_t desc0 = smem_desc_sw128(smem_u32(smem));  // stage 0, A tile
      int s = 0, acc = 0;
      uint32_t ph = 0, aph = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        if (!mbar_wait(&acc_empty[acc], aph ^ 1u, p.limit_ns, p.status, abort_flag)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(acc * C::ACC_STRIDE);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&full[s], ph, p.limit_ns, p.status, abort_flag)) {
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = desc_advance(desc0, (uint32_t)(s * C::STAGE_BYTES));
          const uint64_t bdesc = desc_advance(adesc, (uint32_t)C::A_BYTES);
          if (kb == 0)
            tc_mma_bf16_k<false>(d, adesc, bdesc, IDESC);
          else
            tc_mma_bf16_k<true>(d, adesc, bdesc, IDESC);
#pragma unroll
          for (int j = 1; j < BK / 16; ++j)
            if (kb * BK + j * 16 < p.K)
              tc_mma_bf16_k<true>(d, desc_advance(adesc, 32u * j), desc_advance(bdesc, 32u * j),
                                  IDESC);
          tc_commit(&empty[s]);
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(&acc_full[acc]);
        if (++acc == 2) {
          acc = 0;
          aph ^= 1u;
        }
      }
      // no MMA may still be writing TMEM when it is released
      tc_commit(drain);
      mbar_wait(drain, 0, p.limit_ns, p.status);
    }
  } else if (warp < 2 + EPI_WARPS) {
    // ------------------------------------------------------------ epilogue
    constexpr int HALF = C::HALF, CH = C::CH;
    const int ew = warp - 2;
    const int quarter = warp & 3;          // TMEM lanes 32*quarter .. +31
    const int c_begin = (ew >> 2) * HALF;  // this warp's half of the tile's columns
    const int rt = quarter * 32 + lane;    // tile row == TMEM lane
    int acc = 0;
    uint32_t aph = 0;
    // global row of this thread's TMEM lane in a tile (pooled tiles interleave 4 rows per
    // pooled token)
    auto row_of = [&](int tile) -> long long {
      const int mt = (int)p.fd_ntiles.div((uint32_t)tile);
      if (POOLED) {
        const int per = p.tokens >> 2;
        const int pm = mt * 32 + (rt >> 2);
        const int bb = (int)p.fd_per.div((uint32_t)pm), npp = pm - bb * per;
        return (long long)bb * p.tokens + (rt & 3) * per + npp;
      }
      return (long long)mt * BM + rt;
    };
    // the LayerNorm partials of the next tile's row are loaded while this tile is processed
    float2 part[8];
    auto load_parts = [&](int tile) {
      const long long mm = row_of(tile);
      const int P = p.stats_parts;
      const float2* sp = p.stats_in + (mm < p.M ? mm : 0) * P;
#pragma unroll
      for (int j = 0; j < 8; ++j) part[j] = j < P ? __ldg(sp + j) : make_float2(0.f, 0.f);
    };
    // This warp's column constants (its half of the tile's columns) live in its own
    // shared-memory slots, so moving to the next tile needs no barrier with the other
    // epilogue warps. They are loaded a tile ahead, CPL per lane, and staged at the tile's
    // start.
    constexpr int CPL = (HALF + 31) / 32;
    // (16-byte aligned: CONST_OFF and HALF * 4 are multiples of 16, and so is every chunk
    // start c * 4)
    float* col_sum = reinterpret_cast<float*>(smem + C::CONST_OFF) + ew * 2 * HALF;
    float* col_const = col_sum + HALF;
    float nsum[CPL], nconst[CPL];
    auto load_consts = [&](int tile) {
      const int c0 = (tile - (int)p.fd_ntiles.div((uint32_t)tile) * n_tiles) * BN + c_begin;
#pragma unroll
      for (int k = 0; k < CPL; ++k) {
        const int i = lane + 32 * k;
        nsum[k] = 0.f;
        nconst[k] = 0.f;
        if (i < HALF) {
          const int c = c0 + i;
          nsum[k] = FOLD ? __ldg(p.colsum + c) : 0.f;
          nconst[k] = p.colconst != nullptr ? __ldg(p.colconst + c)
                      : (p.bias16 != nullptr ? __bfloat162float(p.bias16[c]) : 0.f);
        }
      }
    };
    // the store epilogue (residual prefetch already holds many registers, few tiles per
    // CTA) loads them at the tile's start instead
    const LnConsts lnc = ln_consts(p.stats_parts, p.K);
    if ((int)blockIdx.x < num_tiles && FOLD) {
      load_parts(blockIdx.x);
      load_consts(blockIdx.x);
    }
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const int mt = (int)p.fd_ntiles.div((uint32_t)tile), nt = tile - mt * n_tiles;
      const int n0 = nt * BN;
      // row bookkeeping
      const long long m = row_of(tile);
      int b = 0, tok = 0, np = 0;
      if (POOLED) {
        const int per = p.tokens >> 2;
        const int pm = mt * 32 + (rt >> 2);
        b = (int)p.fd_per.div((uint32_t)pm);
        np = pm - b * per;
        tok = (rt & 3) * per + np;
      } else if (EPI == EPI_QKV) {
        b = (int)p.fd_tokens.div((uint32_t)m);  // (M < 2^31)
        tok = (int)m - b * p.tokens;
      }
      const bool row_ok = m < p.M;
      // residual of this row / half, in flight while the mainloop runs
      constexpr int NV = (EPI == EPI_STORE) ? HALF / 8 : 1;
      uint4 res[NV];
      const bool has_res = (EPI == EPI_STORE) && p.residual != nullptr && row_ok;
      if (EPI == EPI_STORE) {
#pragma unroll
        for (int i = 0; i < NV; ++i) {
          res[i] = has_res ? __ldg(reinterpret_cast<const uint4*>(
                                 p.residual + m * p.ldo + n0 + c_begin + 8 * i))
                           : make_uint4(0u, 0u, 0u, 0u);
        }
      }
      // LayerNorm statistics of this row, merged from the producer's partials
      float fa = 1.f, fb = 0.f;  // v = fa * acc + fb * colsum + colconst
      if (FOLD && row_ok) ln_merge_parts(part, p.stats_parts, lnc, p.ln_eps, fa, fb);
      // this warp's column constants of this tile into its slots (loaded a tile ahead)
      if (!FOLD) load_consts(tile);
      __syncwarp();  // every lane is done with the last tile's
#pragma unroll
      for (int k = 0; k < CPL; ++k) {
        const int i = lane + 32 * k;
        if (i < HALF) {
          col_sum[i] = nsum[k];
          col_const[i] = nconst[k];
        }
      }
      __syncwarp();
      if (FOLD && tile + (int)gridDim.x < num_tiles) {
        load_parts(tile + gridDim.x);
        load_consts(tile + gridDim.x);
      }
      if (!warp_wait(&acc_full[acc], aph, p.limit_ns, p.status, abort_flag)) break;
      tc_fence_after();
      const uint32_t tbase = tmem + (uint32_t)(acc * C::ACC_STRIDE) +
                             ((uint32_t)(quarter * 32) << 16) + (uint32_t)c_begin;
      const int which = (EPI == EPI_QKV) ? (int)p.fd_dout.div((uint32_t)n0) : 0;
      const bool pool_this = POOLED && (which == 0 || which == 3);
      const bool writer = row_ok && (!pool_this || (rt & 3) == 0);
      float st_mean = 0.f, st_m2 = 0.f;  // running statistics of the stored half row
#pragma unroll
      for (int c = 0; c < HALF; c += CH) {
        uint32_t r[CH];
        tmem_load<CH>(tbase + (uint32_t)c, r);
        float v[CH];
        // the column constants of this chunk, four per 16-byte shared-memory load (every
        // lane reads the same address: one broadcast per load)
        const float4* cs4 = reinterpret_cast<const float4*>(col_sum + c);
        const float4* cc4 = reinterpret_cast<const float4*>(col_const + c);
#pragma unroll
        for (int g = 0; g < CH / 4; ++g) {
          const float4 k4 = cc4[g];
          const float kc[4] = {k4.x, k4.y, k4.z, k4.w};
          float sc[4] = {0.f, 0.f, 0.f, 0.f};
          if (FOLD) {
            const float4 s4 = cs4[g];
            sc[0] = s4.x;
            sc[1] = s4.y;
            sc[2] = s4.z;
            sc[3] = s4.w;
          }
          if constexpr (EPI == EPI_GELU) {
            // fold and GELU on pairs (packed fp32: the scalar path's bits, half the issues)
            const f32x2 fa2 = f2_pack(fa, fa), fb2 = f2_pack(fb, fb);
#pragma unroll
            for (int e = 0; e < 4; e += 2) {
              const int i = 4 * g + e;
              const f32x2 x = f2_fma(fa2, f2_pack(__uint_as_float(r[i]), __uint_as_float(r[i + 1])),
                                     f2_fma(fb2, f2_pack(sc[e], sc[e + 1]),
                                            f2_pack(kc[e], kc[e + 1])));
              f2_unpack(gelu_fast2(x), v[i], v[i + 1]);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 4; e += 2) {  // (pairs: packed fp32, the scalar bits)
              const int i = 4 * g + e;
              const f32x2 acc2 = f2_pack(__uint_as_float(r[i]), __uint_as_float(r[i + 1]));
              const f32x2 kc2 = f2_pack(kc[e], kc[e + 1]);
              f2_unpack(FOLD ? f2_fma(f2_pack(fa, fa), acc2,
                                      f2_fma(f2_pack(fb, fb), f2_pack(sc[e], sc[e + 1]), kc2))
                             : f2_add(acc2, kc2),
                        v[i], v[i + 1]);
            }
          }
        }
        // ---- finish the values of this chunk (residual; the q / residual pooling of a
        // transition is taken on the packed values when they are copied out)
        static_assert(EPI != EPI_QKV || CH == 56, "q/k/v chunks are whole heads");
        if (EPI == EPI_STORE && has_res) {
#pragma unroll
          for (int g = 0; g < CH / 8; ++g) {
            const uint4 rr = res[(c / 8 + g) < NV ? (c / 8 + g) : 0];
            const uint32_t rw[4] = {rr.x, rr.y, rr.z, rr.w};
#pragma unroll
            for (int q = 0; q < 4; ++q)
              f2_unpack(f2_add(f2_pack(v[8 * g + 2 * q], v[8 * g + 2 * q + 1]),
                               f2_pack(bf16_lo(rw[q]), bf16_hi(rw[q]))),
                        v[8 * g + 2 * q], v[8 * g + 2 * q + 1]);
          }
        }
        // ---- destination of this lane's row for this chunk
        bf16* dst_row = nullptr;
        bool valid = row_ok;
        int nchunk = CH / 8;  // 16-byte chunks per row written
        if (EPI == EPI_QKV) {
          valid = writer;
          const int colw = n0 - which * p.d_out + c_begin + c;  // multiple of 56
          if (which == 3) {
            const int nq = POOLED ? (p.tokens >> 2) : p.tokens;
            const int tq = POOLED ? np : tok;
            dst_row = p.r + ((long long)b * nq + tq) * p.d_out + colw;
          } else {
            const int h = colw / 56;
            const int tt = pool_this ? np : tok;
            const int j = (int)p.fd_nw.div((uint32_t)tt), w = tt - j * p.nW;
            const int T = which == 0 ? p.Tq : p.Tkv;
            bf16* base = which == 0 ? p.q : (which == 1 ? p.k : p.v);
            dst_row = base + ((((long long)b * p.nW + w) * p.heads + h) * T + j) * 64;
            nchunk = 8;  // channels 56..63 of every head row are zero padding
          }
        } else {
          dst_row = p.out + m * p.ldo + n0 + c_begin + c;
        }
        // ---- stage the packed row in shared memory: XOR-swizzled 16-byte chunks for the
        // copy-out below, or dense rows of CH values for a TMA store
        uint8_t* stg = stg_all + (ew << 12);
        // q / k / v rows by TMA tensor store (pooled tiles: k and v only)
        const bool qkv_tma = EPI == EPI_QKV && p.qkv_tma != QKV_TMA_NONE &&
                             (!POOLED || which == 1 || which == 2);
        if (TmaOut<EPI>::value || (EPI == EPI_QKV && p.qkv_tma != QKV_TMA_NONE)) {
          if (lane == 0) tma_store_wait_read();  // the previous chunk's store has read stg
          __syncwarp();
        }
#pragma unroll
        for (int g = 0; g < CH / 8; ++g) {
          const uint4 pk = pack8(&v[8 * g]);
          if (TmaOut<EPI>::value)
            *reinterpret_cast<uint4*>(stg + lane * (CH * 2) + g * 16) = pk;
          else
            *reinterpret_cast<uint4*>(stg + (lane << 7) + ((g ^ (lane & 7)) << 4)) = pk;
          if (EPI == EPI_STORE && p.stats_out != nullptr) {
            // statistics of the values as stored (bf16)
            v[8 * g + 0] = bf16_lo(pk.x);
            v[8 * g + 1] = bf16_hi(pk.x);
            v[8 * g + 2] = bf16_lo(pk.y);
            v[8 * g + 3] = bf16_hi(pk.y);
            v[8 * g + 4] = bf16_lo(pk.z);
            v[8 * g + 5] = bf16_hi(pk.z);
            v[8 * g + 6] = bf16_lo(pk.w);
            v[8 * g + 7] = bf16_hi(pk.w);
          }
        }
        // channels 56..63 of a head row: zero padding for q and k; for v, channel 56 holds
        // 1.0 (bf16 0x3F80) so that the attention's P V product also yields each query
        // row's softmax denominator
        if (EPI == EPI_QKV && CH == 56)
          *reinterpret_cast<uint4*>(stg + (lane << 7) + ((7 ^ (lane & 7)) << 4)) =
              make_uint4(which == 2 ? 0x3F80u : 0u, 0u, 0u, 0u);
        if (EPI == EPI_STORE && p.stats_out != nullptr && row_ok) {
          float cmean, cm2;
          stats_piece<CH>(v, cmean, cm2);
          // merge this chunk into the running (count, mean, M2)
          chan_merge(st_mean, st_m2, cmean, cm2, (float)c, (float)CH);
        }
        if (TmaOut<EPI>::value) {
          fence_proxy_async_smem();  // this lane's staged row before the TMA engine reads it
          __syncwarp();
          if (lane == 0)
            tma_store_2d(&tmO, stg, n0 + c_begin + c, (int)(m - rt + quarter * 32));
          continue;
        }
        if (qkv_tma) {
          // the warp's 32 staged 128-byte rows (128-byte swizzle) are one box of the head's
          // q / k / v layout (QKV_TMA_* in gemm_shared.cuh); lane 0's row is the box origin
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && valid) {
            const int h = (n0 - which * p.d_out + c_begin + c) / 56;
            const CUtensorMap* map = which == 0 ? &tmO : (which == 1 ? &tmK2 : &tmV2);
            if (POOLED) {
              // k / v of a transition: lane 0 holds candidate 0 of pooled position np
              const int jj = (int)p.fd_nw.div((uint32_t)np);
              tma_store_5d(map, stg, 0, jj, 0, h, b * p.nW + np - jj * p.nW);
            } else if (p.qkv_tma == QKV_TMA_WINDOWS) {
              const int j = (int)p.fd_nw.div((uint32_t)tok);
              tma_store_4d(map, stg, 0, j, h, b * p.nW + tok - j * p.nW);
            } else {
              const int T = which == 0 ? p.Tq : p.Tkv;
              tma_store_2d(map, stg, 0, (b * p.heads + h) * T + tok);
            }
          }
          continue;
        }
        __syncwarp();
        // ---- copy out: 8 lanes per row, 4 rows per instruction, whole row segments
        const unsigned long long my_dst = reinterpret_cast<unsigned long long>(dst_row);
        if (POOLED && pool_this) {
          // q / residual of a transition: staged rows 4o..4o+3 are the four pooling
          // candidates of output row o (lanes 4o..4o+3, the first of them the writer). Their
          // max is taken on the bf16 values; rounding to nearest is monotonic, so the max of
          // the rounded values is the rounded max of the fp32 values.
#pragma unroll
          for (int it = 0; it < 2; ++it) {
            const int orow = it * 4 + (lane >> 3), ch = lane & 7;
            const unsigned long long d = __shfl_sync(0xffffffffu, my_dst, 4 * orow);
            const int ok = __shfl_sync(0xffffffffu, valid ? 1 : 0, 4 * orow);
            if (ok && ch < nchunk) {
              uint4 val = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
              for (int c4 = 0; c4 < 4; ++c4) {
                const int row = 4 * orow + c4;
                const uint4 o =
                    *reinterpret_cast<const uint4*>(stg + (row << 7) + ((ch ^ (row & 7)) << 4));
                val = c4 == 0 ? o : bf16x8_max(val, o);
              }
              *reinterpret_cast<uint4*>(reinterpret_cast<bf16*>(d) + ch * 8) = val;
            }
          }
        } else {
#pragma unroll
          for (int it = 0; it < 8; ++it) {
            const int row = it * 4 + (lane >> 3), ch = lane & 7;
            const unsigned long long d = __shfl_sync(0xffffffffu, my_dst, row);
            const int ok = __shfl_sync(0xffffffffu, valid ? 1 : 0, row);
            if (ok && ch < nchunk) {
              const uint4 val =
                  *reinterpret_cast<const uint4*>(stg + (row << 7) + ((ch ^ (row & 7)) << 4));
              *reinterpret_cast<uint4*>(reinterpret_cast<bf16*>(d) + ch * 8) = val;
            }
          }
        }
        __syncwarp();
      }
      if (EPI == EPI_STORE && p.stats_out != nullptr && row_ok)
        p.stats_out[m * p.stats_out_parts + nt * 2 + (ew >> 2)] = make_float2(st_mean, st_m2);
      tc_fence_before();
      mbar_arrive(&acc_empty[acc]);
      if (++acc == 2) {
        acc = 0;
        aph ^= 1u;
      }
    }
    // every TMA store of this warp has completed before the CTA exits
    if ((TmaOut<EPI>::value || (EPI == EPI_QKV && p.qkv_tma != QKV_TMA_NONE)) && lane == 0)
      tma_store_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tc_dealloc(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

bool encode_bf16(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims,
                 const cuuint64_t* strides_bytes, const cuuint32_t* box) {
  return encode_tmap_bf16_sw128(map, base, rank, dims, strides_bytes, box);
}


template <int BN, int EPI, bool FOLD, bool POOLED>
hiera_status run(const TcGemmArgs& a, cudaStream_t stream) {
  using C = Cfg<BN>;
  CUtensorMap tmA, tmB;
  if (POOLED) {
    const int per = a.tokens / 4;
    const int B = a.M / a.tokens;
    cuuint64_t dims[4] = {(cuuint64_t)a.K, 4, (cuuint64_t)per, (cuuint64_t)B};
    cuuint64_t str[3] = {(cuuint64_t)per * a.K * 2, (cuuint64_t)a.K * 2,
                         (cuuint64_t)a.tokens * a.K * 2};
    cuuint32_t box[4] = {BK, 4, (cuuint32_t)(per < 32 ? per : 32), 1};
    if (!encode_bf16(&tmA, a.A, 4, dims, str, box)) return HIERA_ERR_CUDA;
  } else {
    cuuint64_t dims[2] = {(cuuint64_t)a.K, (cuuint64_t)a.M};
    cuuint64_t str[1] = {(cuuint64_t)a.K * 2};
    cuuint32_t box[2] = {BK, BM};
    if (!encode_bf16(&tmA, a.A, 2, dims, str, box)) return HIERA_ERR_CUDA;
  }
  {
    cuuint64_t dims[2] = {(cuuint64_t)a.K, (cuuint64_t)a.N};
    cuuint64_t str[1] = {(cuuint64_t)a.K * 2};
    cuuint32_t box[2] = {BK, BN};
    if (!encode_bf16(&tmB, a.W, 2, dims, str, box)) return HIERA_ERR_CUDA;
  }
  CUtensorMap tmO = tmA, tmK2 = tmA, tmV2 = tmA;  // (unused unless set below)
  if (TmaOut<EPI>::value &&
      !encode_bf16_plain(&tmO, a.out, (cuuint64_t)a.N, (cuuint64_t)a.M, (cuuint64_t)a.ldo * 2,
                         (cuuint32_t)C::CH, 32))
    return HIERA_ERR_CUDA;
  // q / k / v head rows leave through TMA tensor stores where a warp's 32 rows form one box
  // (QKV_TMA_* in gemm_shared.cuh); every map covers the whole [B][nW][heads][T][64] layout
  int qkv_tma = QKV_TMA_NONE;
  if (EPI == EPI_QKV && a.tokens % 32 == 0 && a.nW >= 1 && a.tokens % a.nW == 0) {
    const int B = a.M / a.tokens;
    const int T = a.tokens / a.nW;  // keys per window
    const cuuint64_t bw = (cuuint64_t)B * a.nW;
    if (!POOLED && a.nW == 1 && a.Tq == T && a.Tkv == T && a.N == 3 * a.d_out) {
      const cuuint64_t dims[2] = {64, bw * a.heads * T};
      const cuuint64_t str[1] = {128};
      const cuuint32_t box[2] = {64, 32};
      if (!encode_bf16(&tmO, a.q, 2, dims, str, box) ||
          !encode_bf16(&tmK2, a.k, 2, dims, str, box) || !encode_bf16(&tmV2, a.v, 2, dims, str, box))
        return HIERA_ERR_CUDA;
      qkv_tma = QKV_TMA_GLOBAL;
    } else if (!POOLED && a.nW % 32 == 0 && a.Tq == T && a.Tkv == T && a.N == 3 * a.d_out) {
      const cuuint64_t dims[4] = {64, (cuuint64_t)T, (cuuint64_t)a.heads, bw};
      const cuuint64_t str[3] = {128, (cuuint64_t)T * 128, (cuuint64_t)a.heads * T * 128};
      const cuuint32_t box[4] = {64, 1, 1, 32};
      if (!encode_bf16(&tmO, a.q, 4, dims, str, box) ||
          !encode_bf16(&tmK2, a.k, 4, dims, str, box) || !encode_bf16(&tmV2, a.v, 4, dims, str, box))
        return HIERA_ERR_CUDA;
      qkv_tma = QKV_TMA_WINDOWS;
    } else if (POOLED && a.nW % 8 == 0 && (a.tokens / 4) % a.nW == 0 && (a.tokens / 4) % 8 == 0 &&
               a.Tkv == T) {
      const int TP = a.tokens / 4 / a.nW;  // in-window rows per pooling candidate
      const cuuint64_t dims[5] = {64, (cuuint64_t)TP, 4, (cuuint64_t)a.heads, bw};
      const cuuint64_t str[4] = {128, (cuuint64_t)TP * 128, (cuuint64_t)T * 128,
                                 (cuuint64_t)a.heads * T * 128};
      const cuuint32_t box[5] = {64, 1, 4, 1, 8};
      if (!encode_bf16(&tmK2, a.k, 5, dims, str, box) || !encode_bf16(&tmV2, a.v, 5, dims, str, box))
        return HIERA_ERR_CUDA;
      qkv_tma = QKV_TMA_POOLED;
    }
  }
  KParams p;
  p.M = a.M;
  p.N = a.N;
  p.K = a.K;
  p.colsum = a.colsum;
  p.colconst = a.colconst;
  p.bias16 = static_cast<const bf16*>(a.bias_bf16);
  p.ln_eps = a.ln_eps;
  p.out = static_cast<bf16*>(a.out);
  p.residual = static_cast<const bf16*>(a.residual);
  p.ldo = a.ldo;
  p.q = static_cast<bf16*>(a.q);
  p.k = static_cast<bf16*>(a.k);
  p.v = static_cast<bf16*>(a.v);
  p.r = static_cast<bf16*>(a.r);
  p.tokens = a.tokens;
  p.nW = a.nW;
  p.heads = a.heads;
  p.d_out = a.d_out;
  p.Tq = a.Tq;
  p.Tkv = a.Tkv;
  p.limit_ns = g_wait_limit_ns();
  p.status = g_status_ptr();
  p.stats_in = static_cast<const float2*>(a.stats_in);
  p.stats_parts = a.stats_parts;
  p.stats_out = static_cast<float2*>(a.stats_out);
  p.stats_out_parts = a.stats_out_parts;
  p.w_static = a.w_static;
  p.qkv_tma = qkv_tma;
  p.fd_ntiles = make_fastdiv((uint32_t)(a.N / BN));
  p.fd_tokens = make_fastdiv((uint32_t)a.tokens);
  p.fd_per = make_fastdiv((uint32_t)(a.tokens / 4));
  p.fd_nw = make_fastdiv((uint32_t)a.nW);
  p.fd_dout = make_fastdiv((uint32_t)a.d_out);

  auto kern = tc_gemm_kernel<BN, EPI, FOLD, POOLED>;
  if (!ensure_smem_attr(reinterpret_cast<const void*>(kern), C::SMEM_BYTES)) return HIERA_ERR_CUDA;
  const int m_tiles = POOLED ? (a.M / 4 + 31) / 32 : (a.M + BM - 1) / BM;
  const int tiles = m_tiles * (a.N / BN);
  if (tiles == 0) return HIERA_OK;
  int grid = g_num_sms();
  if (grid > tiles) grid = tiles;
  profile_mark(EPI == EPI_QKV ? K_GEMM_QKV : (EPI == EPI_GELU ? K_GEMM_GELU : K_GEMM_STORE),
               stream);
  launch_k(kern, dim3(grid), dim3(320), C::SMEM_BYTES, stream, tmA, tmB, tmO, tmK2, tmV2, p);
  return cudaGetLastError() == cudaSuccess ? HIERA_OK : HIERA_ERR_CUDA;
}

}  // namespace

bool encode_bf16_plain(CUtensorMap* map, const void* base, cuuint64_t cols, cuuint64_t rows,
                       cuuint64_t row_bytes, cuuint32_t box_cols, cuuint32_t box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t str[1] = {row_bytes};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, str, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_tmap_bf16_sw128(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims,
                            const cuuint64_t* strides_bytes, const cuuint32_t* box) {
  EncodeTiledFn fn = get_encode_fn();
  if (fn == nullptr) return false;
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base),
                  dims, strides_bytes, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

hiera_status launch_tc_gemm(int epi, const TcGemmArgs& a, cudaStream_t stream) {
  if (a.M <= 0 || a.N <= 0 || a.K <= 0) return HIERA_OK;
  if (a.N % 16 != 0 || a.K % 8 != 0) return HIERA_ERR_SHAPE;
  if (a.ln_fold && (a.stats_in == nullptr || a.stats_parts < 1 || a.stats_parts > 8 ||
                    a.K % a.stats_parts != 0))
    return HIERA_ERR_INVALID_ARG;
  if (a.stats_out != nullptr &&
      (epi != EPI_STORE || a.stats_out_parts != 2 * (a.N / store_bn(a.N))))
    return HIERA_ERR_INVALID_ARG;
  if (epi == EPI_QKV) {
    if (!a.ln_fold) return HIERA_ERR_INVALID_ARG;
    const bool pooled = a.pooled != 0;
    if (pooled) {
      // tiles of 32 pooled tokens: whole 32-row slices of one image, or whole images
      const int per = a.tokens / 4;
      if (a.tokens % 4 != 0 || per < 2 || (per >= 32 ? per % 32 != 0 : 32 % per != 0))
        return HIERA_ERR_SHAPE;
    }
    if (a.d_out % 224 == 0) {
      if (pooled) return run<224, EPI_QKV, true, true>(a, stream);
      // (the sixteen-warp kernels write q, k and v only: no residual-projection columns)
      const int mode = a.N == 3 * a.d_out ? g_option(HIERA_OPT_GEMM224) : 0;
      return mode == 1   ? run_wide<EPI_QKV, true, false>(a, stream)
             : mode == 2 ? run_wide<EPI_QKV, true, true>(a, stream)
                         : run<224, EPI_QKV, true, false>(a, stream);
    }
    if (a.d_out % 112 == 0)
      return pooled ? run<112, EPI_QKV, true, true>(a, stream)
                    : run<112, EPI_QKV, true, false>(a, stream);
    return HIERA_ERR_SHAPE;
  }
  if (epi == EPI_GELU) {
    if (!a.ln_fold) return HIERA_ERR_INVALID_ARG;
    if (a.N % 224 == 0) {
      const int mode = g_option(HIERA_OPT_GEMM224);
      return mode == 1   ? run_wide<EPI_GELU, true, false>(a, stream)
             : mode == 2 ? run_wide<EPI_GELU, true, true>(a, stream)
                         : run<224, EPI_GELU, true, false>(a, stream);
    }
    if (a.N % 112 == 0) return run<112, EPI_GELU, true, false>(a, stream);
    return HIERA_ERR_SHAPE;
  }
  if (a.ln_fold) return HIERA_ERR_INVALID_ARG;
  switch (store_bn(a.N)) {
    case 224: {
      const int mode = g_option(HIERA_OPT_GEMM224);
      return mode == 1   ? run_wide<EPI_STORE, false, false>(a, stream)
             : mode == 2 ? run_wide<EPI_STORE, false, true>(a, stream)
                         : run<224, EPI_STORE, false, false>(a, stream);
    }
    case 128: return run<128, EPI_STORE, false, false>(a, stream);
    case 112: return run<112, EPI_STORE, false, false>(a, stream);
    case 64: return run<64, EPI_STORE, false, false>(a, stream);
    case 32: return run<32, EPI_STORE, false, false>(a, stream);
    default: return run<16, EPI_STORE, false, false>(a, stream);
  }
}

}  // namespace hiera
