// tcgen05 GEMMs with a sixteen-warp epilogue for the 224-column tiles of the Hiera block's
// Linear layers ("Phase 4: Hiera Backbone MLX Port", Architecture Summary: qkv =
// Linear(dim, 3 dim), proj = Linear(dim, dim), MLP fc1 -> GELU -> fc2), the same product and
// epilogue arithmetic as the eight-warp kernel of gemm_tcgen05.cu:
//
//   C[M, N] = A[M, K] * W[N, K]^T      bf16 operands, fp32 accumulation in TMEM
//
// Two forms share the epilogue:
//  * tc_gemm_wide_kernel: one CTA per 128 x 224 tile (persistent), M = 128 MMAs.
//  * tc_gemm_pair_kernel: two CTAs of a cluster share one 256 x 224 tile through
//    tcgen05.mma.cta_group::2 (M = 256): rows 0..127 of A come from the first CTA's shared
//    memory and rows 128..255 from the second's, the 224 W rows (output columns) as two
//    halves of 112, one in each CTA, so each CTA loads its 128 A rows but only half of the W
//    tile per stage (30 KB per stage and SM instead of 44 KB). Each CTA's TMEM holds its
//    128 rows x 224 columns.
//
// Roles per CTA (576 threads):
//   warp 0       TMA producer: the CTA's A rows and W tile (or W half) of every stage; in the
//                pair the copies of both CTAs complete on the first CTA's "full" barrier.
//   warp 1       TMEM owner and MMA issuer (in the pair, the first CTA's thread issues the
//                pair's MMAs and commits them to barriers in both CTAs).
//   warps 2-17   epilogue, four warps per TMEM lane quarter, each a quarter (56 columns) of
//                the tile: one 56-column chunk per warp and tile, so an accumulator is read
//                and handed back to the MMA in one step. Rows leave through shared memory in
//                two halves of 16 (a TMA store per half, or the q / k / v head-row scatter),
//                which keeps the staging small enough for four (pair: six) pipeline stages.
//                A store epilogue's row statistics per column half merge two warps'
//                partials through shared memory (the eight-warp kernel's running merge,
//                same formula and rounding).
// With eighteen warps ptxas gives each thread at most 96 registers: the epilogue holds one
// chunk (56 accumulator values) at a time and loads its LayerNorm partials and column
// constants at the start of each tile (sixteen warps hide that latency).
//
// Measured on B200 (CUDA-graph replays, M = 8192, K = 448 / 1792, N = 448 / 1344 / 1792):
// the pair form's main loop runs at ~680 cycles per 64-wide k-block against ~620 for one CTA
// (seven stages did not change it, so the pair's MMA pace, not the L2 traffic it saves, sets
// it) and its set-up costs more (cluster barrier, pair TMEM allocation): it is the slower
// form at these shapes. Every wait is bounded; in the pair a role that gives up raises the
// abort flag of both CTAs.
#include "common.cuh"
#include "gemm_shared.cuh"
#include "internal.h"

namespace hiera {
namespace {

constexpr int WBN = 224;                  // tile columns (N of each MMA)
constexpr int W_EW = 16;                  // epilogue warps
constexpr int W_THREADS = 64 + 32 * W_EW;
constexpr int W_COLS = WBN / 4;           // columns per epilogue warp (one chunk)
constexpr int W_A_BYTES = BM * BK * 2;
constexpr int W_BAR_BYTES = 512;
constexpr int W_CONST_BYTES = W_EW * 2 * W_COLS * 4;  // per warp: colsum, colconst of its columns
constexpr int W_XCH_BUFS = 3;                         // statistics exchange buffers
constexpr int W_ACC_STRIDE = 256;
constexpr int W_TMEM_COLS = 2 * W_ACC_STRIDE;
constexpr int W_HALF_ROWS = 16;                       // rows staged per half

// Shared-memory layout of one CTA: the stage ring, barriers, column constants, the epilogue
// warps' staging (16 rows: dense 112-byte rows for a TMA store, 128-byte swizzled head rows
// for the q / k / v scatter) and, for a store epilogue, the statistics exchange.
template <int EPI, bool PAIR>
struct WideCfg {
  static constexpr int B_ROWS = PAIR ? WBN / 2 : WBN;  // W rows this CTA holds per stage
  static constexpr int B_BYTES = B_ROWS * BK * 2;
  static constexpr int STAGE_BYTES = W_A_BYTES + B_BYTES;
  static constexpr int STG_WARP = EPI == EPI_QKV ? W_HALF_ROWS * 128 : W_HALF_ROWS * W_COLS * 2;
  static constexpr int STG_BYTES = W_EW * STG_WARP;
  static constexpr int XCH_BYTES = EPI == EPI_STORE ? W_XCH_BUFS * 8 * 32 * 8 : 0;
  static constexpr int FIXED = W_BAR_BYTES + W_CONST_BYTES + STG_BYTES + XCH_BYTES + 1024;
  static constexpr int STAGES = cmin(8, (227 * 1024 - FIXED) / STAGE_BYTES);
  static constexpr int BAR_OFF = STAGES * STAGE_BYTES;
  static constexpr int CONST_OFF = BAR_OFF + W_BAR_BYTES;
  static constexpr int STG_OFF = CONST_OFF + W_CONST_BYTES;
  static constexpr int XCH_OFF = STG_OFF + STG_BYTES;
  static constexpr int SMEM = XCH_OFF + XCH_BYTES + 1024;
  static_assert(W_A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "1024-byte operand alignment");
  static_assert(STAGES >= 4, "pipeline depth");
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static_assert(STG_OFF % 128 == 0 && STG_WARP % 128 == 0 && XCH_OFF % 16 == 0, "staging");
  static_assert((2 * STAGES + 4 + 1 + 8 * W_XCH_BUFS) * 8 + 8 <= W_BAR_BYTES, "barrier block");
};

// ------------------------------------------------------------------ cluster primitives
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// address of the same shared-memory location in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t cluster_addr(const void* p, uint32_t rank) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(p)), "r"(rank));
  return a;
}
// arrive on a barrier of the other CTA (default release semantics: the arrive is a fire-
// and-forget message, it does not wait for this thread's earlier memory operations)
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t addr) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(addr) : "memory");
}
__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
// every thread of both CTAs (warps need not be converged)
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
// TMA load into this CTA's shared memory whose completion is counted on a barrier that may
// sit in the other CTA of the pair (no multicast: one destination, this GPU's memory)
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const CUtensorMap* map,
                                                 uint32_t bar_cluster, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tc_alloc_pair(uint32_t* smem_result, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(smem_result)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tc_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
// D (+)= A B^T over the pair: M = 256 (128 rows per CTA), operands at the same shared-memory
// offsets in both CTAs
template <bool ACC>
__device__ __forceinline__ void tc_mma_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.eq.u32 p, %4, 1;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(ACC ? 1u : 0u)
      : "memory");
}
// Arrive on the barrier at this shared-memory offset in every CTA of `mask` once the pair
// MMAs issued so far by this thread have completed.
__device__ __forceinline__ void tc_commit_pair(uint64_t* bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"(mask)
      : "memory");
}

// Barriers of one CTA (in the barrier block, in this order).
struct WideBars {
  uint64_t* full;       // [STAGES] (pair: first CTA, both CTAs' copies)
  uint64_t* empty;      // [STAGES] the MMAs read the stage
  uint64_t* acc_full;   // [2] the accumulator is complete
  uint64_t* acc_empty;  // [2] the epilogue read it (pair: first CTA, both CTAs' epilogues)
  uint64_t* drain;
  uint64_t* xch_full;   // [8 warp pairs][W_XCH_BUFS] statistics exchange
  uint32_t* tmem_slot;
  volatile int* abort_flag;
};

template <int STAGES>
__device__ __forceinline__ WideBars wide_bars(uint8_t* bar_block) {
  WideBars b;
  uint64_t* bars = reinterpret_cast<uint64_t*>(bar_block);
  b.full = bars;
  b.empty = b.full + STAGES;
  b.acc_full = b.empty + STAGES;
  b.acc_empty = b.acc_full + 2;
  b.drain = b.acc_empty + 2;
  b.xch_full = b.drain + 1;
  b.tmem_slot = reinterpret_cast<uint32_t*>(b.xch_full + 8 * W_XCH_BUFS);
  b.abort_flag = reinterpret_cast<volatile int*>(b.tmem_slot + 1);
  return b;
}

// The sixteen epilogue warps (warps 2..17) of either form. Tiles are cl, cl + n_cl, ...;
// tile (mt, nt) covers rows mt * ROWS + rank * 128 + (0..127) of this CTA.
template <int EPI, bool FOLD, bool PAIR>
__device__ __forceinline__ void wide_epilogue(const KParams& p, const CUtensorMap* tmO,
                                              uint8_t* smem, const WideBars& bb, uint32_t tmem,
                                              uint32_t rank, int cl, int n_cl, int num_tiles,
                                              int n_tiles, int warp, int lane) {
  using C = WideCfg<EPI, PAIR>;
  constexpr int CH = W_COLS;
  constexpr int ROWS = PAIR ? 2 * BM : BM;
  const int ew = warp - 2;
  const int quarter = warp & 3;           // TMEM lanes 32*quarter .. +31
  const int colq = ew >> 2;               // this warp's quarter of the tile's columns
  const int c_begin = colq * CH;
  const int half = colq >> 1;             // column half (statistics partial)
  const int rt = quarter * 32 + lane;     // tile row of this CTA == TMEM lane
  int acc = 0, tcount = 0;
  uint32_t aph = 0;
  constexpr int CPL = (CH + 31) / 32;
  float* col_sum = reinterpret_cast<float*>(smem + C::CONST_OFF) + ew * 2 * CH;
  float* col_const = col_sum + CH;
  uint8_t* stg = smem + C::STG_OFF + ew * C::STG_WARP;
  float2* xch = reinterpret_cast<float2*>(smem + C::XCH_OFF);
  auto give_up = [&]() {
    if (lane == 0) {
      *bb.abort_flag = 1;
      if (PAIR) st_cluster_u32(cluster_addr((const void*)bb.abort_flag, rank ^ 1u), 1u);
    }
  };
  const LnConsts lnc = ln_consts(p.stats_parts, p.K);
  for (int tile = cl; tile < num_tiles; tile += n_cl, ++tcount) {
    const int mt = tile / n_tiles, nt = tile - (tile / n_tiles) * n_tiles;
    const int n0 = nt * WBN;
    const long long m = (long long)mt * ROWS + (long long)rank * BM + rt;
    const long long m_warp = m - lane;  // row of lane 0
    int b = 0, tok = 0;
    if (EPI == EPI_QKV) {
      b = (int)(m / p.tokens);
      tok = (int)(m - (long long)b * p.tokens);
    }
    const bool row_ok = m < p.M;
    const bool has_res = (EPI == EPI_STORE) && p.residual != nullptr && row_ok;
    // LayerNorm coefficients of this row (v = fa * acc + fb * colsum + colconst) and this
    // warp's column constants
    float fa = 1.f, fb = 0.f;
    if (FOLD && row_ok) ln_fold_coeffs(p.stats_in + m * p.stats_parts, p.stats_parts, lnc,
                                       p.ln_eps, fa, fb);
    __syncwarp();  // every lane is done with the last tile's constants
#pragma unroll
    for (int k = 0; k < CPL; ++k) {
      const int i = lane + 32 * k;
      if (i < CH) {
        const int c = n0 + c_begin + i;
        col_sum[i] = FOLD ? __ldg(p.colsum + c) : 0.f;
        col_const[i] = p.colconst != nullptr ? __ldg(p.colconst + c)
                       : (p.bias16 != nullptr ? __bfloat162float(p.bias16[c]) : 0.f);
      }
    }
    __syncwarp();
    if (!warp_wait(&bb.acc_full[acc], aph, p.limit_ns, p.status, bb.abort_flag)) {
      give_up();
      break;
    }
    tc_fence_after();
    const uint32_t tbase = tmem + (uint32_t)(acc * W_ACC_STRIDE) +
                           ((uint32_t)(quarter * 32) << 16) + (uint32_t)c_begin;
    const int which = (EPI == EPI_QKV) ? n0 / p.d_out : 0;
    uint32_t r[CH];
    tmem_load<CH>(tbase, r);
    // the accumulator columns are in registers: hand them back to the MMA now
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      if (PAIR)
        mbar_arrive_cluster(cluster_addr(&bb.acc_empty[acc], 0));
      else
        mbar_arrive(&bb.acc_empty[acc]);
    }
    float v[CH];
    {
      const float4* cs4 = reinterpret_cast<const float4*>(col_sum);
      const float4* cc4 = reinterpret_cast<const float4*>(col_const);
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
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = 4 * g + e;
          float x = FOLD ? fmaf(fa, __uint_as_float(r[i]), fmaf(fb, sc[e], kc[e]))
                         : __uint_as_float(r[i]) + kc[e];
          if (EPI == EPI_GELU) x = gelu_fast(x);
          v[i] = x;
        }
      }
    }
    if (EPI == EPI_STORE && has_res) {
      const uint4* rsrc = reinterpret_cast<const uint4*>(p.residual + m * p.ldo + n0 + c_begin);
#pragma unroll
      for (int g = 0; g < CH / 8; ++g) {
        const uint4 rr = __ldg(rsrc + g);
        v[8 * g + 0] += bf16_lo(rr.x);
        v[8 * g + 1] += bf16_hi(rr.x);
        v[8 * g + 2] += bf16_lo(rr.y);
        v[8 * g + 3] += bf16_hi(rr.y);
        v[8 * g + 4] += bf16_lo(rr.z);
        v[8 * g + 5] += bf16_hi(rr.z);
        v[8 * g + 6] += bf16_lo(rr.w);
        v[8 * g + 7] += bf16_hi(rr.w);
      }
    }
    uint4 pk[CH / 8];
#pragma unroll
    for (int g = 0; g < CH / 8; ++g) {
      pk[g] = pack8(&v[8 * g]);
      if (EPI == EPI_STORE && p.stats_out != nullptr) {
        // statistics of the values as stored (bf16)
        v[8 * g + 0] = bf16_lo(pk[g].x);
        v[8 * g + 1] = bf16_hi(pk[g].x);
        v[8 * g + 2] = bf16_lo(pk[g].y);
        v[8 * g + 3] = bf16_hi(pk[g].y);
        v[8 * g + 4] = bf16_lo(pk[g].z);
        v[8 * g + 5] = bf16_hi(pk[g].z);
        v[8 * g + 6] = bf16_lo(pk[g].w);
        v[8 * g + 7] = bf16_hi(pk[g].w);
      }
    }
    if (EPI == EPI_STORE && p.stats_out != nullptr) {
      // (mean, M2) of this warp's 56 columns; the two quarters of a column half are merged by
      // the warp of the first quarter as the eight-warp kernel's running merge of two 56-column
      // chunks. The second quarter's warp writes buffer tcount % 3 only after this tile's MMA,
      // which waited for this warp's accumulator release of the tile before the one where this
      // warp last read that buffer.
      float cmean, cm2;
      stats_piece<CH>(v, cmean, cm2);
      const int pr = quarter * 2 + half, buf = tcount % W_XCH_BUFS;
      float2* slot = xch + (buf * 8 + pr) * 32 + lane;
      uint64_t* xb = &bb.xch_full[pr * W_XCH_BUFS + buf];
      if (colq & 1) {
        *slot = make_float2(cmean, cm2);
        mbar_arrive(xb);
      } else {
        const bool got = mbar_wait(xb, (uint32_t)((tcount / W_XCH_BUFS) & 1), p.limit_ns,
                                   p.status, bb.abort_flag);
        if (got && row_ok) {
          const float2 o = *slot;
          // the first quarter as the running (mean, M2), then the second merged in; for the
          // first chunk the eight-warp kernel's merge into (0, 0) over 0 values gives exactly
          // (cmean, cm2)
          float mean = cmean, m2 = cm2;
          chan_merge(mean, m2, o.x, o.y, (float)CH, (float)CH);
          p.stats_out[m * p.stats_out_parts + nt * 2 + half] = make_float2(mean, m2);
        }
        if (!__all_sync(0xffffffffu, got ? 1 : 0)) {
          give_up();
          break;
        }
      }
    }
    // ---- rows out through shared memory, 16 at a time
    if (TmaOut<EPI>::value) {
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        if (lane == 0) tma_store_wait_read();  // the previous store has read the staging rows
        __syncwarp();
        if ((lane >> 4) == hh) {
#pragma unroll
          for (int g = 0; g < CH / 8; ++g)
            *reinterpret_cast<uint4*>(stg + (lane & 15) * (CH * 2) + g * 16) = pk[g];
        }
        fence_proxy_async_smem();  // the staged rows before the TMA engine reads them
        __syncwarp();
        if (lane == 0)
          tma_store_2d(tmO, stg, n0 + c_begin, (int)(m_warp + W_HALF_ROWS * hh));
      }
    } else {
      // q / k / v scatter: one head row of 64 channels per token (channels 56..63: zero
      // padding for q and k; for v channel 56 holds 1.0, bf16 0x3F80, so that the
      // attention's P V product also yields the softmax denominator), 8 lanes per row
      bf16* dst_row = nullptr;
      {
        const int colw = n0 - which * p.d_out + c_begin;  // multiple of 56: one head
        const int h = colw / 56;
        const int w = tok % p.nW, j = tok / p.nW;
        const int T = which == 0 ? p.Tq : p.Tkv;
        bf16* base = which == 0 ? p.q : (which == 1 ? p.k : p.v);
        dst_row = base + ((((long long)b * p.nW + w) * p.heads + h) * T + j) * 64;
      }
      const unsigned long long my_dst = reinterpret_cast<unsigned long long>(dst_row);
      const uint4 padv = make_uint4(which == 2 ? 0x3F80u : 0u, 0u, 0u, 0u);
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        if ((lane >> 4) == hh) {
          const int sr = lane & 15;
#pragma unroll
          for (int g = 0; g < CH / 8; ++g)
            *reinterpret_cast<uint4*>(stg + (sr << 7) + ((g ^ (sr & 7)) << 4)) = pk[g];
          *reinterpret_cast<uint4*>(stg + (sr << 7) + ((7 ^ (sr & 7)) << 4)) = padv;
        }
        __syncwarp();
#pragma unroll
        for (int it = 0; it < W_HALF_ROWS / 4; ++it) {
          const int row = it * 4 + (lane >> 3), ch = lane & 7;
          const unsigned long long dd = __shfl_sync(0xffffffffu, my_dst, W_HALF_ROWS * hh + row);
          const int ok = __shfl_sync(0xffffffffu, row_ok ? 1 : 0, W_HALF_ROWS * hh + row);
          if (ok) {
            const uint4 val =
                *reinterpret_cast<const uint4*>(stg + (row << 7) + ((ch ^ (row & 7)) << 4));
            *reinterpret_cast<uint4*>(reinterpret_cast<bf16*>(dd) + ch * 8) = val;
          }
        }
        __syncwarp();
      }
    }
    if (++acc == 2) {
      acc = 0;
      aph ^= 1u;
    }
  }
  // every TMA store of this warp has completed before the CTA exits
  if (TmaOut<EPI>::value && lane == 0) tma_store_wait_all();
}

template <int STAGES>
__device__ __forceinline__ void wide_init_bars(const WideBars& bb, uint32_t acc_arrivals) {
  for (int s = 0; s < STAGES; ++s) {
    mbar_init(&bb.full[s], 1);
    mbar_init(&bb.empty[s], 1);
  }
  for (int a = 0; a < 2; ++a) {
    mbar_init(&bb.acc_full[a], 1);
    mbar_init(&bb.acc_empty[a], acc_arrivals);
  }
  mbar_init(bb.drain, 1);
  for (int i = 0; i < 8 * W_XCH_BUFS; ++i) mbar_init(&bb.xch_full[i], 32);
  *bb.abort_flag = 0;
  fence_barrier_init();
}

// ------------------------------------------------------------------ one CTA per tile
template <int EPI, bool FOLD>
__global__ void __launch_bounds__(W_THREADS, 1)
    tc_gemm_wide_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmO, const KParams p) {
  using C = WideCfg<EPI, false>;
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const WideBars bb = wide_bars<STAGES>(smem + C::BAR_OFF);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = p.N / WBN;
  const int num_tiles = ((p.M + BM - 1) / BM) * n_tiles;
  const int kblocks = (p.K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    wide_init_bars<STAGES>(bb, W_EW);
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tc_alloc(bb.tmem_slot, W_TMEM_COLS);
    tc_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *bb.tmem_slot;
  griddep_wait();  // everything below reads or writes data of earlier kernels
  griddep_launch_dependents();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    // consecutive stages' copies come from different lanes (one thread's TMA loads complete
    // in order); every lane walks the same stages and waits on the same barriers
    int s = 0;
    uint32_t ph = 0;
    long long issued = 0;
    bool ok = true;
    int rr = 0;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      const int mt = tile / n_tiles, nt = tile - (tile / n_tiles) * n_tiles;
      for (int kb = 0; kb < kblocks; ++kb) {
        if (!warp_wait(&bb.empty[s], ph ^ 1u, p.limit_ns, p.status, bb.abort_flag)) {
          ok = false;
          break;
        }
        uint8_t* sa = smem + s * C::STAGE_BYTES;
        if (lane == 0) mbar_arrive_expect_tx(&bb.full[s], C::STAGE_BYTES);
        __syncwarp();
        if (lane == rr) tma_load_2d(sa, &tmA, &bb.full[s], kb * BK, mt * BM);
        if (lane == rr + 1) tma_load_2d(sa + W_A_BYTES, &tmB, &bb.full[s], kb * BK, nt * WBN);
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
        mbar_wait(&bb.full[i % STAGES], (uint32_t)((i / STAGES) & 1), p.limit_ns, p.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16_f32(BM, WBN);
      const uint64_t desc0 = smem_desc_sw128(smem_u32(smem));  // stage 0, A tile
      int s = 0, acc = 0;
      uint32_t ph = 0, aph = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        if (!mbar_wait(&bb.acc_empty[acc], aph ^ 1u, p.limit_ns, p.status, bb.abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(acc * W_ACC_STRIDE);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&bb.full[s], ph, p.limit_ns, p.status, bb.abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = desc_advance(desc0, (uint32_t)(s * C::STAGE_BYTES));
          const uint64_t bdesc = desc_advance(adesc, (uint32_t)W_A_BYTES);
          if (kb == 0)
            tc_mma_bf16_k<false>(d, adesc, bdesc, IDESC);
          else
            tc_mma_bf16_k<true>(d, adesc, bdesc, IDESC);
#pragma unroll
          for (int j = 1; j < BK / 16; ++j)
            if (kb * BK + j * 16 < p.K)
              tc_mma_bf16_k<true>(d, desc_advance(adesc, 32u * j), desc_advance(bdesc, 32u * j),
                                  IDESC);
          tc_commit(&bb.empty[s]);
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(&bb.acc_full[acc]);
        if (++acc == 2) {
          acc = 0;
          aph ^= 1u;
        }
      }
      if (!ok) *bb.abort_flag = 1;
      // no MMA may still be writing TMEM when it is released
      tc_commit(bb.drain);
      mbar_wait(bb.drain, 0, p.limit_ns, p.status);
    }
  } else {
    wide_epilogue<EPI, FOLD, false>(p, &tmO, smem, bb, tmem, 0u, (int)blockIdx.x,
                                    (int)gridDim.x, num_tiles, n_tiles, warp, lane);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tc_dealloc(tmem, W_TMEM_COLS);
  }
}

// ------------------------------------------------------------------ CTA pair per tile
template <int EPI, bool FOLD>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(W_THREADS, 1)
    tc_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmO, const KParams p) {
  using C = WideCfg<EPI, true>;
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  // (the same offset in both CTAs: the MMA addresses both CTAs' operands with one descriptor)
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const WideBars bb = wide_bars<STAGES>(smem + C::BAR_OFF);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int n_tiles = p.N / WBN;
  const int num_tiles = ((p.M + 2 * BM - 1) / (2 * BM)) * n_tiles;
  const int kblocks = (p.K + BK - 1) / BK;
  const int cl = (int)blockIdx.x >> 1, n_cl = (int)gridDim.x >> 1;

  if (threadIdx.x == 0) {
    wide_init_bars<STAGES>(bb, 2 * W_EW);  // (the first CTA's acc_empty: both CTAs' warps)
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tc_alloc_pair(bb.tmem_slot, W_TMEM_COLS);
    tc_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers exist before either signals the other's
  tc_fence_after();
  const uint32_t tmem = *bb.tmem_slot;
  griddep_wait();  // everything below reads or writes data of earlier kernels
  griddep_launch_dependents();
  // raise the abort flag of both CTAs (a role of either gave up)
  auto abort_pair = [&]() {
    *bb.abort_flag = 1;
    st_cluster_u32(cluster_addr((const void*)bb.abort_flag, rank ^ 1u), 1u);
  };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    int s = 0;
    uint32_t ph = 0;
    long long issued = 0;
    bool ok = true;
    int rr = 0;
    for (int tile = cl; tile < num_tiles && ok; tile += n_cl) {
      const int mt = tile / n_tiles, nt = tile - (tile / n_tiles) * n_tiles;
      // (a box wholly past the last row of A is never requested: such rows are not stored)
      int row_a = mt * 2 * BM + (int)rank * BM;
      if (row_a >= p.M) row_a = 0;
      const int row_b = nt * WBN + (int)rank * C::B_ROWS;
      for (int kb = 0; kb < kblocks; ++kb) {
        if (!warp_wait(&bb.empty[s], ph ^ 1u, p.limit_ns, p.status, bb.abort_flag)) {
          ok = false;
          break;
        }
        uint8_t* sa = smem + s * C::STAGE_BYTES;
        const uint32_t fb = cluster_addr(&bb.full[s], 0);
        // The first CTA's producer announces the stage's bytes of both CTAs. The other CTA's
        // copies may land before that (the barrier's transaction count goes negative for a
        // while; the phase cannot complete without the arrival), and never early for a later
        // phase: the other CTA reloads a stage only after the MMAs of this phase read it.
        if (lane == 0 && rank == 0) mbar_arrive_expect_tx(&bb.full[s], 2 * C::STAGE_BYTES);
        __syncwarp();
        if (lane == rr) tma_load_2d_pair(sa, &tmA, fb, kb * BK, row_a);
        if (lane == rr + 1) tma_load_2d_pair(sa + W_A_BYTES, &tmB, fb, kb * BK, row_b);
        rr = (rr + 2) & 7;
        ++issued;
        if (++s == STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
    if (!ok) {
      if (lane == 0) abort_pair();
      // copies already in flight (this CTA's and the other's) complete on the first CTA's
      // barriers: let them land before either CTA's shared memory goes away
      if (rank == 0 && lane == 0)
        for (long long i = issued > STAGES ? issued - STAGES : 0; i < issued; ++i)
          mbar_wait(&bb.full[i % STAGES], (uint32_t)((i / STAGES) & 1), p.limit_ns, p.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (first CTA)
    if (rank == 0 && lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16_f32(2 * BM, WBN);
      const uint64_t desc0 = smem_desc_sw128(smem_u32(smem));  // stage 0, A tile
      int s = 0, acc = 0;
      uint32_t ph = 0, aph = 0;
      bool ok = true;
      for (int tile = cl; tile < num_tiles && ok; tile += n_cl) {
        if (!mbar_wait(&bb.acc_empty[acc], aph ^ 1u, p.limit_ns, p.status, bb.abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(acc * W_ACC_STRIDE);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&bb.full[s], ph, p.limit_ns, p.status, bb.abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = desc_advance(desc0, (uint32_t)(s * C::STAGE_BYTES));
          const uint64_t bdesc = desc_advance(adesc, (uint32_t)W_A_BYTES);
          if (kb == 0)
            tc_mma_pair<false>(d, adesc, bdesc, IDESC);
          else
            tc_mma_pair<true>(d, adesc, bdesc, IDESC);
#pragma unroll
          for (int j = 1; j < BK / 16; ++j)
            if (kb * BK + j * 16 < p.K)
              tc_mma_pair<true>(d, desc_advance(adesc, 32u * j), desc_advance(bdesc, 32u * j),
                                IDESC);
          tc_commit_pair(&bb.empty[s], 0x3);
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair(&bb.acc_full[acc], 0x3);
        if (++acc == 2) {
          acc = 0;
          aph ^= 1u;
        }
      }
      if (!ok) abort_pair();
      // no MMA may still be reading either CTA's shared memory or writing TMEM when the
      // pair synchronises for the last time
      tc_commit_pair(bb.drain, 0x1);
      mbar_wait(bb.drain, 0, p.limit_ns, p.status);
    }
  } else {
    wide_epilogue<EPI, FOLD, true>(p, &tmO, smem, bb, tmem, rank, cl, n_cl, num_tiles, n_tiles,
                                   warp, lane);
  }

  tc_fence_before();
  __syncwarp();
  cluster_sync_all();  // the other CTA's MMAs, copies and arrivals are done with this CTA
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tc_dealloc_pair(tmem, W_TMEM_COLS);
  }
}

}  // namespace

template <int EPI, bool FOLD, bool PAIR>
hiera_status run_wide(const TcGemmArgs& a, cudaStream_t stream) {
  using C = WideCfg<EPI, PAIR>;
  CUtensorMap tmA, tmB;
  {
    cuuint64_t dims[2] = {(cuuint64_t)a.K, (cuuint64_t)a.M};
    cuuint64_t str[1] = {(cuuint64_t)a.K * 2};
    cuuint32_t box[2] = {BK, BM};
    if (!encode_tmap_bf16_sw128(&tmA, a.A, 2, dims, str, box)) return HIERA_ERR_CUDA;
  }
  {
    cuuint64_t dims[2] = {(cuuint64_t)a.K, (cuuint64_t)a.N};
    cuuint64_t str[1] = {(cuuint64_t)a.K * 2};
    cuuint32_t box[2] = {BK, (cuuint32_t)C::B_ROWS};
    if (!encode_tmap_bf16_sw128(&tmB, a.W, 2, dims, str, box)) return HIERA_ERR_CUDA;
  }
  CUtensorMap tmO = tmA;  // unused by the q / k / v scatter
  if (TmaOut<EPI>::value &&
      !encode_bf16_plain(&tmO, a.out, (cuuint64_t)a.N, (cuuint64_t)a.M, (cuuint64_t)a.ldo * 2,
                         (cuuint32_t)W_COLS, W_HALF_ROWS))
    return HIERA_ERR_CUDA;
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
  p.w_static = 0;
  p.qkv_tma = 0;
  p.fd_ntiles = make_fastdiv((uint32_t)(a.N / 224));
  p.fd_tokens = make_fastdiv((uint32_t)a.tokens);
  p.fd_per = make_fastdiv((uint32_t)(a.tokens / 4));
  p.fd_nw = make_fastdiv((uint32_t)a.nW);
  p.fd_dout = make_fastdiv((uint32_t)a.d_out);

  auto kern = PAIR ? tc_gemm_pair_kernel<EPI, FOLD> : tc_gemm_wide_kernel<EPI, FOLD>;
  if (!ensure_smem_attr(reinterpret_cast<const void*>(kern), C::SMEM)) return HIERA_ERR_CUDA;
  const int rows = PAIR ? 2 * BM : BM;
  const int tiles = ((a.M + rows - 1) / rows) * (a.N / WBN);
  if (tiles == 0) return HIERA_OK;
  int ctas = PAIR ? g_num_sms() / 2 : g_num_sms();
  if (ctas > tiles) ctas = tiles;
  profile_mark(EPI == EPI_QKV ? K_GEMM_QKV : (EPI == EPI_GELU ? K_GEMM_GELU : K_GEMM_STORE),
               stream);
  launch_k(kern, dim3(PAIR ? 2 * ctas : ctas), dim3(W_THREADS), C::SMEM, stream, tmA, tmB, tmO,
           p);
  return cudaGetLastError() == cudaSuccess ? HIERA_OK : HIERA_ERR_CUDA;
}

template hiera_status run_wide<EPI_STORE, false, false>(const TcGemmArgs&, cudaStream_t);
template hiera_status run_wide<EPI_GELU, true, false>(const TcGemmArgs&, cudaStream_t);
template hiera_status run_wide<EPI_QKV, true, false>(const TcGemmArgs&, cudaStream_t);
template hiera_status run_wide<EPI_STORE, false, true>(const TcGemmArgs&, cudaStream_t);
template hiera_status run_wide<EPI_GELU, true, true>(const TcGemmArgs&, cudaStream_t);
template hiera_status run_wide<EPI_QKV, true, true>(const TcGemmArgs&, cudaStream_t);

}  // namespace hiera
