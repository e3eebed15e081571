// Tensor-core (tcgen05) attention core for the global-attention blocks ("Phase 4: Hiera
// Backbone MLX Port", Architecture Summary, MaskUnitAttention with mask_unit_attn=False:
// scaled dot-product attention over all tokens, heads merged before proj).
//
// One CTA = two 128-row query tiles (A and B) of one (image, window, head) unit:
//   warp 0      TMA: both Q tiles once, then K and V tiles (128 keys x 64 channels each)
//               through a KV_STAGES-deep ring shared by the two query tiles.
//   warp 1      TMEM owner and MMA issuer: S_t(j) = Q_t K_j^T (M=128, N=128, K=64) and
//               O_t += P_t(j) V_j (M=128, N=64, K=128; P_t(j) read from TMEM) for t = A, B.
//   warps 2-5   softmax of tile A, warps 6-9 of tile B, one query row per thread (TMEM lane
//               = row): row max, then the weights P = 2^(s log2(e)/sqrt(56) - m) on the
//               MUFU unit, cut to bf16 by a byte permute per pair, stored as bf16 pairs over
//               the S columns they came from; the PV product reads its A operand (P) from
//               there, so P never goes through shared memory. The running max is raised, and
//               O rescaled in TMEM, only when a tile's max exceeds it by more than 2^8, so P
//               entries stay below 256.
// TMEM holds three S/P buffers and the two O accumulators. Slot k = 2j + t (tile t, key tile
// j) uses buffer k mod 3, so a softmax warpgroup never waits for its own previous P V
// product before writing the next weights: buffer k mod 3 was last used by slot k - 3 (the
// other tile), whose P V the MMA thread issues right before S of slot k (issue order
// P_A(j-1) V, S_B(j), P_B(j-1) V, S_A(j+1); the tensor core executes one thread's MMAs in
// order).
// head_dim 56 is padded to 64: q/k channels 56..63 are zero; v's padding channel 56 is one,
// so column 56 of O accumulates the softmax denominator from the very P values the tensor core
// used; the output is O[:, :56] / O[:, 56]. V is read in its natural [keys][channels] layout
// as an MN-major B operand (channels contiguous), so no transposed copy of v exists.
// Any Tq and Tkv work: query rows and keys past the ends are zero-filled by TMA, masked keys
// take no part in the softmax and rows past Tq are not stored.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace hiera {
namespace {

constexpr int QT = 128;          // query rows per tile, two tiles per CTA
constexpr int KT = 128;          // keys per tile
constexpr int KV_STAGES = 4;
constexpr int Q_BYTES = QT * 128;                // [128 q][64 ch] bf16
constexpr int K_BYTES = KT * 128;                // [128 keys][64 ch]
constexpr int V_BYTES = KT * 128;                // [128 keys][64 ch]
constexpr int KV_BYTES = K_BYTES + V_BYTES;
constexpr int OFF_Q = 0;                         // Q_A, Q_B
constexpr int OFF_KV = OFF_Q + 2 * Q_BYTES;
constexpr int OFF_BAR = OFF_KV + KV_STAGES * KV_BYTES;
constexpr int SMEM_BYTES = OFF_BAR + 256 + 1024;
constexpr uint32_t TMEM_COLS = 512;  // S/P buffers at 0, 128, 256; O_A, O_B at 384, 448
constexpr uint32_t O_COL = 384;      // P as bf16 pairs: 128 keys in the first 64 columns
constexpr float RESCALE_LOG2 = 8.f;              // raise the running max past 2^8 only

struct AParams {
  int Tq, Tkv, nW, heads, d_out;
  float sl2;  // log2(e) / sqrt(56)
  bf16* o;
  uint64_t limit_ns;
  unsigned int* status;
};

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const AParams& p,
                                          volatile int* abort_flag) {
  int ok = mbar_wait(bar, parity, p.limit_ns, p.status, abort_flag) ? 1 : 0;
  ok = __all_sync(0xffffffffu, ok);
  if (!ok) *abort_flag = 1;
  return ok != 0;
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  tc_ld_32x32b_x32(taddr, r);
}

// max(a, b, c) in one instruction (three-input form of max.f32 on sm_100a); the scores
// are finite or -inf.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Softmax weights p in [0, 1] to bf16x2 by truncation (the high half of each fp32, lo
// first): one byte permute per pair. Truncation leaves every weight a fraction of an ulp
// low. The denominator is the sum of the same bf16 weights (v's ones channel), so for
// rows with many comparable weights that bias cancels, and the output error is round-to-
// nearest's. For rows dominated by a few weights it is about twice that, near 2e-3
// relative.
__device__ __forceinline__ uint32_t pack_bf16x2_trunc(float lo, float hi) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, 0x7632;" : "=r"(d) : "r"(__float_as_uint(lo)), "r"(__float_as_uint(hi)));
  return d;
}

__global__ void __launch_bounds__(320, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const AParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t pad = (1024u - (smem_u32(smem_raw) & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + KV_STAGES;
  uint64_t* s_full = kv_empty + KV_STAGES;  // [3]: per S/P buffer
  uint64_t* p_full = s_full + 3;            // [3]
  uint64_t* o_done = p_full + 3;            // [tile][key-tile parity]: that P V has completed
  uint64_t* drain = o_done + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int unit = blockIdx.x;
  const int q0 = blockIdx.y * 2 * QT;
  const int n_tiles = (p.Tkv + KT - 1) / KT;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < KV_STAGES; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int i = 0; i < 3; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
    }
    for (int i = 0; i < 4; ++i) mbar_init(&o_done[i], 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tc_alloc(tmem_slot, TMEM_COLS);
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
    // One thread's TMA loads complete one after another, so the boxes are issued by lanes
    // rotating over 8; every lane walks the same sequence and waits on the same barriers.
    if (lane == 0) mbar_arrive_expect_tx(q_full, 2 * Q_BYTES);
    __syncwarp();
    if (lane == 0) tma_load_3d(smem + OFF_Q, &tmQ, q_full, 0, q0, unit);
    if (lane == 1) tma_load_3d(smem + OFF_Q + Q_BYTES, &tmQ, q_full, 0, q0 + QT, unit);
    long long issued = 0;
    bool ok = true;
    int rr = 2;
    for (int j = 0; j < n_tiles; ++j) {
      const int s = j % KV_STAGES;
      if (!warp_wait(&kv_empty[s], (uint32_t)(((j / KV_STAGES) & 1) ^ 1), p, abort_flag)) {
        ok = false;
        break;
      }
      uint8_t* st = smem + OFF_KV + s * KV_BYTES;
      if (lane == 0) mbar_arrive_expect_tx(&kv_full[s], KV_BYTES);
      __syncwarp();
      if (lane == rr) tma_load_3d(st, &tmK, &kv_full[s], 0, j * KT, unit);
      if (lane == ((rr + 1) & 7)) tma_load_3d(st + K_BYTES, &tmV, &kv_full[s], 0, j * KT, unit);
      rr = (rr + 2) & 7;
      ++issued;
    }
    if (lane == 0) {
      mbar_wait(q_full, 0, p.limit_ns, p.status);
      if (!ok) {
        for (long long i = issued > KV_STAGES ? issued - KV_STAGES : 0; i < issued; ++i)
          mbar_wait(&kv_full[i % KV_STAGES], (uint32_t)((i / KV_STAGES) & 1), p.limit_ns,
                    p.status);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16_f32(128, KT);
      constexpr uint32_t IDESC_O = idesc_bf16_f32(128, 64) | IDESC_B_MN_MAJOR;
      const uint64_t desc0 = smem_desc_sw128(smem_u32(smem));
      // S of slot k = 2j + t into buffer k mod 3
      auto issue_s = [&](int j, int t) {
        const int k = 2 * j + t, buf = k % 3;
        const uint64_t kdesc = desc_advance(desc0, (uint32_t)(OFF_KV + (j % KV_STAGES) * KV_BYTES));
        const uint64_t qdesc = desc_advance(desc0, (uint32_t)(OFF_Q + t * Q_BYTES));
        const uint32_t sd = tmem + (uint32_t)(128 * buf);
        tc_mma_bf16_k<false>(sd, qdesc, kdesc, IDESC_S);
#pragma unroll
        for (int kk = 1; kk < 4; ++kk)
          tc_mma_bf16_k<true>(sd, desc_advance(qdesc, 32u * kk), desc_advance(kdesc, 32u * kk),
                              IDESC_S);
        tc_commit(&s_full[buf]);
      };
      // P of slot k = 2j + t (buffer k mod 3) times V_j into O_t, once the weights are in
      auto issue_pv = [&](int j, int t) -> bool {
        const int k = 2 * j + t, buf = k % 3;
        if (!mbar_wait(&p_full[buf], (uint32_t)((k / 3) & 1), p.limit_ns, p.status, abort_flag))
          return false;
        tc_fence_after();
        const uint64_t vdesc =
            smem_desc_sw128_mn64(smem_u32(smem + OFF_KV + (j % KV_STAGES) * KV_BYTES + K_BYTES));
        const uint32_t pa = tmem + (uint32_t)(128 * buf);
        const uint32_t od = tmem + O_COL + (uint32_t)(t * 64);
        if (j == 0)
          tc_mma_bf16_ta<false>(od, pa, vdesc, IDESC_O);
        else
          tc_mma_bf16_ta<true>(od, pa, vdesc, IDESC_O);
        // K step kk covers keys 16kk..16kk+15: two 8-row groups of the swizzled V tile
#pragma unroll
        for (int kk = 1; kk < 8; ++kk)
          tc_mma_bf16_ta<true>(od, pa + 8u * kk, desc_advance(vdesc, 2048u * kk), IDESC_O);
        tc_commit(&o_done[2 * t + (j & 1)]);
        return true;
      };
      auto wait_kv = [&](int j) -> bool {
        const bool r = mbar_wait(&kv_full[j % KV_STAGES], (uint32_t)((j / KV_STAGES) & 1),
                                 p.limit_ns, p.status, abort_flag);
        tc_fence_after();
        return r;
      };
      // Issue order P_A(j-1) V, S_B(j), P_B(j-1) V, S_A(j+1): each S waits only for the P V
      // that freed its buffer (slot k - 3), so tile A's next scores do not wait for tile B's
      // current weights.
      bool ok = mbar_wait(q_full, 0, p.limit_ns, p.status, abort_flag) && wait_kv(0);
      if (ok) issue_s(0, 0);
      for (int j = 0; ok && j <= n_tiles; ++j) {
        if (j >= 1 && !issue_pv(j - 1, 0)) {
          ok = false;
          break;
        }
        if (j < n_tiles) issue_s(j, 1);  // buffer of slot 2j - 2 (P_A(j-1) V just issued)
        if (j >= 1) {
          if (!issue_pv(j - 1, 1)) {
            ok = false;
            break;
          }
          tc_commit(&kv_empty[(j - 1) % KV_STAGES]);
        }
        if (j + 1 < n_tiles) {  // buffer of slot 2j - 1 (P_B(j-1) V just issued)
          if (!wait_kv(j + 1)) {
            ok = false;
            break;
          }
          issue_s(j + 1, 0);
        }
      }
      if (!ok) *abort_flag = 1;
      tc_commit(drain);
      mbar_wait(drain, 0, p.limit_ns, p.status);
    }
  } else {
    // ------------------------------------------------------------ softmax (row per thread)
    const int t = (warp - 2) >> 2;  // query tile of this warpgroup
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t o_col = O_COL + (uint32_t)(t * 64);
    const float sl2 = p.sl2;
    const float thr = RESCALE_LOG2 / sl2;  // in raw score units
    float m_run = -INFINITY;
    bool ok = true;
    // o_done[t][j & 1] completes once per two key tiles; waiting on key tile j-2's phase at
    // key tile j keeps every wait at most one phase behind (P_t(j) V cannot have run yet)
    auto wait_pv = [&](int jj) -> bool {
      return warp_wait(&o_done[2 * t + (jj & 1)], (uint32_t)((jj >> 1) & 1), p, abort_flag);
    };
    for (int j = 0; j < n_tiles; ++j) {
      const int k = 2 * j + t, buf = k % 3;
      const uint32_t s_col = (uint32_t)(128 * buf);
      if (!warp_wait(&s_full[buf], (uint32_t)((k / 3) & 1), p, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[KT];
#pragma unroll
      for (int c = 0; c < KT / 32; ++c)
        tmem_ld32(lane_base + s_col + (uint32_t)(32 * c),
                  *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * c]));
      tc_wait_ld();
#pragma unroll
      for (int i = 0; i < KT; ++i) asm volatile("" : "+r"(sr[i]));
      const int kv_valid = min(KT, p.Tkv - j * KT);
      if (kv_valid < KT) {  // ragged last tile: masked keys take no part
#pragma unroll
        for (int i = 0; i < KT; ++i)
          if (i >= kv_valid) sr[i] = __float_as_uint(-INFINITY);
      }
      // row max as a tree of three-input maxima: 128 -> 43 -> 15 -> 5 -> 2 -> 1 (depth 5;
      // the 43 first-level maxima are independent)
      static_assert(KT == 128, "max tree over 128 keys");
      float m1[43];
#pragma unroll
      for (int i = 0; i < 42; ++i)
        m1[i] = fmax3(__uint_as_float(sr[3 * i]), __uint_as_float(sr[3 * i + 1]),
                      __uint_as_float(sr[3 * i + 2]));
      m1[42] = fmaxf(__uint_as_float(sr[126]), __uint_as_float(sr[127]));
      float m2[15];
#pragma unroll
      for (int i = 0; i < 14; ++i) m2[i] = fmax3(m1[3 * i], m1[3 * i + 1], m1[3 * i + 2]);
      m2[14] = m1[42];
      const float m3[5] = {fmax3(m2[0], m2[1], m2[2]), fmax3(m2[3], m2[4], m2[5]),
                           fmax3(m2[6], m2[7], m2[8]), fmax3(m2[9], m2[10], m2[11]),
                           fmax3(m2[12], m2[13], m2[14])};
      const float mt = fmaxf(fmax3(m3[0], m3[1], m3[2]), fmaxf(m3[3], m3[4]));
      float alpha = 1.f;
      bool resc = false;
      if (mt > m_run + thr) {
        alpha = (m_run == -INFINITY) ? 0.f : ex2_approx((m_run - mt) * sl2);
        m_run = mt;
        resc = j > 0;
      }
      const float ms = m_run * sl2;
      // bookkeeping: P_t(j-2) V was issued before S_t(j), which has completed
      if (j >= 2 && !wait_pv(j - 2)) {
        ok = false;
        break;
      }
      // P of this row as bf16 pairs over the S columns just read (lane = row), 64 keys per
      // store
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t pw[32];
        const f32x2 sl2x2 = f2_pack(sl2, sl2), nms2 = f2_pack(-ms, -ms);
#pragma unroll
        for (int u = 0; u < 32; ++u) {
          // s log2(e)/sqrt(56) - m for a pair of keys in one packed FMA (-inf -> 0 below)
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[64 * h + 2 * u]),
                                   __uint_as_float(sr[64 * h + 2 * u + 1])), sl2x2, nms2), x0, x1);
          pw[u] = pack_bf16x2_trunc(ex2_approx(x0), ex2_approx(x1));
        }
        tc_st_32x32b_x32(lane_base + s_col + (uint32_t)(32 * h), pw);
      }
      if (__any_sync(0xffffffffu, resc)) {
        // O_t holds the sum through tile j-1 once that P V has completed: rescale these rows
        if (!wait_pv(j - 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float f = resc ? alpha : 1.f;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t ov[32];
          tmem_ld32(lane_base + o_col + (uint32_t)(32 * c), ov);
          tc_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            asm volatile("" : "+r"(ov[i]));
            ov[i] = __float_as_uint(__uint_as_float(ov[i]) * f);
          }
          tc_st_32x32b_x32(lane_base + o_col + (uint32_t)(32 * c), ov);
        }
        tc_wait_st();
      }
      tc_wait_st();  // P (and any rescaled O) written before the tensor core reads them
      tc_fence_before();
      mbar_arrive(&p_full[buf]);
    }
    // ---- normalise and store this row: merged head layout, token j*nW + w, once the last
    // two P V products have completed
    bool done = ok;
    if (done && n_tiles >= 2) done = wait_pv(n_tiles - 2);
    if (done) done = wait_pv(n_tiles - 1);
    if (done) {
      tc_fence_after();
      uint32_t ov[64];
      tmem_ld32(lane_base + o_col, *reinterpret_cast<uint32_t(*)[32]>(&ov[0]));
      tmem_ld32(lane_base + o_col + 32, *reinterpret_cast<uint32_t(*)[32]>(&ov[32]));
      tc_wait_ld();
#pragma unroll
      for (int i = 0; i < 64; ++i) asm volatile("" : "+r"(ov[i]));
      const int qrow = q0 + t * QT + r;
      if (qrow < p.Tq) {
        const float inv = 1.f / __uint_as_float(ov[56]);  // softmax denominator (ones channel)
        const int h = unit % p.heads;
        const int w = (unit / p.heads) % p.nW;
        const int bimg = unit / (p.heads * p.nW);
        const long long Nq = (long long)p.Tq * p.nW;
        bf16* dst = p.o + ((long long)bimg * Nq + (long long)qrow * p.nW + w) * p.d_out + h * 56;
        const f32x2 inv2 = f2_pack(inv, inv);
#pragma unroll
        for (int c = 0; c < 7; ++c) {
          float f[8];
#pragma unroll
          for (int e = 0; e < 8; e += 2)
            f2_unpack(f2_mul(f2_pack(__uint_as_float(ov[8 * c + e]), __uint_as_float(ov[8 * c + e + 1])),
                             inv2), f[e], f[e + 1]);
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
    tc_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

hiera_status launch_attention_tc(const AttnArgs& a, cudaStream_t stream) {
  const long long units_ll = (long long)a.B * a.nW * a.heads;
  if (units_ll <= 0 || a.Tq <= 0 || a.Tkv <= 0) return HIERA_OK;
  if (units_ll > (1ll << 30)) return HIERA_ERR_SHAPE;
  const int units = (int)units_ll;
  CUtensorMap tmQ, tmK, tmV;
  {
    cuuint64_t dims[3] = {64, (cuuint64_t)a.Tq, (cuuint64_t)units};
    cuuint64_t str[2] = {128, (cuuint64_t)a.Tq * 128};
    cuuint32_t box[3] = {64, QT, 1};
    if (!encode_tmap_bf16_sw128(&tmQ, a.q, 3, dims, str, box)) return HIERA_ERR_CUDA;
  }
  {
    cuuint64_t dims[3] = {64, (cuuint64_t)a.Tkv, (cuuint64_t)units};
    cuuint64_t str[2] = {128, (cuuint64_t)a.Tkv * 128};
    cuuint32_t box[3] = {64, KT, 1};
    if (!encode_tmap_bf16_sw128(&tmK, a.k, 3, dims, str, box)) return HIERA_ERR_CUDA;
  }
  {
    cuuint64_t dims[3] = {64, (cuuint64_t)a.Tkv, (cuuint64_t)units};
    cuuint64_t str[2] = {128, (cuuint64_t)a.Tkv * 128};
    cuuint32_t box[3] = {64, KT, 1};
    if (!encode_tmap_bf16_sw128(&tmV, a.v, 3, dims, str, box)) return HIERA_ERR_CUDA;
  }
  AParams p;
  p.Tq = a.Tq;
  p.Tkv = a.Tkv;
  p.nW = a.nW;
  p.heads = a.heads;
  p.d_out = a.d_out;
  p.sl2 = (float)(1.4426950408889634 / sqrt(56.0));
  p.o = static_cast<bf16*>(a.o);
  p.limit_ns = g_wait_limit_ns();
  p.status = g_status_ptr();
  if (!ensure_smem_attr(reinterpret_cast<const void*>(attn_tc_kernel), SMEM_BYTES))
    return HIERA_ERR_CUDA;
  dim3 grid(units, (a.Tq + 2 * QT - 1) / (2 * QT));
  if (grid.y > 65535) return HIERA_ERR_SHAPE;
  profile_mark(K_ATTN_TC, stream);
  launch_k(attn_tc_kernel, grid, dim3(320), SMEM_BYTES, stream, tmQ, tmK, tmV, p);
  return cudaGetLastError() == cudaSuccess ? HIERA_OK : HIERA_ERR_CUDA;
}

}  // namespace hiera
