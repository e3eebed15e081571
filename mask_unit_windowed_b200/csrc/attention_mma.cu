// Mask-unit windowed / global attention core for head_dim 56 (bf16 in, fp32 softmax and
// accumulation) - "Phase 4: Hiera Backbone MLX Port", Architecture Summary,
// MaskUnitAttention: scaled dot-product attention inside each window (or over all
// tokens), heads merged before proj.
//
// Inputs are head-major q/k/v [B][windows][heads][T][64] (channels 56..63 zero) as the
// qkv GEMM epilogue writes them, q already max-pooled over q_stride. The output is
// the merged [B, Tq*windows, heads*56] token sequence (token j*windows + w, channel
// h*56 + e) that the attention proj Linear consumes.
//
// Flash-style, one warp per 16 query rows: S = Q K^T and O += P V on mma.sync
// m16n8k16 (bf16 -> fp32), the running row max / row sum kept in registers and
// reduced across the 4 lanes of a quad with shuffles, exponentials in base 2 with
// log2(e)/sqrt(56) folded into one multiply. K/V tiles of 64 keys stream through
// shared memory (cp.async, XOR-swizzled 16-byte chunks for conflict-free ldmatrix).
//   * tiled mode (Tq > 16): a CTA = 4 warps = 64 query rows of one (image, window,
//     head), K/V double-buffered and shared by the 4 warps;
//   * packed mode (Tq <= 16, Tkv <= 64, e.g. stage 1's 16-token units): a CTA = 4
//     independent (image, window, head) units, one per warp.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace hiera {
namespace {

__device__ __forceinline__ uint32_t swz(int row, int chunk) {
  return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// rows [row0, row0 + nrows) of a [T][64] bf16 matrix -> swizzled smem tile; rows >= T zero
__device__ __forceinline__ void load_rows(uint32_t s_base, const bf16* g, int row0, int nrows,
                                          int T, int tid, int nthr) {
  for (int i = tid; i < nrows * 8; i += nthr) {
    const int r = i >> 3, c = i & 7;
    const int gr = row0 + r;
    const bool valid = gr < T;
    cp_async16(s_base + swz(r, c), g + (long long)(valid ? gr : 0) * 64 + c * 8, valid);
  }
}

// Q fragments (4 k-steps of 16 channels) of the 16 rows starting at smem row `r0`.
__device__ __forceinline__ void load_q_frags(uint32_t sQ, int r0, uint32_t (&qf)[4][4]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int ks = 0; ks < 4; ++ks) {
    const int row = r0 + (lane & 7) + 8 * ((lane >> 3) & 1);
    const int chunk = 2 * ks + (lane >> 4);
    ldsm_x4(sQ + swz(row, chunk), qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3]);
  }
}

// One tile of KEYS keys for this warp's 16 query rows (online softmax update).
template <int KEYS>
__device__ __forceinline__ void attend_tile(const uint32_t (&qf)[4][4], uint32_t sK, uint32_t sV,
                                            int kv_valid, float (&o)[8][4], float (&mrow)[2],
                                            float (&lrow)[2], float sl2) {
  constexpr int NT = KEYS / 8;
  const int lane = threadIdx.x & 31;
  const int t4 = lane & 3;
  float s[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
    for (int kp = 0; kp < 2; ++kp) {
      const int row = nt * 8 + (lane & 7);
      const int chunk = 4 * kp + (lane >> 3);
      uint32_t b0, b1, b2, b3;
      ldsm_x4(sK + swz(row, chunk), b0, b1, b2, b3);
      mma16816(s[nt], qf[2 * kp], b0, b1);
      mma16816(s[nt], qf[2 * kp + 1], b2, b3);
    }
  }
  if (kv_valid < KEYS) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        if (nt * 8 + 2 * t4 + (e & 1) >= kv_valid) s[nt][e] = -INFINITY;
  }
  float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    mx0 = fmaxf(mx0, fmaxf(s[nt][0], s[nt][1]));
    mx1 = fmaxf(mx1, fmaxf(s[nt][2], s[nt][3]));
  }
  mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
  mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
  mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
  mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
  const float mn0 = fmaxf(mrow[0], mx0), mn1 = fmaxf(mrow[1], mx1);
  const float al0 = exp2f((mrow[0] - mn0) * sl2), al1 = exp2f((mrow[1] - mn1) * sl2);
  mrow[0] = mn0;
  mrow[1] = mn1;
  const float ms0 = mn0 * sl2, ms1 = mn1 * sl2;
  float ls0 = 0.f, ls1 = 0.f;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    s[nt][0] = exp2f(fmaf(s[nt][0], sl2, -ms0));
    s[nt][1] = exp2f(fmaf(s[nt][1], sl2, -ms0));
    s[nt][2] = exp2f(fmaf(s[nt][2], sl2, -ms1));
    s[nt][3] = exp2f(fmaf(s[nt][3], sl2, -ms1));
    ls0 += s[nt][0] + s[nt][1];
    ls1 += s[nt][2] + s[nt][3];
  }
  lrow[0] = lrow[0] * al0 + ls0;
  lrow[1] = lrow[1] * al1 + ls1;
#pragma unroll
  for (int dt = 0; dt < 8; ++dt) {
    o[dt][0] *= al0;
    o[dt][1] *= al0;
    o[dt][2] *= al1;
    o[dt][3] *= al1;
  }
#pragma unroll
  for (int kk = 0; kk < KEYS / 16; ++kk) {
    uint32_t pa[4];
    pa[0] = pack_bf16x2(s[2 * kk][0], s[2 * kk][1]);
    pa[1] = pack_bf16x2(s[2 * kk][2], s[2 * kk][3]);
    pa[2] = pack_bf16x2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
    pa[3] = pack_bf16x2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
    for (int dp = 0; dp < 4; ++dp) {
      const int mi = lane >> 3;
      const int row = 16 * kk + (lane & 7) + 8 * (mi & 1);
      const int chunk = 2 * dp + (mi >> 1);
      uint32_t v0, v1, v2, v3;
      ldsm_x4_t(sV + swz(row, chunk), v0, v1, v2, v3);
      mma16816(o[2 * dp], pa, v0, v1);
      if (dp < 3) mma16816(o[2 * dp + 1], pa, v2, v3);  // channels 56..63 are padding
    }
  }
}

// Normalise and write this warp's 16 rows (rows >= Tq dropped) through a warp-private
// [16][64] staging tile at smem `sO`.
__device__ __forceinline__ void store_rows(float (&o)[8][4], float (&lrow)[2], uint32_t sO,
                                           bf16* sOp, bf16* out, int q0, int Tq, int b, int w,
                                           int h, int nW, int d_out) {
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, t4 = lane & 3;
  float l0 = lrow[0], l1 = lrow[1];
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  const float i0 = 1.f / l0, i1 = 1.f / l1;
  (void)sO;
#pragma unroll
  for (int dt = 0; dt < 7; ++dt) {
    const uint32_t a0 = pack_bf16x2(o[dt][0] * i0, o[dt][1] * i0);
    const uint32_t a1 = pack_bf16x2(o[dt][2] * i1, o[dt][3] * i1);
    *reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(sOp) + swz(g, dt) + 4 * t4) = a0;
    *reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(sOp) + swz(g + 8, dt) + 4 * t4) = a1;
  }
  __syncwarp();
  const int Nq = Tq * nW;
  for (int i = lane; i < 16 * 7; i += 32) {
    const int r = i / 7, c = i - (i / 7) * 7;
    const int j = q0 + r;
    if (j >= Tq) continue;
    const uint4 val = *reinterpret_cast<const uint4*>(reinterpret_cast<uint8_t*>(sOp) + swz(r, c));
    bf16* dst = out + ((long long)b * Nq + (long long)j * nW + w) * d_out + h * 56 + c * 8;
    *reinterpret_cast<uint4*>(dst) = val;
  }
}

struct KArgs {
  const bf16* q;
  const bf16* k;
  const bf16* v;
  bf16* o;
  int units, nW, heads, Tq, Tkv, d_out;
  float sl2;
};

// tiled mode: blockIdx.x = unit (b, w, h), blockIdx.y = 64-row query tile
__global__ void __launch_bounds__(128) attn_tiled_kernel(const KArgs p) {
  griddep_wait();  // everything below reads or writes data of earlier kernels
  griddep_launch_dependents();
  __shared__ __align__(1024) uint8_t smem[8192 + 2 * 2 * 8192];
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sKV = sQ + 8192;  // [buf][K|V] 8 KB each
  const int tid = threadIdx.x, warp = tid >> 5;
  const int unit = blockIdx.x;
  const int h = unit % p.heads;
  const int w = (unit / p.heads) % p.nW;
  const int b = unit / (p.heads * p.nW);
  const bf16* qg = p.q + (long long)unit * p.Tq * 64;
  const bf16* kg = p.k + (long long)unit * p.Tkv * 64;
  const bf16* vg = p.v + (long long)unit * p.Tkv * 64;
  const int q0 = blockIdx.y * 64;

  load_rows(sQ, qg, q0, 64, p.Tq, tid, 128);
  load_rows(sKV, kg, 0, 64, p.Tkv, tid, 128);
  load_rows(sKV + 8192, vg, 0, 64, p.Tkv, tid, 128);
  cp_async_commit();

  float o[8][4];
#pragma unroll
  for (int dt = 0; dt < 8; ++dt) o[dt][0] = o[dt][1] = o[dt][2] = o[dt][3] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
  uint32_t qf[4][4];

  const int ntiles = (p.Tkv + 63) / 64;
  for (int t = 0; t < ntiles; ++t) {
    if (t + 1 < ntiles) {
      const uint32_t nb = sKV + (uint32_t)(((t + 1) & 1) * 16384);
      load_rows(nb, kg, (t + 1) * 64, 64, p.Tkv, tid, 128);
      load_rows(nb + 8192, vg, (t + 1) * 64, 64, p.Tkv, tid, 128);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (t == 0) load_q_frags(sQ, warp * 16, qf);
    const uint32_t cb = sKV + (uint32_t)((t & 1) * 16384);
    attend_tile<64>(qf, cb, cb + 8192, min(64, p.Tkv - t * 64), o, mrow, lrow, p.sl2);
    __syncthreads();
  }
  bf16* sOp = reinterpret_cast<bf16*>(smem + warp * 2048);  // rows 16*warp.. of the Q tile
  store_rows(o, lrow, sQ + warp * 2048, sOp, p.o, q0 + warp * 16, p.Tq, b, w, h, p.nW, p.d_out);
}

// packed mode: 4 units per CTA, one per warp; Tq <= 16 and Tkv <= KEYS
template <int KEYS>
__global__ void __launch_bounds__(128) attn_packed_kernel(const KArgs p) {
  griddep_wait();  // everything below reads or writes data of earlier kernels
  griddep_launch_dependents();
  constexpr int WARP_BYTES = 2048 + 2 * KEYS * 128;
  extern __shared__ __align__(1024) uint8_t smem[];  // 4 * WARP_BYTES
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int unit = blockIdx.x * 4 + warp;
  if (unit >= p.units) return;
  const uint32_t sQ = smem_u32(smem + warp * WARP_BYTES);
  const uint32_t sK = sQ + 2048, sV = sK + KEYS * 128;
  const int h = unit % p.heads;
  const int w = (unit / p.heads) % p.nW;
  const int b = unit / (p.heads * p.nW);
  load_rows(sQ, p.q + (long long)unit * p.Tq * 64, 0, 16, p.Tq, lane, 32);
  load_rows(sK, p.k + (long long)unit * p.Tkv * 64, 0, KEYS, p.Tkv, lane, 32);
  load_rows(sV, p.v + (long long)unit * p.Tkv * 64, 0, KEYS, p.Tkv, lane, 32);
  cp_async_commit();
  cp_async_wait<0>();
  __syncwarp();
  uint32_t qf[4][4];
  load_q_frags(sQ, 0, qf);
  float o[8][4];
#pragma unroll
  for (int dt = 0; dt < 8; ++dt) o[dt][0] = o[dt][1] = o[dt][2] = o[dt][3] = 0.f;
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
  attend_tile<KEYS>(qf, sK, sV, p.Tkv, o, mrow, lrow, p.sl2);
  __syncwarp();
  store_rows(o, lrow, sQ, reinterpret_cast<bf16*>(smem + warp * WARP_BYTES), p.o, 0, p.Tq, b, w,
             h, p.nW, p.d_out);
}

}  // namespace

hiera_status launch_attention_bf16(const AttnArgs& a, cudaStream_t stream) {
  KArgs p;
  p.q = static_cast<const bf16*>(a.q);
  p.k = static_cast<const bf16*>(a.k);
  p.v = static_cast<const bf16*>(a.v);
  p.o = static_cast<bf16*>(a.o);
  p.units = a.B * a.nW * a.heads;
  p.nW = a.nW;
  p.heads = a.heads;
  p.Tq = a.Tq;
  p.Tkv = a.Tkv;
  p.d_out = a.d_out;
  p.sl2 = (float)(1.4426950408889634 / sqrt(56.0));
  if (p.units <= 0 || a.Tq <= 0 || a.Tkv <= 0) return HIERA_OK;
  profile_mark(a.Tq <= 16 && a.Tkv <= 64 ? K_ATTN_PACKED : K_ATTN_TILED, stream);
  if (a.Tq <= 16 && a.Tkv <= 16) {
    launch_k(attn_packed_kernel<16>, dim3((p.units + 3) / 4), dim3(128), 4 * (2048 + 2 * 16 * 128), stream, p);
  } else if (a.Tq <= 16 && a.Tkv <= 64) {
    constexpr int bytes = 4 * (2048 + 2 * 64 * 128);
    static bool attr_done[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_done[dev]) {
      if (cudaFuncSetAttribute(attn_packed_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               bytes) != cudaSuccess)
        return HIERA_ERR_CUDA;
      attr_done[dev] = true;
    }
    launch_k(attn_packed_kernel<64>, dim3((p.units + 3) / 4), dim3(128), bytes, stream, p);
  } else {
    dim3 grid(p.units, (a.Tq + 63) / 64);
    if (grid.y > 65535) return HIERA_ERR_SHAPE;
    launch_k(attn_tiled_kernel, grid, dim3(128), 0, stream, p);
  }
  return cudaGetLastError() == cudaSuccess ? HIERA_OK : HIERA_ERR_CUDA;
}

}  // namespace hiera
