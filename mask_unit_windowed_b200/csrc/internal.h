// Internal (non-ABI) declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "hiera.h"

namespace hiera {

int g_num_sms();                         // SM count of the current device (cached per device)
uint64_t g_wait_limit_ns();              // bound on every device-side wait
unsigned int* g_status_ptr();            // device address of the status word (current device)

// kernel ids reported by the launch profiler (hiera_profile_begin)
enum KernelId {
  K_PATCH_EMBED = 0, K_PERMUTE = 1, K_GEMM_QKV = 2, K_GEMM_GELU = 3, K_GEMM_STORE = 4,
  K_ATTN_WIN = 5, K_F32_GEMM = 6, K_F32_ATTN = 7, K_F32_STATS = 8, K_PACK = 9, K_PROBE = 10,
  K_ROW_STATS = 11, K_ATTN_TC = 12, K_MLP_FUSED = 13, K_ATTN_BLOCK = 14, K_COUNT = 15
};
void profile_mark(int kind, cudaStream_t stream);  // no-op unless a session is open

cudaError_t launch_permute(bool unroll, const void* x, void* y, int B, int G, int C, int L,
                           int elem_bytes, cudaStream_t stream);

// ---------------------------------------------------------------- tcgen05 GEMM (bf16)
enum EpiKind { EPI_STORE = 0, EPI_GELU = 1, EPI_QKV = 2 };

struct TcGemmArgs {
  int M, N, K;            // C[M, N] = A[M, K] * W[N, K]^T  (M = rows of A)
  const void* A;          // bf16 [M, K]
  const void* W;          // bf16 [N, K]
  // epilogue: v = ln_fold ? rstd*(acc - mean*colsum[n]) + colconst[n] : acc + colconst[n]
  const float* colsum;    // [N] (ln_fold only)
  const float* colconst;  // [N] or nullptr
  const void* bias_bf16;  // [N] bf16 bias used when colconst is nullptr (may be nullptr)
  float ln_eps;
  int ln_fold;            // 1: LayerNorm of A's rows folded into the epilogue
  const void* stats_in;   // ln_fold: float2 [M][stats_parts] partial (mean, M2) of A's rows,
  int stats_parts;        //          each over K / stats_parts columns (1..8 parts)
  void* stats_out;        // EPI_STORE: float2 [M][stats_out_parts] partials of the output
  int stats_out_parts;    //          (= 2 * N / store_bn(N)), or nullptr
  // EPI_STORE / EPI_GELU: out[m * ldo + n] (+ residual[m * ldo + n])
  void* out;
  const void* residual;
  int ldo;
  // EPI_QKV: scatter into head-major q/k/v [B][nW][heads][T][64], channels 56..63 zero
  // except v's channel 56 = 1 (+ pooled residual r)
  void* q;
  void* k;
  void* v;
  void* r;                // transition residual [B, tokens/4, d_out] (columns 3*d_out..)
  int tokens, nW, heads, d_out, Tq, Tkv;
  int pooled;             // 1: rows n, n+T/4, n+T/2, n+3T/4 of each image loaded together and
                          //    q / r columns max-pooled over them (q_stride 4)
  int w_static;           // 1: W is never written by a kernel this launch can overlap (packed
                          //    weights), so its first stages are requested before the wait for
                          //    the previous kernel
};

hiera_status launch_tc_gemm(int epi, const TcGemmArgs& a, cudaStream_t stream);

// ---------------------------------------------------------------- fused MLP (bf16, tcgen05)
// out = x + GELU(LN(x) W1'^T folded) W2^T + b2 with the hidden kept on chip (D = 112, 224)
struct MlpArgs {
  int M, D;
  const void* x;            // bf16 [M, D] input and residual
  const void* w1;           // bf16 [4D, D] LayerNorm-folded fc1 weight
  const float* colsum1;     // [4D]
  const float* colconst1;   // [4D]
  const void* w2;           // bf16 [D, 4D]
  const float* bias2;       // [D]
  const void* stats_in;     // float2 [M][stats_parts] partials of x's rows
  int stats_parts;
  float ln_eps;
  void* out;                // bf16 [M, D]
  void* stats_out;          // float2 [M][2] partials of out (row halves), or nullptr
};
bool mlp_fused_supported(int d);
hiera_status launch_mlp_fused(const MlpArgs& a, cudaStream_t stream);
int g_option(int opt);      // library options (hiera_set_option)

// Launch on `stream`, with programmatic dependent launch unless HIERA_OPT_PDL is off. A
// kernel launched this way must execute griddep_wait() (common.cuh) before it reads or
// writes global memory that another kernel of the stream writes or reads.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                     cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = g_option(HIERA_OPT_PDL) ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args&&>(args)...);
}

// N-tile width the plain-store GEMM uses for N output columns (N a multiple of 16).
inline int store_bn(int N) {
  return N % 224 == 0 ? 224 : N % 128 == 0 ? 128 : N % 112 == 0 ? 112 : N % 64 == 0 ? 64
         : N % 32 == 0 ? 32 : 16;
}
// Partial statistics per row written by a plain-store GEMM with N columns.
inline int store_stats_parts(int N) { return 2 * (N / store_bn(N)); }

// Per-row (mean, M2) of a bf16 [M, K] matrix as one partial per row.
hiera_status launch_row_partials_bf16(const void* x, int M, int K, float2* out,
                                      cudaStream_t stream);

// ---------------------------------------------------------------- attention (bf16, tcgen05)
struct AttnArgs {
  const void* q;  // [B][nW][heads][Tq][64], channels 56..63 zero
  const void* k;  // [B][nW][heads][Tkv][64], channels 56..63 zero
  const void* v;  // [B][nW][heads][Tkv][64], channel 56 = 1, 57..63 zero
  void* o;        // [B][Tq*nW][d_out], token j*nW + w, channel h*56 + e
  int B, nW, heads, Tq, Tkv, d_out;
};
// Small mask-unit windows (Tkv a power of two in 4..64, Tq = Tkv or Tkv / 4): several units
// per 128-row tile, one exact softmax pass.
bool attention_win_supported(int Tq, int Tkv);
hiera_status launch_attention_win(const AttnArgs& a, cudaStream_t stream);
// Any Tq, Tkv: 128-key tiles with an online softmax (global attention).
hiera_status launch_attention_tc(const AttnArgs& a, cudaStream_t stream);
// The windowed kernel where it applies, else the general one.
hiera_status launch_attention(const AttnArgs& a, cudaStream_t stream);

// The attention half of a stage-0 block in one kernel (dim 112, 2 heads, windows of 64,
// q_stride 1): x1 = x + proj(attention(norm1(x))) and x1's norm2 partials.
struct AttnBlockArgs {
  int B, tokens;
  const void* x;            // bf16 [B, tokens, 112]
  const void* stats_in;     // float2 [B * tokens][stats_parts] partials of x's rows
  int stats_parts;
  float ln_eps;
  const void* w1;           // bf16 [336, 112] norm1-folded q | k | v weight
  const float* colsum1;     // [336]
  const float* colconst1;   // [336]
  const void* wo;           // bf16 [112, 112] attention proj weight
  const float* bias_o;      // [112]
  void* x1;                 // bf16 [B, tokens, 112]
  void* stats_out;          // float2 [B * tokens][2] (column halves), or nullptr
};
bool attention_block_supported(int B, int tokens, int d_in, int d_out, int heads, int q_stride,
                               int window_tokens, int mask_unit_attn);
hiera_status launch_attention_block(const AttnBlockArgs& a, cudaStream_t stream);

// Raise `kern`'s dynamic shared-memory limit to `bytes` on the current device, once per
// (kernel, device); thread-safe. False if the runtime refused.
bool ensure_smem_attr(const void* kern, int bytes);

// TMA descriptor of a bf16 tensor with 128-byte swizzle (cuTensorMapEncodeTiled).
bool encode_tmap_bf16_sw128(CUtensorMap* map, const void* base, int rank, const cuuint64_t* dims,
                            const cuuint64_t* strides_bytes, const cuuint32_t* box);

// ---------------------------------------------------------------- fp32 SIMT path
hiera_status launch_row_stats_f32(const float* x, int M, int K, float eps, float2* stats,
                                  cudaStream_t stream);
struct F32GemmArgs {
  int M, N, K;
  const float* A; int lda;
  const float* W;              // [N, K]
  const float2* stats;         // per-row (mean, rstd) for the LayerNorm fold, or nullptr
  const float* colsum;         // [N] (fold only)
  const float* colconst;       // [N] or nullptr
  int gelu;
  const float* residual; int ldr;
  int resid_pool_tokens;       // >0: residual row m = max over 4 chunk rows of an image
                               //     with this many (un-pooled) tokens
  float* out; int ldo;
};
hiera_status launch_gemm_f32(const F32GemmArgs& a, cudaStream_t stream);
struct F32AttnArgs {
  const float* T; int ldT;     // token-major [B, tokens, ldT]; q/k/v at channel offsets
  int q_off, k_off, v_off;
  float* o;                    // [B, tokens/q_stride, d_out]
  int B, tokens, nW, heads, q_stride, d_out;
};
hiera_status launch_attention_f32(const F32AttnArgs& a, cudaStream_t stream);

// ---------------------------------------------------------------- pack / patch embed
hiera_status launch_fold_pack(const void* w, const void* gamma, const void* beta,
                              const void* bias, int N, int K, int dtype_bf16, void* w_out,
                              float* colsum, float* colconst, cudaStream_t stream);
hiera_status launch_copy_pack(const void* w, const void* bias, int N, int K, int dtype_bf16,
                              void* w_out, float* bias_out, cudaStream_t stream);
// Packed patch-embedding weights (HIERA_PATCH_PACKED_BYTES): fp32 [196][112] (k-major), fp32
// bias [112], bf16 [112][208] (co-major, k zero-padded to 208).
constexpr int PATCH_K = 196, PATCH_KP = 208, PATCH_CO = 112;
constexpr int PATCH_OFF_BIAS = PATCH_K * PATCH_CO * 4;
constexpr int PATCH_OFF_W16 = PATCH_OFF_BIAS + PATCH_CO * 4;
hiera_status launch_patch_pack(const void* w, const void* bias, int dtype_bf16, void* packed,
                               cudaStream_t stream);
// stats_out (bf16 only, may be nullptr): float2 [B*N][2] partial (mean, M2) of each output
// token's two 56-channel halves.
hiera_status launch_patch_embed(const void* img, const void* packed, const void* pos, void* out,
                                float2* stats_out, int B, int img_side, int dtype_bf16,
                                cudaStream_t stream);

}  // namespace hiera
