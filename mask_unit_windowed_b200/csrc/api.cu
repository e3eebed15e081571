// The C ABI (include/hiera.h): argument checks, packed-weight and workspace layouts,
// and the launch sequences of the block and the backbone. Every arithmetic step runs
// in this library's kernels; this file only validates and schedules.
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <set>
#include <utility>

#include "common.cuh"
#include "internal.h"

namespace hiera {

// First error recorded by any kernel since the last hiera_get_device_status().
__device__ unsigned int g_device_status = 0;

namespace {

constexpr int kMaxDev = 64;

struct DevInfo {
  int sms = 0;
  int ok = -1;  // -1 unknown, 0 not sm_100, 1 sm_100
  unsigned int* status = nullptr;
};
DevInfo g_dev[kMaxDev];
std::mutex g_dev_mu;

DevInfo& dev_info() {
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= kMaxDev) dev = 0;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DevInfo& d = g_dev[dev];
  if (d.ok < 0) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
      d.ok = 0;
    } else {
      d.ok = (major == 10 && minor == 0) ? 1 : 0;
      d.sms = sms;
      void* sp = nullptr;
      if (d.ok == 1 && cudaGetSymbolAddress(&sp, g_device_status) == cudaSuccess)
        d.status = static_cast<unsigned int*>(sp);
      else
        d.ok = 0;
    }
  }
  return d;
}

hiera_status check_device() { return dev_info().ok == 1 ? HIERA_OK : HIERA_ERR_DEVICE; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

#define HIERA_TRY(expr)                   \
  do {                                    \
    hiera_status _s = (expr);             \
    if (_s != HIERA_OK) return _s;        \
  } while (0)

// ---------------------------------------------------------------- block geometry
struct Geom {
  int B, tokens, d_in, d_out, heads, qs, nW, Tkv, Tq, Nq, hid, N1;
  bool transition, bf16;
  float eps;
};

hiera_status make_geom(const hiera_block_desc* d, Geom* g) {
  if (d == nullptr) return HIERA_ERR_INVALID_ARG;
  if (d->dtype != HIERA_F32 && d->dtype != HIERA_BF16) return HIERA_ERR_DTYPE;
  if (d->B < 1 || d->tokens < 1 || d->dim_in < 1 || d->dim_out < 1 || d->heads < 1)
    return HIERA_ERR_INVALID_ARG;
  if (!(d->ln_eps > 0.f) || d->ln_eps > 1.f) return HIERA_ERR_INVALID_ARG;
  if (d->head_dim != 56 || d->dim_out != d->heads * 56) return HIERA_ERR_SHAPE;
  if (d->dim_in % 16 != 0 || d->dim_out % 16 != 0) return HIERA_ERR_SHAPE;
  if (d->q_stride != 1 && d->q_stride != 4) return HIERA_ERR_SHAPE;
  if (d->tokens % d->q_stride != 0) return HIERA_ERR_SHAPE;
  if (d->q_stride == 4 && d->dim_in == d->dim_out) return HIERA_ERR_SHAPE;
  g->B = d->B;
  g->tokens = d->tokens;
  g->d_in = d->dim_in;
  g->d_out = d->dim_out;
  g->heads = d->heads;
  g->qs = d->q_stride;
  if (d->mask_unit_attn) {
    if (d->window_tokens < 1 || d->tokens % d->window_tokens != 0 ||
        d->window_tokens % d->q_stride != 0)
      return HIERA_ERR_SHAPE;
    g->nW = d->tokens / d->window_tokens;
  } else {
    g->nW = 1;
  }
  g->Tkv = d->tokens / g->nW;
  g->Tq = g->Tkv / g->qs;
  g->Nq = d->tokens / g->qs;
  g->hid = 4 * d->dim_out;
  g->transition = d->dim_in != d->dim_out;
  g->N1 = 3 * d->dim_out + (g->transition ? d->dim_out : 0);
  g->bf16 = d->dtype == HIERA_BF16;
  g->eps = d->ln_eps;
  if (g->bf16 && g->qs == 4) {
    const int per = d->tokens / 4;
    if (per < 2 || (per >= 32 ? per % 32 != 0 : 32 % per != 0)) return HIERA_ERR_SHAPE;
  }
  const long long rows = (long long)g->B * g->tokens;
  if (rows * (long long)std::max(g->N1, g->hid) > (1ll << 40)) return HIERA_ERR_SHAPE;
  return HIERA_OK;
}

struct PackLayout {
  size_t W1, s1, c1, Wo, bo, W2, s2, c2, W3, b3, total;
};

PackLayout pack_layout(const Geom& g) {
  const size_t es = g.bf16 ? 2 : 4;
  PackLayout L;
  size_t o = 0;
  L.W1 = o; o = up256(o + (size_t)g.N1 * g.d_in * es);
  L.s1 = o; o = up256(o + (size_t)g.N1 * 4);
  L.c1 = o; o = up256(o + (size_t)g.N1 * 4);
  L.Wo = o; o = up256(o + (size_t)g.d_out * g.d_out * es);
  L.bo = o; o = up256(o + (size_t)g.d_out * 4);
  L.W2 = o; o = up256(o + (size_t)g.hid * g.d_out * es);
  L.s2 = o; o = up256(o + (size_t)g.hid * 4);
  L.c2 = o; o = up256(o + (size_t)g.hid * 4);
  L.W3 = o; o = up256(o + (size_t)g.d_out * g.hid * es);
  L.b3 = o; o = up256(o + (size_t)g.d_out * 4);
  L.total = o;
  return L;
}

// bf16: q k v o r x1 h ; f32: t(=q slot) stats1 o x1 stats2 h
struct WsLayout {
  long long q, k, v, o, r, x1, h, st1, st2;
  size_t total;
};

WsLayout ws_layout(const Geom& g) {
  WsLayout L;
  size_t o = 0;
  const long long rows = (long long)g.B * g.tokens, qrows = (long long)g.B * g.Nq;
  if (g.bf16) {
    const long long units = (long long)g.B * g.nW * g.heads;
    L.q = o; o = up256(o + (size_t)units * g.Tq * 64 * 2);
    L.k = o; o = up256(o + (size_t)units * g.Tkv * 64 * 2);
    L.v = o; o = up256(o + (size_t)units * g.Tkv * 64 * 2);
    L.o = o; o = up256(o + (size_t)qrows * g.d_out * 2);
    if (g.transition) {
      L.r = o;
      o = up256(o + (size_t)(g.qs == 4 ? qrows : rows) * g.d_out * 2);
    } else {
      L.r = -1;
    }
    L.x1 = o; o = up256(o + (size_t)qrows * g.d_out * 2);
    L.h = o; o = up256(o + (size_t)qrows * g.hid * 2);
    // LayerNorm statistics: norm1's (one partial per row, from a statistics pass when the
    // caller's x did not come with partials) and norm2's (written by the proj epilogue)
    L.st1 = o; o = up256(o + (size_t)rows * 8);
    L.st2 = o; o = up256(o + (size_t)qrows * store_stats_parts(g.d_out) * 8);
  } else {
    L.q = o; o = up256(o + (size_t)rows * g.N1 * 4);
    L.k = L.v = -1;
    L.st1 = o; o = up256(o + (size_t)rows * 8);
    L.o = o; o = up256(o + (size_t)qrows * g.d_out * 4);
    L.r = -1;
    L.x1 = o; o = up256(o + (size_t)qrows * g.d_out * 4);
    L.st2 = o; o = up256(o + (size_t)qrows * 8);
    L.h = o; o = up256(o + (size_t)qrows * g.hid * 4);
  }
  L.total = o;
  return L;
}

hiera_status pack_block(const Geom& g, const hiera_block_weights* w, uint8_t* packed,
                        cudaStream_t st) {
  const PackLayout L = pack_layout(g);
  const size_t es = g.bf16 ? 2 : 4;
  const int bf = g.bf16 ? 1 : 0;
  HIERA_TRY(launch_fold_pack(w->qkv_w, w->norm1_w, w->norm1_b, w->qkv_b, 3 * g.d_out, g.d_in, bf,
                             packed + L.W1, (float*)(packed + L.s1), (float*)(packed + L.c1), st));
  if (g.transition) {
    HIERA_TRY(launch_fold_pack(w->proj_w, w->norm1_w, w->norm1_b, w->proj_b, g.d_out, g.d_in, bf,
                               packed + L.W1 + (size_t)3 * g.d_out * g.d_in * es,
                               (float*)(packed + L.s1) + 3 * g.d_out,
                               (float*)(packed + L.c1) + 3 * g.d_out, st));
  }
  HIERA_TRY(launch_copy_pack(w->attn_proj_w, w->attn_proj_b, g.d_out, g.d_out, bf, packed + L.Wo,
                             (float*)(packed + L.bo), st));
  HIERA_TRY(launch_fold_pack(w->fc1_w, w->norm2_w, w->norm2_b, w->fc1_b, g.hid, g.d_out, bf,
                             packed + L.W2, (float*)(packed + L.s2), (float*)(packed + L.c2), st));
  HIERA_TRY(launch_copy_pack(w->fc2_w, w->fc2_b, g.d_out, g.hid, bf, packed + L.W3,
                             (float*)(packed + L.b3), st));
  return HIERA_OK;
}

bool weights_ok(const Geom& g, const hiera_block_weights* w) {
  const void* req[] = {w->norm1_w, w->norm1_b, w->qkv_w, w->qkv_b, w->attn_proj_w,
                       w->attn_proj_b, w->norm2_w, w->norm2_b, w->fc1_w, w->fc1_b,
                       w->fc2_w, w->fc2_b};
  for (const void* p : req)
    if (p == nullptr) return false;
  if (g.transition && (w->proj_w == nullptr || w->proj_b == nullptr)) return false;
  return true;
}

bool weights_aligned(const hiera_block_weights* w) {
  const void* all[] = {w->norm1_w, w->norm1_b, w->qkv_w,  w->qkv_b,   w->proj_w,
                       w->proj_b,  w->attn_proj_w, w->attn_proj_b, w->norm2_w, w->norm2_b,
                       w->fc1_w,   w->fc1_b,   w->fc2_w,  w->fc2_b};
  for (const void* p : all)
    if (p != nullptr && !aligned16(p)) return false;
  return true;
}

// (a3-a9) norm1 + qkv (+ transition proj) with window scatter and q / r pooling, attention,
// heads merged, proj + residual: x1 and its norm2 partials in the workspace, as separate
// kernels (q, k, v and the attention output pass through the workspace).
hiera_status attention_half_unfused(const Geom& g, const uint8_t* packed, const void* x,
                                    uint8_t* ws, cudaStream_t st, const float2* stats_x,
                                    int parts_x, int parts_out) {
  const PackLayout P = pack_layout(g);
  const WsLayout W = ws_layout(g);
  const long long rows = (long long)g.B * g.tokens, qrows = (long long)g.B * g.Nq;
  // (a3-a6, a8 folded) norm1 + qkv (+ transition proj) with window scatter and q / r pooling
  TcGemmArgs a{};
  a.w_static = 1;  // packed block weights
  a.M = (int)rows;
  a.N = g.N1;
  a.K = g.d_in;
  a.A = x;
  a.W = packed + P.W1;
  a.colsum = (const float*)(packed + P.s1);
  a.colconst = (const float*)(packed + P.c1);
  a.ln_eps = g.eps;
  a.ln_fold = 1;
  a.stats_in = stats_x;
  a.stats_parts = parts_x;
  a.q = ws + W.q;
  a.k = ws + W.k;
  a.v = ws + W.v;
  a.r = g.transition ? ws + W.r : nullptr;
  a.tokens = g.tokens;
  a.nW = g.nW;
  a.heads = g.heads;
  a.d_out = g.d_out;
  a.Tq = g.Tq;
  a.Tkv = g.Tkv;
  a.pooled = g.qs == 4;
  HIERA_TRY(launch_tc_gemm(EPI_QKV, a, st));
  // (a7, a8) attention core, heads merged
  AttnArgs at{};
  at.q = ws + W.q;
  at.k = ws + W.k;
  at.v = ws + W.v;
  at.o = ws + W.o;
  at.B = g.B;
  at.nW = g.nW;
  at.heads = g.heads;
  at.Tq = g.Tq;
  at.Tkv = g.Tkv;
  at.d_out = g.d_out;
  HIERA_TRY(launch_attention(at, st));
  // (a9) attention proj + residual
  TcGemmArgs pj{};
  pj.w_static = 1;  // packed block weights
  pj.M = (int)qrows;
  pj.N = g.d_out;
  pj.K = g.d_out;
  pj.A = ws + W.o;
  pj.W = packed + P.Wo;
  pj.colconst = (const float*)(packed + P.bo);
  pj.out = ws + W.x1;
  pj.residual = g.transition ? (const void*)(ws + W.r) : x;
  pj.ldo = g.d_out;
  pj.stats_out = ws + W.st2;
  pj.stats_out_parts = parts_out;
  return launch_tc_gemm(EPI_STORE, pj, st);
}

// stats_x: partial (mean, M2) of x's rows from x's producer ([rows][parts_x]), or nullptr
// to compute them here; stats_y: where to write y's partials for the next LayerNorm
// ([qrows][store_stats_parts(d_out)]), or nullptr.
hiera_status forward_bf16(const Geom& g, const uint8_t* packed, const void* x, void* y,
                          uint8_t* ws, cudaStream_t st, const float2* stats_x = nullptr,
                          int parts_x = 0, float2* stats_y = nullptr) {
  const PackLayout P = pack_layout(g);
  const WsLayout W = ws_layout(g);
  const long long rows = (long long)g.B * g.tokens, qrows = (long long)g.B * g.Nq;
  if (stats_x == nullptr) {
    HIERA_TRY(launch_row_partials_bf16(x, (int)rows, g.d_in, (float2*)(ws + W.st1), st));
    stats_x = (const float2*)(ws + W.st1);
    parts_x = 1;
  }
  const int parts_out = store_stats_parts(g.d_out);
  const bool fused_attn =
      g_option(HIERA_OPT_FUSED_ATTN) &&
      attention_block_supported(g.B, g.tokens, g.d_in, g.d_out, g.heads, g.qs, g.Tkv,
                                g.nW > 1 ? 1 : 0) &&
      parts_out == 2;
  if (fused_attn) {
    // (a3-a9) norm1 + qkv + windowed attention + heads merged + proj + residual, one kernel
    AttnBlockArgs ab{};
    ab.B = g.B;
    ab.tokens = g.tokens;
    ab.x = x;
    ab.stats_in = stats_x;
    ab.stats_parts = parts_x;
    ab.ln_eps = g.eps;
    ab.w1 = packed + P.W1;
    ab.colsum1 = (const float*)(packed + P.s1);
    ab.colconst1 = (const float*)(packed + P.c1);
    ab.wo = packed + P.Wo;
    ab.bias_o = (const float*)(packed + P.bo);
    ab.x1 = ws + W.x1;
    ab.stats_out = ws + W.st2;
    HIERA_TRY(launch_attention_block(ab, st));
  } else {
    HIERA_TRY(attention_half_unfused(g, packed, x, ws, st, stats_x, parts_x, parts_out));
  }
  if (g_option(HIERA_OPT_FUSED_MLP) && mlp_fused_supported(g.d_out) && parts_out == 2) {
    // (a10-a12) norm2 + fc1 + GELU + fc2 + residual in one kernel, hidden kept on chip
    MlpArgs ml{};
    ml.M = (int)qrows;
    ml.D = g.d_out;
    ml.x = ws + W.x1;
    ml.w1 = packed + P.W2;
    ml.colsum1 = (const float*)(packed + P.s2);
    ml.colconst1 = (const float*)(packed + P.c2);
    ml.w2 = packed + P.W3;
    ml.bias2 = (const float*)(packed + P.b3);
    ml.stats_in = ws + W.st2;
    ml.stats_parts = parts_out;
    ml.ln_eps = g.eps;
    ml.out = y;
    ml.stats_out = stats_y;
    return launch_mlp_fused(ml, st);
  }
  // (a10, a11) norm2 + fc1 + GELU
  TcGemmArgs f1{};
  f1.w_static = 1;  // packed block weights
  f1.M = (int)qrows;
  f1.N = g.hid;
  f1.K = g.d_out;
  f1.A = ws + W.x1;
  f1.W = packed + P.W2;
  f1.colsum = (const float*)(packed + P.s2);
  f1.colconst = (const float*)(packed + P.c2);
  f1.ln_eps = g.eps;
  f1.ln_fold = 1;
  f1.stats_in = ws + W.st2;
  f1.stats_parts = parts_out;
  f1.out = ws + W.h;
  f1.ldo = g.hid;
  HIERA_TRY(launch_tc_gemm(EPI_GELU, f1, st));
  // (a12) fc2 + residual
  TcGemmArgs f2{};
  f2.w_static = 1;  // packed block weights
  f2.M = (int)qrows;
  f2.N = g.d_out;
  f2.K = g.hid;
  f2.A = ws + W.h;
  f2.W = packed + P.W3;
  f2.colconst = (const float*)(packed + P.b3);
  f2.out = y;
  f2.residual = ws + W.x1;
  f2.ldo = g.d_out;
  f2.stats_out = stats_y;
  f2.stats_out_parts = stats_y != nullptr ? parts_out : 0;
  return launch_tc_gemm(EPI_STORE, f2, st);
}

hiera_status forward_f32(const Geom& g, const uint8_t* packed, const void* x, void* y,
                         uint8_t* ws, cudaStream_t st) {
  const PackLayout P = pack_layout(g);
  const WsLayout W = ws_layout(g);
  const int rows = g.B * g.tokens, qrows = g.B * g.Nq;
  float* T = (float*)(ws + W.q);
  float2* st1 = (float2*)(ws + W.st1);
  float2* st2 = (float2*)(ws + W.st2);
  float* O = (float*)(ws + W.o);
  float* X1 = (float*)(ws + W.x1);
  float* H = (float*)(ws + W.h);
  HIERA_TRY(launch_row_stats_f32((const float*)x, rows, g.d_in, g.eps, st1, st));
  F32GemmArgs a{};
  a.M = rows;
  a.N = g.N1;
  a.K = g.d_in;
  a.A = (const float*)x;
  a.lda = g.d_in;
  a.W = (const float*)(packed + P.W1);
  a.stats = st1;
  a.colsum = (const float*)(packed + P.s1);
  a.colconst = (const float*)(packed + P.c1);
  a.out = T;
  a.ldo = g.N1;
  HIERA_TRY(launch_gemm_f32(a, st));
  F32AttnArgs at{};
  at.T = T;
  at.ldT = g.N1;
  at.q_off = 0;
  at.k_off = g.d_out;
  at.v_off = 2 * g.d_out;
  at.o = O;
  at.B = g.B;
  at.tokens = g.tokens;
  at.nW = g.nW;
  at.heads = g.heads;
  at.q_stride = g.qs;
  at.d_out = g.d_out;
  HIERA_TRY(launch_attention_f32(at, st));
  F32GemmArgs pj{};
  pj.M = qrows;
  pj.N = g.d_out;
  pj.K = g.d_out;
  pj.A = O;
  pj.lda = g.d_out;
  pj.W = (const float*)(packed + P.Wo);
  pj.colconst = (const float*)(packed + P.bo);
  if (g.transition) {
    pj.residual = T + 3 * g.d_out;
    pj.ldr = g.N1;
    pj.resid_pool_tokens = g.qs == 4 ? g.tokens : 0;
  } else {
    pj.residual = (const float*)x;
    pj.ldr = g.d_out;
  }
  pj.out = X1;
  pj.ldo = g.d_out;
  HIERA_TRY(launch_gemm_f32(pj, st));
  HIERA_TRY(launch_row_stats_f32(X1, qrows, g.d_out, g.eps, st2, st));
  F32GemmArgs f1{};
  f1.M = qrows;
  f1.N = g.hid;
  f1.K = g.d_out;
  f1.A = X1;
  f1.lda = g.d_out;
  f1.W = (const float*)(packed + P.W2);
  f1.stats = st2;
  f1.colsum = (const float*)(packed + P.s2);
  f1.colconst = (const float*)(packed + P.c2);
  f1.gelu = 1;
  f1.out = H;
  f1.ldo = g.hid;
  HIERA_TRY(launch_gemm_f32(f1, st));
  F32GemmArgs f2{};
  f2.M = qrows;
  f2.N = g.d_out;
  f2.K = g.hid;
  f2.A = H;
  f2.lda = g.hid;
  f2.W = (const float*)(packed + P.W3);
  f2.colconst = (const float*)(packed + P.b3);
  f2.residual = X1;
  f2.ldr = g.d_out;
  f2.out = (float*)y;
  f2.ldo = g.d_out;
  return launch_gemm_f32(f2, st);
}

// ---------------------------------------------------------------- backbone schedule
constexpr int kDepth = 24;
const int kStageDepth[4] = {2, 3, 16, 3};
const int kStageDim[4] = {112, 224, 448, 896};
const int kStageHeads[4] = {2, 4, 8, 16};
const int kStageEnds[4] = {1, 4, 20, 23};

struct BlockPlan {
  hiera_block_desc d;
  int stage;
};

hiera_status backbone_plan(const hiera_backbone_desc* bd, BlockPlan plan[kDepth]) {
  if (bd == nullptr) return HIERA_ERR_INVALID_ARG;
  if (bd->dtype != HIERA_F32 && bd->dtype != HIERA_BF16) return HIERA_ERR_DTYPE;
  if (bd->B < 1 || bd->img < 32) return HIERA_ERR_INVALID_ARG;
  if (bd->img % 32 != 0) return HIERA_ERR_SHAPE;
  const int G0 = bd->img / 4;
  int i = 0, prev_dim = kStageDim[0];
  for (int s = 0; s < 4; ++s) {
    const int Gs = G0 >> s;
    for (int j = 0; j < kStageDepth[s]; ++j, ++i) {
      const bool trans = s > 0 && j == 0;
      const int tokens_in = trans ? (Gs * 2) * (Gs * 2) : Gs * Gs;
      const int flat_mu = 64 >> (2 * s);  // q tokens per unit after this block
      hiera_block_desc& d = plan[i].d;
      d.B = bd->B;
      d.tokens = tokens_in;
      d.dim_in = trans ? prev_dim : kStageDim[s];
      d.dim_out = kStageDim[s];
      d.heads = kStageHeads[s];
      d.head_dim = 56;
      d.q_stride = trans ? 4 : 1;
      d.window_tokens = flat_mu * d.q_stride;
      d.mask_unit_attn = (s < 2) || (i == 5 && bd->mask_unit_attn_stage2_first) ? 1 : 0;
      d.ln_eps = 1e-6f;
      d.dtype = bd->dtype;
      plan[i].stage = s;
      Geom g;
      HIERA_TRY(make_geom(&d, &g));
    }
    prev_dim = kStageDim[s];
  }
  return HIERA_OK;
}

struct BackbonePack {
  size_t patch_w, patch_b, pos, blocks[kDepth], total;
};

BackbonePack backbone_pack_layout(const hiera_backbone_desc* bd, const BlockPlan plan[kDepth]) {
  BackbonePack L;
  const size_t es = bd->dtype == HIERA_BF16 ? 2 : 4;
  const size_t G0 = bd->img / 4;
  size_t o = 0;
  L.patch_w = o;
  L.patch_b = o + PATCH_OFF_BIAS;
  o = up256(o + HIERA_PATCH_PACKED_BYTES);
  L.pos = o; o = up256(o + G0 * G0 * 112 * es);
  for (int i = 0; i < kDepth; ++i) {
    Geom g;
    make_geom(&plan[i].d, &g);
    L.blocks[i] = o;
    o = up256(o + pack_layout(g).total);
  }
  L.total = o;
  return L;
}

struct BackboneWs {
  size_t act0, act1, st0, st1, block, total;
};

BackboneWs backbone_ws_layout(const hiera_backbone_desc* bd, const BlockPlan plan[kDepth]) {
  BackboneWs L;
  const size_t es = bd->dtype == HIERA_BF16 ? 2 : 4;
  const size_t G0 = bd->img / 4;
  const size_t act = (size_t)bd->B * G0 * G0 * 112 * es;  // largest stage activation
  size_t blk = 0;
  for (int i = 0; i < kDepth; ++i) {
    Geom g;
    make_geom(&plan[i].d, &g);
    blk = std::max(blk, ws_layout(g).total);
  }
  // LayerNorm partials passed from block to block: at most 2 per stage-0 token
  const size_t stb = (size_t)bd->B * G0 * G0 * 2 * 8;
  L.act0 = 0;
  L.act1 = up256(act);
  L.st0 = L.act1 + up256(act);
  L.st1 = L.st0 + up256(stb);
  L.block = L.st1 + up256(stb);
  L.total = L.block + blk;
  return L;
}

// A call's images are independent, and every kernel of the forward sizes its grid to the SM
// count: run as two concurrent half batches on two streams, the halves' kernels take the SMs
// that a single chain of kernels leaves idle in its kernel tails and partial waves
// (HIERA_OPT_SPLIT_BATCH). The second stream and the fork / join events belong to the
// calling thread (one set per device), so calls from other threads never share them.
struct AuxStreams {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
thread_local AuxStreams t_aux[kMaxDev];

// The calling thread's second stream on the current device, created on first use (never
// inside a stream capture: with `capturing` set and no stream yet, *out stays nullptr and
// the call runs as one batch). hiera_backbone_pack creates it ahead of time.
hiera_status aux_streams(AuxStreams** out, bool capturing) {
  *out = nullptr;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return HIERA_ERR_CUDA;
  AuxStreams& a = t_aux[dev];
  if (a.s == nullptr) {
    if (capturing) return HIERA_OK;
    if (cudaStreamCreateWithFlags(&a.s, cudaStreamNonBlocking) != cudaSuccess) {
      a.s = nullptr;
      return HIERA_ERR_CUDA;
    }
    if (cudaEventCreateWithFlags(&a.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&a.join, cudaEventDisableTiming) != cudaSuccess)
      return HIERA_ERR_CUDA;
  }
  *out = &a;
  return HIERA_OK;
}

// the two halves of a split batch: images [0, B1) and [B1, B)
void split_descs(const hiera_backbone_desc* d, hiera_backbone_desc* h1, hiera_backbone_desc* h2) {
  *h1 = *d;
  *h2 = *d;
  h1->B = (d->B + 1) / 2;
  h2->B = d->B - h1->B;
}

bool profile_open();
// (not while a launch profile is open: its events bracket consecutive launches on one stream)
bool split_applies(const hiera_backbone_desc* d) {
  return g_option(HIERA_OPT_SPLIT_BATCH) != 0 && d->B >= 2 && !profile_open();
}

// workspace of a split call: the first half's, then (256-byte aligned) the second half's
size_t split_ws_bytes(const hiera_backbone_desc* d, size_t* second_off) {
  hiera_backbone_desc h1, h2;
  split_descs(d, &h1, &h2);
  BlockPlan p1[kDepth], p2[kDepth];
  if (backbone_plan(&h1, p1) != HIERA_OK || backbone_plan(&h2, p2) != HIERA_OK) return 0;
  const size_t a = up256(backbone_ws_layout(&h1, p1).total);
  if (second_off != nullptr) *second_off = a;
  return a + backbone_ws_layout(&h2, p2).total;
}

// One forward of the backbone for desc->B images, enqueued on one stream.
hiera_status backbone_run(const hiera_backbone_desc* desc, const BlockPlan plan[kDepth],
                          const uint8_t* pk, const void* img_nhwc, void* const feats[4],
                          uint8_t* ws, cudaStream_t st) {
  const BackbonePack P = backbone_pack_layout(desc, plan);
  const BackboneWs W = backbone_ws_layout(desc, plan);
  const int bf = desc->dtype == HIERA_BF16 ? 1 : 0;
  const int es = bf ? 2 : 4;
  const int G0 = desc->img / 4;
  uint8_t* act[2] = {ws + W.act0, ws + W.act1};
  float2* stp[2] = {(float2*)(ws + W.st0), (float2*)(ws + W.st1)};
  // (a0-a2) patch embedding + pos_embed + Unroll, fused; in bf16 it also emits the LayerNorm
  // partials of its output (two 56-channel halves per token) for block 0's norm1
  HIERA_TRY(launch_patch_embed(img_nhwc, pk + P.patch_w, pk + P.pos, act[0],
                               bf ? stp[0] : nullptr, desc->B, desc->img, bf, st));
  int cur = 0, s_idx = 0, parts = 2;
  for (int i = 0; i < kDepth; ++i) {
    Geom g;
    make_geom(&plan[i].d, &g);
    const uint8_t* bp = pk + P.blocks[i];
    uint8_t* out = act[cur ^ 1];
    HIERA_TRY(g.bf16 ? forward_bf16(g, bp, act[cur], out, ws + W.block, st, stp[cur], parts,
                                    stp[cur ^ 1])
                     : forward_f32(g, bp, act[cur], out, ws + W.block, st));
    parts = store_stats_parts(g.d_out);
    cur ^= 1;
    if (s_idx < 4 && i == kStageEnds[s_idx]) {
      // (a13) Reroll the stage output to NHWC
      const int s = plan[i].stage;
      const int Gs = G0 >> s;
      if (launch_permute(false, act[cur], feats[s_idx], desc->B, Gs, kStageDim[s], 3 - s, es,
                         st) != cudaSuccess)
        return HIERA_ERR_CUDA;
      ++s_idx;
    }
  }
  return HIERA_OK;
}

// Library-owned scratch for hiera_block_forward_noalloc (see include/hiera.h): a static
// device array, so calls through that entry point allocate nothing. Host code needs the
// array's device address, looked up once per device with that device current.
static __device__ __align__(256) unsigned char g_static_scratch[HIERA_STATIC_SCRATCH_BYTES];
void* g_static_scratch_addr[kMaxDev] = {};
std::mutex g_static_scratch_mu;

hiera_status static_scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return HIERA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_static_scratch_mu);
  if (g_static_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr)
      return HIERA_ERR_CUDA;
    g_static_scratch_addr[dev] = p;
  }
  *out = g_static_scratch_addr[dev];
  return HIERA_OK;
}

// The tensor-core path's GELU as its epilogues evaluate it: on pairs with the packed fp32
// instructions (an odd n's last value alone, through the scalar form, which gives the same
// bits).
__global__ void gelu_probe_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i + 1 < n) {
    f2_unpack(gelu_fast2(f2_pack(x[i], x[i + 1])), y[i], y[i + 1]);
  } else if (i < n) {
    y[i] = gelu_fast(x[i]);
  }
}

__global__ void timeout_probe_kernel(uint64_t limit_ns, unsigned int* status) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  // nothing ever arrives on `bar`: phase 0 never completes and the bounded wait gives up
  if (threadIdx.x == 0) mbar_wait(&bar, 0, limit_ns, status);
}

}  // namespace

int g_num_sms() {
  const int s = dev_info().sms;
  return s > 0 ? s : 148;
}

unsigned int* g_status_ptr() { return dev_info().status; }

bool ensure_smem_attr(const void* kern, int bytes) {
  static std::mutex mu;
  static std::set<std::pair<const void*, int>> done;  // (kernel, device)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  std::lock_guard<std::mutex> lk(mu);
  if (done.count({kern, dev})) return true;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess)
    return false;
  done.insert({kern, dev});
  return true;
}

namespace {
// Under stream capture a plain cudaEventRecord only orders the capture; the external
// flag makes it an event-record node that re-records on every graph replay.
void record_profile_event(cudaEvent_t ev, cudaStream_t stream) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  cudaStreamIsCapturing(stream, &cs);
  if (cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(ev, stream, cudaEventRecordExternal);
  else
    cudaEventRecord(ev, stream);
}

struct ProfileSession {
  void* const* events = nullptr;
  int* kinds = nullptr;
  int capacity = 0;
  int count = 0;
  bool open = false;
} g_prof;

bool profile_open() { return g_prof.open; }
}  // namespace

void profile_mark(int kind, cudaStream_t stream) {
  if (!g_prof.open) return;
  if (g_prof.count < g_prof.capacity) {
    record_profile_event(static_cast<cudaEvent_t>(g_prof.events[g_prof.count]), stream);
    g_prof.kinds[g_prof.count] = kind;
  }
  ++g_prof.count;
}

namespace {
// fused MLP, programmatic dependent launch and fused attention half on; the eight-warp
// 224-column GEMM
int g_options[HIERA_OPT_COUNT] = {1, 1, 1, 0, 1};
}  // namespace

int g_option(int opt) { return (opt >= 0 && opt < HIERA_OPT_COUNT) ? g_options[opt] : 0; }

uint64_t g_wait_limit_ns() {
  static uint64_t limit = [] {
    const char* e = getenv("HIERA_WAIT_LIMIT_MS");
    long ms = e != nullptr ? atol(e) : 0;
    if (ms <= 0) ms = 2000;
    return (uint64_t)ms * 1000000ull;
  }();
  return limit;
}

}  // namespace hiera

using namespace hiera;

extern "C" {

const char* hiera_status_string(hiera_status s) {
  switch (s) {
    case HIERA_OK: return "HIERA_OK";
    case HIERA_ERR_INVALID_ARG: return "HIERA_ERR_INVALID_ARG";
    case HIERA_ERR_SHAPE: return "HIERA_ERR_SHAPE";
    case HIERA_ERR_DTYPE: return "HIERA_ERR_DTYPE";
    case HIERA_ERR_ALIGNMENT: return "HIERA_ERR_ALIGNMENT";
    case HIERA_ERR_WORKSPACE: return "HIERA_ERR_WORKSPACE";
    case HIERA_ERR_CUDA: return "HIERA_ERR_CUDA";
    case HIERA_ERR_TIMEOUT: return "HIERA_ERR_TIMEOUT";
    case HIERA_ERR_DEVICE: return "HIERA_ERR_DEVICE";
  }
  return "HIERA_ERR_UNKNOWN";
}

hiera_status hiera_get_device_status(hiera_stream_t stream) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return HIERA_ERR_CUDA;
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(v)) != cudaSuccess) return HIERA_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero)) != cudaSuccess)
    return HIERA_ERR_CUDA;
  return (hiera_status)v;
}

static hiera_status permute_common(bool unroll, const void* x, void* y, int B, int G, int C,
                                   int levels, hiera_dtype dt, hiera_stream_t stream) {
  if (x == nullptr || y == nullptr || x == y) return HIERA_ERR_INVALID_ARG;
  if (dt != HIERA_F32 && dt != HIERA_BF16) return HIERA_ERR_DTYPE;
  if (B < 1 || G < 1 || C < 1 || levels < 0 || levels > 5) return HIERA_ERR_INVALID_ARG;
  const int es = dt == HIERA_BF16 ? 2 : 4;
  if (G % (1 << levels) != 0 || (C * es) % 16 != 0) return HIERA_ERR_SHAPE;
  if ((long long)G * G > (1ll << 30)) return HIERA_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(y)) return HIERA_ERR_ALIGNMENT;
  HIERA_TRY(check_device());
  return launch_permute(unroll, x, y, B, G, C, levels, es, (cudaStream_t)stream) == cudaSuccess
             ? HIERA_OK
             : HIERA_ERR_CUDA;
}

hiera_status hiera_unroll(const void* x, void* y, int B, int G, int C, int levels,
                          hiera_dtype dtype, hiera_stream_t stream) {
  return permute_common(true, x, y, B, G, C, levels, dtype, stream);
}

hiera_status hiera_reroll(const void* x, void* y, int B, int G, int C, int levels,
                          hiera_dtype dtype, hiera_stream_t stream) {
  return permute_common(false, x, y, B, G, C, levels, dtype, stream);
}

hiera_status hiera_linear(const void* x, const void* w, const void* bias, const void* residual,
                          void* y, int M, int N, int K, hiera_dtype dtype,
                          hiera_stream_t stream) {
  if (x == nullptr || w == nullptr || y == nullptr) return HIERA_ERR_INVALID_ARG;
  if (dtype != HIERA_F32 && dtype != HIERA_BF16) return HIERA_ERR_DTYPE;
  if (M < 1 || N < 1 || K < 1) return HIERA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w) || !aligned16(y) || (bias && !aligned16(bias)) ||
      (residual && !aligned16(residual)))
    return HIERA_ERR_ALIGNMENT;
  HIERA_TRY(check_device());
  if (dtype == HIERA_BF16) {
    if (N % 16 != 0 || K % 8 != 0) return HIERA_ERR_SHAPE;
    TcGemmArgs a{};
    a.M = M;
    a.N = N;
    a.K = K;
    a.A = x;
    a.W = w;
    a.bias_bf16 = bias;
    a.out = y;
    a.residual = residual;
    a.ldo = N;
    return launch_tc_gemm(EPI_STORE, a, (cudaStream_t)stream);
  }
  F32GemmArgs a{};
  a.M = M;
  a.N = N;
  a.K = K;
  a.A = (const float*)x;
  a.lda = K;
  a.W = (const float*)w;
  a.colconst = (const float*)bias;
  a.residual = (const float*)residual;
  a.ldr = N;
  a.out = (float*)y;
  a.ldo = N;
  return launch_gemm_f32(a, (cudaStream_t)stream);
}

size_t hiera_block_packed_bytes(const hiera_block_desc* desc) {
  Geom g;
  if (make_geom(desc, &g) != HIERA_OK) return 0;
  return pack_layout(g).total;
}

hiera_status hiera_block_pack(const hiera_block_desc* desc, const hiera_block_weights* w,
                              void* packed, size_t packed_bytes, hiera_stream_t stream) {
  Geom g;
  HIERA_TRY(make_geom(desc, &g));
  if (w == nullptr || packed == nullptr || !weights_ok(g, w)) return HIERA_ERR_INVALID_ARG;
  if (!aligned16(packed) || !weights_aligned(w)) return HIERA_ERR_ALIGNMENT;
  if (packed_bytes < pack_layout(g).total) return HIERA_ERR_WORKSPACE;
  HIERA_TRY(check_device());
  return pack_block(g, w, static_cast<uint8_t*>(packed), (cudaStream_t)stream);
}

size_t hiera_block_workspace_bytes(const hiera_block_desc* desc) {
  Geom g;
  if (make_geom(desc, &g) != HIERA_OK) return 0;
  return ws_layout(g).total;
}

hiera_status hiera_block_workspace_layout(const hiera_block_desc* desc, long long offsets[7]) {
  Geom g;
  HIERA_TRY(make_geom(desc, &g));
  if (offsets == nullptr) return HIERA_ERR_INVALID_ARG;
  const WsLayout L = ws_layout(g);
  offsets[0] = L.q;
  offsets[1] = L.k;
  offsets[2] = L.v;
  offsets[3] = L.o;
  offsets[4] = L.r;
  offsets[5] = L.x1;
  offsets[6] = L.h;
  return HIERA_OK;
}

hiera_status hiera_block_forward(const hiera_block_desc* desc, const void* packed, const void* x,
                                 void* y, void* workspace, size_t workspace_bytes,
                                 hiera_stream_t stream) {
  Geom g;
  HIERA_TRY(make_geom(desc, &g));
  if (packed == nullptr || x == nullptr || y == nullptr || workspace == nullptr)
    return HIERA_ERR_INVALID_ARG;
  if (!aligned16(packed) || !aligned16(x) || !aligned16(y) || !aligned16(workspace))
    return HIERA_ERR_ALIGNMENT;
  if (workspace_bytes < ws_layout(g).total) return HIERA_ERR_WORKSPACE;
  HIERA_TRY(check_device());
  const cudaStream_t st = (cudaStream_t)stream;
  return g.bf16 ? forward_bf16(g, (const uint8_t*)packed, x, y, (uint8_t*)workspace, st)
                : forward_f32(g, (const uint8_t*)packed, x, y, (uint8_t*)workspace, st);
}

size_t hiera_static_scratch_bytes(void) { return HIERA_STATIC_SCRATCH_BYTES; }

hiera_status hiera_block_forward_noalloc(const hiera_block_desc* desc, const void* packed,
                                         const void* x, void* y, hiera_stream_t stream) {
  Geom g;
  HIERA_TRY(make_geom(desc, &g));
  if (packed == nullptr || x == nullptr || y == nullptr) return HIERA_ERR_INVALID_ARG;
  if (!aligned16(packed) || !aligned16(x) || !aligned16(y)) return HIERA_ERR_ALIGNMENT;
  if (ws_layout(g).total > HIERA_STATIC_SCRATCH_BYTES) return HIERA_ERR_WORKSPACE;
  HIERA_TRY(check_device());
  void* scratch = nullptr;
  HIERA_TRY(static_scratch_address(&scratch));
  const cudaStream_t st = (cudaStream_t)stream;
  return g.bf16 ? forward_bf16(g, (const uint8_t*)packed, x, y, (uint8_t*)scratch, st)
                : forward_f32(g, (const uint8_t*)packed, x, y, (uint8_t*)scratch, st);
}

hiera_status hiera_attention(const void* q, const void* k, const void* v, void* o, int B,
                             int windows, int heads, int Tq, int Tkv, hiera_stream_t stream) {
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) return HIERA_ERR_INVALID_ARG;
  if (B < 1 || windows < 1 || heads < 1 || Tq < 1 || Tkv < 1) return HIERA_ERR_INVALID_ARG;
  if ((long long)B * windows * heads * std::max(Tq, Tkv) > (1ll << 31)) return HIERA_ERR_SHAPE;
  if ((long long)heads * 56 > (1 << 20)) return HIERA_ERR_SHAPE;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return HIERA_ERR_ALIGNMENT;
  HIERA_TRY(check_device());
  AttnArgs at{};
  at.q = q;
  at.k = k;
  at.v = v;
  at.o = o;
  at.B = B;
  at.nW = windows;
  at.heads = heads;
  at.Tq = Tq;
  at.Tkv = Tkv;
  at.d_out = heads * 56;
  return launch_attention(at, (cudaStream_t)stream);
}

hiera_status hiera_patch_pack(const void* patch_w, const void* patch_b, void* packed,
                              hiera_dtype dtype, hiera_stream_t stream) {
  if (patch_w == nullptr || packed == nullptr) return HIERA_ERR_INVALID_ARG;
  if (dtype != HIERA_F32 && dtype != HIERA_BF16) return HIERA_ERR_DTYPE;
  if (!aligned16(patch_w) || !aligned16(packed) || (patch_b != nullptr && !aligned16(patch_b)))
    return HIERA_ERR_ALIGNMENT;
  HIERA_TRY(check_device());
  return launch_patch_pack(patch_w, patch_b, dtype == HIERA_BF16 ? 1 : 0, packed,
                           (cudaStream_t)stream);
}

hiera_status hiera_patch_embed(const void* img, const void* packed_patch, const void* pos_embed,
                               void* out, int B, int img_side, hiera_dtype dtype,
                               hiera_stream_t stream) {
  if (img == nullptr || packed_patch == nullptr || pos_embed == nullptr || out == nullptr)
    return HIERA_ERR_INVALID_ARG;
  if (dtype != HIERA_F32 && dtype != HIERA_BF16) return HIERA_ERR_DTYPE;
  if (B < 1 || img_side < 32) return HIERA_ERR_INVALID_ARG;
  if (img_side % 32 != 0) return HIERA_ERR_SHAPE;
  if (!aligned16(img) || !aligned16(packed_patch) || !aligned16(pos_embed) || !aligned16(out))
    return HIERA_ERR_ALIGNMENT;
  HIERA_TRY(check_device());
  return launch_patch_embed(img, packed_patch, pos_embed, out, nullptr, B, img_side,
                            dtype == HIERA_BF16 ? 1 : 0, (cudaStream_t)stream);
}

size_t hiera_backbone_packed_bytes(const hiera_backbone_desc* desc) {
  BlockPlan plan[kDepth];
  if (backbone_plan(desc, plan) != HIERA_OK) return 0;
  return backbone_pack_layout(desc, plan).total;
}

hiera_status hiera_backbone_pack(const hiera_backbone_desc* desc, const hiera_backbone_weights* w,
                                 void* packed, size_t packed_bytes, hiera_stream_t stream) {
  BlockPlan plan[kDepth];
  HIERA_TRY(backbone_plan(desc, plan));
  if (w == nullptr || packed == nullptr || w->patch_w == nullptr || w->pos_embed == nullptr)
    return HIERA_ERR_INVALID_ARG;
  if (!aligned16(packed) || !aligned16(w->patch_w) || !aligned16(w->pos_embed) ||
      (w->patch_b != nullptr && !aligned16(w->patch_b)))
    return HIERA_ERR_ALIGNMENT;
  const BackbonePack L = backbone_pack_layout(desc, plan);
  if (packed_bytes < L.total) return HIERA_ERR_WORKSPACE;
  for (int i = 0; i < kDepth; ++i) {
    Geom g;
    make_geom(&plan[i].d, &g);
    if (!weights_ok(g, &w->blocks[i])) return HIERA_ERR_INVALID_ARG;
    if (!weights_aligned(&w->blocks[i])) return HIERA_ERR_ALIGNMENT;
  }
  HIERA_TRY(check_device());
  {
    // the calling thread's second stream for split-batch forwards, made here, outside any
    // capture the forward may later be enqueued in
    AuxStreams* aux = nullptr;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing((cudaStream_t)stream, &cap) != cudaSuccess) return HIERA_ERR_CUDA;
    HIERA_TRY(aux_streams(&aux, cap != cudaStreamCaptureStatusNone));
  }
  const cudaStream_t st = (cudaStream_t)stream;
  uint8_t* p = static_cast<uint8_t*>(packed);
  const int bf = desc->dtype == HIERA_BF16 ? 1 : 0;
  HIERA_TRY(launch_patch_pack(w->patch_w, w->patch_b, bf, p + L.patch_w, st));
  const int G0 = desc->img / 4;
  HIERA_TRY(launch_copy_pack(w->pos_embed, nullptr, G0 * G0, 112, bf, p + L.pos, nullptr, st));
  for (int i = 0; i < kDepth; ++i) {
    Geom g;
    make_geom(&plan[i].d, &g);
    HIERA_TRY(pack_block(g, &w->blocks[i], p + L.blocks[i], st));
  }
  return HIERA_OK;
}

size_t hiera_backbone_workspace_bytes(const hiera_backbone_desc* desc) {
  BlockPlan plan[kDepth];
  if (backbone_plan(desc, plan) != HIERA_OK) return 0;
  // enough for the call as one batch and as two concurrent halves, whatever the option
  const size_t whole = backbone_ws_layout(desc, plan).total;
  return desc->B >= 2 ? std::max(whole, split_ws_bytes(desc, nullptr)) : whole;
}

hiera_status hiera_backbone_forward(const hiera_backbone_desc* desc, const void* packed,
                                    const void* img_nhwc, void* const feats[4], void* workspace,
                                    size_t workspace_bytes, hiera_stream_t stream) {
  BlockPlan plan[kDepth];
  HIERA_TRY(backbone_plan(desc, plan));
  if (packed == nullptr || img_nhwc == nullptr || feats == nullptr || workspace == nullptr)
    return HIERA_ERR_INVALID_ARG;
  for (int s = 0; s < 4; ++s) {
    if (feats[s] == nullptr) return HIERA_ERR_INVALID_ARG;
    if (!aligned16(feats[s])) return HIERA_ERR_ALIGNMENT;
  }
  if (!aligned16(packed) || !aligned16(img_nhwc) || !aligned16(workspace))
    return HIERA_ERR_ALIGNMENT;
  const cudaStream_t st = (cudaStream_t)stream;
  const uint8_t* pk = static_cast<const uint8_t*>(packed);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (!split_applies(desc)) {
    if (workspace_bytes < backbone_ws_layout(desc, plan).total) return HIERA_ERR_WORKSPACE;
    HIERA_TRY(check_device());
    return backbone_run(desc, plan, pk, img_nhwc, feats, ws, st);
  }
  size_t off2 = 0;
  if (workspace_bytes < split_ws_bytes(desc, &off2)) return HIERA_ERR_WORKSPACE;
  HIERA_TRY(check_device());
  hiera_backbone_desc h1, h2;
  split_descs(desc, &h1, &h2);
  BlockPlan p1[kDepth], p2[kDepth];
  HIERA_TRY(backbone_plan(&h1, p1));
  HIERA_TRY(backbone_plan(&h2, p2));
  // the second half's image and feature rows follow the first half's B1 images
  const size_t es = desc->dtype == HIERA_BF16 ? 2 : 4;
  const size_t G0 = (size_t)desc->img / 4;
  const uint8_t* img2 = static_cast<const uint8_t*>(img_nhwc) +
                        (size_t)h1.B * desc->img * desc->img * 4 * es;
  void* feats2[4];
  for (int s = 0; s < 4; ++s) {
    const size_t Gs = G0 >> s;
    feats2[s] = static_cast<uint8_t*>(feats[s]) + (size_t)h1.B * Gs * Gs * kStageDim[s] * es;
  }
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cap) != cudaSuccess) return HIERA_ERR_CUDA;
  AuxStreams* aux = nullptr;
  HIERA_TRY(aux_streams(&aux, cap != cudaStreamCaptureStatusNone));
  if (aux == nullptr) {
    if (workspace_bytes < backbone_ws_layout(desc, plan).total) return HIERA_ERR_WORKSPACE;
    return backbone_run(desc, plan, pk, img_nhwc, feats, ws, st);
  }
  // fork: the second stream starts after everything the caller's stream holds so far
  if (cudaEventRecord(aux->fork, st) != cudaSuccess ||
      cudaStreamWaitEvent(aux->s, aux->fork, 0) != cudaSuccess)
    return HIERA_ERR_CUDA;
  const hiera_status r1 = backbone_run(&h1, p1, pk, img_nhwc, feats, ws, st);
  const hiera_status r2 = backbone_run(&h2, p2, pk, img2, feats2, ws + off2, aux->s);
  // join (also after a failed launch, so that the streams, or a capture, stay consistent)
  if (cudaEventRecord(aux->join, aux->s) != cudaSuccess ||
      cudaStreamWaitEvent(st, aux->join, 0) != cudaSuccess)
    return HIERA_ERR_CUDA;
  return r1 != HIERA_OK ? r1 : r2;
}

hiera_status hiera_profile_begin(void* const* events, int capacity, int* kinds) {
  if (events == nullptr || kinds == nullptr || capacity < 1) return HIERA_ERR_INVALID_ARG;
  g_prof.events = events;
  g_prof.kinds = kinds;
  g_prof.capacity = capacity;
  g_prof.count = 0;
  g_prof.open = true;
  return HIERA_OK;
}

int hiera_profile_end(hiera_stream_t stream) {
  if (!g_prof.open) return 0;
  g_prof.open = false;
  if (g_prof.count < g_prof.capacity)
    record_profile_event(static_cast<cudaEvent_t>(g_prof.events[g_prof.count]),
                         (cudaStream_t)stream);
  return g_prof.count;
}

hiera_status hiera_set_option(hiera_option opt, int value) {
  if (opt < 0 || opt >= HIERA_OPT_COUNT) return HIERA_ERR_INVALID_ARG;
  const int max_value = opt == HIERA_OPT_GEMM224 ? 2 : 1;
  if (value < 0 || value > max_value) return HIERA_ERR_INVALID_ARG;
  g_options[opt] = value;
  return HIERA_OK;
}

int hiera_get_option(hiera_option opt) { return g_option(opt); }

const char* hiera_kernel_name(int kind) {
  static const char* names[K_COUNT] = {
      "patch_embed", "unroll_reroll", "gemm_qkv_lnfold", "gemm_fc1_lnfold_gelu",
      "gemm_bias_residual", "attention_window", "f32_gemm", "f32_attention",
      "f32_row_stats", "pack", "timeout_probe", "row_stats", "attention_tcgen05",
      "mlp_fused", "attention_block_fused"};
  return (kind >= 0 && kind < K_COUNT) ? names[kind] : "unknown";
}

hiera_status hiera_debug_gelu(const float* x, float* y, int n, hiera_stream_t stream) {
  if (x == nullptr || y == nullptr || n < 1) return HIERA_ERR_INVALID_ARG;
  HIERA_TRY(check_device());
  profile_mark(K_PROBE, (cudaStream_t)stream);
  gelu_probe_kernel<<<((n + 1) / 2 + 255) / 256, 256, 0, (cudaStream_t)stream>>>(x, y, n);
  return cudaGetLastError() == cudaSuccess ? HIERA_OK : HIERA_ERR_CUDA;
}

hiera_status hiera_debug_timeout_probe(int limit_us, hiera_stream_t stream) {
  if (limit_us < 1 || limit_us > 10000000) return HIERA_ERR_INVALID_ARG;
  HIERA_TRY(check_device());
  profile_mark(K_PROBE, (cudaStream_t)stream);
  timeout_probe_kernel<<<1, 32, 0, (cudaStream_t)stream>>>((uint64_t)limit_us * 1000ull,
                                                           g_status_ptr());
  return cudaGetLastError() == cudaSuccess ? HIERA_OK : HIERA_ERR_CUDA;
}

}  // extern "C"
