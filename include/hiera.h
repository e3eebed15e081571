/*
 * hiera.h - C ABI of the B200 (sm_100a) Hiera mask-unit windowed block library.
 *
 * What it computes. The forward pass of the Hiera block and of the 24-block Hiera-B+
 * backbone as the "Phase 4: Hiera Backbone MLX Port" plan describes them (section
 * "Architecture Summary": PatchEmbed, pos_embed, Unroll, 24 HieraBlocks in 4 stages,
 * Reroll, stage transitions, MaskUnitAttention, MLP; section "Sub-phase 4a: Core
 * backbone module": unroll, reroll, undo_windowing, MaskUnitAttention, HieraMLP,
 * HieraBlock, HieraBackbone). All tensors are [B, N, C] token sequences, with NHWC
 * only at the backbone's input image and output features (Key Decisions item 5).
 *
 * Conventions shared by every entry point.
 *   Ownership  The caller owns every buffer. All tensor pointers are DEVICE pointers
 *              (cudaMalloc / PyTorch allocations) to dense, contiguous, row-major
 *              arrays, 16-byte aligned. The library allocates no device memory, keeps
 *              no pointer after a call returns and never frees anything.
 *   Dtype      HIERA_BF16: activations and weights are bfloat16, arithmetic
 *              accumulates in fp32 (tensor cores). HIERA_F32: everything fp32 with
 *              fp32 SIMT arithmetic. One dtype per call applies to every tensor
 *              argument of that call.
 *   Stream     Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *              stream) and runs asynchronously; nothing synchronises the host.
 *   Errors     Arguments are checked on the host before anything is launched; a bad
 *              argument returns an error code and launches nothing. A failed launch
 *              returns HIERA_ERR_CUDA. Kernels never trap: a device-side bounded wait
 *              that runs out records HIERA_ERR_TIMEOUT in a per-device status word,
 *              which hiera_get_device_status() reads. No CPU fallback exists.
 *   Device     The current CUDA device must be sm_100 (B200); otherwise
 *              HIERA_ERR_DEVICE.
 *   Linear     Weights follow the Linear convention [out, in] (Checkpoint Details:
 *              block weights are Linear, no transpose); the patch kernel is OHWI
 *              (112, 7, 7, 4).
 */
#ifndef HIERA_H_
#define HIERA_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define HIERA_API __attribute__((visibility("default")))
#else
#define HIERA_API
#endif

typedef struct CUstream_st* hiera_stream_t; /* identical to cudaStream_t */

typedef enum {
  HIERA_OK = 0,
  HIERA_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, unknown enum value */
  HIERA_ERR_SHAPE = 2,       /* a shape outside what the kernels support (see each call) */
  HIERA_ERR_DTYPE = 3,       /* dtype not HIERA_F32 / HIERA_BF16 */
  HIERA_ERR_ALIGNMENT = 4,   /* a pointer is not 16-byte aligned */
  HIERA_ERR_WORKSPACE = 5,   /* workspace or packed-weight buffer smaller than required */
  HIERA_ERR_CUDA = 6,        /* a CUDA runtime / driver call or a launch failed */
  HIERA_ERR_TIMEOUT = 7,     /* a device-side bounded wait ran out (kernel wound down) */
  HIERA_ERR_DEVICE = 8       /* current device is not an sm_100 GPU */
} hiera_status;

typedef enum { HIERA_F32 = 0, HIERA_BF16 = 1 } hiera_dtype;

/* Human-readable name of a status code (static string, never NULL). */
HIERA_API const char* hiera_status_string(hiera_status s);

/* Synchronises `stream`, then returns and clears the first device-side error recorded
 * on the current device since the previous call (HIERA_OK if none). */
HIERA_API hiera_status hiera_get_device_status(hiera_stream_t stream);

/* --------------------------------------------------------------------------------
 * Unroll / Reroll ("Architecture Summary": Unroll permutes tokens for mask-unit
 * windowed attention; Reroll undoes the permutation to spatial [B, H, W, C]; Sub-phase
 * 4a items 2-4).
 *
 * x and y: [B, G*G, C] of `dtype`. Unroll reads raster order (token y*G + x) and
 * writes unrolled order; Reroll reads unrolled order and writes raster (NHWC) order.
 * With L = levels and M = G / 2^L, spatial (y, x) with y = my*2^L + sum_k a_k 2^(k-1),
 * x = mx*2^L + sum_k b_k 2^(k-1) sits at unrolled token
 *   u = (sum_{k=1..L} (2 a_k + b_k) * 4^(L-k)) * M^2 + my*M + mx,
 * i.e. the finest 2x2 offset is the outermost index and the mask unit (my, mx) the
 * innermost. Requirements: B, G, C >= 1; 0 <= levels <= 5; G divisible by 2^levels;
 * C*sizeof(dtype) a multiple of 16 bytes (HIERA_ERR_SHAPE otherwise); x != y.
 * Bit-exact (a pure copy).
 * -------------------------------------------------------------------------------- */
HIERA_API hiera_status hiera_unroll(const void* x, void* y, int B, int G, int C, int levels,
                          hiera_dtype dtype, hiera_stream_t stream);
HIERA_API hiera_status hiera_reroll(const void* x, void* y, int B, int G, int C, int levels,
                          hiera_dtype dtype, hiera_stream_t stream);

/* --------------------------------------------------------------------------------
 * Linear ("Architecture Summary", MaskUnitAttention / MLP: every projection is a
 * Linear): y[M, N] = x[M, K] * w[N, K]^T + bias[N] (+ residual[M, N]).
 * bias and residual may be NULL. HIERA_BF16 runs on the tcgen05 tensor cores with fp32
 * accumulation; it needs N a multiple of 16 and K a multiple of 8 (HIERA_ERR_SHAPE).
 * HIERA_F32 runs fp32 SIMT. residual may alias y (in-place accumulate).
 * -------------------------------------------------------------------------------- */
HIERA_API hiera_status hiera_linear(const void* x, const void* w, const void* bias, const void* residual,
                          void* y, int M, int N, int K, hiera_dtype dtype,
                          hiera_stream_t stream);

/* --------------------------------------------------------------------------------
 * One HieraBlock (Sub-phase 4a item 7): norm1 -> [proj + max-pool if transition] ->
 * MaskUnitAttention + residual -> norm2 -> MLP + residual.
 *
 * Fields of hiera_block_desc:
 *   B              batch
 *   tokens         tokens per image at the block input (N)
 *   dim_in         channels of the input; dim_out channels of the output.
 *                  dim_in != dim_out marks a transition block, whose residual branch is
 *                  proj = Linear(dim_in, dim_out) of norm1's output, max-pooled over the
 *                  q_stride outermost token chunks.
 *   heads, head_dim  dim_out = heads * head_dim; head_dim must be 56.
 *   q_stride       1, or 4 (queries max-pooled over the 4 outermost chunks of each
 *                  window's token axis: "q_stride > 1 at transitions: max-pool over
 *                  q_stride dim in queries").
 *   window_tokens  keys per mask-unit window at the block input (64 at stage 0, 64 for
 *                  the stage-1 transition, 16 at stage 1); token n belongs to window
 *                  n mod (tokens / window_tokens). Ignored if mask_unit_attn == 0.
 *   mask_unit_attn 1 = attention inside each mask unit; 0 = global (one window).
 *   ln_eps         LayerNorm epsilon (1e-6 for Hiera), population variance.
 *   dtype          HIERA_BF16 or HIERA_F32.
 * Output tokens: tokens / q_stride, in the same unrolled order, dim_out channels.
 * Shape limits (HIERA_ERR_SHAPE): head_dim 56; dim_in and dim_out multiples of 16;
 * q_stride divides tokens; with mask_unit_attn, window_tokens divides tokens and
 * q_stride divides window_tokens; for bf16 with q_stride 4, tokens a multiple of 128.
 *
 * Weights (hiera_block_weights): all of `dtype`, Linear [out, in]:
 *   norm1_w/b [dim_in]; qkv_w [3*dim_out, dim_in], qkv_b [3*dim_out] with output
 *   channel c = which*dim_out + head*56 + e (which 0/1/2 = q/k/v); proj_w [dim_out,
 *   dim_in], proj_b [dim_out] (transition blocks only, else NULL); attn_proj_w
 *   [dim_out, dim_out], attn_proj_b; norm2_w/b [dim_out]; fc1_w [4*dim_out, dim_out],
 *   fc1_b; fc2_w [dim_out, 4*dim_out], fc2_b.
 *
 * hiera_block_pack() converts the weights once into `packed` (caller memory of
 * hiera_block_packed_bytes() bytes): LayerNorm's gamma is folded into the following
 * Linear (W' = W diag(gamma)) together with the column sums of W' and the constant
 * beta W^T + b, so that the forward pass applies LayerNorm inside the GEMM epilogue
 * (bf16: from per-row (mean, M2) partials written by the kernel that produced the
 * LayerNorm's input, merged in the epilogue; x itself is reduced once by a small
 * statistics kernel). The raw weights may be freed after the pack has run.
 *
 * hiera_block_forward(): x [B, tokens, dim_in] -> y [B, tokens/q_stride, dim_out];
 * workspace of hiera_block_workspace_bytes() bytes holds the intermediates. x, y,
 * packed and workspace must not overlap.
 * -------------------------------------------------------------------------------- */
typedef struct {
  int B;
  int tokens;
  int dim_in;
  int dim_out;
  int heads;
  int head_dim;
  int q_stride;
  int window_tokens;
  int mask_unit_attn;
  float ln_eps;
  hiera_dtype dtype;
} hiera_block_desc;

typedef struct {
  const void* norm1_w;
  const void* norm1_b;
  const void* qkv_w;
  const void* qkv_b;
  const void* proj_w;
  const void* proj_b;
  const void* attn_proj_w;
  const void* attn_proj_b;
  const void* norm2_w;
  const void* norm2_b;
  const void* fc1_w;
  const void* fc1_b;
  const void* fc2_w;
  const void* fc2_b;
} hiera_block_weights;

HIERA_API size_t hiera_block_packed_bytes(const hiera_block_desc* desc);
HIERA_API hiera_status hiera_block_pack(const hiera_block_desc* desc, const hiera_block_weights* w,
                              void* packed, size_t packed_bytes, hiera_stream_t stream);
HIERA_API size_t hiera_block_workspace_bytes(const hiera_block_desc* desc);
HIERA_API hiera_status hiera_block_forward(const hiera_block_desc* desc, const void* packed, const void* x,
                                 void* y, void* workspace, size_t workspace_bytes,
                                 hiera_stream_t stream);

/* Byte offsets of the block's intermediates inside its workspace, for inspection:
 * [0] q, [1] k, [2] v (head-major: bf16 [B][windows][heads][T][64] with channels 56..63
 * zero, except v's channel 56, which holds 1.0 (the layout hiera_attention() takes); f32
 * token-major [B, tokens, 4*dim_out] holding q|k|v|proj in [0] and -1 in [1],[2]), [3] merged
 * attention output [B, tokens/q_stride, dim_out], [4] transition residual (or -1), [5] x
 * after the attention residual, [6] MLP hidden [B, tokens/q_stride, 4*dim_out] (left
 * unwritten when the bf16 MLP runs fused: dim_out 112 or 224 with HIERA_OPT_FUSED_MLP).
 * Returns HIERA_ERR_SHAPE on a bad desc. */
HIERA_API hiera_status hiera_block_workspace_layout(const hiera_block_desc* desc, long long offsets[7]);

/* --------------------------------------------------------------------------------
 * Attention core of MaskUnitAttention ("Architecture Summary", MaskUnitAttention:
 * scaled dot-product attention per mask-unit window, or over all tokens, then the heads
 * merged before proj), on the head-major q/k/v the block's qkv projection writes.
 *
 *   o[b, j*windows + w, h*56 + e] = sum_t softmax_t(q_j . k_t / sqrt(56)) v_t[e]
 *
 * for every image b, window w, head h and query j < Tq, over the window's Tkv keys t.
 * All tensors are bf16:
 *   q  [B][windows][heads][Tq][64]   channels 56..63 zero (head_dim 56, padded);
 *   k  [B][windows][heads][Tkv][64]  channels 56..63 zero;
 *   v  [B][windows][heads][Tkv][64]  channel 56 = 1.0 and 57..63 zero (the kernels sum the
 *                                    softmax denominator through that channel);
 *   o  [B, Tq*windows, heads*56]     written; token j*windows + w, channel h*56 + e.
 * Queries are already max-pooled where the block pools them (Tq = Tkv / q_stride). The
 * softmax is max-subtracted in fp32 with fp32 accumulation; the weights enter the P V
 * product as bf16. Windows of 4..64 keys (a power of two) with Tq = Tkv or Tkv / 4 run
 * several windows per tensor-core tile; every other size runs the 128-key-tile kernel.
 * Any B, windows, heads >= 1 with B*windows*heads*max(Tq, Tkv) <= 2^31.
 * -------------------------------------------------------------------------------- */
HIERA_API hiera_status hiera_attention(const void* q, const void* k, const void* v, void* o,
                                       int B, int windows, int heads, int Tq, int Tkv,
                                       hiera_stream_t stream);

/* --------------------------------------------------------------------------------
 * Allocation-free variant of hiera_block_forward (no counterpart on the pages: it exists
 * for callers, not for the method).
 *
 * Some callers cannot provide a workspace because they cannot allocate device memory at
 * all: a plug-in running inside a host framework that owns every device allocation and
 * hands the plug-in only its input and output buffers, or a real-time loop whose policy
 * forbids cudaMalloc once it has started. hiera_block_forward_noalloc() computes exactly
 * what hiera_block_forward() computes, but its intermediates live in one library-owned
 * device array of HIERA_STATIC_SCRATCH_BYTES bytes (32 MiB), declared statically in the
 * library: every GPU that loads the library holds that array until the process exits.
 * The call itself allocates and frees nothing.
 *
 * The caller still passes the packed weights, the input x and the output y (as for
 * hiera_block_forward). A block whose hiera_block_workspace_bytes() exceeds
 * HIERA_STATIC_SCRATCH_BYTES is rejected with HIERA_ERR_WORKSPACE before anything runs.
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress,
 * with that device current) and caches it; make that first call before any stream
 * capture. All calls share the one array, which keeps the last call's contents: calls
 * whose GPU work overlaps (different streams, or different host threads) race on it and
 * must be serialised by the caller. Nothing in the array needs to start at zero: every
 * byte a call reads was written earlier in the same call.
 * -------------------------------------------------------------------------------- */
#define HIERA_STATIC_SCRATCH_BYTES ((size_t)32 << 20)
/* The size of that array as compiled into the library (HIERA_STATIC_SCRATCH_BYTES), for
 * callers that load the library without this header. */
HIERA_API size_t hiera_static_scratch_bytes(void);
HIERA_API hiera_status hiera_block_forward_noalloc(const hiera_block_desc* desc,
                                                   const void* packed, const void* x, void* y,
                                                   hiera_stream_t stream);

/* --------------------------------------------------------------------------------
 * PatchEmbed + pos_embed + Unroll ("Architecture Summary": Conv2d(4 -> 112, 7x7,
 * stride 4) reshaped to [B, N, C]; learned pos_embed (1, N, 112) added; Unroll).
 *
 * hiera_patch_pack(): patch_w OHWI [112, 7, 7, 4] and patch_b [112] (may be NULL = 0) of
 * `dtype` -> `packed` (caller memory of HIERA_PATCH_PACKED_BYTES bytes): fp32 [196][112]
 * with k = (ky*7 + kx)*4 + c, then at byte 87808 the fp32 bias [112], then at byte 88256
 * the weight as bf16 [112][208] (k fastest, zero for k >= 196) for the tensor-core path.
 * hiera_patch_embed(): img NHWC [B, img, img, 4]; pos_embed [(img/4)^2, 112] in raster
 * order; out [B, (img/4)^2, 112] in the unrolled order of hiera_unroll with levels = 3.
 * Padding 3, bias included; img a multiple of 32. fp32 accumulation in both dtypes.
 * -------------------------------------------------------------------------------- */
#define HIERA_PATCH_PACKED_BYTES ((196 * 112 + 112) * 4 + 112 * 208 * 2)
HIERA_API hiera_status hiera_patch_pack(const void* patch_w, const void* patch_b, void* packed,
                              hiera_dtype dtype, hiera_stream_t stream);
HIERA_API hiera_status hiera_patch_embed(const void* img, const void* packed_patch, const void* pos_embed,
                               void* out, int B, int img_side, hiera_dtype dtype,
                               hiera_stream_t stream);

/* --------------------------------------------------------------------------------
 * Hiera-B+ backbone (Sub-phase 4a item 8: patch_embed + pos_embed + unroll + 24 blocks
 * + reroll at stage ends [1, 4, 20, 23]). Stage table built in: dims 112/224/448/896,
 * heads 2/4/8/16, depths 2/3/16/3, mask-unit windows of 64 tokens (stage 0) and 16
 * (stage 1), global attention in stages 2-3, transitions at blocks 2, 5, 21.
 * mask_unit_attn_stage2_first: 0 = block 5 global (as the plan's table lists stage 2);
 * 1 = block 5 keeps mask-unit attention (16 keys, 4 pooled queries per unit).
 * Features: feats[s] is NHWC [B, img/2^(s+2), img/2^(s+2), 112*2^s].
 * hiera_backbone_workspace_bytes is enough for the call as one batch and as two
 * concurrent halves (HIERA_OPT_SPLIT_BATCH below), whichever the option selects. With
 * the split, hiera_backbone_forward enqueues images [0, ceil(B/2)) on `stream` and the
 * rest on a second stream owned by the calling thread (one per device), forked from and
 * joined back into `stream` with events: the call stays ordered with the caller's work on
 * `stream` and may be captured into a CUDA graph from it (the second stream joins the
 * capture). The second stream is created by the thread's first hiera_backbone_pack (or,
 * failing that, its first split call outside a capture; a call made inside a capture
 * before the thread has one runs as one batch). A call is not to be made while a capture
 * begun by the same thread on another stream is still open.
 * -------------------------------------------------------------------------------- */
typedef struct {
  int B;
  int img;
  int mask_unit_attn_stage2_first;
  hiera_dtype dtype;
} hiera_backbone_desc;

typedef struct {
  const void* patch_w;
  const void* patch_b;
  const void* pos_embed;
  hiera_block_weights blocks[24];
} hiera_backbone_weights;

HIERA_API size_t hiera_backbone_packed_bytes(const hiera_backbone_desc* desc);
HIERA_API hiera_status hiera_backbone_pack(const hiera_backbone_desc* desc, const hiera_backbone_weights* w,
                                 void* packed, size_t packed_bytes, hiera_stream_t stream);
HIERA_API size_t hiera_backbone_workspace_bytes(const hiera_backbone_desc* desc);
HIERA_API hiera_status hiera_backbone_forward(const hiera_backbone_desc* desc, const void* packed,
                                    const void* img_nhwc, void* const feats[4], void* workspace,
                                    size_t workspace_bytes, hiera_stream_t stream);

/* --------------------------------------------------------------------------------
 * Library options (process-wide, host-side; read when a forward call enqueues its
 * launches, so change them between calls, not while another thread is enqueuing).
 *   HIERA_OPT_FUSED_MLP  1 (default): for bf16 blocks with dim_out 112 or 224 (stages 0
 *                        and 1), norm2 + fc1 + GELU + fc2 + residual run as one kernel
 *                        that keeps the 4*dim hidden activation on chip (the block's
 *                        HieraMLP, "Phase 4: Hiera Backbone MLX Port", Architecture
 *                        Summary). 0: the two stand-alone GEMMs with the hidden
 *                        activation in the workspace. Both give the same values (same
 *                        tensor-core K order, same epilogue arithmetic).
 *   HIERA_OPT_PDL        1 (default): the bf16 path's kernels are launched with programmatic
 *                        dependent launch, so each one's launch and set-up (barrier init,
 *                        TMEM allocation, descriptor prefetch) overlap the tail of the
 *                        kernel before it; every kernel waits (griddepcontrol.wait) for
 *                        its predecessor's completion before it reads or writes any data
 *                        a previous kernel touches. 0: ordinary stream-ordered launches.
 *   HIERA_OPT_FUSED_ATTN 1 (default): for bf16 stage-0 blocks (dim 112, 2 heads, mask-unit
 *                        windows of 64 tokens, no pooling, an even number of windows), norm1
 *                        + qkv + windowed attention + proj + residual run as one kernel with
 *                        q, k, v and the attention output kept on chip (the attention half
 *                        of the plan's HieraBlock, Sub-phase 4a item 7); workspace slots
 *                        [0]-[3] of hiera_block_workspace_layout are then left unwritten.
 *                        0: the separate qkv GEMM, attention and proj GEMM. The two agree
 *                        to rounding (the fused P V product sums the window's keys in
 *                        another order).
 *   HIERA_OPT_GEMM224    the kernel for the bf16 Linear layers whose output columns come in
 *                        tiles of 224 (dims 224, 448, 896; not the transition's pooled qkv).
 *                        0 (default): one CTA per 128 x 224 tile with eight epilogue warps.
 *                        1: one CTA per 128 x 224 tile with sixteen epilogue warps (one
 *                        56-column chunk each). 2: a CTA pair per 256 x 224 tile
 *                        (tcgen05.mma.cta_group::2, each SM loading its 128 input rows and
 *                        half of the weight tile) with the sixteen-warp epilogue. All three
 *                        give the same bits.
 *   HIERA_OPT_SPLIT_BATCH 1 (default): hiera_backbone_forward with B >= 2 runs its images as
 *                        two concurrent half batches on two streams (each kernel sizes its
 *                        grid to the SM count; the halves' kernels fill the SMs one chain
 *                        leaves idle in kernel tails and partial waves). 0: one batch on
 *                        `stream`. Every image's features are the same bits either way.
 * hiera_set_option returns HIERA_ERR_INVALID_ARG for an unknown option or value (0 or
 * 1; 0 to 2 for HIERA_OPT_GEMM224);
 * hiera_get_option returns the current value (0 for an unknown option).
 * -------------------------------------------------------------------------------- */
typedef enum {
  HIERA_OPT_FUSED_MLP = 0,
  HIERA_OPT_PDL = 1,
  HIERA_OPT_FUSED_ATTN = 2,
  HIERA_OPT_GEMM224 = 3,
  HIERA_OPT_SPLIT_BATCH = 4,
  HIERA_OPT_COUNT = 5
} hiera_option;
HIERA_API hiera_status hiera_set_option(hiera_option opt, int value);
HIERA_API int hiera_get_option(hiera_option opt);

/* --------------------------------------------------------------------------------
 * Launch profiling (host-side bookkeeping only). Between hiera_profile_begin() and
 * hiera_profile_end(), every kernel launch the library makes, on whatever stream the
 * call was given, is preceded by cudaEventRecord(events[i], stream) and its kernel id is
 * stored in kinds[i] (i counts launches from 0; launches beyond `capacity` are not
 * marked). `events` are cudaEvent_t handles created by the caller with timing enabled.
 * hiera_profile_end() records events[n] on `stream` (n = launches seen, if n <
 * capacity) and returns n, so launch i took elapsed(events[i], events[i+1]) when all
 * launches went to one stream; while a session is open hiera_backbone_forward therefore
 * does not split its batch (HIERA_OPT_SPLIT_BATCH). Works under CUDA-graph stream capture
 * (the records become event nodes). Not thread-safe: one session at a time per process.
 * hiera_kernel_name() names a kernel id (static string).
 * -------------------------------------------------------------------------------- */
HIERA_API hiera_status hiera_profile_begin(void* const* events, int capacity, int* kinds);
HIERA_API int hiera_profile_end(hiera_stream_t stream);
HIERA_API const char* hiera_kernel_name(int kind);

/* --------------------------------------------------------------------------------
 * Self-test of the bounded-wait machinery: launches one kernel that waits on an
 * mbarrier nothing will complete, for at most limit_us microseconds; the wait records
 * HIERA_ERR_TIMEOUT in the device status word and the kernel returns normally.
 * -------------------------------------------------------------------------------- */
HIERA_API hiera_status hiera_debug_timeout_probe(int limit_us, hiera_stream_t stream);

/* Self-test of the tensor-core path's GELU: y[i] = GELU(x[i]) for n fp32 device values,
 * computed exactly as the fc1 epilogue does (x * sigmoid of a fitted odd polynomial for
 * logit(Phi(x)), the sigmoid evaluated through tanh.approx; |error| <= 4e-5 against
 * x Phi(x)). */
HIERA_API hiera_status hiera_debug_gelu(const float* x, float* y, int n, hiera_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* HIERA_H_ */
