/*
 * moe_b200.h -- C ABI of the single-GPU MoE layer forward for NVIDIA B200
 * (sm_100a).
 *
 * The layer, as the pages define it (MoE Align & Sort article on
 * dignews.cc, opening definition of the MoE layer and its "FasterTransformer",
 * "Megatron", "CK" and D-C-P sections; aiter issue 1248 "[Feature]: Add more
 * configuration options for MoE assembly kernels", "Suggestion Description"):
 *
 *   gate     : softmax top-k over E expert logits per token, weights
 *              renormalised over the k chosen experts          (moe_topk_gate)
 *   align    : counting sort of the T*k (token, choice) slots by expert,
 *              each expert's segment padded to a multiple of block_size
 *                                                             (moe_align_sort)
 *   FFN      : per block of sorted slots, the owning expert's gated FFN
 *              h = silu(x Wg^T) * (x Wu^T), y = h Wd^T, in bf16 or with
 *              per-token FP8 E4M3 activations and per-channel FP8 weights
 *                                                            (moe_grouped_ffn)
 *   combine  : out[t] = sum_j w[t,j] * y[t*k+j]                  (moe_combine)
 *   all four : moe_forward
 *
 * Also: the layer's gradients (moe_backward), the per-rank steps of an
 * expert-parallel layer (moe_ep_route, moe_permute_rows, moe_scatter_rows;
 * the exchange between ranks is the caller's), MX block-scaled weights
 * (moe_mx_tile_scales lays out their scales; moe_mx_quantize_rows is the
 * activation quantiser), and align & sort without a caller workspace
 * (moe_align_sort_noalloc).
 *
 * Conventions (every entry point):
 *   - All tensor pointers are DEVICE pointers unless stated otherwise.  The
 *     caller owns every buffer and the stream; the library allocates no
 *     device memory and keeps no per-call state between calls.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Calls are asynchronous and stream-ordered; none synchronises
 *     the host.
 *   - Arguments are validated synchronously; a bad argument returns an error
 *     and launches nothing.  Errors found on the device (an expert id out of
 *     range, a bounded wait that ran out) are OR-ed into *dev_status (bit
 *     flags MOE_DEV_*) when dev_status is non-NULL; the caller reads it after
 *     synchronising.  With dev_status NULL they are dropped and the outputs
 *     are unspecified.
 *   - Layouts are row-major and contiguous.  Flat slot i = t*k + j names
 *     token t's j-th choice.
 *   - Requires an sm_100a device.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* null pointer, negative size, k > E, ...     */
  MOE_ERR_UNSUPPORTED = 2,   /* valid but not handled (e.g. H % 128 != 0)   */
  MOE_ERR_WORKSPACE = 3,     /* workspace smaller than the size query says  */
  MOE_ERR_CUDA = 4,          /* a CUDA runtime call failed (see moe_last_cuda_error) */
  MOE_ERR_DEVICE = 5         /* no sm_100 device: none current, no GPU or
                                driver at all, or another architecture      */
} moe_status_t;

/* MOE_MXFP8 / MOE_MXFP4: MX block-scaled weights (OCP Microscaling: one E8M0
 * scale per 32 consecutive elements along K; E4M3 or E2M1 elements); the
 * activations are then MXFP8 too (see moe_grouped_ffn). */
typedef enum { MOE_BF16 = 0, MOE_FP8_E4M3 = 1, MOE_F32 = 2, MOE_MXFP8 = 3, MOE_MXFP4 = 4 } moe_dtype_t;

/* Device-side status bits (OR-ed into *dev_status). */
#define MOE_DEV_BAD_EXPERT_ID 0x1  /* an expert id outside [0, E): slot skipped */
#define MOE_DEV_TIMEOUT       0x2  /* a bounded wait ran out; outputs unspecified */
#define MOE_DEV_BAD_PLAN      0x4  /* routing metadata inconsistent with sizes,
                                      or an expert's blocks not one run in
                                      expert_ids: no GEMM tile runs          */
#define MOE_DEV_BOUNDS        0x10 /* libraries built with MOE_DEBUG only
                                      (libmoe_b200_debug.so): an index a kernel
                                      computed or read fell outside its buffer
                                      (a negative sorted id, a GEMM tile past
                                      num_post); the access was skipped, and a
                                      GEMM CTA stopped at its tile */
#define MOE_DEV_DRAIN_TIMEOUT 0x8  /* after a timeout, a GEMM CTA also gave up
                                      waiting for its own copies or MMAs in
                                      flight before freeing its tensor memory:
                                      the device state is undefined; do not call
                                      the library again in this CUDA context    */

/* Human-readable name of a status code.  Host only; never fails. */
MOE_API const char* moe_status_string(int status);
/* Text of the last CUDA error seen by this thread inside the library. */
MOE_API const char* moe_last_cuda_error(void);
/* ABI version (major*100 + minor); equals MOE_ABI_VERSION of the header the
 * library was built with.  Major 2: moe_topk_gate takes bias_mode and
 * n_shared, moe_forward_args ends with n_shared and bias_mode.  Major 3:
 * moe_ffn_args and moe_forward_args end with the MX weight scales; MX weight
 * types; moe_mx_tile_scales, moe_mx_quantize_rows; moe_backward; the
 * expert-parallel steps moe_ep_route, moe_permute_rows, moe_scatter_rows. */
#define MOE_ABI_VERSION 300
MOE_API int moe_version(void);

/* ---------------------------------------------------------------------------
 * moe_topk_gate -- softmax top-k gating.
 * Passage: MoE Align & Sort article, "FasterTransformer" (moe_softmax +
 * moe_top_k fused as topk_gating_softmax; "biased" variant) and the opening
 * definition (Top-K gating scores; DeepSeek V3's gating bias for
 * auxiliary-loss-free balancing and its shared expert).
 *
 *   logits    f32 [T, E]  router logits (the router GEMM is the caller's)
 *   bias      f32 [E]     nullable; added to the logits in fp32
 *   bias_mode             MOE_BIAS_LOGITS: the biased logits are both the
 *                         selection score and the softmax input;
 *                         MOE_BIAS_SELECT: they only select, the weights use
 *                         the raw logits (DeepSeek-V3 style)
 *   n_shared              shared experts appended to every token's row
 *   topk_ids  i32 [T, k+n_shared]  out: chosen experts by descending score
 *                         (equal scores go to the lower expert index), then
 *                         the shared experts E, E+1, ..., E+n_shared-1
 *   topk_w    f32 [T, k+n_shared]  out: softmax(l)[chosen] /
 *                         sum(softmax(l)[chosen]), then 1 per shared expert
 * Limits: 0 <= T, 1 <= E, E + n_shared <= 1024, 1 <= k <= E,
 * k + n_shared <= 32, n_shared >= 0.  Logits must be finite.  Errors:
 * MOE_ERR_INVALID_ARG on a bad size, mode or NULL output.
 * ------------------------------------------------------------------------- */
#define MOE_BIAS_LOGITS 0
#define MOE_BIAS_SELECT 1
MOE_API moe_status_t moe_topk_gate(const float* logits, const float* bias, int bias_mode, int T, int E, int k,
                                   int n_shared, int32_t* topk_ids, float* topk_w, void* stream);

/* ---------------------------------------------------------------------------
 * moe_align_sort -- block-aligned MoE Align & Sort.
 * Passage: MoE Align & Sort article, the D-C-P section (distributed
 * concurrent counting; unaligned local cumsum, merge, aligned global cumsum;
 * parallel placement) and the paragraph on aligned sorting for Group GEMM.
 *
 *   topk_ids   i32 [T*k]  expert of every flat slot
 *   sorted_ids i32 [P]    out: slots grouped by expert (ascending expert,
 *                         ascending slot inside an expert), every expert's
 *                         segment padded with the sentinel T*k to a multiple
 *                         of block_size; experts with no slot get no block.
 *                         Entries [num_post, P) are not written.
 *   expert_ids i32 [NB]   out: expert owning each block of block_size
 *                         entries; entries [num_post/block_size, NB) are not
 *                         written.
 *   num_post   i32 [1]    out: padded length = sum_e ceil(c_e/bs)*bs
 *   ws, ws_bytes          device workspace of at least the size
 *                         moe_align_sort_sizes returns; contents on entry are
 *                         irrelevant.
 * P = T*k + E*(block_size-1), NB = ceil(P / block_size) (host values from
 * moe_align_sort_sizes).  Limits: 1 <= E <= 1024, 1 <= block_size <= 1024,
 * T*k < 2^31 - 1.  Out-of-range ids are skipped and flagged with
 * MOE_DEV_BAD_EXPERT_ID.  The kernel runs as one cooperative grid with a
 * bounded grid-wide wait (MOE_DEV_TIMEOUT if it runs out).
 * ------------------------------------------------------------------------- */
MOE_API moe_status_t moe_align_sort_sizes(int T, int k, int E, int block_size,
                                  size_t* P, size_t* NB, size_t* ws_bytes);
MOE_API moe_status_t moe_align_sort(const int32_t* topk_ids, int T, int k, int E, int block_size,
                            int32_t* sorted_ids, int32_t* expert_ids, int32_t* num_post,
                            void* ws, size_t ws_bytes, int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * moe_align_sort_noalloc -- moe_align_sort without a caller workspace.
 * The pages have no counterpart: this entry point exists for callers that
 * cannot allocate device memory (code running while another framework's
 * memory pool is frozen, plain C hosts that only receive pointers, runtimes
 * that forbid cudaMalloc after start-up).  Inputs, outputs, results and
 * device-status bits are exactly those of moe_align_sort; only the scratch
 * differs: a fixed device array inside the library (MOE_NOALLOC_SCRATCH_BYTES,
 * held by every GPU that loads the library until the process exits).
 * Limit: E <= MOE_NOALLOC_MAX_EXPERTS, otherwise MOE_ERR_UNSUPPORTED and
 * nothing is launched.  The first call on a device looks up the array's
 * device address and keeps it per device ordinal (make that call before any
 * stream capture).  The kept address belongs to the device's primary context,
 * the one the CUDA runtime uses by default: do not call this entry point from
 * another context of the device, nor after cudaDeviceReset on it (the address
 * would then name memory that is gone).  All calls share the array: calls
 * that overlap on the GPU race; order them on one stream.  Allocates nothing.
 * CUDA failures return MOE_ERR_CUDA with the text in moe_last_cuda_error.
 * ------------------------------------------------------------------------- */
#define MOE_NOALLOC_MAX_EXPERTS 256
#define MOE_NOALLOC_SCRATCH_BYTES (256 + 256 * 256 * 4)
MOE_API moe_status_t moe_align_sort_noalloc(const int32_t* topk_ids, int T, int k, int E, int block_size,
                                            int32_t* sorted_ids, int32_t* expert_ids, int32_t* num_post,
                                            int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * moe_grouped_ffn -- gated grouped expert FFN over the sorted slots.
 * Passage: MoE Align & Sort article, opening definition (expert FFNs on the
 * chosen tokens computed by a Group GEMM) and "AITER" (the grouped GEMM
 * multiplies each expert's FFN weights with a block of token hidden states);
 * aiter issue 1248, "Suggestion Description" (g1u1 SiLU, per-token FP8
 * activations with bf16 in/out); GC-MoE abstract (fused SwiGLU and
 * requantisation between the two GEMMs).
 *
 * For every sorted row r < num_post with slot s = sorted_ids[r] in [0, T*k)
 * and expert e = expert_ids[r / block_size], token t = s / k (other ids are
 * padding: T*k as moe_align_sort writes it; a negative id is an error that
 * the debug build reports as MOE_DEV_BOUNDS, and both builds skip the row):
 *   BF16:  g = Wg[e] x_t, u = Wu[e] x_t (fp32 accumulation),
 *          h = bf16(silu(g) * u), y_s = Wd[e] h
 *   FP8:   (q_x, s_x) = e4m3 per-token quantisation of x_t (s = amax/448),
 *          g = (Wg_q[e] q_x) * s_x * w13_scale[e], u likewise,
 *          h = bf16(silu(g) * u), (q_h, s_h) = per-row requantisation,
 *          y_s = (Wd_q[e] q_h) * s_h * w2_scale[e]
 *   MX (MOE_MXFP8 / MOE_MXFP4 weights; GC-MoE abstract: block-scaled MMAs
 *   with FP4 weights on Blackwell):
 *          x_t is MXFP8-quantised (per 32 elements along H: X = 2^(floor(log2
 *          amax) - 8), E4M3 codes of x / X), g and u are the block sums
 *          sum_b X_x[b] X_w[n,b] (q_x[b] . q_w[n,b]) accumulated in fp32,
 *          h = bf16(silu(g) * u) is MXFP8-quantised along I in the gate/up
 *          GEMM's epilogue (no separate requantisation), y_s likewise.
 * ------------------------------------------------------------------------- */
typedef struct {
  int T, H, I, E, k, block_size;
  int wdtype;                 /* MOE_BF16 or MOE_FP8_E4M3                       */
  const void* x;              /* bf16 [T, H]                                     */
  const void* w13;            /* [E, 2I, H]: rows 0..I-1 gate, I..2I-1 up;
                                 bf16, or E4M3 codes when wdtype is FP8          */
  const float* w13_scale;     /* f32 [E, 2I] per output channel (FP8 only)       */
  const void* w2;             /* [E, H, I] bf16 or E4M3 codes                    */
  const float* w2_scale;      /* f32 [E, H] (FP8 only)                           */
  const int32_t* sorted_ids;  /* [P]  from moe_align_sort                        */
  const int32_t* expert_ids;  /* [NB] from moe_align_sort                        */
  const int32_t* num_post;    /* [1]  from moe_align_sort                        */
  int tile_tokens;            /* tokens per GEMM tile: 0 = automatic, else one
                                 of 16, 32, 64, 128, 256 (MX: at most 128)        */
  /* MX weights only (else NULL): E8M0 scale codes in the tiled layout of
   * moe_mx_tile_scales, from [E * 2I, H/32] and [E * H, I/32].  With MX
   * weights w13 / w2 hold E4M3 codes [E, 2I, H] / [E, H, I] (MOE_MXFP8) or E2M1
   * codes packed two per byte, element 2j in the low nibble, [E, 2I, H/2] /
   * [E, H, I/2] (MOE_MXFP4; 32-byte aligned). */
  const uint8_t* w13_mx_scale;
  const uint8_t* w2_mx_scale;
} moe_ffn_args;

/* Limits: H % 128 == 0, I % 128 == 0, 1 <= E <= 1024, 1 <= k <= 32,
 * 1 <= block_size <= 1024; device pointers 16-byte aligned (MXFP4 weights:
 * 32-byte).  Missing scales for the weight type: MOE_ERR_INVALID_ARG. */
MOE_API moe_status_t moe_ffn_workspace(const moe_ffn_args* args, size_t* ws_bytes);
/*   y  f32 [T*k, H]  out: per-slot expert output y_s (rows of slots that were
 *                    skipped are not written) */
MOE_API moe_status_t moe_grouped_ffn(const moe_ffn_args* args, float* y, void* ws, size_t ws_bytes,
                             int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * moe_combine -- top-k weighted combine (unpermute).
 * Passage: MoE Align & Sort article, "Megatron" (unpermute) and
 * "FasterTransformer" (permute before the group GEMM).
 *   y       f32 [T*k, H];  topk_w f32 [T, k]
 *   out     [T, H] in out_dtype (MOE_BF16 or MOE_F32):
 *           out[t] = sum_j topk_w[t,j] * y[t*k+j], summed in fp32 in
 *           ascending j, rounded once.
 * ------------------------------------------------------------------------- */
MOE_API moe_status_t moe_combine(const float* y, const float* topk_w, int T, int k, int H,
                         void* out, int out_dtype, void* stream);

/* ---------------------------------------------------------------------------
 * moe_forward -- gate, align & sort, grouped FFN and combine in one call:
 * the same arithmetic as moe_topk_gate, moe_align_sort, moe_grouped_ffn and
 * moe_combine in sequence.  With k + n_shared >= 4 slots per token the
 * combine is fused into the down GEMM: each slot's w * y is added into an
 * fp32 row per token (in L2, in no fixed order, so the last bits of the
 * output may differ between calls), then rounded once to out_dtype.  With
 * fewer slots the per-slot outputs are summed by the combine kernel in
 * ascending j (deterministic).
 * Shared experts (n_shared > 0; MoE Align & Sort article, opening: DeepSeek's
 * shared expert) are stored after the E routed experts in w13/w2 and their
 * scales ([E + n_shared, ...]); every token goes to each of them with weight
 * 1, so they are scheduled in the same grouped GEMM launches as the routed
 * experts (align & sort sees k + n_shared slots per token over
 * E + n_shared experts).
 * ------------------------------------------------------------------------- */
typedef struct {
  int T, H, I, E, k, block_size;
  int wdtype;                 /* MOE_BF16 or MOE_FP8_E4M3                 */
  int out_dtype;              /* MOE_BF16 or MOE_F32                      */
  const void* x;              /* bf16 [T, H]                              */
  const float* logits;        /* f32 [T, E]                               */
  const float* bias;          /* f32 [E], nullable (see bias_mode)        */
  const void* w13;            /* as in moe_ffn_args, E + n_shared experts */
  const float* w13_scale;
  const void* w2;
  const float* w2_scale;
  void* out;                  /* [T, H] out_dtype                         */
  int32_t* topk_ids;          /* nullable: routing also written here
                                 [T, k + n_shared] (as moe_topk_gate)      */
  float* topk_w;              /* nullable [T, k + n_shared]               */
  int tile_tokens;            /* as in moe_ffn_args                       */
  void** stage_events;        /* nullable: MOE_NUM_STAGES + 1 cudaEvent_t
                                 handles; event 0 is recorded before the first
                                 stage and event i+1 after stage i, on
                                 `stream` (for per-stage timing)           */
  int n_shared;               /* shared experts after the E routed ones (0..) */
  int bias_mode;              /* MOE_BIAS_LOGITS or MOE_BIAS_SELECT        */
  const uint8_t* w13_mx_scale;  /* MX weights only: as in moe_ffn_args      */
  const uint8_t* w2_mx_scale;
} moe_forward_args;

/* Stages of moe_forward, in launch order (stage_events indices). */
#define MOE_STAGE_GATE 0      /* top-k gating                              */
#define MOE_STAGE_ALIGN 1     /* align & sort                              */
#define MOE_STAGE_PLAN 2      /* tile list for the grouped GEMMs           */
#define MOE_STAGE_GATHER 3    /* token rows to sorted order (+FP8 quant)   */
#define MOE_STAGE_GATEUP 4    /* gate/up GEMM with SiLU*mul                */
#define MOE_STAGE_REQUANT 5   /* FP8 requantisation of h (empty for bf16)  */
#define MOE_STAGE_DOWN 6      /* down GEMM (with the combine when fused)    */
#define MOE_STAGE_COMBINE 7   /* combine kernel, or the fp32 -> bf16 rounding
                                 of the fused accumulator (empty for f32)    */
#define MOE_NUM_STAGES 8

MOE_API moe_status_t moe_forward_workspace(const moe_forward_args* args, size_t* ws_bytes);
MOE_API moe_status_t moe_forward(const moe_forward_args* args, void* ws, size_t ws_bytes,
                         int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------------------
 * moe_backward -- gradients of the layer forward (bf16 weights).
 * Passage: MoE Align & Sort article, "Megatron" (the combine's gradient is the
 * unpermute of the output gradient) and the opening definition of the layer;
 * the pages print no backward formulas, these are the chain rule through
 * moe_forward's arithmetic.  With L = sum(out * dout):
 *   dx       f32 [T, H]          dL/dx
 *   dlogits  f32 [T, E]          dL/dlogits: the renormalised top-k softmax's
 *                                gradient at the chosen experts, 0 elsewhere
 *                                (the choice itself is piecewise constant)
 *   dw13     f32 [E+S, 2I, H]    dL/dW13 (gate rows, then up rows); zero for
 *                                experts that no token reached
 *   dw2      f32 [E+S, H, I]     dL/dW2
 * Conventions as the forward's reference: the bf16 rounding of h passes the
 * gradient through unchanged (dh is the gradient of silu(g) * u, dW2 uses
 * the rounded h); shared experts' weight 1 is a constant.  Routing is
 * recomputed from the logits (the same arithmetic as moe_topk_gate and
 * moe_align_sort), and so is the gate/up projection (activations are not
 * kept by the forward).  Intermediate operands of the gradient GEMMs are bf16
 * (dout, [dg; du], w * h), accumulation fp32.  All outputs are overwritten.
 * Limits: as moe_forward with bf16 weights, and block_size % 16 == 0
 * (MOE_ERR_UNSUPPORTED otherwise).
 * ------------------------------------------------------------------------- */
typedef struct {
  int T, H, I, E, k, block_size;
  int n_shared;               /* shared experts after the E routed ones       */
  int bias_mode;              /* MOE_BIAS_LOGITS or MOE_BIAS_SELECT           */
  const void* x;              /* bf16 [T, H]                                  */
  const float* logits;        /* f32 [T, E]                                   */
  const float* bias;          /* f32 [E], nullable                            */
  const void* w13;            /* bf16 [E + n_shared, 2I, H]                   */
  const void* w2;             /* bf16 [E + n_shared, H, I]                    */
  const void* dout;           /* bf16 [T, H] gradient of the layer output      */
  float* dx;                  /* out [T, H]                                   */
  float* dlogits;             /* out [T, E]                                   */
  float* dw13;                /* out [E + n_shared, 2I, H]                    */
  float* dw2;                 /* out [E + n_shared, H, I]                     */
} moe_backward_args;
MOE_API moe_status_t moe_backward_workspace(const moe_backward_args* args, size_t* ws_bytes);
MOE_API moe_status_t moe_backward(const moe_backward_args* args, void* ws, size_t ws_bytes, int32_t* dev_status,
                                  void* stream);

/* ---------------------------------------------------------------------------
 * Expert parallelism (EP): the layer's experts sharded over R ranks (rank r
 * holds experts [r*E/R, (r+1)*E/R)), every rank gating its own tokens.
 * Passage: X-MoE abstract and GC-MoE abstract (expert-parallel dispatch and
 * combine across GPUs).  These calls are the per-rank steps; the exchange
 * between ranks (all-to-all of counts, token rows and expert outputs) is the
 * caller's collective (NCCL through torch.distributed in the Python binding).
 *
 * moe_ep_route: destination ranks of the T*k slots.
 *   topk_ids    i32 [T*k]  global expert of every slot
 *   order       i32 [T*k]  out: the flat slots grouped by destination rank
 *                          (ascending rank, ascending slot inside a rank)
 *   send_counts i32 [R]    out: slots per destination rank
 *   local_ids   i32 [T*k]  out: order's slots' expert ids local to their rank
 *                          (expert % (E/R))
 *   ws          device workspace of moe_ep_route_workspace's size
 * Limits: 1 <= R <= 1024, E % R == 0.  Out-of-range ids are skipped and
 * flagged with MOE_DEV_BAD_EXPERT_ID (order then holds fewer real entries).
 * ------------------------------------------------------------------------- */
MOE_API moe_status_t moe_ep_route_workspace(int T, int k, int R, size_t* ws_bytes);
MOE_API moe_status_t moe_ep_route(const int32_t* topk_ids, int T, int k, int E, int R, int32_t* order,
                                  int32_t* send_counts, int32_t* local_ids, void* ws, size_t ws_bytes,
                                  int32_t* dev_status, void* stream);
/* moe_permute_rows: dst row i = src row map[i] / div for i < n (the permute
 * before the exchange: div = k turns slots into tokens).  moe_scatter_rows:
 * dst row map[i] = src row i (the un-permute after it).  Rows of row_bytes
 * bytes (a multiple of 16), 16-byte-aligned buffers; map entries whose row
 * falls outside [0, src_rows) / [0, dst_rows) move nothing.
 * Passage: MoE Align & Sort article, "FasterTransformer" (permute) and
 * "Megatron" (unpermute). */
MOE_API moe_status_t moe_permute_rows(const void* src, int row_bytes, const int32_t* map, int n, int div,
                                      int src_rows, void* dst, void* stream);
MOE_API moe_status_t moe_scatter_rows(const void* src, int row_bytes, const int32_t* map, int n, int dst_rows,
                                      void* dst, void* stream);

/* ---------------------------------------------------------------------------
 * moe_mx_tile_scales -- lay out MX weight scales for the block-scaled GEMM.
 * Model preparation, done once per weight tensor (GC-MoE abstract: block-
 * scaled MMAs; the scale layout is the one the tensor cores' scale-factor
 * copies read, 128 rows x 4 K-blocks per 512-byte chunk).
 *   sf   u8 [rows, K/32]  E8M0 scale codes, one per 32 elements of a row
 *   out  u8 [rows * K/32] chunk (rt, w) = rows 128*rt.. x K-blocks 4w..4w+3
 *        holds at byte (r % 32) * 16 + ((r % 128) / 32) * 4 + b the scale of
 *        row 128*rt + r, K-block 4w + b; chunks ordered rt-major.
 * Limits: rows % 128 == 0, K % 128 == 0, 16-byte aligned pointers.
 * ------------------------------------------------------------------------- */
MOE_API moe_status_t moe_mx_tile_scales(const uint8_t* sf, long long rows, int K, uint8_t* out, void* stream);

/* ---------------------------------------------------------------------------
 * moe_mx_quantize_rows -- MXFP8 quantisation of bf16 rows (the activation
 * quantiser of the MX path, also usable on its own).
 *   x       bf16 [R, C];  codes u8 [R, C] out: E4M3 codes of x / X
 *   scales  u8 [R, C/32] out: E8M0 code 127 + floor(log2 amax) - 8 of every
 *           32-element block (clamped to >= 0; 127 for an all-zero block)
 * Rounding: nearest even, saturating to +-448.  Limits: C % 32 == 0, R >= 0,
 * 16-byte aligned x and codes.
 * ------------------------------------------------------------------------- */
MOE_API moe_status_t moe_mx_quantize_rows(const void* x, int R, int C, uint8_t* codes, uint8_t* scales,
                                          void* stream);

/* ---------------------------------------------------------------------------
 * Diagnostics.
 * moe_test_wait_timeout runs the grid-wide wait of moe_align_sort on a
 * barrier that can never fill (it expects one more arrival than the grid
 * has) with the given limit in nanoseconds, so that the timeout path can be
 * exercised without a fault: it must OR MOE_DEV_TIMEOUT into *dev_status and
 * return.  ws: at least 256 bytes of device memory.
 * ------------------------------------------------------------------------- */
MOE_API moe_status_t moe_test_wait_timeout(void* ws, int32_t* dev_status, long long timeout_ns,
                                   void* stream);

/* moe_test_quant_division checks the E4M3 quantiser's quotient path (one
 * reciprocal per row plus a fused-multiply-add correction per element) against
 * an IEEE fp32 division for every pair of bf16 values (v, amax) with
 * 0 < amax <= the largest finite bf16 and |v| <= amax: it compares the E4M3
 * codes of v / s, s = amax / 448.  ws: at least 32 bytes of device memory,
 * cleared by the call; on completion of the stream it holds uint64 pairs
 * checked, uint64 mismatches and uint32 (v bits << 16 | amax bits) of one
 * mismatch (0 if none).  Test hook; the method's pages have no counterpart. */
MOE_API moe_status_t moe_test_quant_division(void* ws, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
