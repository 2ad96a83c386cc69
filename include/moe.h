/*
 * moe.h -- C ABI of the B200 (sm_100a) token-choice Mixture-of-Experts layer.
 *
 * One forward pass of the layer is
 *
 *     s_t = h_t W_r^T (+ b)                 router scores
 *     E_t = TopK(s_t, k)                     expert choice
 *     g_t = softmax(s_t) renormalised over E_t
 *     y_t = sum_{e in E_t} g_{t,e} f_e(h_t)  combine
 *
 * ("How Does Mixture-of-Experts Routing Affect LLM Repeatability?", the
 * simplified token-choice layer), carried out as the stages of "MoE Token
 * Dispatch: Why an All-Reduce Result Does Not Describe the Exchange", section
 * "Follow one documented dispatch and return path": per-expert counts from the
 * routing map, a permutation that groups token rows by expert, the experts,
 * and the return of every output to its original token position. On one GPU
 * the dispatch and the return are on-device permutations. moe_layer_backward
 * differentiates the same layer (bf16, SwiGLU experts).
 *
 * Conventions for every entry point:
 *  - Tensor arguments are DEVICE pointers owned by the caller. The library
 *    never allocates, frees or keeps device memory; scratch comes from the
 *    caller's `workspace` (size from moe_workspace_size). Pointers must be
 *    16-byte aligned.
 *  - Row-major throughout. Weights are "out x in" (the reduction index is the
 *    contiguous one), i.e. W_r [E, d], W_gate/W_up [E, F, d], W_down [E, d, F].
 *  - `dtype` (MOE_DTYPE_*) is the storage type of h, the expert weights, the
 *    permuted rows and y. The router weight has the same type; the router bias
 *    is always fp32. Logits and gates are fp32, indices int32. Arithmetic
 *    accumulates in fp32 on both paths.
 *  - Every call only enqueues work on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream) and never synchronises. Counts and offsets stay on
 *    the device.
 *  - Return value: MOE_OK or a host-side error (MOE_ERR_*), detected before
 *    anything is enqueued, except MOE_ERR_CUDA, which reports a failed launch.
 *  - Data errors found on the device never trap: they are OR-ed into
 *    *status_dev (MOE_STATUS_* bits) when status_dev is not NULL. The caller
 *    zeroes it and reads it when convenient.
 *
 * Limits: 1 <= E <= 256, 1 <= k <= min(E, 8), T >= 0, T*k < 2^31, E*capacity < 2^31 (PADDED).
 * bf16 path: d and F multiples of 128. fp32 path: d a multiple of 4.
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

/* host-side return codes */
#define MOE_OK              0
#define MOE_ERR_INVALID_ARG 1  /* NULL where a pointer is required, bad sizes */
#define MOE_ERR_UNSUPPORTED 2  /* outside the limits above, misaligned pointer */
#define MOE_ERR_WORKSPACE   3  /* workspace too small or misaligned */
#define MOE_ERR_CUDA        4  /* a kernel launch or CUDA runtime call failed */
#define MOE_ERR_NO_DEVICE   5  /* no usable sm_100 device / driver entry point */

/* asynchronous status bits, OR-ed into *status_dev */
#define MOE_STATUS_NAN_LOGIT 1  /* a router logit was NaN (treated as -inf) */
#define MOE_STATUS_BAD_ROUTE 2  /* an index out of [0,E) or repeated within a token (slot dropped) */
#define MOE_STATUS_TIMEOUT   4  /* a bounded on-chip wait gave up (output invalid) */
/* MXFP8 precision only, informational (the output is valid): */
#define MOE_STATUS_MX_SATURATED 8   /* an element was clamped to +-448 when quantised; the OCP scale
                                       rule does this whenever a block's largest magnitude has a
                                       mantissa above 1.75, so it is expected on most calls */
#define MOE_STATUS_MX_UNDERFLOW 16  /* a non-zero element was quantised to 0 */

#define MOE_DTYPE_BF16 0
#define MOE_DTYPE_F32  1

#define MOE_EXPERT_SWIGLU   0  /* f_e(x) = W_down,e (silu(W_gate,e x) * (W_up,e x)) */
#define MOE_EXPERT_IDENTITY 1  /* f_e(x) = x       (test expert) */
#define MOE_EXPERT_SCALE    2  /* f_e(x) = (e+1) x (test expert) */

/* Grouped-GEMM tiles (bf16 path). SINGLE: 128x256 tiles, one SM each. PAIR:
 * 256x256 tiles shared by two SMs of a cluster (tcgen05 cta_group::2), which
 * halves the operand bytes each SM stages. Both give the same bits. AUTO
 * picks PAIR where it measured faster on B200: bf16 SwiGLU experts of at
 * least 1024 rows on average (T*k/E, or the capacity if smaller; the
 * capacity in the padded layout) with at most 128 MiB of weights each
 * (3*d*d_ff bf16), and none of the options that need single tiles (MXFP8,
 * gather dispatch, fused combine, kept pre-activations). Larger experts (the
 * Mixtral 8x7B shape, 352 MB each) measured about 5% slower on pair tiles
 * under the 1 kW power cap, smaller ones pad more. moe_gemm_tiles_used
 * reports the choice. */
#define MOE_GEMM_TILES_AUTO   0
#define MOE_GEMM_TILES_SINGLE 1
#define MOE_GEMM_TILES_PAIR   2

/* Row layout of the permuted buffers (x_perm, y_perm, perm_src) when a
 * capacity is set. COMPACT: kept rows only, expert e at [offsets[e],
 * offsets[e+1]) with offsets the prefix sum of the kept counts; P = T*k rows.
 * PADDED: every expert owns exactly `capacity` rows, expert e at
 * [e*capacity, (e+1)*capacity), kept rows first and the rest zero padding
 * that the grouped FFN computes like any other row; P = E*capacity rows. This
 * is the fixed-capacity padded arm that the evaluation in "Dropless MoE Is a
 * Runtime Problem as Much as a Model Design" compares the dropless grouped
 * computation against; y is the same in both layouts. PADDED needs
 * capacity >= 0. */
#define MOE_LAYOUT_COMPACT 0
#define MOE_LAYOUT_PADDED  1

/* How moe_layer_forward moves token rows to the grouped FFN. COPY: the
 * dispatch writes x_perm (a bulk row copy) and GEMM1 reads it. GATHER: no
 * x_perm; GEMM1's loader fetches each A row straight from h through the
 * permutation (TMA tile::gather4, four rows per load), the fused dispatch of
 * "Dropless MoE Is a Runtime Problem as Much as a Model Design" (fusing
 * dispatch to cut intermediate writes). GATHER needs bf16, SwiGLU experts, the
 * COMPACT layout and single-CTA tiles (gemm_tiles SINGLE, or AUTO, which then
 * keeps them). The result is the same bit for bit.
 * AUTO is COPY: a tile reloads its A rows once per column tile, so the
 * gather repeats for every column tile, and GATHER measured 2.2-2.4x slower
 * per layer on B200. The stage entry points (moe_permute, moe_grouped_ffn)
 * always use x_perm. */
#define MOE_DISPATCH_AUTO   0
#define MOE_DISPATCH_COPY   1
#define MOE_DISPATCH_GATHER 2

/* Arithmetic of the grouped expert GEMMs (moe_grouped_ffn, moe_layer_forward).
 * BF16: bf16 operands (the default).
 * MXFP8: block-scaled 8-bit operands, the MXFP8 variant of "Dropless MoE Is a
 * Runtime Problem as Much as a Model Design" (its MXFP8 paragraph), with the
 * format of the OCP Microscaling specification: every 32 consecutive
 * elements along the reduction axis of a row share one scale 2^E (an E8M0
 * byte E + 127), E = floor(log2 max|v|) - 8 clamped to [-127, 127], and every
 * element is FP8 E4M3 of v / 2^E, rounded to nearest even and clamped at
 * +-448. The permuted token rows are quantised along d, the weights along
 * their reduction axis (moe_pack_weights_mxfp8), and silu(gate) * up along F
 * in GEMM1's epilogue before GEMM2; accumulation is fp32 and y_perm, y stay
 * bf16. Routing, dispatch and combine are unchanged. Needs bf16 storage,
 * SwiGLU experts, single-CTA tiles and the COPY dispatch; the backward is
 * bf16 only. In this precision the w13_packed and w_down arguments of
 * moe_grouped_ffn and moe_layer_forward are the two blobs written by
 * moe_pack_weights_mxfp8, and the first 16 bytes of their workspace receive
 * four uint32 counters of the call: token-row elements saturated and
 * underflowed (once per permuted row), then h_mid elements saturated and
 * underflowed. */
#define MOE_PRECISION_BF16  0
#define MOE_PRECISION_MXFP8 1

/* Where moe_layer_forward applies the combine. SEPARATE: its own kernel reads
 * y_perm back and writes y. FUSED (k <= 2 only): the down projection's
 * epilogue writes y itself: a token with one kept slot gets gate * row at
 * once, and for a token with two the epilogue that stores the later of its
 * two rows of a column tile (a per-token counter decides) reads both back
 * from y_perm and writes y in slot order. y is bit-identical either way, and
 * y_perm is still written (the backward reads it). Needs bf16 SwiGLU
 * experts, single-CTA tiles (gemm_tiles SINGLE, or AUTO, which then keeps
 * them) and bf16 precision. AUTO is SEPARATE: on B200
 * the fused form measured 1-3% slower per layer (its epilogue re-reads both
 * rows of a token while the GEMM runs), so it is opt-in. */
#define MOE_COMBINE_AUTO     0
#define MOE_COMBINE_SEPARATE 1
#define MOE_COMBINE_FUSED    2

/* What moe_layer_forward keeps for moe_layer_backward. RECOMPUTE: nothing
 * extra; the backward recomputes the gate/up pre-activations with a grouped
 * GEMM (4 A d F flops) and applies the SwiGLU backward in its epilogue. SAVE:
 * GEMM1's epilogue also stores the pre-activations a = x W_gate^T and
 * u = x W_up^T as bf16 [P, 2F] in the layer workspace (w13's interleaved
 * column order), and the backward applies the SwiGLU backward in the epilogue
 * of its dh_mid GEMM from them, with no recompute. The forward then writes
 * 4 P F more bytes; the backward's gradients use the bf16-rounded a and u.
 * SAVE needs bf16 SwiGLU experts, single-CTA tiles (gemm_tiles SINGLE, or
 * AUTO, which then keeps them), bf16 precision and the COPY dispatch. */
#define MOE_PREACT_RECOMPUTE 0
#define MOE_PREACT_SAVE      1

#define MOE_OP_ROUTE       0
#define MOE_OP_PERMUTE     1
#define MOE_OP_GROUPED_FFN 2
#define MOE_OP_LAYER       3
#define MOE_OP_BACKWARD    4

#define MOE_MAX_E 256
#define MOE_MAX_K 8
#define MOE_PACK_BLOCK 128

typedef struct moe_config {
  int32_t T;            /* tokens */
  int32_t d;            /* hidden size */
  int32_t E;            /* experts */
  int32_t k;            /* experts per token */
  int32_t d_ff;         /* expert FFN width F */
  int32_t dtype;        /* MOE_DTYPE_* */
  int32_t expert_kind;  /* MOE_EXPERT_* */
  int32_t capacity;     /* -1: dropless; >= 0: per-expert cap in assignments */
  int32_t gemm_tiles;   /* MOE_GEMM_TILES_*: tile shape of the bf16 grouped GEMMs */
  int32_t layout;       /* MOE_LAYOUT_*: row layout of the permuted buffers (P rows) */
  int32_t dispatch;     /* MOE_DISPATCH_*: x_perm row copy or gather inside GEMM1 (layer only) */
  int32_t precision;    /* MOE_PRECISION_*: operands of the grouped expert GEMMs */
  int32_t combine;      /* MOE_COMBINE_*: separate combine kernel or fused into the down projection (layer only) */
  int32_t preact;       /* MOE_PREACT_*: gate/up pre-activations recomputed or kept for the backward (layer only) */
} moe_config;

typedef void* moe_stream_t; /* cudaStream_t */

/* Bytes of workspace the given operation needs (MOE_OP_*). 0 on invalid cfg. */
MOE_API size_t moe_workspace_size(const moe_config* cfg, int32_t op);

/* Text for a MOE_OK / MOE_ERR_* code. Never NULL. */
MOE_API const char* moe_status_string(int32_t code);

/* ABI version, (major << 16) | minor. */
MOE_API int32_t moe_version(void);

/* moe_gemm_tiles_used -- writes to *tiles the tile shape
 * (MOE_GEMM_TILES_SINGLE or MOE_GEMM_TILES_PAIR) that the bf16 grouped GEMMs
 * of moe_grouped_ffn and moe_layer_forward take for cfg, with AUTO resolved.
 * Returns MOE_OK, MOE_ERR_INVALID_ARG (NULL tiles, invalid cfg) or
 * MOE_ERR_UNSUPPORTED (a cfg the library rejects); *tiles is then untouched.
 * Host only: no GPU work, no CUDA call. */
MOE_API int32_t moe_gemm_tiles_used(const moe_config* cfg, int32_t* tiles);

/* moe_pack_weights -- lay out the gate and up projections for the grouped FFN.
 * w_gate, w_up: [E, F, d]. w13_packed: [E, 2F, d], written. For each expert,
 * rows are interleaved in blocks of MOE_PACK_BLOCK (128) rows: block b holds
 * gate rows [128b, 128b+n) followed by up rows [128b, 128b+n), n = min(128,
 * F-128b). This lets one output tile of the first expert GEMM see matching
 * gate and up columns, so the SwiGLU product is formed in its epilogue.
 * W_down is used as given, [E, d, F]. Runs once per set of weights. */
MOE_API int32_t moe_pack_weights(const moe_config* cfg, const void* w_gate, const void* w_up,
                         void* w13_packed, moe_stream_t stream);

/* moe_route -- router scores, softmax and top-k.
 * ("How Does Mixture-of-Experts Routing Affect LLM Repeatability?": s_t =
 * h_t W_r, E_t = TopK(s_t, k), gate g_{t,e}; deterministic tie handling.)
 * h [T, d], w_router [E, d] (dtype), bias [E] fp32 or NULL.
 * logits_out [T, E] fp32 or NULL: s_t with the bias added.
 * topk_idx [T, k] int32: slot j holds the expert with the (j+1)-th highest
 *   score; equal scores go to the lower expert index; NaN counts as -inf.
 * topk_gate [T, k] fp32: softmax over all E experts renormalised over the k
 *   picks (= softmax over the k picked scores). A token whose scores are all
 *   -inf gets experts 0..k-1 with gate 0.
 * Scores are accumulated in fp32 (bf16 products on tensor cores for bf16). */
MOE_API int32_t moe_route(const moe_config* cfg, const void* h, const void* w_router, const float* bias,
                  float* logits_out, int32_t* topk_idx, float* topk_gate,
                  void* workspace, size_t ws_bytes, int32_t* status_dev, moe_stream_t stream);

/* moe_permute -- per-expert counts, offsets, drop decisions and the dispatch
 * permutation ("MoE Token Dispatch ...", "Follow one documented dispatch and
 * return path"; capacity resolved in token order as in "How Does
 * Mixture-of-Experts Routing Affect LLM Repeatability?").
 * topk_idx [T, k] int32 may come from moe_route or be supplied by the caller
 * (route replay). Slots with an index outside [0,E) or repeating an earlier
 * slot's expert are dropped and flag MOE_STATUS_BAD_ROUTE.
 * rank(t,j) = number of tokens t' < t that picked the same expert. The slot is
 * kept iff capacity < 0 or rank < capacity.
 * Outputs (all written; P rows as given by cfg->layout):
 *   routed_counts [E]  assignments per expert before drops
 *   counts [E]         kept assignments per expert
 *   offsets [E+1]      COMPACT: exclusive prefix sum of counts, offsets[E] = kept
 *                      total; PADDED: offsets[e] = e*capacity
 *   dest_row [T, k]    row of x_perm holding slot (t,j), -1 if dropped
 *   perm_src [P]       token of each x_perm row (COMPACT: first offsets[E]
 *                      entries valid; PADDED: -1 on padding rows)
 *   x_perm [P, d]      x_perm[dest_row[t,j]] = h[t], bitwise; the kept rows of
 *                      expert e start at offsets[e], in ascending token order;
 *                      COMPACT: rows past offsets[E] are left untouched;
 *                      PADDED: the padding rows are written as zeros. */
MOE_API int32_t moe_permute(const moe_config* cfg, const void* h, const int32_t* topk_idx,
                    int32_t* routed_counts, int32_t* counts, int32_t* offsets,
                    int32_t* dest_row, int32_t* perm_src, void* x_perm,
                    void* workspace, size_t ws_bytes, int32_t* status_dev, moe_stream_t stream);

/* moe_grouped_ffn -- all experts over their variable-length row groups in one
 * grouped computation ("Dropless MoE Is a Runtime Problem as Much as a Model
 * Design": one implementation over a collection of expert shapes, no padding).
 * x_perm [P, d] and offsets [E+1] as written by moe_permute; the group sizes
 * are read on the device (no host synchronisation).
 * w13_packed [E, 2F, d] from moe_pack_weights, w_down [E, d, F] (SwiGLU only;
 * may be NULL for the identity and scale experts).
 * y_perm [P, d]: y_perm[r] = f_e(x_perm[r]) for r in [offsets[e], offsets[e+1]).
 * bf16 path: silu(gate) * up is rounded to bf16 before the down projection. */
MOE_API int32_t moe_grouped_ffn(const moe_config* cfg, const void* x_perm, const int32_t* offsets,
                        const void* w13_packed, const void* w_down, void* y_perm,
                        void* workspace, size_t ws_bytes, int32_t* status_dev, moe_stream_t stream);

/* moe_unpermute_combine -- return every expert output to its token and
 * weight it (archcrux "moe-unpermute-wrong-token": outputs restored to their
 * original positions; top-k weights tied to the same token).
 * y[t] = sum_{j=0..k-1, dest_row[t,j] >= 0} topk_gate[t,j] * y_perm[dest_row[t,j]],
 * accumulated in fp32 in slot order, stored in dtype. Dropped slots add
 * nothing and the kept gates are not renormalised. */
MOE_API int32_t moe_unpermute_combine(const moe_config* cfg, const void* y_perm, const int32_t* dest_row,
                              const float* topk_gate, void* y, int32_t* status_dev,
                              moe_stream_t stream);

/* moe_layer_forward -- the whole layer on one stream: route, permute, grouped
 * FFN, unpermute/combine. Intermediates live in the workspace
 * (moe_workspace_size(cfg, MOE_OP_LAYER)). Optional outputs (NULL to skip):
 * topk_idx [T,k], topk_gate [T,k], routed_counts [E], counts [E]. */
MOE_API int32_t moe_layer_forward(const moe_config* cfg, const void* h, const void* w_router,
                          const float* bias, const void* w13_packed, const void* w_down, void* y,
                          int32_t* topk_idx, float* topk_gate, int32_t* routed_counts,
                          int32_t* counts, void* workspace, size_t ws_bytes,
                          int32_t* status_dev, moe_stream_t stream);

/* moe_layer_forward_timed -- moe_layer_forward that also records caller-owned
 * CUDA events between its stages, so a caller can time each stage inside a
 * real layer step (the stand-alone stage calls differ: moe_permute counts the
 * routes itself, while in the layer the router does). The pages have no
 * counterpart for this entry point; it is a measurement hook.
 * stage_events: NULL (then this is moe_layer_forward), or an array of 5
 * cudaEvent_t handles, each may be NULL. Recorded on `stream`:
 *   [0] before the router, [1] after the router, [2] after the dispatch
 *   (rank + row copy), [3] after the expert stage, [4] after the combine.
 * The events stay owned by the caller and must be created on the current
 * device; a failed record returns MOE_ERR_CUDA and enqueues no later stage. */
MOE_API int32_t moe_layer_forward_timed(const moe_config* cfg, const void* h, const void* w_router,
                                        const float* bias, const void* w13_packed, const void* w_down, void* y,
                                        int32_t* topk_idx, float* topk_gate, int32_t* routed_counts,
                                        int32_t* counts, void* workspace, size_t ws_bytes,
                                        int32_t* status_dev, moe_stream_t stream, void* const* stage_events);

/* moe_pack_weights_backward -- the transposed expert weights the backward
 * dgrad GEMMs read (once per weight update, like moe_pack_weights):
 *   w13_t [E, d, 2F]     w13_t[e] = w13_packed[e]^T (packed column order kept)
 *   w_down_t [E, F, d]   w_down_t[e] = w_down[e]^T
 * bf16 only; d and F multiples of 128. */
MOE_API int32_t moe_pack_weights_backward(const moe_config* cfg, const void* w13_packed, const void* w_down,
                                          void* w13_t, void* w_down_t, moe_stream_t stream);

/* moe_layer_backward -- gradients of L = sum_t <dy_t, y_t> for the layer
 * computed by the moe_layer_forward call that last used `fwd_workspace` with
 * the same cfg, h and weights: the chain rule through the forward
 * definition ("How Does Mixture-of-Experts Routing Affect LLM
 * Repeatability?", the token-choice layer) with the routing decision held
 * fixed. It reads the routing, gates, permutation, x_perm, h_mid and y_perm
 * that the forward left in fwd_workspace; nothing may touch it in between.
 *   dy [T, d] (bf16)          upstream gradient
 *   dh [T, d] (bf16)          through the experts and the router scores
 *   dw_router [E, d] (fp32)   dL/dW_r;  dbias [E] (fp32, may be NULL)
 *   dw13 [E, 2F, d] (fp32)    dL/dw13_packed: rows in w13_packed's interleaved
 *                             order (block b of 128 gate rows, then the
 *                             matching 128 up rows)
 *   dw_down [E, d, F] (fp32)  dL/dW_down
 * Gate gradient: ds_{t,j} = g_j (dgate_j - sum_i g_i dgate_i) over the picked
 * slots (dgate_j = <dy_t, f_e(h_t)> for kept slots, 0 for dropped ones).
 * Needs bf16, SwiGLU experts and a forward that wrote x_perm (dispatch COPY
 * or AUTO); else MOE_ERR_UNSUPPORTED. Both layouts are supported (in the
 * PADDED one the padding rows are computed as zero rows). Scratch:
 * moe_workspace_size(cfg, MOE_OP_BACKWARD). Deterministic. */
MOE_API int32_t moe_layer_backward(const moe_config* cfg, const void* h, const void* w_router,
                                   const void* w13_packed, const void* w13_t, const void* w_down_t,
                                   const void* dy, void* dh, float* dw_router, float* dbias, float* dw13,
                                   float* dw_down, const void* fwd_workspace, size_t fwd_ws_bytes,
                                   void* workspace, size_t ws_bytes, int32_t* status_dev, moe_stream_t stream);

/* moe_mxfp8_quantize -- MXFP8 quantisation of a bf16 matrix along its rows
 * (the format described at MOE_PRECISION_MXFP8).
 * x [rows, cols] bf16, cols a multiple of 128. q [rows, cols]: one E4M3 byte
 * per element. sf: the E8M0 scale bytes in the order the block-scaled tensor
 * cores read them: for every 128-row block R and 128-column slice kt one
 * 512-byte atom at (kt * ceil(rows/128) + R) * 512, in which the scale of row
 * r (within the block) and 32-column block j (within the slice) is byte
 * (r % 32) * 16 + (r / 32) * 4 + j; (cols/128) * ceil(rows/128) * 512 bytes.
 * Bytes of the last atom row that belong to rows past `rows` are left
 * untouched. counts [2] uint32 (may be NULL): saturated and underflowed
 * elements are ADDED to counts[0] and counts[1]. status_dev as elsewhere
 * (MOE_STATUS_MX_* bits). */
MOE_API int32_t moe_mxfp8_quantize(const void* x, int32_t rows, int32_t cols, void* q, void* sf, uint32_t* counts,
                                   int32_t* status_dev, moe_stream_t stream);

/* Bytes of the MXFP8 weight blobs for cfg: which = 0 for w13 (GEMM1's B,
 * [E*2F, d]), 1 for w_down (GEMM2's B, [E*d, F]). A blob holds the E4M3
 * bytes [rows, cols], then at the next 256-byte boundary the scale atoms of
 * moe_mxfp8_quantize's layout with one extra (zero) 128-row block per
 * 128-column slice: (cols/128) * (rows/128 + 1) * 512 bytes. 0 on an
 * invalid cfg. */
MOE_API size_t moe_mxfp8_weights_size(const moe_config* cfg, int32_t which);

/* moe_pack_weights_mxfp8 -- quantise the expert weights once for
 * MOE_PRECISION_MXFP8: w13_packed [E, 2F, d] (from moe_pack_weights) along d
 * into w13_mx, and w_down [E, d, F] along F into w_down_mx (blobs sized by
 * moe_mxfp8_weights_size). counts [2] (may be NULL): saturated and
 * underflowed weight elements are added. bf16, SwiGLU experts. */
MOE_API int32_t moe_pack_weights_mxfp8(const moe_config* cfg, const void* w13_packed, const void* w_down,
                                       void* w13_mx, void* w_down_mx, uint32_t* counts, moe_stream_t stream);

/* moe_debug_stall_next_gemms -- testing hook for the timeout path. The pages
 * have no counterpart. The next n launches (process-wide, any stream) of the
 * bf16 grouped GEMM kernels (single-CTA or CTA-pair tiles) make their
 * MMA-issuing thread first wait on a barrier that nothing signals. That wait gives up after the library's
 * on-chip limit (2 s), the kernel unwinds as after any timeout (no MMA was
 * issued; the operand loads already issued are waited for and TMEM is freed)
 * and MOE_STATUS_TIMEOUT is OR-ed into the status word; that call's outputs
 * are invalid and the context stays usable. n = 0 cancels. */
MOE_API int32_t moe_debug_stall_next_gemms(int32_t n);

/* moe_permute_static_scratch -- moe_permute for callers that cannot allocate.
 * The paper has no counterpart for this entry point. It is for code that has
 * no way to pass a workspace: a host framework or memory pool that owns all
 * device memory and forbids allocations outside it, or a latency-critical
 * path that must not allocate. Inputs, outputs and results are exactly those
 * of moe_permute; the permute scratch lives instead in a fixed 1 MiB array in
 * the library's device image, which every GPU that loads the library holds
 * until the process exits.
 * Limit: 2 * roundup256(4 * E * ceil(T/128)) bytes must fit in 1 MiB
 * (E * ceil(T/128) <= 131072, e.g. T <= 65536 at E = 256); larger problems
 * return MOE_ERR_WORKSPACE and enqueue nothing.
 * All calls share the array: calls that may overlap on the GPU (streams with
 * no ordering between them) race and give wrong results. Nothing in the array
 * needs to start at zero. A call outside stream capture looks up the
 * array's address on the current device and remembers it; a call made while
 * `stream` is being captured uses the remembered address, so make one call on
 * each device before capturing (else MOE_ERR_CUDA). No cudaMalloc, cudaFree
 * or other allocating call is made. */
MOE_API int32_t moe_permute_static_scratch(const moe_config* cfg, const void* h, const int32_t* topk_idx,
                                           int32_t* routed_counts, int32_t* counts, int32_t* offsets,
                                           int32_t* dest_row, int32_t* perm_src, void* x_perm,
                                           int32_t* status_dev, moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
