// Internal launch interface between the C ABI layer and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

// Tokens per dispatch chunk (one CTA of the count and rank kernels).
constexpr int kChunkTokens = 128;
// Rows per tile of the tensor-core kernels.
constexpr int kTileM = 128;
// Columns per output tile of the grouped expert GEMM.
constexpr int kGemmTileN = 256;

int device_sm_count();

// router.cu
// Padded expert count of the router's score tile: a multiple of 16, or of 32
// from 49 experts on, where a CTA pair splits the reduction over d and each
// CTA ranks half of the experts.
constexpr int kRouterSplitMin = 64;
inline int router_npad(int E) { return E > 48 ? (E + 31) / 32 * 32 : (E + 15) / 16 * 16; }
inline bool router_splits_experts(int npad) { return npad >= kRouterSplitMin; }
// chunk_counts (may be NULL): per-128-token-tile expert histogram [ceil(T/128)][E].
cudaError_t launch_router_tc(const CUtensorMap& tm_h, const CUtensorMap& tm_w, int T, int d, int E, int k,
                             int npad, const float* bias, float* logits, int32_t* idx, float* gate,
                             int32_t* chunk_counts, int32_t* status, cudaStream_t s);
cudaError_t launch_router_f32(const float* h, const float* w, int T, int d, int E, int k, const float* bias,
                              float* logits, int32_t* idx, float* gate, int32_t* status, cudaStream_t s);

// dispatch.cu
// padded: every expert owns `cap` rows of x_perm (offsets[e] = e * cap); the
// rows past its kept count are zero-filled and their perm_src set to -1.
// copy_rows: false skips the x_perm row copy (the grouped GEMM gathers the
// rows itself); everything else is still written.
// pair_cnt / pair_tiles / y_zero (the combine fused into the down projection;
// NULL / 0 / NULL otherwise): the rank kernel zeroes pair_cnt [T][pair_tiles]
// and the y rows (row_bytes each) of tokens that keep no slot.
cudaError_t launch_permute(const void* h, size_t row_bytes, const int32_t* idx, int T, int k, int E, int cap,
                           bool padded, bool copy_rows, int32_t* chunk_counts, int32_t* chunk_base, int32_t* routed, int32_t* kept,
                           int32_t* offsets, int32_t* dest_row, int32_t* perm_src, void* x_perm,
                           bool counts_ready, bool pdl, int32_t* status, cudaStream_t s, int32_t* pair_cnt = nullptr,
                           int pair_tiles = 0, void* y_zero = nullptr);
cudaError_t launch_combine(int dtype, const void* y_perm, const int32_t* dest_row, const float* gate, void* y,
                           int T, int k, int d, bool pdl, cudaStream_t s, int32_t* status = nullptr);

// grouped_ffn.cu
// Launch flags `pdl` (here and in launch_permute / launch_combine): launch as
// a programmatic dependent of the previous kernel on the stream. Only set it
// when that kernel belongs to the same library call.
// gather_rows (may be NULL): A row r is row gather_rows[r] of the tensor behind
// tm_a, whose box must then be 64 columns by one row.
// preact (swiglu only, may be NULL): also store the gate/up pre-activations
// [rows, n_per_expert] bf16 in w13's interleaved column order.
// tm_d (may be NULL): D as a store tensor map (make_map_store: bf16, 32 x 32
// boxes, 64-byte swizzle); the epilogue then writes whole 32-row blocks of
// the tile with TMA stores.
cudaError_t launch_grouped_gemm_tc(const CUtensorMap& tm_a, const CUtensorMap& tm_b, bool swiglu,
                                   const int32_t* offsets, int E, int K, int n_per_expert, int n_tiles,
                                   int out_cols, int ldd, void* D, const int32_t* gather_rows, int32_t* status,
                                   bool pdl, cudaStream_t s, void* preact = nullptr,
                                   const CUtensorMap* tm_d = nullptr);
// The backward's dh_mid GEMM (dy_perm rows against W_down^T rows, K = d) with
// the SwiGLU backward in its epilogue from the saved pre-activations
// preact [rows, 2F]: writes dgu [rows, 2F] = [dgate | dup] (interleaved) and
// its transposed copy dgu_t as launch_grouped_gemm_swiglu_bwd does.
cudaError_t launch_grouped_gemm_dh_swiglu_bwd(const CUtensorMap& tm_a, const CUtensorMap& tm_b,
                                              const int32_t* offsets, int E, int K, int F, const void* preact,
                                              void* dgu, void* dgu_t, const int32_t* col_off, int ldt, int32_t* status,
                                              bool pdl, cudaStream_t s,
                                              const CUtensorMap* tm_d = nullptr);
// The down projection with the combine fused into its epilogue (k <= 2): y_perm
// rows as launch_grouped_gemm_tc, and y [T, d] = sum over each token's kept
// slots, in slot order, of gate * bf16 row (bit-identical to launch_combine).
// pair_cnt [T][2 * ceil(d/256)] must be zero and the y rows of tokens that keep
// no slot written beforehand (launch_permute does both).
cudaError_t launch_grouped_gemm_combine(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const int32_t* offsets, int E,
                                        int K, int d, void* y_perm, const int32_t* perm_src, const int32_t* dest_row,
                                        const float* gate, int32_t* pair_cnt, void* y, int k, int32_t* status, bool pdl,
                                        cudaStream_t s);
// Testing hook: the next n launches of the bf16 grouped GEMM kernel stall their
// MMA issuer on a barrier nothing signals until the bounded wait gives up.
void debug_stall_next_gemms(int n);
// GEMM1 recomputed with the SwiGLU backward in its epilogue: from the gate and
// up pre-activations of each row (x_perm rows against w13) and dh_mid [rows, F]
// it writes dgu [rows, 2F] = [dgate | dup] in w13's interleaved column order,
// and, when dgu_t is set, the same values transposed: dgu_t [2F, ldt] with
// expert e's rows at columns col_off[e] + i and zeros up to col_off[e+1].
cudaError_t launch_grouped_gemm_swiglu_bwd(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const int32_t* offsets,
                                           int E, int K, int F, void* dgu, const void* dh_mid, void* dgu_t,
                                           const int32_t* col_off, int ldt, int32_t* status, bool pdl,
                                           cudaStream_t s,
                                           const CUtensorMap* tm_d = nullptr);
// Weight gradients: for each expert e, D32[e] [M, N] (fp32) = A_e B_e^T where
// A [M, cols] and B [N, cols] are transposed activations whose columns
// [col_offsets[e], col_offsets[e+1]) (multiples of 64, zero padded) belong to
// expert e. tm_a has boxes of 128 rows, tm_b of 256 rows (64 columns each).
cudaError_t launch_grouped_gemm_wgrad(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const int32_t* col_offsets,
                                      int E, int M, int N, float* D32, int32_t* status, bool pdl, cudaStream_t s);
cudaError_t launch_grouped_gemm_pair(const CUtensorMap& tm_a, const CUtensorMap& tm_b, bool swiglu,
                                     const int32_t* offsets, int E, int K, int n_per_expert, int n_tiles, int out_cols,
                                     int ldd, void* D, int32_t* status, bool pdl, cudaStream_t s,
                                     const CUtensorMap* tm_d = nullptr);
cudaError_t launch_ffn_f32(const float* x_perm, const int32_t* offsets, const float* w13, const float* wd,
                           float* h_mid, float* y_perm, int rows_max, int d, int F, int E, cudaStream_t s);
cudaError_t launch_scale_rows(int dtype, int kind, const void* x_perm, const int32_t* offsets, void* y_perm,
                              int rows_max, int d, int E, cudaStream_t s);
cudaError_t launch_pack_w13(const void* w_gate, const void* w_up, void* w13, int E, int F, size_t row_bytes,
                            cudaStream_t s);

// grouped_ffn_mx.cu (MXFP8: E4M3 elements, one E8M0 scale per 32 along the
// reduction axis; scales in 512-byte atoms per 128 rows x 128 columns)
// Quantises rows of a bf16 matrix. offsets != NULL: grouped mode, the output
// rows are the padded layout (every expert's rows start on a 128-row
// boundary, rows past its count are zeros) and `rows` only bounds the grid.
// sf_row_blocks: 128-row blocks per 128-column slice of the atom array.
cudaError_t launch_mx_quantize(const void* src, int rows, int cols, const int32_t* offsets, int E, void* q, void* sf,
                               int sf_row_blocks, uint32_t* counts, int32_t* status, bool pdl, cudaStream_t s);
// The layer's dispatch fused with the quantisation: token rows of h [T, d]
// straight to the padded quantised layout (every kept slot's destination from
// dest_row, idx and offsets), padding rows zeroed.
cudaError_t launch_mx_dispatch(const void* h, int T, int d, int k, const int32_t* idx, const int32_t* dest_row,
                               const int32_t* offsets, int E, void* q, void* sf, int sf_row_blocks, uint32_t* counts,
                               int32_t* status, bool pdl, cudaStream_t s);
// Block-scaled grouped GEMM over the padded groups. swiglu_quant: GEMM1, D is
// the quantised silu(gate) * up in the padded layout (q_out, sf_out with
// ra_blocks row blocks, ldq = F); else GEMM2, bf16 D in the compact layout.
// sfb: the B scale atoms with rb_blocks + 1 row blocks per slice.
cudaError_t launch_grouped_gemm_mx(const CUtensorMap& tm_a, const CUtensorMap& tm_b, bool swiglu_quant,
                                   const int32_t* offsets, int E, int K, int n_per_expert, int out_cols,
                                   const void* sfa, int ra_blocks, const void* sfb, void* q_out, void* sf_out, int ldq,
                                   uint32_t* counts, void* D, int ldd, int32_t* status, bool pdl, cudaStream_t s,
                                   const CUtensorMap* tm_d = nullptr);

// backward.cu
cudaError_t launch_combine_bwd(const void* dy, const void* y_perm, const int32_t* dest_row, const float* gate,
                               void* dy_perm, float* ds, int T, int k, int d, cudaStream_t s);
cudaError_t launch_token_grad(const void* dx_perm, const int32_t* dest_row, const int32_t* idx, const float* ds,
                              const void* w_router, void* dh, int T, int k, int d, cudaStream_t s);
// scratch: router_wgrad_scratch(T, E, d) bytes (per-chunk partial sums).
size_t router_wgrad_scratch(int T, int E, int d);
cudaError_t launch_router_wgrad(const void* h, const int32_t* idx, const float* ds, int T, int k, int d, int E,
                                float* dw_router, float* dbias, float* scratch, cudaStream_t s);
cudaError_t launch_col_offsets(const int32_t* offsets, int E, int32_t* col_off, cudaStream_t s);
// XT [C, ppad_max] from X [rows, C]: expert e's rows become columns
// [col_off[e], col_off[e+1]) (multiples of 64), zero padded.
cudaError_t launch_transpose_grouped(const void* X, int C, const int32_t* offsets, const int32_t* col_off, int E,
                                     int ppad_max, void* XT, cudaStream_t s);
// [E][R][C] -> [E][C][R], bf16, R and C multiples of 64.
cudaError_t launch_transpose_batched(const void* X, int E, int R, int C, void* XT, cudaStream_t s);

}  // namespace moe
