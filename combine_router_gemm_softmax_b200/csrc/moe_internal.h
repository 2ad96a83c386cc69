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
cudaError_t launch_permute(const void* h, size_t row_bytes, const int32_t* idx, int T, int k, int E, int cap,
                           bool padded, bool copy_rows, int32_t* chunk_counts, int32_t* chunk_base, int32_t* routed, int32_t* kept,
                           int32_t* offsets, int32_t* dest_row, int32_t* perm_src, void* x_perm,
                           bool counts_ready, bool pdl, int32_t* status, cudaStream_t s);
cudaError_t launch_combine(int dtype, const void* y_perm, const int32_t* dest_row, const float* gate, void* y,
                           int T, int k, int d, bool pdl, cudaStream_t s);

// grouped_ffn.cu
// Launch flags `pdl` (here and in launch_permute / launch_combine): launch as
// a programmatic dependent of the previous kernel on the stream. Only set it
// when that kernel belongs to the same library call.
// gather_rows (may be NULL): A row r is row gather_rows[r] of the tensor behind
// tm_a, whose box must then be 64 columns by one row.
cudaError_t launch_grouped_gemm_tc(const CUtensorMap& tm_a, const CUtensorMap& tm_b, bool swiglu,
                                   const int32_t* offsets, int E, int K, int n_per_expert, int n_tiles,
                                   int out_cols, int ldd, void* D, const int32_t* gather_rows, int32_t* status,
                                   bool pdl, cudaStream_t s);
cudaError_t launch_grouped_gemm_pair(const CUtensorMap& tm_a, const CUtensorMap& tm_b, bool swiglu,
                                     const int32_t* offsets, int E, int K, int n_per_expert, int n_tiles, int out_cols,
                                     int ldd, void* D, int32_t* status, bool pdl, cudaStream_t s);
cudaError_t launch_ffn_f32(const float* x_perm, const int32_t* offsets, const float* w13, const float* wd,
                           float* h_mid, float* y_perm, int rows_max, int d, int F, int E, cudaStream_t s);
cudaError_t launch_scale_rows(int dtype, int kind, const void* x_perm, const int32_t* offsets, void* y_perm,
                              int rows_max, int d, int E, cudaStream_t s);
cudaError_t launch_pack_w13(const void* w_gate, const void* w_up, void* w13, int E, int F, size_t row_bytes,
                            cudaStream_t s);

}  // namespace moe
