// Backward pass of the layer: gradients of L = sum_t <dy_t, y_t> by the chain
// rule through the forward definition ("How Does Mixture-of-Experts Routing
// Affect LLM Repeatability?", the simplified token-choice layer; the routing
// decision is piecewise constant and held fixed). "Dropless MoE Is a Runtime
// Problem as Much as a Model Design" treats the dropless layer as a training
// workload; this is the training half of the same path.
//
// The expert GEMMs run on the grouped tcgen05 kernel (grouped_ffn.cu); this
// file holds the memory-bound pieces around them:
//   combine_bwd   dgate_{t,j} = <dy_t, y_perm[r]>, dy_perm[r] = g_{t,j} dy_t and
//                 ds = g (dgate - sum_i g_i dgate_i)  (softmax over the picks)
//   token_grad    dh_t = sum over kept slots of dx_perm[r] + sum_j ds_j W_r[e_j]
//   router_wgrad  dW_r[e] = sum ds_{t,j} h_t, db[e] = sum ds_{t,j} over (t,j) with e_j = e
//   transposes    the weight-gradient GEMMs reduce over each expert's rows, so
//                 their operands are transposed into [channels, rows] with each
//                 expert's rows starting at a multiple of 64 (zero padded)
// All reductions run in a fixed order, so the gradients are deterministic.
#include <algorithm>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

MOE_DEV float warp_sum_f(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

MOE_DEV float bf_lo(uint32_t p) { return __uint_as_float(p << 16); }
MOE_DEV float bf_hi(uint32_t p) { return __uint_as_float(p & 0xffff0000u); }

// One warp per token. Rows are bf16, vpr 16-byte vectors (8 values) each.
template <int K>
__global__ void __launch_bounds__(256) combine_bwd_kernel(const uint4* __restrict__ dy,
                                                          const uint4* __restrict__ y_perm,
                                                          const int32_t* __restrict__ dest_row,
                                                          const float* __restrict__ gate, uint4* __restrict__ dy_perm,
                                                          float* __restrict__ ds, int T, int vpr) {
  const int lane = threadIdx.x & 31;
  const int nw = gridDim.x * (blockDim.x >> 5);
  for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += nw) {
    int dst[K];
    float g[K], dg[K];
#pragma unroll
    for (int j = 0; j < K; ++j) {
      dst[j] = dest_row[static_cast<size_t>(t) * K + j];
      g[j] = gate[static_cast<size_t>(t) * K + j];
      dg[j] = 0.f;
    }
    for (int v = lane; v < vpr; v += 32) {
      const uint4 q = dy[static_cast<size_t>(t) * vpr + v];
      const uint32_t dq[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int j = 0; j < K; ++j) {
        if (dst[j] < 0) continue;
        const uint4 w = y_perm[static_cast<size_t>(dst[j]) * vpr + v];
        const uint32_t wq[4] = {w.x, w.y, w.z, w.w};
        float acc = 0.f;
        uint32_t out[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc = fmaf(bf_lo(dq[i]), bf_lo(wq[i]), acc);
          acc = fmaf(bf_hi(dq[i]), bf_hi(wq[i]), acc);
          out[i] = pack_bf16x2(g[j] * bf_lo(dq[i]), g[j] * bf_hi(dq[i]));
        }
        dg[j] += acc;
        dy_perm[static_cast<size_t>(dst[j]) * vpr + v] = make_uint4(out[0], out[1], out[2], out[3]);
      }
    }
    float sum = 0.f;
#pragma unroll
    for (int j = 0; j < K; ++j) {
      dg[j] = warp_sum_f(dg[j]);
      sum = fmaf(g[j], dg[j], sum);
    }
    if (lane < K) {
      float mine = 0.f;
#pragma unroll
      for (int j = 0; j < K; ++j)
        if (j == lane) mine = g[j] * (dg[j] - sum);
      ds[static_cast<size_t>(t) * K + lane] = mine;
    }
  }
}

// One warp per token: dh_t = sum_j dx_perm[dest_j] (kept slots, in slot order)
// + sum_j ds_j W_r[e_j], accumulated in fp32 and stored as bf16.
template <int K>
__global__ void __launch_bounds__(256) token_grad_kernel(const uint4* __restrict__ dx_perm,
                                                         const int32_t* __restrict__ dest_row,
                                                         const int32_t* __restrict__ idx, const float* __restrict__ ds,
                                                         const uint4* __restrict__ w_router, uint4* __restrict__ dh,
                                                         int T, int vpr) {
  const int lane = threadIdx.x & 31;
  const int nw = gridDim.x * (blockDim.x >> 5);
  for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += nw) {
    int dst[K], ex[K];
    float s[K];
#pragma unroll
    for (int j = 0; j < K; ++j) {
      dst[j] = dest_row[static_cast<size_t>(t) * K + j];
      ex[j] = idx[static_cast<size_t>(t) * K + j];
      s[j] = ds[static_cast<size_t>(t) * K + j];
    }
    for (int v = lane; v < vpr; v += 32) {
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
      for (int j = 0; j < K; ++j) {
        if (dst[j] < 0) continue;
        const uint4 q = dx_perm[static_cast<size_t>(dst[j]) * vpr + v];
        const uint32_t p[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[2 * i] += bf_lo(p[i]);
          acc[2 * i + 1] += bf_hi(p[i]);
        }
      }
#pragma unroll
      for (int j = 0; j < K; ++j) {
        const uint4 q = w_router[static_cast<size_t>(ex[j]) * vpr + v];
        const uint32_t p[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[2 * i] = fmaf(s[j], bf_lo(p[i]), acc[2 * i]);
          acc[2 * i + 1] = fmaf(s[j], bf_hi(p[i]), acc[2 * i + 1]);
        }
      }
      dh[static_cast<size_t>(t) * vpr + v] =
          make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]), pack_bf16x2(acc[4], acc[5]),
                     pack_bf16x2(acc[6], acc[7]));
    }
  }
}

// Router weight gradient in two fixed-order passes. Pass 1: CTA (token chunk
// of kRwChunk tokens, 128 columns) keeps a [E][128] fp32 partial in shared
// memory, each thread one column, adding ds_{t,j} h[t, c] into row e_j for the
// chunk's tokens in order (thread 0 also sums ds into a [E] bias partial);
// it writes the partials out. Pass 2 adds the partials over chunks in chunk
// order.
constexpr int kRwChunk = 512;
constexpr int kRwCols = 128;

__global__ void __launch_bounds__(kRwCols) router_wgrad_partial_kernel(const __nv_bfloat16* __restrict__ h,
                                                                       const int32_t* __restrict__ idx,
                                                                       const float* __restrict__ ds, int T, int k,
                                                                       int d, int E, float* __restrict__ part,
                                                                       float* __restrict__ part_b) {
  extern __shared__ float sp[];  // [E][kRwCols], then [E] bias partial
  float* spb = sp + E * kRwCols;
  const int chunk = blockIdx.x;
  const int c = blockIdx.y * kRwCols + threadIdx.x;
  for (int i = threadIdx.x; i < E * kRwCols; i += blockDim.x) sp[i] = 0.f;
  for (int i = threadIdx.x; i < E; i += blockDim.x) spb[i] = 0.f;
  __syncthreads();
  const int t0 = chunk * kRwChunk, t1 = min(T, t0 + kRwChunk);
  for (int t = t0; t < t1; ++t) {
    const float hv = c < d ? __bfloat162float(h[static_cast<size_t>(t) * d + c]) : 0.f;
    for (int j = 0; j < k; ++j) {
      const int e = idx[static_cast<size_t>(t) * k + j];
      const float w = ds[static_cast<size_t>(t) * k + j];
      sp[e * kRwCols + threadIdx.x] = fmaf(w, hv, sp[e * kRwCols + threadIdx.x]);
      if (threadIdx.x == 0 && blockIdx.y == 0) spb[e] += w;
    }
  }
  __syncthreads();
  float* out = part + static_cast<size_t>(chunk) * E * d;
  for (int e = 0; e < E; ++e)
    if (c < d) out[static_cast<size_t>(e) * d + c] = sp[e * kRwCols + threadIdx.x];
  if (blockIdx.y == 0)
    for (int e = threadIdx.x; e < E; e += blockDim.x) part_b[static_cast<size_t>(chunk) * E + e] = spb[e];
}

__global__ void __launch_bounds__(256) router_wgrad_reduce_kernel(const float* __restrict__ part,
                                                                  const float* __restrict__ part_b, int n_chunks,
                                                                  int E, int d, float* __restrict__ dw_router,
                                                                  float* __restrict__ dbias) {
  const size_t n = static_cast<size_t>(E) * d;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    float acc = 0.f;
    for (int ch = 0; ch < n_chunks; ++ch) acc += part[static_cast<size_t>(ch) * n + i];
    dw_router[i] = acc;
  }
  if (dbias != nullptr && blockIdx.x == 0)
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      float acc = 0.f;
      for (int ch = 0; ch < n_chunks; ++ch) acc += part_b[static_cast<size_t>(ch) * E + e];
      dbias[e] = acc;
    }
}

// col_off[e] = sum over e' < e of roundup64(offsets[e'+1] - offsets[e']).
__global__ void col_offsets_kernel(const int32_t* __restrict__ offsets, int E, int32_t* __restrict__ col_off) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  int run = 0;
  for (int e = 0; e < E; ++e) {
    col_off[e] = run;
    run += (offsets[e + 1] - offsets[e] + 63) / 64 * 64;
  }
  col_off[E] = run;
}

constexpr int kTr = 64;    // transpose tile edge
constexpr int kTrLd = 72;  // shared row stride in bf16 (144 bytes: 16-byte aligned, spreads the column reads)

// Fills tile[r][0..63] from 64 bf16 of row r (16-byte loads), rows from `src`
// (nullptr: a zero row); 256 threads, two 16-byte pieces each.
MOE_DEV void tr_load(__nv_bfloat16 (*tile)[kTrLd], const __nv_bfloat16* const* src_rows) {
  for (int i = threadIdx.x; i < kTr * 8; i += blockDim.x) {
    const int r = i >> 3, seg = i & 7;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (src_rows[r] != nullptr) v = *reinterpret_cast<const uint4*>(src_rows[r] + seg * 8);
    *reinterpret_cast<uint4*>(&tile[r][seg * 8]) = v;
  }
}

// Writes column c of the tile (64 values, rows 0..63) as row c of the output:
// dst_rows[c] + [0, 64), 16-byte stores. A warp takes 32 consecutive columns
// of the same 8 rows, so each of its shared-memory reads is one contiguous
// 64-byte row segment (no bank conflicts).
MOE_DEV void tr_store(__nv_bfloat16 (*tile)[kTrLd], __nv_bfloat16* const* dst_rows) {
  for (int i = threadIdx.x; i < kTr * 8; i += blockDim.x) {
    const int c = i & (kTr - 1), rseg = i >> 6;
    if (dst_rows[c] == nullptr) continue;
    uint32_t p[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint16_t lo = __bfloat16_as_ushort(tile[rseg * 8 + 2 * q][c]);
      const uint16_t hi = __bfloat16_as_ushort(tile[rseg * 8 + 2 * q + 1][c]);
      p[q] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
    }
    *reinterpret_cast<uint4*>(dst_rows[c] + rseg * 8) = make_uint4(p[0], p[1], p[2], p[3]);
  }
}

// XT [C, ldt] from X [rows, C] (bf16, C a multiple of 64): column j of XT in
// expert e's padded range [col_off[e], col_off[e+1]) is row
// offsets[e] + (j - col_off[e]) of X, or zero past the expert's rows. One 64 x
// 64 tile per CTA through shared memory.
__global__ void __launch_bounds__(256) transpose_grouped_kernel(const __nv_bfloat16* __restrict__ X, int C,
                                                                const int32_t* __restrict__ offsets,
                                                                const int32_t* __restrict__ col_off, int E,
                                                                __nv_bfloat16* __restrict__ XT, int ldt) {
  __shared__ __align__(16) __nv_bfloat16 tile[kTr][kTrLd];
  __shared__ const __nv_bfloat16* src[kTr];
  __shared__ __nv_bfloat16* dst[kTr];
  const int j0 = blockIdx.x * kTr;  // first padded column (= row of X) of this tile
  const int c0 = blockIdx.y * kTr;  // first channel
  if (j0 >= col_off[E]) return;
  int lo = 0, hi = E;  // col_off[lo] <= j0 < col_off[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (col_off[mid] <= j0)
      lo = mid;
    else
      hi = mid;
  }
  const int e = lo;
  const int i0 = j0 - col_off[e];
  const int rows_e = offsets[e + 1] - offsets[e];
  if (threadIdx.x < kTr) {
    const int r = threadIdx.x;
    src[r] = i0 + r < rows_e ? X + static_cast<size_t>(offsets[e] + i0 + r) * C + c0 : nullptr;
    dst[r] = XT + static_cast<size_t>(c0 + r) * ldt + j0;
  }
  __syncthreads();
  tr_load(tile, src);
  __syncthreads();
  tr_store(tile, dst);
}

// Per-expert transpose of a weight [E][R][C] into [E][C][R] (R, C multiples of 64).
__global__ void __launch_bounds__(256) transpose_batched_kernel(const __nv_bfloat16* __restrict__ X, int R, int C,
                                                                __nv_bfloat16* __restrict__ XT) {
  __shared__ __align__(16) __nv_bfloat16 tile[kTr][kTrLd];
  __shared__ const __nv_bfloat16* src[kTr];
  __shared__ __nv_bfloat16* dst[kTr];
  const size_t base = static_cast<size_t>(blockIdx.z) * R * C;
  const int r0 = blockIdx.x * kTr, c0 = blockIdx.y * kTr;
  if (threadIdx.x < kTr) {
    src[threadIdx.x] = X + base + static_cast<size_t>(r0 + threadIdx.x) * C + c0;
    dst[threadIdx.x] = XT + base + static_cast<size_t>(c0 + threadIdx.x) * R + r0;
  }
  __syncthreads();
  tr_load(tile, src);
  __syncthreads();
  tr_store(tile, dst);
}

int warp_grid_bwd(int T) {
  const int want = (T + 7) / 8;
  const int cap = device_sm_count() * 8;
  return want < cap ? (want > 0 ? want : 1) : cap;
}

}  // namespace

cudaError_t launch_combine_bwd(const void* dy, const void* y_perm, const int32_t* dest_row, const float* gate,
                               void* dy_perm, float* ds, int T, int k, int d, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int vpr = d / 8;
  const int grid = warp_grid_bwd(T);
  auto* a = static_cast<const uint4*>(dy);
  auto* b = static_cast<const uint4*>(y_perm);
  auto* o = static_cast<uint4*>(dy_perm);
  switch (k) {
#define MOE_CB_K(KK) \
  case KK:           \
    combine_bwd_kernel<KK><<<grid, 256, 0, s>>>(a, b, dest_row, gate, o, ds, T, vpr); \
    break;
    MOE_CB_K(1)
    MOE_CB_K(2)
    MOE_CB_K(3)
    MOE_CB_K(4)
    MOE_CB_K(5)
    MOE_CB_K(6)
    MOE_CB_K(7)
    MOE_CB_K(8)
#undef MOE_CB_K
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

cudaError_t launch_token_grad(const void* dx_perm, const int32_t* dest_row, const int32_t* idx, const float* ds,
                              const void* w_router, void* dh, int T, int k, int d, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int vpr = d / 8;
  const int grid = warp_grid_bwd(T);
  auto* x = static_cast<const uint4*>(dx_perm);
  auto* w = static_cast<const uint4*>(w_router);
  auto* o = static_cast<uint4*>(dh);
  switch (k) {
#define MOE_TG_K(KK) \
  case KK:           \
    token_grad_kernel<KK><<<grid, 256, 0, s>>>(x, dest_row, idx, ds, w, o, T, vpr); \
    break;
    MOE_TG_K(1)
    MOE_TG_K(2)
    MOE_TG_K(3)
    MOE_TG_K(4)
    MOE_TG_K(5)
    MOE_TG_K(6)
    MOE_TG_K(7)
    MOE_TG_K(8)
#undef MOE_TG_K
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

size_t router_wgrad_scratch(int T, int E, int d) {
  const size_t chunks = (static_cast<size_t>(T) + kRwChunk - 1) / kRwChunk;
  return chunks * E * (static_cast<size_t>(d) + 1) * 4;
}

cudaError_t launch_router_wgrad(const void* h, const int32_t* idx, const float* ds, int T, int k, int d, int E,
                                float* dw_router, float* dbias, float* scratch, cudaStream_t s) {
  const int chunks = (T + kRwChunk - 1) / kRwChunk;
  float* part = scratch;
  float* part_b = scratch + static_cast<size_t>(chunks) * E * d;
  if (chunks > 0) {
    const size_t smem = static_cast<size_t>(E) * (kRwCols + 1) * 4;
    cudaError_t err = cudaFuncSetAttribute(router_wgrad_partial_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    router_wgrad_partial_kernel<<<dim3(chunks, (d + kRwCols - 1) / kRwCols), kRwCols, smem, s>>>(
        static_cast<const __nv_bfloat16*>(h), idx, ds, T, k, d, E, part, part_b);
  }
  const long long n = static_cast<long long>(E) * d;
  const int grid = static_cast<int>(std::min<long long>((n + 255) / 256, device_sm_count() * 8LL));
  router_wgrad_reduce_kernel<<<grid > 0 ? grid : 1, 256, 0, s>>>(part, part_b, chunks, E, d, dw_router, dbias);
  return cudaGetLastError();
}

cudaError_t launch_col_offsets(const int32_t* offsets, int E, int32_t* col_off, cudaStream_t s) {
  col_offsets_kernel<<<1, 32, 0, s>>>(offsets, E, col_off);
  return cudaGetLastError();
}

cudaError_t launch_transpose_grouped(const void* X, int C, const int32_t* offsets, const int32_t* col_off, int E,
                                     int ppad_max, void* XT, cudaStream_t s) {
  if (ppad_max == 0) return cudaSuccess;
  transpose_grouped_kernel<<<dim3(ppad_max / kTr, (C + kTr - 1) / kTr), 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(X), C, offsets, col_off, E, static_cast<__nv_bfloat16*>(XT), ppad_max);
  return cudaGetLastError();
}

cudaError_t launch_transpose_batched(const void* X, int E, int R, int C, void* XT, cudaStream_t s) {
  transpose_batched_kernel<<<dim3(R / kTr, C / kTr, E), 256, 0, s>>>(static_cast<const __nv_bfloat16*>(X), R, C,
                                                                     static_cast<__nv_bfloat16*>(XT));
  return cudaGetLastError();
}

}  // namespace moe
