// Router: scores s_t = h_t W_r^T + b, top-k with lowest-index ties, and gates
// renormalised over the picks ("How Does Mixture-of-Experts Routing Affect
// LLM Repeatability?", the simplified token-choice layer and its note on
// stable score ordering and deterministic tie handling).
//
// bf16 path: one CTA per 128 tokens. The score tile (128 tokens x E padded to
// a multiple of 16) is a tcgen05 GEMM: TMA brings 128x64 slices of h and the
// whole router weight slice into shared memory through a 4-stage mbarrier
// pipeline, one thread issues the MMAs, the fp32 accumulator lives in TMEM.
// The epilogue reads TMEM with the 32x32b shape, so each thread owns one
// token's full score row and does bias, NaN handling, top-k and gates in
// registers. The kernel streams h once: it is bound by HBM reads of h.
#include <math.h>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

constexpr int kRouterStages = 4;
constexpr int kRouterBK = 64;
constexpr uint32_t kRouterABytes = kTileM * kRouterBK * 2;

// Running top-k of one token, sorted by (score descending, expert ascending).
// Empty slots hold NaN, which compares false against everything, so they are
// never ranked ahead of a candidate. An insertion counts the held entries
// that stay ahead of the candidate (independent compares) and shifts the
// tail down by one: no loop-carried chain through the k slots.
struct TopList {
  float v[kMaxK];
  int i[kMaxK];

  MOE_DEV void init() {
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      v[j] = __int_as_float(0x7fffffff);
      i[j] = -1;
    }
  }

  MOE_DEV void insert_at(int p, float x, int e) {
#pragma unroll
    for (int j = kMaxK - 1; j >= 0; --j) {
      const float pv = j > 0 ? v[j - 1] : x;
      const int pi = j > 0 ? i[j - 1] : e;
      const bool move = j > p, put = j == p;
      v[j] = move ? pv : (put ? x : v[j]);
      i[j] = move ? pi : (put ? e : i[j]);
    }
  }

  // Candidates of one list arrive in ascending expert index, so a held entry
  // with an equal score stays ahead (lower index wins).
  MOE_DEV void push_ascending(float x, int e, int k) {
    int p = 0;
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) p += (j < k && v[j] >= x) ? 1 : 0;
    insert_at(p, x, e);
  }

  // Candidate in any index order (merging another list); e < 0 is an empty slot.
  MOE_DEV void push_any(float x, int e, int k) {
    int p = 0;
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) p += (j < k && (v[j] > x || (v[j] == x && i[j] < e))) ? 1 : 0;
    insert_at(e < 0 ? k : p, x, e);
  }

  // Writes slot indices and gates: softmax over the picked scores.
  MOE_DEV void write(int32_t* idx, float* gate, int k) const {
    const float m = v[0];
    float w[kMaxK];
    float sum = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      w[j] = 0.f;
      if (j < k && m > -INFINITY) w[j] = expf(v[j] - m);
      sum += w[j];
    }
#pragma unroll
    for (int j = 0; j < kMaxK; ++j)
      if (j < k) {
        idx[j] = i[j];
        gate[j] = sum > 0.f ? w[j] / sum : 0.f;
      }
  }
};

struct RouterArgs {
  int T, d, E, k, npad, tmem_cols;
  const float* bias;
  float* logits;
  int32_t* idx;
  float* gate;
  int32_t* chunk_counts;  // [n_tiles][E] expert histogram per 128-token tile, or NULL
  int n_tiles;
  int32_t* status;
};

__global__ void __launch_bounds__(256, 2) router_tc_kernel(const __grid_constant__ CUtensorMap tm_h,
                                                        const __grid_constant__ CUtensorMap tm_w,
                                                        const RouterArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_1024(smem_raw);
  const uint32_t b_bytes = static_cast<uint32_t>(a.npad) * kRouterBK * 2;
  const uint32_t stage_bytes = kRouterABytes + b_bytes;  // a multiple of 2048
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kRouterStages * stage_bytes);
  uint64_t* empty = full + kRouterStages;
  uint64_t* done = empty + kRouterStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* consumed_slot = reinterpret_cast<int*>(tmem_slot + 2);
  float* sbias = reinterpret_cast<float*>(tmem_slot + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nkb = a.d / kRouterBK;
  const int tile = blockIdx.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRouterStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    *consumed_slot = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_h);
    tma_prefetch_desc(&tm_w);
  }
  __shared__ int s_hist[kMaxE];
  for (int e = threadIdx.x; e < a.npad; e += blockDim.x)
    sbias[e] = e >= a.E ? -INFINITY : (a.bias ? a.bias[e] : 0.f);
  for (int e = threadIdx.x; e < a.E; e += blockDim.x) s_hist[e] = 0;
  if (warp == 0) {
    tmem_alloc(tmem_slot, a.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  int issued = 0;
  if (warp == 0 && lane == 0) {
    // TMA producer
    for (int kb = 0; kb < nkb; ++kb) {
      const int s = kb % kRouterStages;
      const uint32_t round = kb / kRouterStages;
      if (!mbar_wait(&empty[s], (round & 1) ^ 1, abort_flag)) {
        *abort_flag = 1;
        break;
      }
      uint8_t* st = smem + s * stage_bytes;
      mbar_expect_tx(&full[s], stage_bytes);
      tma_load_2d(st, &tm_h, &full[s], kb * kRouterBK, tile * kTileM);
      tma_load_2d(st + kRouterABytes, &tm_w, &full[s], kb * kRouterBK, 0);
      ++issued;
    }
  } else if (warp == 1 && lane == 0) {
    // MMA issuer
    const uint32_t idesc = idesc_bf16_f32(kTileM, a.npad);
    int kb = 0;
    for (; kb < nkb; ++kb) {
      const int s = kb % kRouterStages;
      const uint32_t round = kb / kRouterStages;
      if (!mbar_wait(&full[s], round & 1, abort_flag)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t sa = smem_addr(smem + s * stage_bytes);
      const uint32_t sb = sa + kRouterABytes;
#pragma unroll
      for (int kk = 0; kk < kRouterBK / 16; ++kk)
        umma_bf16(tmem, sw128_kmajor_desc(sa + kk * 32), sw128_kmajor_desc(sb + kk * 32), idesc,
                  (kb | kk) != 0);
      umma_commit(&empty[s]);
    }
    *consumed_slot = kb;
    umma_commit(done);  // also drains everything issued so far
  }
  __syncwarp();

  bool ok = mbar_wait(done, 0, nullptr);
  tc_fence_after();
  ok = __syncthreads_and(ok && !*abort_flag);  // the same decision in every thread

  if (ok) {
    // 8 warps: warp w reads TMEM lane quadrant (w & 3), i.e. token rows
    // 32*(w&3) .. +31, and every other 16-column chunk starting at 16*(w>>2).
    // The two partial lists of a row are merged through shared memory.
    const int q = warp & 3, half = warp >> 2;
    const int row = q * 32 + lane;
    const int t = tile * kTileM + row;
    TopList top;
    top.init();
    bool nan = false;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16);
    float* lrow = (a.logits != nullptr && t < a.T) ? a.logits + static_cast<size_t>(t) * a.E : nullptr;
    for (int c0 = half * 16; c0 < a.npad; c0 += 32) {
      uint32_t r[16];
      tmem_ld16(lane_base + c0, r);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        float x = __uint_as_float(r[j]) + sbias[c0 + j];  // padded experts carry -inf
        if (lrow != nullptr && c0 + j < a.E) lrow[c0 + j] = x;
        nan |= x != x;
        x = x != x ? -INFINITY : x;
        top.push_ascending(x, c0 + j, a.k);
      }
    }
    float* xv = reinterpret_cast<float*>(smem);  // stage buffers are free once the MMAs are done
    int* xi = reinterpret_cast<int*>(smem + kTileM * kMaxK * 4);
    int* xn = reinterpret_cast<int*>(smem + 2 * kTileM * kMaxK * 4);
    if (half == 1) {
#pragma unroll
      for (int j = 0; j < kMaxK; ++j) {
        xv[row * kMaxK + j] = top.v[j];
        xi[row * kMaxK + j] = top.i[j];
      }
      xn[row] = nan;
    }
    __syncthreads();
    if (half == 0) {
#pragma unroll
      for (int j = 0; j < kMaxK; ++j)
        if (j < a.k) top.push_any(xv[row * kMaxK + j], xi[row * kMaxK + j], a.k);
      nan |= xn[row] != 0;
      if (t < a.T) {
        top.write(a.idx + static_cast<size_t>(t) * a.k, a.gate + static_cast<size_t>(t) * a.k, a.k);
        if (nan) report_status(a.status, MOE_STATUS_NAN_LOGIT);
        if (a.chunk_counts != nullptr) {
#pragma unroll
          for (int j = 0; j < kMaxK; ++j)
            if (j < a.k) atomicAdd(&s_hist[top.i[j]], 1);
        }
      }
    }
    if (a.chunk_counts != nullptr) {
      __syncthreads();
      for (int e = threadIdx.x; e < a.E; e += blockDim.x)
        a.chunk_counts[static_cast<size_t>(tile) * a.E + e] = s_hist[e];
    }
  } else if (threadIdx.x == 0) {
    report_status(a.status, MOE_STATUS_TIMEOUT);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0 && lane == 0 && *abort_flag) {
    // loads issued but never consumed must land before the CTA leaves
    for (int kb = *consumed_slot; kb < issued; ++kb)
      mbar_wait(&full[kb % kRouterStages], (kb / kRouterStages) & 1, nullptr);
  }
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, a.tmem_cols);
}

// fp32 path: one warp per token, lanes over experts, fp32 FMA in index order.
__global__ void __launch_bounds__(256) router_f32_kernel(const float* __restrict__ h, const float* __restrict__ w,
                                                         const RouterArgs a) {
  extern __shared__ float slog[];  // [8 warps][E]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* mine = slog + warp * a.E;
  for (int t = blockIdx.x * 8 + warp; t < a.T; t += gridDim.x * 8) {
    const float* ht = h + static_cast<size_t>(t) * a.d;
    for (int e = lane; e < a.E; e += 32) {
      const float* we = w + static_cast<size_t>(e) * a.d;
      float acc = 0.f;
      for (int c = 0; c < a.d; ++c) acc = fmaf(ht[c], we[c], acc);
      acc += a.bias ? a.bias[e] : 0.f;
      mine[e] = acc;
      if (a.logits) a.logits[static_cast<size_t>(t) * a.E + e] = acc;
    }
    __syncwarp();
    if (lane == 0) {
      TopList top;
      top.init();
      bool nan = false;
      for (int e = 0; e < a.E; ++e) {
        float x = mine[e];
        if (x != x) {
          nan = true;
          x = -INFINITY;
        }
        top.push_ascending(x, e, a.k);
      }
      top.write(a.idx + static_cast<size_t>(t) * a.k, a.gate + static_cast<size_t>(t) * a.k, a.k);
      if (nan) report_status(a.status, MOE_STATUS_NAN_LOGIT);
    }
    __syncwarp();
  }
}

uint32_t pow2_at_least(uint32_t x, uint32_t lo) {
  uint32_t p = lo;
  while (p < x) p <<= 1;
  return p;
}

}  // namespace

cudaError_t launch_router_tc(const CUtensorMap& tm_h, const CUtensorMap& tm_w, int T, int d, int E, int k,
                             int npad, const float* bias, float* logits, int32_t* idx, float* gate,
                             int32_t* chunk_counts, int32_t* status, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int grid = (T + kTileM - 1) / kTileM;
  RouterArgs a{T,    d,      E,   k,    npad,         static_cast<int>(pow2_at_least(npad, 32)),
               bias, logits, idx, gate, chunk_counts, grid,
               status};
  const size_t stage_bytes = kRouterABytes + static_cast<size_t>(npad) * kRouterBK * 2;
  const size_t smem = 1024 + kRouterStages * stage_bytes + (2 * kRouterStages + 1) * 8 + 16 + kMaxE * 4;
  cudaError_t err = cudaFuncSetAttribute(router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  router_tc_kernel<<<grid, 256, smem, s>>>(tm_h, tm_w, a);
  return cudaGetLastError();
}

cudaError_t launch_router_f32(const float* h, const float* w, int T, int d, int E, int k, const float* bias,
                              float* logits, int32_t* idx, float* gate, int32_t* status, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  RouterArgs a{T, d, E, k, E, 0, bias, logits, idx, gate, nullptr, 0, status};
  const int grid = (T + 7) / 8 < 4096 ? (T + 7) / 8 : 4096;
  router_f32_kernel<<<grid, 256, 8 * E * sizeof(float), s>>>(h, w, a);
  return cudaGetLastError();
}

}  // namespace moe
