// Router: scores s_t = h_t W_r^T + b, top-k with lowest-index ties, and gates
// renormalised over the picks ("How Does Mixture-of-Experts Routing Affect
// LLM Repeatability?", the simplified token-choice layer and its note on
// stable score ordering and deterministic tie handling).
//
// bf16 path: one CTA per 128 tokens computes the score tile (128 tokens x E
// padded) as a tcgen05 GEMM: TMA brings 128x64 slices of h and the matching
// slice of W_r into shared memory through an mbarrier ring, one thread issues
// the MMAs, the fp32 accumulator lives in TMEM. The epilogue reads TMEM with
// the 32x32b shape, so each thread owns one token row: bias, NaN handling,
// top-k and gates happen in registers (8 warps: two per TMEM lane quadrant,
// each taking every other 16-column chunk, their lists merged through shared
// memory). The kernel streams h once and is bound by HBM reads of h.
//
// From 49 experts on, a pair of CTAs (a cluster of two) shares each tile and
// splits the reduction: CTA r multiplies the r-th half of d for all experts,
// so each CTA streams half of the tile's h and W_r. Each CTA then hands the
// partner the partial scores of the experts the partner owns (through
// distributed shared memory), adds the partner's half to its own experts'
// scores, ranks its half of the experts, and rank 1 hands its top-k lists to
// rank 0, which merges them and writes the result.
#include <limits.h>
#include <math.h>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

constexpr int kRouterMaxStages = 8;
constexpr int kRouterBK = 64;
constexpr uint32_t kRouterABytes = kTileM * kRouterBK * 2;

// Top-K of one token under the order (score descending, expert ascending):
// an unsorted set of K entries plus its worst entry (lowest score, ties to
// the highest expert index). A candidate that does not beat the worst entry
// costs one comparison; one that does replaces it, and the new worst entry is
// found again. sort() puts the set in slot order at the end. Empty slots hold
// (-inf, INT_MAX), which any real candidate beats.
template <int K>
struct TopList {
  float v[K];
  int i[K];
  float wv;
  int wi;

  MOE_DEV void init() {
#pragma unroll
    for (int j = 0; j < K; ++j) {
      v[j] = -INFINITY;
      i[j] = INT_MAX;
    }
    wv = -INFINITY;
    wi = INT_MAX;
  }

  MOE_DEV void push(float x, int e) {
    if (!(x > wv || (x == wv && e < wi))) return;
    bool done = false;
#pragma unroll
    for (int j = 0; j < K; ++j) {
      const bool here = !done && v[j] == wv && i[j] == wi;
      v[j] = here ? x : v[j];
      i[j] = here ? e : i[j];
      done = done || here;
    }
    float nv = v[0];
    int ni = i[0];
#pragma unroll
    for (int j = 1; j < K; ++j) {
      const bool worse = v[j] < nv || (v[j] == nv && i[j] > ni);
      nv = worse ? v[j] : nv;
      ni = worse ? i[j] : ni;
    }
    wv = nv;
    wi = ni;
  }

  MOE_DEV void sort() {
#pragma unroll
    for (int x = 1; x < K; ++x)
#pragma unroll
      for (int y = x; y > 0; --y) {
        const bool sw = v[y] > v[y - 1] || (v[y] == v[y - 1] && i[y] < i[y - 1]);
        const float tv = v[y];
        const int ti = i[y];
        v[y] = sw ? v[y - 1] : v[y];
        i[y] = sw ? i[y - 1] : i[y];
        v[y - 1] = sw ? tv : v[y - 1];
        i[y - 1] = sw ? ti : i[y - 1];
      }
  }

  // Slot indices and gates (softmax over the picked scores); call after sort().
  MOE_DEV void write(int32_t* idx, float* gate) const {
    const float m = v[0];
    float w[K];
    float sum = 0.f;
#pragma unroll
    for (int j = 0; j < K; ++j) {
      w[j] = m > -INFINITY ? expf(v[j] - m) : 0.f;
      sum += w[j];
    }
#pragma unroll
    for (int j = 0; j < K; ++j) {
      idx[j] = i[j];
      gate[j] = sum > 0.f ? w[j] / sum : 0.f;
    }
  }
};

// Order-preserving 64-bit key of (score, expert) for the tensor-core path:
// a larger key ranks first, i.e. a higher score, then the lower expert index.
// The high word maps the fp32 score onto unsigned order (-0 ranks as +0, as
// it compares in fp32); the low word is the complemented expert index. Key 0
// is below every real key (-inf maps to 0x007fffff) and marks an empty slot.
MOE_DEV uint64_t rank_key(float x, int e) {
  uint32_t u = __float_as_uint(x);
  u = u == 0x80000000u ? 0u : u;
  u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
  return (static_cast<uint64_t>(u) << 32) | static_cast<uint32_t>(~static_cast<uint32_t>(e));
}
MOE_DEV float key_score(uint64_t k) {
  const uint32_t u = static_cast<uint32_t>(k >> 32);
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}
MOE_DEV int key_expert(uint64_t k) { return static_cast<int>(~static_cast<uint32_t>(k)); }

// Compare-exchange: the larger key to slot i, the smaller to slot l.
MOE_DEV void cx(uint64_t& i, uint64_t& l) {
  const uint64_t a = i, b = l;
  const bool s = a < b;
  i = s ? b : a;
  l = s ? a : b;
}

// Bitonic sort of N keys (N a power of two) into descending order. All loops
// unroll, so every index is a compile-time constant and the keys stay in
// registers; each layer is N/2 independent compare-exchanges.
template <int N>
MOE_DEV void sort_desc(uint64_t* v) {
#pragma unroll
  for (int k = 2; k <= N; k <<= 1)
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1)
#pragma unroll
      for (int i = 0; i < N; ++i) {
        const int l = i ^ j;
        if (l > i) {
          if ((i & k) == 0)
            cx(v[i], v[l]);
          else
            cx(v[l], v[i]);
        }
      }
}

// a, b sorted descending: a becomes the N largest keys of both, descending.
// max(a[i], b[N-1-i]) is a bitonic sequence holding the N largest keys; a
// half-cleaner network then sorts it.
template <int N>
MOE_DEV void merge_top(uint64_t* a, const uint64_t* b) {
#pragma unroll
  for (int i = 0; i < N; ++i) a[i] = a[i] > b[N - 1 - i] ? a[i] : b[N - 1 - i];
#pragma unroll
  for (int j = N >> 1; j > 0; j >>= 1)
#pragma unroll
    for (int i = 0; i < N; ++i) {
      const int l = i ^ j;
      if (l > i) cx(a[i], a[l]);
    }
}

struct RouterArgs {
  int T, d, E, npad, tmem_cols;
  int ncols;   // experts this CTA ranks: npad, or npad/2 when a CTA pair splits the reduction
  int stages;  // depth of the TMA ring (<= kRouterMaxStages)
  int split;   // 1: CTA pairs split the reduction over d (clusters of two)
  const float* bias;
  float* logits;
  int32_t* idx;
  float* gate;
  int32_t* chunk_counts;  // [n_tiles][E] expert histogram per 128-token tile, or NULL
  int n_tiles;
  int32_t* status;
};

// Candidate lists hold KP keys, K rounded up to a power of two (<= 8), so
// they merge with bitonic networks; the first K entries are the result.
template <int K>
__host__ __device__ constexpr int list_len() {
  return K <= 1 ? 1 : K <= 2 ? 2 : K <= 4 ? 4 : 8;
}

template <int K>
__global__ void __launch_bounds__(256, 1) router_tc_kernel(const __grid_constant__ CUtensorMap tm_h,
                                                           const __grid_constant__ CUtensorMap tm_w,
                                                           const RouterArgs a) {
  constexpr int KP = list_len<K>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_1024(smem_raw);
  const uint32_t b_bytes = static_cast<uint32_t>(a.npad) * kRouterBK * 2;
  const uint32_t stage_bytes = kRouterABytes + b_bytes;  // a multiple of 2048
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + a.stages * stage_bytes);
  uint64_t* empty = full + kRouterMaxStages;
  uint64_t* done = empty + kRouterMaxStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* consumed_slot = reinterpret_cast<int*>(tmem_slot + 2);
  float* sbias = reinterpret_cast<float*>(tmem_slot + 4);         // [kMaxE]
  // Per-token arrays are stored token-minor ([slot][128]) so a warp's 32
  // tokens touch consecutive words.
  uint64_t* pair_k = reinterpret_cast<uint64_t*>(sbias + kMaxE);   // [KP][128] keys handed over by rank 1
  int* pair_nan = reinterpret_cast<int*>(pair_k + kTileM * KP);     // [128]
  // [128][rs] partner's partial scores, 16-byte aligned; the row stride
  // rs = ncols + 4 puts the 8 rows of a quarter warp's 16-byte accesses in
  // distinct bank groups
  float* recv = reinterpret_cast<float*>(
      (reinterpret_cast<uintptr_t>(pair_nan + kTileM) + 15) & ~static_cast<uintptr_t>(15));
  const int rs = a.ncols + 4;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = a.split ? cluster_ctarank() : 0u;
  const int tile = a.split ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int col0 = static_cast<int>(rank) * a.ncols;  // first expert this CTA ranks
  const int nkb_all = a.d / kRouterBK;
  const int nkb = a.split ? nkb_all / 2 : nkb_all;     // k-blocks this CTA multiplies
  const int kb0 = static_cast<int>(rank) * nkb;

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
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
  pdl_wait();  // h, W_r, bias and the outputs may belong to the kernel before this one
  for (int j = threadIdx.x; j < a.ncols; j += blockDim.x) {
    const int e = col0 + j;
    sbias[j] = e >= a.E ? -INFINITY : (a.bias ? a.bias[e] : 0.f);
  }
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
      const int s = kb % a.stages;
      const uint32_t round = kb / a.stages;
      if (!mbar_wait(&empty[s], (round & 1) ^ 1, abort_flag)) {
        *abort_flag = 1;
        break;
      }
      uint8_t* st = smem + s * stage_bytes;
      mbar_expect_tx(&full[s], stage_bytes);
      tma_load_2d(st, &tm_h, &full[s], (kb0 + kb) * kRouterBK, tile * kTileM);
      tma_load_2d(st + kRouterABytes, &tm_w, &full[s], (kb0 + kb) * kRouterBK, 0);
      ++issued;
    }
  } else if (warp == 1 && lane == 0) {
    // MMA issuer: all npad expert columns over this CTA's k-blocks
    const uint32_t idesc = idesc_bf16_f32(kTileM, a.npad);
    int kb = 0;
    for (; kb < nkb; ++kb) {
      const int s = kb % a.stages;
      const uint32_t round = kb / a.stages;
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

  // Thread layout of the epilogue: warp w reads TMEM lane quadrant (w & 3),
  // i.e. token rows 32*(w&3) .. +31; the two warps of a quadrant take every
  // other 16-column chunk (starting at 16*(w>>2)).
  const int q = warp & 3, half = warp >> 2;
  const int row = q * 32 + lane;
  const int t = tile * kTileM + row;
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16);

  if (a.split) {
    // hand the partner the partial scores of the experts it ranks
    if (ok) {
      const int pcol0 = static_cast<int>(rank ^ 1u) * a.ncols;
      const uint32_t dst = mapa_shared(smem_addr(recv + row * rs), rank ^ 1u);
      for (int c0 = half * 16; c0 < a.ncols; c0 += 32) {
        uint32_t r[16];
        tmem_ld16(lane_base + pcol0 + c0, r);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; j += 4)
          st_shared_cluster_v4(dst + 4 * (c0 + j), r[j], r[j + 1], r[j + 2], r[j + 3]);
      }
    }
    cluster_sync();  // every thread of both CTAs, whatever happened above
  }

  // Each 16-column chunk: bitonic-sort groups of KP keys, merge the groups
  // down to the chunk's best KP, merge those into the running list.
  uint64_t top[KP];
#pragma unroll
  for (int j = 0; j < KP; ++j) top[j] = 0;
  bool nan = false;
  if (ok) {
    float* lrow = (a.logits != nullptr && t < a.T) ? a.logits + static_cast<size_t>(t) * a.E : nullptr;
    for (int c0 = half * 16; c0 < a.ncols; c0 += 32) {
      uint32_t r[16];
      tmem_ld16(lane_base + col0 + c0, r);
      float part[16];  // the partner's partial scores, read while the TMEM load is in flight
#pragma unroll
      for (int j = 0; j < 16; j += 4) {
        float4 p = make_float4(0.f, 0.f, 0.f, 0.f);
        if (a.split) p = *reinterpret_cast<const float4*>(recv + row * rs + c0 + j);
        part[j] = p.x;
        part[j + 1] = p.y;
        part[j + 2] = p.z;
        part[j + 3] = p.w;
      }
      tmem_ld_wait();
      uint64_t key[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int e = col0 + c0 + j;
        float x = __uint_as_float(r[j]) + part[j];
        x += sbias[c0 + j];  // padded experts carry -inf
        if (lrow != nullptr && e < a.E) lrow[e] = x;
        nan |= x != x;
        key[j] = rank_key(x != x ? -INFINITY : x, e);
      }
#pragma unroll
      for (int g = 0; g < 16; g += KP) sort_desc<KP>(key + g);
#pragma unroll
      for (int w = KP; w < 16; w <<= 1)
#pragma unroll
        for (int g = 0; g + w < 16; g += 2 * w) merge_top<KP>(key + g, key + g + w);
      merge_top<KP>(top, key);
    }
    uint64_t* xk = reinterpret_cast<uint64_t*>(smem);  // stage buffers are free once the MMAs are done
    int* xn = reinterpret_cast<int*>(smem + kTileM * KP * 8);
    if (half == 1) {
#pragma unroll
      for (int j = 0; j < KP; ++j) xk[j * kTileM + row] = top[j];
      xn[row] = nan;
    }
    __syncthreads();
    if (half == 0) {
      uint64_t other[KP];
#pragma unroll
      for (int j = 0; j < KP; ++j) other[j] = xk[j * kTileM + row];
      merge_top<KP>(top, other);
      nan |= xn[row] != 0;
      if (a.split && rank == 1) {
        const uint32_t dk = mapa_shared(smem_addr(pair_k + row), 0);
#pragma unroll
        for (int j = 0; j < KP; ++j) st_shared_cluster_u64(dk + 8 * j * kTileM, top[j]);
        st_shared_cluster_u32(mapa_shared(smem_addr(pair_nan + row), 0), nan ? 1u : 0u);
      }
    }
  } else if (threadIdx.x == 0) {
    report_status(a.status, MOE_STATUS_TIMEOUT);
  }
  if (a.split) cluster_sync();  // every thread of both CTAs, whatever happened above
  if (ok && rank == 0) {
    if (half == 0) {
      if (a.split) {
        uint64_t other[KP];
#pragma unroll
        for (int j = 0; j < KP; ++j) other[j] = pair_k[j * kTileM + row];
        merge_top<KP>(top, other);
        nan |= pair_nan[row] != 0;
      }
      if (t < a.T) {
        // gates: softmax over the K picked scores (slot 0 holds the largest)
        const float m = key_score(top[0]);
        float w[K];
        float sum = 0.f;
#pragma unroll
        for (int j = 0; j < K; ++j) {
          w[j] = m > -INFINITY ? expf(key_score(top[j]) - m) : 0.f;
          sum += w[j];
        }
        int32_t* it = a.idx + static_cast<size_t>(t) * K;
        float* gt = a.gate + static_cast<size_t>(t) * K;
#pragma unroll
        for (int j = 0; j < K; ++j) {
          it[j] = key_expert(top[j]);
          gt[j] = sum > 0.f ? w[j] / sum : 0.f;
        }
        if (nan) report_status(a.status, MOE_STATUS_NAN_LOGIT);
        if (a.chunk_counts != nullptr) {
#pragma unroll
          for (int j = 0; j < K; ++j) atomicAdd(&s_hist[key_expert(top[j])], 1);
        }
      }
    }
    if (a.chunk_counts != nullptr) {
      __syncthreads();
      for (int e = threadIdx.x; e < a.E; e += blockDim.x)
        a.chunk_counts[static_cast<size_t>(tile) * a.E + e] = s_hist[e];
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0 && lane == 0 && *abort_flag) {
    // loads issued but never consumed must land before the CTA leaves
    for (int kb = *consumed_slot; kb < issued; ++kb)
      mbar_wait(&full[kb % a.stages], (kb / a.stages) & 1, nullptr);
  }
  __syncthreads();
  if (warp == 0) tmem_dealloc(tmem, a.tmem_cols);
}

// fp32 path: one warp per token, lanes over experts, fp32 FMA in index order.
template <int K>
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
      TopList<K> top;
      top.init();
      bool nan = false;
      for (int e = 0; e < a.E; ++e) {
        float x = mine[e];
        if (x != x) {
          nan = true;
          x = -INFINITY;
        }
        top.push(x, e);
      }
      top.sort();
      top.write(a.idx + static_cast<size_t>(t) * K, a.gate + static_cast<size_t>(t) * K);
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

template <int K>
cudaError_t launch_router_tc_k(const CUtensorMap& tm_h, const CUtensorMap& tm_w, RouterArgs a, int tiles,
                               cudaStream_t s) {
  const size_t stage_bytes = kRouterABytes + static_cast<size_t>(a.npad) * kRouterBK * 2;
  const size_t fixed = 1024 + (2 * kRouterMaxStages + 1) * 8 + 16 + kMaxE * 4 + static_cast<size_t>(kTileM) * list_len<K>() * 8 +
                       kTileM * 4 + 16 + (a.split ? static_cast<size_t>(kTileM) * (a.ncols + 4) * 4 : 0);
  const size_t budget = 227 * 1024 - 1024 /* static histogram */ - fixed;
  int fit = static_cast<int>(budget / stage_bytes);
  fit = fit > kRouterMaxStages ? kRouterMaxStages : fit;
  // every CTA on its own SM: the deepest ring that fits; otherwise a ring
  // small enough for two CTAs per SM (at most 4 stages)
  const int ctas = (a.split ? 2 : 1) * tiles;
  if (ctas <= device_sm_count()) {
    a.stages = fit;
  } else {
    const size_t half_budget = 113 * 1024 - 1024 - fixed;
    const int two = static_cast<int>(half_budget / stage_bytes);
    a.stages = two >= 2 ? (two < 4 ? two : 4) : (fit < 4 ? fit : 4);
  }
  if (a.stages < 2) return cudaErrorInvalidConfiguration;
  const size_t smem = fixed + a.stages * stage_bytes;
  cudaError_t err = cudaFuncSetAttribute(router_tc_kernel<K>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  // Launched as a programmatic dependent of whatever kernel precedes it on the
  // stream: its barrier set-up overlaps that kernel's tail, and pdl_wait()
  // (griddepcontrol.wait: the previous grid has completed and its memory is
  // visible) comes before it reads h, W_r or the bias or writes anything.
  // Back-to-back moe_route calls: 55.5 -> 53.7 us (Mixtral 8x7B shape).
  err = launch_kernel(router_tc_kernel<K>, dim3((a.split ? 2 : 1) * tiles), dim3(256), smem, s, true,
                      a.split ? 2u : 1u, tm_h, tm_w, a);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_router_tc(const CUtensorMap& tm_h, const CUtensorMap& tm_w, int T, int d, int E, int k,
                             int npad, const float* bias, float* logits, int32_t* idx, float* gate,
                             int32_t* chunk_counts, int32_t* status, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  const int tiles = (T + kTileM - 1) / kTileM;
  const int split = router_splits_experts(npad) ? 1 : 0;
  RouterArgs a{};
  a.T = T;
  a.d = d;
  a.E = E;
  a.npad = npad;
  a.tmem_cols = static_cast<int>(pow2_at_least(npad, 32));
  a.ncols = split ? npad / 2 : npad;
  a.stages = 4;
  a.split = split;
  a.bias = bias;
  a.logits = logits;
  a.idx = idx;
  a.gate = gate;
  a.chunk_counts = chunk_counts;
  a.n_tiles = tiles;
  a.status = status;
  switch (k) {
#define MOE_ROUTER_K(KK) \
  case KK:               \
    return launch_router_tc_k<KK>(tm_h, tm_w, a, tiles, s);
    MOE_ROUTER_K(1)
    MOE_ROUTER_K(2)
    MOE_ROUTER_K(3)
    MOE_ROUTER_K(4)
    MOE_ROUTER_K(5)
    MOE_ROUTER_K(6)
    MOE_ROUTER_K(7)
    MOE_ROUTER_K(8)
#undef MOE_ROUTER_K
    default:
      return cudaErrorInvalidValue;
  }
}

cudaError_t launch_router_f32(const float* h, const float* w, int T, int d, int E, int k, const float* bias,
                              float* logits, int32_t* idx, float* gate, int32_t* status, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  RouterArgs a{};
  a.T = T;
  a.d = d;
  a.E = E;
  a.npad = E;
  a.ncols = E;
  a.bias = bias;
  a.logits = logits;
  a.idx = idx;
  a.gate = gate;
  a.status = status;
  const int grid = (T + 7) / 8 < 4096 ? (T + 7) / 8 : 4096;
  const size_t smem = 8 * static_cast<size_t>(E) * sizeof(float);
  switch (k) {
#define MOE_ROUTER_F32_K(KK)                                \
  case KK:                                                  \
    router_f32_kernel<KK><<<grid, 256, smem, s>>>(h, w, a); \
    break;
    MOE_ROUTER_F32_K(1)
    MOE_ROUTER_F32_K(2)
    MOE_ROUTER_F32_K(3)
    MOE_ROUTER_F32_K(4)
    MOE_ROUTER_F32_K(5)
    MOE_ROUTER_F32_K(6)
    MOE_ROUTER_F32_K(7)
    MOE_ROUTER_F32_K(8)
#undef MOE_ROUTER_F32_K
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace moe
