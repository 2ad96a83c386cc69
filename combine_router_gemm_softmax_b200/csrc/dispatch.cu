// Dispatch and return: per-expert counts and offsets from the routing map,
// the stable permutation that groups token rows by expert (with the optional
// capacity drop), and the weighted unpermute/combine.
// ("MoE Token Dispatch: Why an All-Reduce Result Does Not Describe the
// Exchange", "Follow one documented dispatch and return path"; capacity
// resolved in token order as in "How Does Mixture-of-Experts Routing Affect
// LLM Repeatability?"; archcrux "moe-unpermute-wrong-token" for the return.)
//
// Everything stays on the device, no host synchronisation:
//   count : per 128-token chunk, a histogram over experts (shared atomics;
//           only the totals are used, so their order does not matter). In
//           the whole-layer path the router's epilogue writes these counts.
//   scan  : per expert an exclusive scan over chunks (the stable base rank of
//           each chunk), then kept counts and offsets. Done inside every rank
//           CTA when the counts matrix is small, else by one separate CTA.
//   rank  : per chunk, every slot's rank among earlier tokens of the same
//           expert, from per-warp bitmasks (popc), giving dest_row/perm_src
//   copy  : TMA bulk copies: each token row is bulk-loaded into shared memory
//           once and bulk-stored to each kept destination row
//   pad   : padded layout only: rows past each expert's kept count are zeroed
// Nothing decides an order with atomics, so the permutation is deterministic.
// Kernels after the first of a call are launched as programmatic dependents
// and wait (griddepcontrol.wait) before touching earlier kernels' memory.
#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

// Raw expert indices of token t and a bitmask of its valid slots: in range
// and not repeating an earlier slot of the same token.
MOE_DEV uint32_t load_route(const int32_t* __restrict__ idx, int t, int k, int E, int (&ev)[kMaxK]) {
  uint32_t valid = 0;
#pragma unroll
  for (int j = 0; j < kMaxK; ++j) {
    ev[j] = -1;
    if (j < k) {
      const int v = idx[static_cast<size_t>(t) * k + j];
      bool ok = v >= 0 && v < E;
#pragma unroll
      for (int jj = 0; jj < j; ++jj) ok = ok && (ev[jj] != v);
      ev[j] = v;
      if (ok) valid |= 1u << j;
    }
  }
  return valid;
}

__global__ void __launch_bounds__(kChunkTokens) count_kernel(const int32_t* __restrict__ idx, int T, int k, int E,
                                                             int n_chunks, int32_t* __restrict__ chunk_counts) {
  pdl_wait();
  __shared__ int hist[kMaxE];
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int t = blockIdx.x * kChunkTokens + threadIdx.x;
  if (t < T) {
    int ev[kMaxK];
    const uint32_t valid = load_route(idx, t, k, E, ev);
#pragma unroll
    for (int j = 0; j < kMaxK; ++j)
      if (valid & (1u << j)) atomicAdd(&hist[ev[j]], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x)
    chunk_counts[static_cast<size_t>(blockIdx.x) * E + e] = hist[e];
}

constexpr int kScanPerLane = 8;

__global__ void __launch_bounds__(1024) scan_kernel(const int32_t* __restrict__ chunk_counts,
                                                    int32_t* __restrict__ chunk_base, int n_chunks, int E, int cap,
                                                    int padded, int32_t* __restrict__ routed,
                                                    int32_t* __restrict__ kept, int32_t* __restrict__ offsets) {
  pdl_wait();
  __shared__ int s_kept[kMaxE];
  __shared__ int s_warp[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // one warp per expert column: exclusive scan over chunks (tables are [chunk][E])
  for (int e = warp; e < E; e += 32) {
    int carry = 0;
    for (int c0 = 0; c0 < n_chunks; c0 += 32 * kScanPerLane) {
      int vals[kScanPerLane];
      int sum = 0;
#pragma unroll
      for (int v = 0; v < kScanPerLane; ++v) {
        const int c = c0 + lane * kScanPerLane + v;
        vals[v] = c < n_chunks ? chunk_counts[static_cast<size_t>(c) * E + e] : 0;
        sum += vals[v];
      }
      int inc = sum;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, inc, off);
        if (lane >= off) inc += n;
      }
      int run = carry + inc - sum;
#pragma unroll
      for (int v = 0; v < kScanPerLane; ++v) {
        const int c = c0 + lane * kScanPerLane + v;
        if (c < n_chunks) chunk_base[static_cast<size_t>(c) * E + e] = run;
        run += vals[v];
      }
      carry += __shfl_sync(0xffffffffu, inc, 31);
    }
    if (lane == 0) {
      const int kk = cap < 0 ? carry : min(carry, cap);
      routed[e] = carry;
      kept[e] = kk;
      s_kept[e] = kk;
    }
  }
  __syncthreads();
  // offsets = exclusive scan of kept counts over experts (threads 0..255)
  if (threadIdx.x < kMaxE) {
    const int e = threadIdx.x;
    const int v = e < E ? s_kept[e] : 0;
    int inc = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, inc, off);
      if (lane >= off) inc += n;
    }
    if (lane == 31) s_warp[warp] = inc;
    __syncwarp();
    asm volatile("bar.sync 1, 256;" ::: "memory");
    int before = 0;
    for (int w = 0; w < warp; ++w) before += s_warp[w];
    if (e < E) offsets[e] = padded ? e * cap : before + inc - v;
    if (e == E - 1) offsets[E] = padded ? E * cap : before + inc;
  }
}

// Chunk-counts matrices up to this many entries are scanned inside every rank
// CTA (each CTA needs its chunk's base rank for every expert and the offsets);
// larger ones go through scan_kernel first.
constexpr int kFusedScanMax = 8192;

// Ranks of one 128-token chunk: rank(t,j) = tokens before t (in earlier
// chunks, then in earlier warps of this chunk, then in lower lanes) that
// picked the same expert. With kFusedScan the chunk bases and offsets are
// computed here from the per-chunk counts, and CTA 0 writes the counts and
// offsets; otherwise they come from scan_kernel.
template <bool kFusedScan>
__global__ void __launch_bounds__(kChunkTokens) rank_kernel(
    const int32_t* __restrict__ idx, int T, int k, int E, int cap, int padded, int n_chunks,
    const int32_t* __restrict__ chunk_table,  // counts [n_chunks][E] (fused) or bases [n_chunks][E]
    const int32_t* __restrict__ offsets_in, int32_t* __restrict__ routed_out, int32_t* __restrict__ kept_out,
    int32_t* __restrict__ offsets_out, int32_t* __restrict__ dest_row, int32_t* __restrict__ perm_src,
    int32_t* status, int32_t* __restrict__ pair_cnt, int pair_tiles, uint4* __restrict__ y_zero, int y_vpr) {
  constexpr int kWarps = kChunkTokens / 32;
  __shared__ uint32_t mask[kWarps][kMaxE];
  __shared__ int wbase[kWarps][kMaxE];
  __shared__ int s_base[kMaxE];
  __shared__ int s_kept[kMaxE];
  __shared__ int s_off[kMaxE + 1];
  __shared__ int s_warp[kWarps];
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x;
  for (int i = threadIdx.x; i < kWarps * kMaxE; i += blockDim.x) (&mask[0][0])[i] = 0u;
  // this thread's token's route, loaded first so that its latency overlaps
  // the count-table pass below
  const int t = chunk * kChunkTokens + threadIdx.x;
  int ev[kMaxK];
  uint32_t valid = 0;
  if (t < T) valid = load_route(idx, t, k, E, ev);

  if constexpr (kFusedScan) {
    // The whole counts matrix (at most kFusedScanMax entries, 32 KB) comes
    // into shared memory in one coalesced pass of 16-byte loads, all in
    // flight at once; then, per expert: tokens of earlier chunks (this
    // chunk's base rank) and the total, each expert's chunks split over
    // 128/E threads.
    __shared__ __align__(16) int s_tab[kFusedScanMax];
    __shared__ int p_before[kChunkTokens], p_tot[kChunkTokens];
    {
      const int n = n_chunks * E;
      const int n4 = n >> 2;
      const int4* src4 = reinterpret_cast<const int4*>(chunk_table);
      int4* dst4 = reinterpret_cast<int4*>(s_tab);
#pragma unroll 16
      for (int i = threadIdx.x; i < n4; i += blockDim.x) dst4[i] = src4[i];
      for (int i = 4 * n4 + threadIdx.x; i < n; i += blockDim.x) s_tab[i] = chunk_table[i];
      __syncthreads();
    }
    for (int e_base = 0; e_base < E; e_base += kChunkTokens) {
      const int ne = min(E - e_base, kChunkTokens);
      const int groups = kChunkTokens / ne;
      int before = 0, tot = 0;
      if (threadIdx.x < groups * ne) {
        const int e = e_base + threadIdx.x % ne, g = threadIdx.x / ne;
#pragma unroll 8
        for (int c = g; c < n_chunks; c += groups) {
          const int v = s_tab[c * E + e];
          tot += v;
          before += c < chunk ? v : 0;
        }
      }
      p_before[threadIdx.x] = before;
      p_tot[threadIdx.x] = tot;
      __syncthreads();
      if (threadIdx.x < ne) {
        int b = 0, tt = 0;
        for (int g = 0; g < groups; ++g) {
          b += p_before[g * ne + threadIdx.x];
          tt += p_tot[g * ne + threadIdx.x];
        }
        const int e = e_base + threadIdx.x;
        s_base[e] = b;
        s_kept[e] = cap < 0 ? tt : min(tt, cap);
        if (chunk == 0) {
          routed_out[e] = tt;
          kept_out[e] = s_kept[e];
        }
      }
      __syncthreads();
    }
    __syncthreads();
    // offsets: exclusive scan of kept counts, two experts per thread
    const int e0 = 2 * threadIdx.x;
    const int v0 = e0 < E ? s_kept[e0] : 0, v1 = e0 + 1 < E ? s_kept[e0 + 1] : 0;
    int inc = v0 + v1;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int nb = __shfl_up_sync(0xffffffffu, inc, off);
      if (lane >= off) inc += nb;
    }
    if (lane == 31) s_warp[warp] = inc;
    __syncthreads();
    int before = 0;
    for (int w = 0; w < warp; ++w) before += s_warp[w];
    const int excl = before + inc - v0 - v1;
    if (e0 < E) s_off[e0] = padded ? e0 * cap : excl;
    if (e0 + 1 < E) s_off[e0 + 1] = padded ? (e0 + 1) * cap : excl + v0;
    if (threadIdx.x == blockDim.x - 1) s_off[E] = padded ? E * cap : before + inc;
    __syncthreads();
    if (chunk == 0)
      for (int e = threadIdx.x; e <= E; e += blockDim.x) offsets_out[e] = s_off[e];
  } else {
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
      s_base[e] = chunk_table[static_cast<size_t>(chunk) * E + e];
      s_off[e] = offsets_in[e];
    }
  }
  __syncthreads();

  if (t < T) {
#pragma unroll
    for (int j = 0; j < kMaxK; ++j)
      if (valid & (1u << j)) atomicOr(&mask[warp][ev[j]], 1u << lane);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      wbase[w][e] = run;
      run += __popc(mask[w][e]);
    }
  }
  __syncthreads();
  if (t < T) {
    const uint32_t lt = lanemask_lt();
    int n_kept = 0;
#pragma unroll
    for (int j = 0; j < kMaxK; ++j) {
      if (j >= k) break;
      int dest = -1;
      if (valid & (1u << j)) {
        const int e = ev[j];
        const int r = s_base[e] + wbase[warp][e] + __popc(mask[warp][e] & lt);
        if (cap < 0 || r < cap) {
          dest = s_off[e] + r;
          perm_src[dest] = t;
          ++n_kept;
        }
      }
      dest_row[static_cast<size_t>(t) * k + j] = dest;
    }
    if (valid != ((1u << k) - 1u)) report_status(status, MOE_STATUS_BAD_ROUTE);
    // combine fused into the down projection: this call's per-token counters
    // start at zero, and a token with no kept slot gets its zero output row
    // here (no expert row will write it)
    if (pair_cnt != nullptr)
      for (int i = 0; i < pair_tiles; ++i) pair_cnt[static_cast<size_t>(t) * pair_tiles + i] = 0;
    if (y_zero != nullptr && n_kept == 0)
      for (int v = 0; v < y_vpr; ++v) y_zero[static_cast<size_t>(t) * y_vpr + v] = make_uint4(0, 0, 0, 0);
  }
}

// Padded layout: rows e*cap + i with i >= kept[e] are padding. One warp per
// row writes zeros (16-byte stores) and marks perm_src -1; kept rows are
// skipped (the row copy writes them).
__global__ void __launch_bounds__(256) pad_rows_kernel(const int32_t* __restrict__ kept, int E, int cap,
                                                       uint4* __restrict__ x_perm, int vpr,
                                                       int32_t* __restrict__ perm_src) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const long long rows = static_cast<long long>(E) * cap;
  const long long nw = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  for (long long r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += nw) {
    const int e = static_cast<int>(r / cap);
    const int i = static_cast<int>(r - static_cast<long long>(e) * cap);
    if (i < kept[e]) continue;
    uint4* row = x_perm + r * vpr;
    for (int v = lane; v < vpr; v += 32) row[v] = make_uint4(0, 0, 0, 0);
    if (lane == 0) perm_src[r] = -1;
  }
}

constexpr int kCopyBuffers = 8;     // shared-memory row buffers per CTA
constexpr int kCopyLead = 4;        // row loads kept in flight ahead of the stores
constexpr int kCopyPiece = 8192;    // bytes per bulk transfer
// Tokens per CTA: small blocks give many CTAs per SM and the most row loads in
// flight. With buffers reserved per block, 2 tokens (2 buffers for rows of up
// to 8 KiB, about 26 CTAs per SM) beat 4 in A/B runs on B200: many_small
// 65.6 -> 57.9 us, skewed 85.0 -> 82.2 us, Mixtral 8x7B unchanged.
constexpr int kCopyTokensPerCta = 2;
static_assert(kCopyTokensPerCta <= 32, "one lane stages the active-token list");

// Row copy with the TMA engine. Each CTA owns a contiguous block of tokens and
// stages their dest_row entries in shared memory; one thread then runs a
// pipeline: bulk-load a row (or a piece of it) into one of up to 8 buffers,
// and when it lands, bulk-store it to every kept destination row. Each row is
// read from HBM once; a few instructions move a whole row. A block reserves
// only the buffers its rows can use (2 tokens of one piece: 2 buffers), so
// many more blocks fit on an SM than with 8 (A/B on B200, 4 tokens and 4
// buffers against 8 buffers: the Mixtral 8x7B dispatch 152 -> 139 us, skewed
// with capacity 39.6 -> 33.8 us).
__global__ void __launch_bounds__(32) permute_copy_bulk_kernel(const uint8_t* __restrict__ h,
                                                               const int32_t* __restrict__ dest_row,
                                                               uint8_t* __restrict__ x_perm, int T, int k, int rb,
                                                               int tokens_per_cta, int32_t* status) {
  pdl_wait();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((128u - (smem_addr(smem_raw) & 127u)) & 127u);
  const int piece = rb < kCopyPiece ? rb : kCopyPiece;
  const int n_pieces = (rb + piece - 1) / piece;
  const int nbuf = min(kCopyBuffers, tokens_per_cta * n_pieces);
  uint8_t* buf = smem;                                                    // nbuf x piece
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + nbuf * piece);
  int* dests = reinterpret_cast<int*>(bars + kCopyBuffers);               // tokens_per_cta x k
  const int lane = threadIdx.x;
  const int t0 = blockIdx.x * tokens_per_cta;
  const int nt = min(tokens_per_cta, T - t0);
  if (nt <= 0) return;
  for (int i = lane; i < nt * k; i += 32) dests[i] = dest_row[static_cast<size_t>(t0) * k + i];
  if (lane == 0) {
    for (int b = 0; b < kCopyBuffers; ++b) mbar_init(&bars[b], 1);
    fence_mbar_init();
  }
  __syncwarp();
  if (lane != 0) return;

  // tokens of this block that keep at least one slot (a token whose slots
  // were all dropped is not read)
  int act[kCopyTokensPerCta];
  int n_act = 0;
  for (int tl = 0; tl < nt; ++tl) {
    bool any = false;
    for (int j = 0; j < k; ++j) any = any || dests[tl * k + j] >= 0;
    if (any) act[n_act++] = tl;
  }
  const int n = n_act * n_pieces;
  int issued = 0;
  auto issue = [&](int m) {
    const int b = m % kCopyBuffers;
    const int off = (m % n_pieces) * piece;
    const uint32_t bytes = static_cast<uint32_t>(min(piece, rb - off));
    mbar_expect_tx(&bars[b], bytes);
    bulk_load(buf + b * piece, h + static_cast<size_t>(t0 + act[m / n_pieces]) * rb + off, bytes, &bars[b]);
    ++issued;
  };
  for (int m = 0; m < kCopyLead && m < n; ++m) issue(m);
  int m = 0;
  for (; m < n; ++m) {
    const int b = m % kCopyBuffers;
    if (!mbar_wait(&bars[b], (m / kCopyBuffers) & 1, nullptr)) {
      report_status(status, MOE_STATUS_TIMEOUT);
      break;
    }
    const int tl = act[m / n_pieces];
    const int off = (m % n_pieces) * piece;
    const uint32_t bytes = static_cast<uint32_t>(min(piece, rb - off));
    for (int j = 0; j < k; ++j) {
      const int dest = dests[tl * k + j];
      if (dest >= 0) bulk_store(x_perm + static_cast<size_t>(dest) * rb + off, buf + b * piece, bytes);
    }
    bulk_commit();
    if (m + kCopyLead < n) {
      // buffer (m + lead) % 8 was last used by unit m + lead - 8, whose stores
      // were committed 8 - lead groups ago
      bulk_wait_read<kCopyBuffers - kCopyLead>();
      issue(m + kCopyLead);
    }
  }
  for (int r = m + 1; r < issued; ++r)  // only after a timeout: let issued loads land
    mbar_wait(&bars[r % kCopyBuffers], (r / kCopyBuffers) & 1, nullptr);
  bulk_wait_all();
}

// 16-byte vector <-> fp32 lanes for the two storage types.
template <int DT>
struct Vec;

template <>
struct Vec<MOE_DTYPE_BF16> {
  static constexpr int N = 8;
  MOE_DEV static void load(const uint4& q, float (&f)[8]) {
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 x = __bfloat1622float2(p[i]);
      f[2 * i] = x.x;
      f[2 * i + 1] = x.y;
    }
  }
  MOE_DEV static uint4 store(const float (&f)[8]) {
    uint4 q;
    q.x = pack_bf16x2(f[0], f[1]);
    q.y = pack_bf16x2(f[2], f[3]);
    q.z = pack_bf16x2(f[4], f[5]);
    q.w = pack_bf16x2(f[6], f[7]);
    return q;
  }
};

template <>
struct Vec<MOE_DTYPE_F32> {
  static constexpr int N = 4;
  MOE_DEV static void load(const uint4& q, float (&f)[4]) {
    f[0] = __uint_as_float(q.x);
    f[1] = __uint_as_float(q.y);
    f[2] = __uint_as_float(q.z);
    f[3] = __uint_as_float(q.w);
  }
  MOE_DEV static uint4 store(const float (&f)[4]) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]), __float_as_uint(f[3]));
  }
};

// 16-byte segments per row that a lane loads before using any, by the number
// of kept rows: 15-16 loads in flight up to four rows, 10-12 for five and
// six, one segment per row for seven and eight (interleaved A/B on B200:
// tokens that kept few rows gain most; at k = 6 two segments per row beat
// one by 9%, at k = 8 one beats two by 5%).
constexpr int combine_batch(int nk) {
  return nk == 1 ? 16 : nk == 2 ? 8 : nk == 3 ? 5 : nk == 4 ? 4 : nk <= 6 ? 2 : 1;
}
// Resident CTAs per SM the register budget is sized for: three (80 registers
// a thread) up to k = 6, four (64) for k = 7 and 8, where the loads in flight
// per lane are capped at 8 so that the budget holds without spills. Against
// two CTAs per SM, A/B runs on B200 gave 5-13% faster combines at k = 6 and 8,
// the same at k = 2.
template <int K>
constexpr int kCombineCtasPerSm = K >= 7 ? 4 : 3;
constexpr int combine_batch_k(int nk, int k) {
  return k >= 7 && combine_batch(nk) * nk > 8 ? (8 / nk > 0 ? 8 / nk : 1) : combine_batch(nk);
}

// y[t] from the token's NK kept rows (slot order), one warp: all NK rows of U
// 16-byte segments per lane are loaded before any is used.
template <int DT, int NK, int U, int K>
MOE_DEV void combine_rows(const uint4* __restrict__ y_perm, const int (&dst)[K], const float (&g)[K],
                          uint4* __restrict__ yrow, int vpr, int lane) {
  using V = Vec<DT>;
  for (int v0 = 0; v0 < vpr; v0 += 32 * U) {
    uint4 q[NK][U];
#pragma unroll
    for (int j = 0; j < NK; ++j)
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int v = v0 + u * 32 + lane;
        q[j][u] = v < vpr ? __ldg(y_perm + static_cast<size_t>(dst[j]) * vpr + v) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float acc[V::N];
#pragma unroll
      for (int i = 0; i < V::N; ++i) acc[i] = 0.f;
#pragma unroll
      for (int j = 0; j < NK; ++j) {
        float f[V::N];
        V::load(q[j][u], f);
#pragma unroll
        for (int i = 0; i < V::N; ++i) acc[i] = fmaf(g[j], f[i], acc[i]);
      }
      const int v = v0 + u * 32 + lane;
      if (v < vpr) yrow[v] = V::store(acc);
    }
  }
}

// One warp per token: y[t] = sum_j gate[t,j] * y_perm[dest_row[t,j]] in fp32,
// slots in order 0..k-1, dropped slots skipped. The kept slots are listed
// first (in slot order) and the loads are batched by their number, so a token
// that kept few of its k slots still has about 16 loads per lane in flight.
template <int DT, int K>
__global__ void __launch_bounds__(256, kCombineCtasPerSm<K>) combine_kernel(const uint4* __restrict__ y_perm,
                                                      const int32_t* __restrict__ dest_row,
                                                      const float* __restrict__ gate, uint4* __restrict__ y, int T,
                                                      int vpr) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int nw = gridDim.x * (blockDim.x >> 5);
  for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += nw) {
    const int my_dest = lane < K ? dest_row[static_cast<size_t>(t) * K + lane] : -1;
    const float my_gate = lane < K ? gate[static_cast<size_t>(t) * K + lane] : 0.f;
    const uint32_t kept = __ballot_sync(0xffffffffu, my_dest >= 0);
    // kept slots in slot order: the j-th set bit of `kept`
    int dst[K];
    float g[K];
    uint32_t rest = kept;
#pragma unroll
    for (int j = 0; j < K; ++j) {
      const int src = rest ? __ffs(rest) - 1 : 0;
      rest &= rest - 1;
      dst[j] = __shfl_sync(0xffffffffu, my_dest, src);
      g[j] = __shfl_sync(0xffffffffu, my_gate, src);
    }
    uint4* yrow = y + static_cast<size_t>(t) * vpr;
    switch (__popc(kept)) {
      case 0:
        for (int v = lane; v < vpr; v += 32) yrow[v] = make_uint4(0, 0, 0, 0);
        break;
#define MOE_COMBINE_NK(NKK)                                                              \
  case NKK:                                                                              \
    if constexpr (NKK <= K) combine_rows<DT, NKK, combine_batch_k(NKK, K), K>(y_perm, dst, g, yrow, vpr, lane); \
    break;
      MOE_COMBINE_NK(1)
      MOE_COMBINE_NK(2)
      MOE_COMBINE_NK(3)
      MOE_COMBINE_NK(4)
      MOE_COMBINE_NK(5)
      MOE_COMBINE_NK(6)
      MOE_COMBINE_NK(7)
      MOE_COMBINE_NK(8)
#undef MOE_COMBINE_NK
      default:
        break;
    }
  }
}

template <int DT>
cudaError_t launch_combine_k(const uint4* y_perm, const int32_t* dest_row, const float* gate, uint4* y, int T, int k,
                             int vpr, int grid, bool pdl, cudaStream_t s) {
  cudaError_t err = cudaSuccess;
  switch (k) {
#define MOE_COMBINE_K(KK)                                                                                       \
  case KK:                                                                                                     \
    err = launch_kernel(combine_kernel<DT, KK>, dim3(grid), dim3(256), 0, s, pdl, 1, y_perm, dest_row, gate, y, T, \
                        vpr);                                                                                  \
    break;
    MOE_COMBINE_K(1)
    MOE_COMBINE_K(2)
    MOE_COMBINE_K(3)
    MOE_COMBINE_K(4)
    MOE_COMBINE_K(5)
    MOE_COMBINE_K(6)
    MOE_COMBINE_K(7)
    MOE_COMBINE_K(8)
#undef MOE_COMBINE_K
    default:
      return cudaErrorInvalidValue;
  }
  return err != cudaSuccess ? err : cudaGetLastError();
}

int warp_grid(int T) {
  const int want = (T + 7) / 8;
  const int cap = device_sm_count() * 8;
  return want < cap ? (want > 0 ? want : 1) : cap;
}

}  // namespace

cudaError_t launch_permute(const void* h, size_t row_bytes, const int32_t* idx, int T, int k, int E, int cap,
                           bool padded, bool copy_rows, int32_t* chunk_counts, int32_t* chunk_base, int32_t* routed,
                           int32_t* kept,
                           int32_t* offsets, int32_t* dest_row, int32_t* perm_src, void* x_perm,
                           bool counts_ready, bool pdl, int32_t* status, cudaStream_t s, int32_t* pair_cnt,
                           int pair_tiles, void* y_zero) {
  const int y_vpr = static_cast<int>(row_bytes / 16);
  // the first kernel launches as the caller asks; the later ones always as
  // programmatic dependents of the one before
  bool first = pdl;
  auto next = [&]() {
    const bool p = first;
    first = true;
    return p;
  };
  cudaError_t err = cudaSuccess;
  const int n_chunks = (T + kChunkTokens - 1) / kChunkTokens;
  if (n_chunks > 0 && !counts_ready)
    err = launch_kernel(count_kernel, dim3(n_chunks), dim3(kChunkTokens), 0, s, next(), 1, idx, T, k, E, n_chunks,
                        chunk_counts);
  if (err != cudaSuccess) return err;
  const bool fused = n_chunks > 0 && static_cast<long long>(E) * n_chunks <= kFusedScanMax;
  if (fused) {
    err = launch_kernel(rank_kernel<true>, dim3(n_chunks), dim3(kChunkTokens), 0, s, next(), 1, idx, T, k, E, cap,
                        static_cast<int>(padded), n_chunks, static_cast<const int32_t*>(chunk_counts), static_cast<const int32_t*>(nullptr),
                        routed, kept, offsets, dest_row, perm_src, status, pair_cnt, pair_tiles,
                        static_cast<uint4*>(y_zero), y_vpr);
  } else {
    err = launch_kernel(scan_kernel, dim3(1), dim3(1024), 0, s, next(), 1, static_cast<const int32_t*>(chunk_counts),
                        chunk_base, n_chunks, E, cap, static_cast<int>(padded), routed, kept, offsets);
    if (err == cudaSuccess && n_chunks > 0)
      err = launch_kernel(rank_kernel<false>, dim3(n_chunks), dim3(kChunkTokens), 0, s, next(), 1, idx, T, k, E, cap,
                          static_cast<int>(padded), n_chunks, static_cast<const int32_t*>(chunk_base), static_cast<const int32_t*>(offsets),
                          static_cast<int32_t*>(nullptr), static_cast<int32_t*>(nullptr),
                          static_cast<int32_t*>(nullptr), dest_row, perm_src, status, pair_cnt, pair_tiles,
                          static_cast<uint4*>(y_zero), y_vpr);
  }
  if (err != cudaSuccess) return err;
  if (n_chunks > 0 && copy_rows) {
    const int tpc = kCopyTokensPerCta;
    const int piece = static_cast<int>(row_bytes < kCopyPiece ? row_bytes : kCopyPiece);
    const int n_pieces = static_cast<int>((row_bytes + piece - 1) / piece);
    const int nbuf = tpc * n_pieces < kCopyBuffers ? tpc * n_pieces : kCopyBuffers;
    const size_t smem = 128 + static_cast<size_t>(nbuf) * piece + kCopyBuffers * 8 + tpc * k * 4;
    err = cudaFuncSetAttribute(permute_copy_bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    err = launch_kernel(permute_copy_bulk_kernel, dim3((T + tpc - 1) / tpc), dim3(32), smem, s, next(), 1,
                        static_cast<const uint8_t*>(h), static_cast<const int32_t*>(dest_row),
                        static_cast<uint8_t*>(x_perm), T, k, static_cast<int>(row_bytes), tpc, status);
    if (err != cudaSuccess) return err;
  }
  if (padded && cap > 0) {
    const long long rows = static_cast<long long>(E) * cap;
    const long long want = (rows + 7) / 8;
    const int grid = static_cast<int>(want < device_sm_count() * 8LL ? want : device_sm_count() * 8LL);
    err = launch_kernel(pad_rows_kernel, dim3(grid), dim3(256), 0, s, next(), 1, static_cast<const int32_t*>(kept), E,
                        cap, static_cast<uint4*>(x_perm), static_cast<int>(row_bytes / 16), perm_src);
    if (err != cudaSuccess) return err;
  }
  return cudaGetLastError();
}

cudaError_t launch_combine(int dtype, const void* y_perm, const int32_t* dest_row, const float* gate, void* y,
                           int T, int k, int d, bool pdl, cudaStream_t s, int32_t* status) {
  (void)status;  // the combine has no wait that could time out
  if (T == 0) return cudaSuccess;
  const int elem = dtype == MOE_DTYPE_BF16 ? 2 : 4;
  const int vpr = d * elem / 16;
  if (dtype == MOE_DTYPE_BF16)
    return launch_combine_k<MOE_DTYPE_BF16>(static_cast<const uint4*>(y_perm), dest_row, gate,
                                            static_cast<uint4*>(y), T, k, vpr, warp_grid(T), pdl, s);
  return launch_combine_k<MOE_DTYPE_F32>(static_cast<const uint4*>(y_perm), dest_row, gate, static_cast<uint4*>(y),
                                         T, k, vpr, warp_grid(T), pdl, s);
}

}  // namespace moe
