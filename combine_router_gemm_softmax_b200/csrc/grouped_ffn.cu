// Grouped expert FFN over variable-length groups ("Dropless MoE Is a Runtime
// Problem as Much as a Model Design": one computation over a collection of
// expert shapes instead of one GEMM per expert or padding to a capacity).
//
// bf16 path, two launches of one persistent tcgen05 kernel:
//   GEMM1  [rows_e x d] x [2F x d]^T per expert, SwiGLU in the epilogue:
//          h_mid = silu(x W_gate^T) * (x W_up^T), rounded to bf16
//   GEMM2  [rows_e x F] x [d x F]^T per expert -> y_perm (bf16)
// Tiles are 128 rows x 256 columns x 64-deep K slices. The tile list is built
// on the device from the expert offsets (no host synchronisation): every CTA
// reads offsets, counts ceil(rows_e / 128) row tiles per expert, and walks the
// (row tile, column tile) grid in bands of row tiles so that a wave of CTAs
// shares A and B tiles in L2. A band holds about 64 MB of A (8 to 32 row
// tiles: 32 for the Mixtral-sized gate/up GEMM with K = 4096, 16 for its down
// projection with K = 14336), so the band stays in L2 while the weights stream
// through it once. grid = number of SMs; CTA c takes tiles c, c + grid, ...
//
// Inside a CTA (320 threads): warp 0 issues TMA loads into a 4-stage ring of
// shared-memory buffers, warp 1 allocates TMEM and one of its threads issues
// tcgen05.mma into one of two 256-column fp32 accumulators, warps 2..9 (two
// per TMEM lane quadrant, each taking half of the columns) drain the other
// accumulator (tcgen05.ld, 32x32b: one thread per output row), so the
// epilogue of tile i overlaps the main loop of tile i+1. A warp whose 32 rows
// all belong to the expert writes each 32-column block into its own staging
// buffer in shared memory and stores it with one TMA store; the others store
// row by row. Rows past the end of an expert's group are computed on whatever
// the buffer holds there and never stored.
//
// CTA-pair variant (grouped_gemm_pair_kernel): 256 x 256 tiles on a cluster
// of two SMs with tcgen05.mma.cta_group::2, each CTA staging its own 128 A
// rows and half of B, so each SM stages a third fewer operand bytes per
// flop; same epilogue, same bits. The layer takes it for mid-sized experts
// (the rule is use_pair_tiles in api.cu).
//
// The same kernel, by template arguments, also serves the layer's backward:
// a plain bf16 store (the down projection and both dgrad GEMMs), the gate/up
// GEMM recomputed with the SwiGLU backward in its epilogue (it reads dh_mid
// and writes [dgate | dup]), and a reduction-grouped mode for the weight
// gradients, where each expert owns a fixed grid of output tiles and its token
// rows are the K range (operands transposed with 64-aligned per-expert
// columns), stored in fp32. In gather mode GEMM1's producer loads A rows
// straight from the token matrix through the permutation (tile::gather4).
#include <atomic>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

constexpr int kBM = kTileM;       // 128
constexpr int kBN = kGemmTileN;   // 256
constexpr int kBK = 64;
constexpr int kStages = 4;
// warp 0: TMA producer, warp 1: TMEM allocation and MMA issue, warps 2..9:
// epilogue, two warps per TMEM lane quadrant, each draining half of a
// tile's columns (the SwiGLU epilogue is as long as a short-K main loop)
constexpr int kGemmThreads = 320;
constexpr int kEpiWarps = 8;
constexpr int kPairThreads = 320;  // the same warp roles as the single-CTA kernel
constexpr uint32_t kABytes = kBM * kBK * 2;
constexpr uint32_t kBBytes = kBN * kBK * 2;
constexpr uint32_t kStageBytes = kABytes + kBBytes;
constexpr uint32_t kTmemCols = 2 * kBN;

// Epilogue store staging: one 32-row x 32-column bf16 block (2 KB) per
// epilogue warp, in the 64-byte-swizzled layout of the store tensor map's box.
constexpr uint32_t kStgBytes = 32 * 32 * 2;

constexpr size_t gemm_smem_bytes() {
  return 1024 + kStages * static_cast<size_t>(kStageBytes) + kEpiWarps * kStgBytes + (2 * kStages + 5) * 8 + 16 +
         2 * (kMaxE + 1) * 4 + kBM * 4;
}
static_assert(gemm_smem_bytes() <= 227 * 1024, "shared memory");

struct GemmArgs {
  const int32_t* offsets;
  int E;
  int K;             // reduction length, a multiple of 64
  int n_per_expert;  // rows of B per expert (2F for GEMM1, d for GEMM2)
  int n_tiles;       // column tiles per expert
  int out_cols;      // columns of D
  int ldd;           // row stride of D in elements
  __nv_bfloat16* D;
  int32_t* status;
  int band;          // row tiles per band of the tile walk
  // Gather mode (single-CTA kernel only): when set, A row r of the grouped
  // problem is row gather_rows[r] of the tensor behind tm_a (a box of one
  // row); rows at or past offsets[E] read row 0 and are never stored.
  const int32_t* gather_rows;
  // SwiGLU-backward epilogue: the gradient dL/dh_mid [rows, aux_ld] (bf16).
  const __nv_bfloat16* aux;
  int aux_ld;
  // Reduction-grouped mode (weight gradients): offsets are the 64-aligned
  // column offsets of each expert in the transposed operands, every expert
  // owns an m_tiles x n_tiles grid of output tiles, and D32 receives the fp32
  // result [E][m_tiles * 128][out_cols].
  float* D32;
  int m_tiles;
  // SwiGLU-backward epilogue, optional: also write [dgate | dup] transposed,
  // DT[column][col_off[e] + row within expert] (ldt columns per row), with
  // the rows up to col_off[e+1] past the expert's end written as zeros.
  __nv_bfloat16* DT;
  const int32_t* col_off;
  int ldt;
  // Combine fused into the down projection (k <= 2, kEpiStoreCombine): every
  // row is stored to D (y_perm) as usual; a token with one kept slot gets
  // y[t] = gate * row written at once; for a token with two kept slots the
  // epilogue that finishes the second of its rows in this column tile (a
  // counter per token and column tile decides which) reads both rows back
  // and writes y[t] in slot order, bit-identical to the separate combine.
  const int32_t* perm_src;
  const int32_t* dest_row;
  const float* gate;
  int32_t* pair_cnt;  // [T][n_tiles][2 column halves], zeroed by the rank kernel of the same call
  __nv_bfloat16* Y;
  int k;
  // Testing hook (moe_debug_stall_next_gemms): the MMA issuer first waits on a
  // barrier that nothing signals, so its bounded wait runs out and the
  // kernel takes its timeout path.
  int stall;
  // Gate/up pre-activations [rows, preact_ld] (bf16, w13's interleaved column
  // order): written by the SwiGLU epilogue when set (kept for the backward),
  // read by the kEpiDhSwiGLUBwd epilogue.
  __nv_bfloat16* preact;
  int preact_ld;
  // kEpiSwiGLU / kEpiStore: D is also described by the kernel's tm_d (bf16,
  // boxes of 32 rows x 32 columns, 64-byte swizzle). A warp whose 32 rows of
  // the tile all belong to the expert stores each 32-column block through its
  // staging buffer with one TMA store; other warps store row by row.
  int tma_store;
};

// Epilogues and tile groupings of grouped_gemm_kernel.
constexpr int kEpiStore = 0;       // D (bf16) = accumulator
constexpr int kEpiSwiGLU = 1;      // D (bf16) = silu(gate) * up, half-width
constexpr int kEpiSwiGLUBwd = 2;   // D (bf16) = [dgate | dup] from gate, up and aux = dL/dh_mid
constexpr int kEpiStoreF32 = 3;    // D32 (fp32) = accumulator
constexpr int kEpiStoreCombine = 4;  // D (bf16) = accumulator, and the combine into Y for k <= 2
// The dh_mid GEMM of the backward with the SwiGLU backward in its epilogue,
// from saved pre-activations: the accumulator is dL/dh_mid for 256 channels;
// D (bf16) = [dgate | dup] in w13's interleaved order, from the accumulator
// and the saved a, u (preact), and optionally the transposed copy DT.
constexpr int kEpiDhSwiGLUBwd = 5;
constexpr int kGroupRows = 0;      // groups of rows (experts' token rows), same K for all
constexpr int kGroupReduce = 1;    // groups along K (experts' token rows are the reduction)
constexpr int kReduceBand = 16;    // row tiles per band in the reduction-grouped tile walk

// tile -> (expert, row tile within the expert, column tile)
MOE_DEV void decode_tile(long long tile, int m_total, int n_tiles, int band_rows, const int* prefix, int E, int& e,
                         int& m, int& n) {
  const long long band_size = static_cast<long long>(band_rows) * n_tiles;
  const int band = static_cast<int>(tile / band_size);
  const int within = static_cast<int>(tile - band * band_size);
  const int m0 = band * band_rows;
  const int rows = min(band_rows, m_total - m0);
  n = within / rows;
  const int gm = m0 + within % rows;
  int lo = 0, hi = E;  // prefix[lo] <= gm < prefix[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] <= gm)
      lo = mid;
    else
      hi = mid;
  }
  e = lo;
  m = gm - prefix[lo];
}

// One warp's 32 rows x 32 bf16 columns (p: this lane's row) to D with a TMA
// store through the warp's staging buffer.
MOE_DEV void stage_store(uint8_t* stg, const uint32_t (&p)[16], int lane, const CUtensorMap* tm_d, int x, int y) {
  const uint4 v[4] = {make_uint4(p[0], p[1], p[2], p[3]), make_uint4(p[4], p[5], p[6], p[7]),
                      make_uint4(p[8], p[9], p[10], p[11]), make_uint4(p[12], p[13], p[14], p[15])};
  stage_store_rows<64>(stg, v, lane, tm_d, x, y);
}

template <int kEpi, int kMode>
__global__ void __launch_bounds__(kGemmThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                        const __grid_constant__ CUtensorMap tm_d, const GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages * kABytes;
  uint8_t* stg_all = smem + kStages * kStageBytes;  // kEpiWarps x kStgBytes, 1024-aligned
  uint64_t* full = reinterpret_cast<uint64_t*>(stg_all + kEpiWarps * kStgBytes);
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* consumed_slot = reinterpret_cast<int*>(tmem_slot + 2);
  int* s_off = reinterpret_cast<int*>(tmem_slot + 4);  // [E+1]
  int* prefix = s_off + (kMaxE + 1);                   // [E+1]
  int* s_rows = prefix + (kMaxE + 1);                  // [128] source rows of the A tile (gather mode)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = a.E;
  const int nkb = a.K / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], kEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    *consumed_slot = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
    if (a.tma_store) tma_prefetch_desc(&tm_d);
  }
  pdl_wait();  // offsets and the A rows come from the kernels before this one
  for (int e = threadIdx.x; e <= E; e += blockDim.x) s_off[e] = a.offsets[e];
  __syncthreads();
  if (warp == 0) {
    // row tiles per expert, exclusive prefix over experts (8 experts per lane)
    int loc[8];
    int sum = 0;
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      const int e = lane * 8 + v;
      loc[v] = e < E ? (s_off[e + 1] - s_off[e] + kBM - 1) / kBM : 0;
      sum += loc[v];
    }
    int inc = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int nb = __shfl_up_sync(0xffffffffu, inc, off);
      if (lane >= off) inc += nb;
    }
    int run = inc - sum;
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      const int e = lane * 8 + v;
      if (e < E) prefix[e] = run;
      run += loc[v];
    }
    if (lane == 31) prefix[E] = inc;
  } else if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int m_total = kMode == kGroupRows ? prefix[E] : E * a.m_tiles;
  const long long total = static_cast<long long>(m_total) * a.n_tiles;
  // tile -> (expert, row tile, column tile) and its K-block range
  auto coords = [&](long long tile, int& e, int& m, int& n, int& kb0, int& kb1) {
    if constexpr (kMode == kGroupRows) {
      decode_tile(tile, m_total, a.n_tiles, a.band, prefix, E, e, m, n);
      kb0 = 0;
      kb1 = nkb;
    } else {
      // within an expert: bands of kReduceBand row tiles, each band sweeping
      // all column tiles, so a band's A rows stay in L2 while B streams
      const int per = a.m_tiles * a.n_tiles;
      e = static_cast<int>(tile / per);
      const int rem = static_cast<int>(tile - static_cast<long long>(e) * per);
      const int band = rem / (kReduceBand * a.n_tiles);
      const int m0 = band * kReduceBand;
      const int rows = min(kReduceBand, a.m_tiles - m0);
      const int within = rem - band * kReduceBand * a.n_tiles;
      m = m0 + within % rows;
      n = within / rows;
      kb0 = s_off[e] / kBK;
      kb1 = s_off[e + 1] / kBK;
    }
  };

  int issued = 0;
  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    // lane 0 issues the loads; in gather mode the whole warp first stages the
    // tile's 128 source rows in shared memory
    const bool gather = a.gather_rows != nullptr;
    const int kept_total = s_off[E];
    int stage = 0;
    uint32_t phase = 0;
    bool stop = false;
    for (long long tile = blockIdx.x; tile < total && !stop; tile += gridDim.x) {
      int e, m, n, kb0, kb1;
      coords(tile, e, m, n, kb0, kb1);
      const int a_row = kMode == kGroupRows ? s_off[e] + m * kBM : m * kBM;
      const int b_row = kMode == kGroupRows ? e * a.n_per_expert + n * kBN : n * kBN;
      if (gather) {
        __syncwarp();  // the previous tile's rows were read by lane 0's last issue
        for (int i = lane; i < kBM; i += 32) {
          const int r = a_row + i;
          s_rows[i] = r < kept_total ? a.gather_rows[r] : 0;
        }
        __syncwarp();
      }
      if (lane == 0) {
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) {
            *abort_flag = 1;
            stop = true;
            break;
          }
          mbar_expect_tx(&full[stage], kStageBytes);
          if (gather) {
            uint8_t* dst = sA + stage * kABytes;
#pragma unroll 4
            for (int i = 0; i < kBM; i += 4)
              tma_gather4(dst + i * (kBK * 2), &tm_a, &full[stage], kb * kBK, s_rows[i], s_rows[i + 1],
                          s_rows[i + 2], s_rows[i + 3]);
          } else {
            tma_load_2d(sA + stage * kABytes, &tm_a, &full[stage], kb * kBK, a_row);
          }
          tma_load_2d(sB + stage * kBBytes, &tm_b, &full[stage], kb * kBK, b_row);
          ++issued;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      stop = __shfl_sync(0xffffffffu, stop, 0);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      const uint32_t idesc = idesc_bf16_f32(kBM, kBN);
      int stage = 0;
      uint32_t phase = 0;
      int consumed = 0, local = 0;
      bool stop = false;
      if (a.stall && !mbar_wait(drain, 0, abort_flag)) {  // nothing arrives on `drain` before the end
        *abort_flag = 1;
        stop = true;
      }
      for (long long tile = blockIdx.x; tile < total && !stop; tile += gridDim.x, ++local) {
        const int acc = local & 1;
        const uint32_t acc_phase = (local >> 1) & 1;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1, abort_flag)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + acc * kBN;
        int te, tm, tn, kb0, kb1;
        coords(tile, te, tm, tn, kb0, kb1);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag)) {
            *abort_flag = 1;
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_addr(sA + stage * kABytes);
          const uint32_t sb = smem_addr(sB + stage * kBBytes);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            umma_bf16(d_tmem, sw128_kmajor_desc(sa + kk * 32), sw128_kmajor_desc(sb + kk * 32), idesc,
                      (kb != kb0) || (kk != 0));
          umma_commit(&empty[stage]);
          ++consumed;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!stop) umma_commit(&tfull[acc]);
      }
      *consumed_slot = consumed;
      umma_commit(drain);
      mbar_wait(drain, 0, nullptr);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;            // TMEM lane quadrant this warp may read
    const int half = (warp - 2) >> 2;  // which half of the tile's columns it drains
    const int row = q * 32 + lane;
    uint8_t* stg = stg_all + (warp - 2) * kStgBytes;
    int local = 0;
    for (long long tile = blockIdx.x; tile < total; tile += gridDim.x, ++local) {
      int e, m, n, kb0, kb1;
      coords(tile, e, m, n, kb0, kb1);
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      if (!mbar_wait(&tfull[acc], acc_phase, abort_flag)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem + acc * kBN + (static_cast<uint32_t>(q * 32) << 16);
      if constexpr (kMode == kGroupReduce) {
        // fp32 weight-gradient tile of expert e; an expert with no rows has no
        // K blocks, its accumulator was never written and the tile is zero
        float* out = a.D32 + (static_cast<size_t>(e) * a.m_tiles * kBM + m * kBM + row) * a.ldd + n * kBN;
        const bool empty_k = kb1 == kb0;
#pragma unroll 1
        for (int c = half * (kBN / 2); c < (half + 1) * (kBN / 2); c += 32) {
          if (n * kBN + c >= a.out_cols) break;
          uint32_t v[32];
          if (!empty_k) {
            tmem_ld32(tbase + c, v);
            tmem_ld_wait();
          }
          float4* dst = reinterpret_cast<float4*>(out + c);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = empty_k ? make_float4(0.f, 0.f, 0.f, 0.f)
                             : make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                           __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[acc]);
        continue;
      }
      const int rows_valid = min(kBM, s_off[e + 1] - s_off[e] - m * kBM);
      const bool valid = row < rows_valid;
      const size_t grow = static_cast<size_t>(s_off[e] + m * kBM + row);
      // this warp's 32 rows all belong to the expert: stage and TMA-store them
      const bool staged = a.tma_store != 0 && q * 32 + 32 <= rows_valid;
      const int srow = s_off[e] + m * kBM + q * 32;
      if constexpr (kEpi == kEpiSwiGLUBwd) {
        // columns [0,128) of the tile are the gate pre-activations a, [128,256)
        // the matching up pre-activations u, for channels n*128 + [0,128):
        // dgate = dh * u * silu'(a), dup = dh * silu(a)
        __nv_bfloat16* out = a.D + grow * a.ldd + n * kBN;
        const __nv_bfloat16* dh = a.aux + grow * a.aux_ld + n * (kBN / 2);
        // transposed copy: lanes are consecutive rows, so each 2-byte store of
        // a warp covers 32 consecutive columns of one DT row
        const int pcol = a.DT != nullptr ? a.col_off[e] + m * kBM + row : 0;
        const bool twrite = a.DT != nullptr && pcol < a.col_off[e + 1];
#pragma unroll 1
        for (int c = half * (kBN / 4); c < (half + 1) * (kBN / 4); c += 32) {
          uint32_t g[32], u[32];
          tmem_ld32(tbase + c, g);
          tmem_ld32(tbase + kBN / 2 + c, u);
          uint4 dq[4];
          if (valid) {
            const uint4* src = reinterpret_cast<const uint4*>(dh + c);
#pragma unroll
            for (int i = 0; i < 4; ++i) dq[i] = src[i];
          }
          tmem_ld_wait();
          uint32_t pg[16], pu[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) pg[i] = pu[i] = 0u;
          if (valid) {
            const __nv_bfloat16* dv = reinterpret_cast<const __nv_bfloat16*>(dq);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float dg2[2], du2[2];
#pragma unroll
              for (int h2 = 0; h2 < 2; ++h2) {
                const float av = __uint_as_float(g[2 * i + h2]);
                const float uv = __uint_as_float(u[2 * i + h2]);
                const float d0 = __bfloat162float(dv[2 * i + h2]);
                const float sg = 1.0f / (1.0f + expf(-av));
                dg2[h2] = d0 * uv * (sg * (1.0f + av * (1.0f - sg)));
                du2[h2] = d0 * av * sg;
              }
              pg[i] = pack_bf16x2(dg2[0], dg2[1]);
              pu[i] = pack_bf16x2(du2[0], du2[1]);
            }
            if (staged) {
              stage_store(stg, pg, lane, &tm_d, n * kBN + c, srow);
              stage_store(stg, pu, lane, &tm_d, n * kBN + kBN / 2 + c, srow);
            } else {
              uint4* dg_dst = reinterpret_cast<uint4*>(out + c);
              uint4* du_dst = reinterpret_cast<uint4*>(out + kBN / 2 + c);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                dg_dst[i] = make_uint4(pg[4 * i], pg[4 * i + 1], pg[4 * i + 2], pg[4 * i + 3]);
                du_dst[i] = make_uint4(pu[4 * i], pu[4 * i + 1], pu[4 * i + 2], pu[4 * i + 3]);
              }
            }
          }
          if (twrite) {
            uint16_t* tg = reinterpret_cast<uint16_t*>(a.DT) + static_cast<size_t>(n * kBN + c) * a.ldt + pcol;
            uint16_t* tu = tg + static_cast<size_t>(kBN / 2) * a.ldt;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              tg[static_cast<size_t>(2 * i) * a.ldt] = static_cast<uint16_t>(pg[i] & 0xffffu);
              tg[static_cast<size_t>(2 * i + 1) * a.ldt] = static_cast<uint16_t>(pg[i] >> 16);
              tu[static_cast<size_t>(2 * i) * a.ldt] = static_cast<uint16_t>(pu[i] & 0xffffu);
              tu[static_cast<size_t>(2 * i + 1) * a.ldt] = static_cast<uint16_t>(pu[i] >> 16);
            }
          }
        }
      } else if constexpr (kEpi == kEpiSwiGLU) {
        // columns [0,128) of the tile are gate, [128,256) the matching up
        __nv_bfloat16* out = a.D + grow * a.ldd + n * (kBN / 2);
#pragma unroll 1
        for (int c = half * (kBN / 4); c < (half + 1) * (kBN / 4); c += 32) {
          uint32_t g[32], u[32];
          tmem_ld32(tbase + c, g);
          tmem_ld32(tbase + kBN / 2 + c, u);
          tmem_ld_wait();
          if (valid) {
            uint32_t p[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float h0 = silu_fast(__uint_as_float(g[2 * i])) * __uint_as_float(u[2 * i]);
              const float h1 = silu_fast(__uint_as_float(g[2 * i + 1])) * __uint_as_float(u[2 * i + 1]);
              p[i] = pack_bf16x2(h0, h1);
            }
            if (staged) {
              stage_store(stg, p, lane, &tm_d, n * (kBN / 2) + c, srow);
            } else {
              uint4* dst = reinterpret_cast<uint4*>(out + c);
#pragma unroll
              for (int i = 0; i < 4; ++i) dst[i] = make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
            }
            if (a.preact != nullptr) {  // the pre-activations themselves, for the backward
              uint32_t pg[16], pu[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                pg[i] = pack_bf16x2(__uint_as_float(g[2 * i]), __uint_as_float(g[2 * i + 1]));
                pu[i] = pack_bf16x2(__uint_as_float(u[2 * i]), __uint_as_float(u[2 * i + 1]));
              }
              uint4* pgd = reinterpret_cast<uint4*>(a.preact + grow * a.preact_ld + n * kBN + c);
              uint4* pud = reinterpret_cast<uint4*>(a.preact + grow * a.preact_ld + n * kBN + kBN / 2 + c);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                pgd[i] = make_uint4(pg[4 * i], pg[4 * i + 1], pg[4 * i + 2], pg[4 * i + 3]);
                pud[i] = make_uint4(pu[4 * i], pu[4 * i + 1], pu[4 * i + 2], pu[4 * i + 3]);
              }
            }
          }
        }
      } else if constexpr (kEpi == kEpiDhSwiGLUBwd) {
        // this half of the tile's 256 channels is pack block b of w13: its
        // gate pre-activations at columns [256 b, 256 b + 128) of preact and
        // of the output, the up ones at [256 b + 128, 256 b + 256)
        const int b = 2 * n + half;
        const bool live = b * MOE_PACK_BLOCK < a.out_cols;
        const int pcol = a.DT != nullptr ? a.col_off[e] + m * kBM + row : 0;
        const bool twrite = live && a.DT != nullptr && pcol < a.col_off[e + 1];
        const __nv_bfloat16* pre = a.preact + grow * a.preact_ld + b * kBN;
        __nv_bfloat16* out = a.D + grow * a.ldd + b * kBN;
#pragma unroll 1
        for (int c = 0; c < kBN / 2 && live; c += 32) {
          uint32_t dh[32];
          tmem_ld32(tbase + half * (kBN / 2) + c, dh);
          uint4 ga[4], ua[4];
          if (valid) {
            const uint4* gsrc = reinterpret_cast<const uint4*>(pre + c);
            const uint4* usrc = reinterpret_cast<const uint4*>(pre + kBN / 2 + c);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              ga[i] = gsrc[i];
              ua[i] = usrc[i];
            }
          }
          tmem_ld_wait();
          uint32_t pg[16], pu[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) pg[i] = pu[i] = 0u;
          if (valid) {
            const __nv_bfloat16* av = reinterpret_cast<const __nv_bfloat16*>(ga);
            const __nv_bfloat16* uv = reinterpret_cast<const __nv_bfloat16*>(ua);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float dg2[2], du2[2];
#pragma unroll
              for (int h2 = 0; h2 < 2; ++h2) {
                const float av1 = __bfloat162float(av[2 * i + h2]);
                const float uv1 = __bfloat162float(uv[2 * i + h2]);
                const float d0 = __uint_as_float(dh[2 * i + h2]);
                const float sg = 1.0f / (1.0f + expf(-av1));
                dg2[h2] = d0 * uv1 * (sg * (1.0f + av1 * (1.0f - sg)));
                du2[h2] = d0 * av1 * sg;
              }
              pg[i] = pack_bf16x2(dg2[0], dg2[1]);
              pu[i] = pack_bf16x2(du2[0], du2[1]);
            }
            if (staged) {
              stage_store(stg, pg, lane, &tm_d, b * kBN + c, srow);
              stage_store(stg, pu, lane, &tm_d, b * kBN + kBN / 2 + c, srow);
            } else {
              uint4* dg_dst = reinterpret_cast<uint4*>(out + c);
              uint4* du_dst = reinterpret_cast<uint4*>(out + kBN / 2 + c);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                dg_dst[i] = make_uint4(pg[4 * i], pg[4 * i + 1], pg[4 * i + 2], pg[4 * i + 3]);
                du_dst[i] = make_uint4(pu[4 * i], pu[4 * i + 1], pu[4 * i + 2], pu[4 * i + 3]);
              }
            }
          }
          if (twrite) {
            uint16_t* tg = reinterpret_cast<uint16_t*>(a.DT) + static_cast<size_t>(b * kBN + c) * a.ldt + pcol;
            uint16_t* tu = tg + static_cast<size_t>(kBN / 2) * a.ldt;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              tg[static_cast<size_t>(2 * i) * a.ldt] = static_cast<uint16_t>(pg[i] & 0xffffu);
              tg[static_cast<size_t>(2 * i + 1) * a.ldt] = static_cast<uint16_t>(pg[i] >> 16);
              tu[static_cast<size_t>(2 * i) * a.ldt] = static_cast<uint16_t>(pu[i] & 0xffffu);
              tu[static_cast<size_t>(2 * i + 1) * a.ldt] = static_cast<uint16_t>(pu[i] >> 16);
            }
          }
        }
      } else if constexpr (kEpi == kEpiStoreCombine) {
        __nv_bfloat16* out = a.D + grow * a.ldd + n * kBN;
        // this row's token, its slot, its gate and the token's other kept row
        int t = -1, slot = 0, other = -1;
        float g_own = 0.f, g_other = 0.f;
        if (valid) {
          t = a.perm_src[grow];
          if (t >= 0) {
            slot = a.dest_row[static_cast<size_t>(t) * a.k] == static_cast<int>(grow) ? 0 : 1;
            g_own = a.gate[static_cast<size_t>(t) * a.k + slot];
            if (a.k == 2) {
              other = a.dest_row[static_cast<size_t>(t) * 2 + (1 - slot)];
              if (other >= 0) g_other = a.gate[static_cast<size_t>(t) * 2 + (1 - slot)];
            }
          }
        }
        __nv_bfloat16* yrow = a.Y + static_cast<size_t>(t < 0 ? 0 : t) * a.ldd + n * kBN;
#pragma unroll 1
        for (int c = half * (kBN / 2); c < (half + 1) * (kBN / 2); c += 32) {
          if (n * kBN + c >= a.out_cols) break;
          uint32_t v[32];
          tmem_ld32(tbase + c, v);
          tmem_ld_wait();
          if (valid) {
            uint32_t p[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) p[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
            uint4* dst = reinterpret_cast<uint4*>(out + c);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
            if (t >= 0 && other < 0) {
              // the token's only kept slot: y = gate * row (the row rounded to bf16 first)
              uint32_t yq[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&p[i]));
                yq[i] = pack_bf16x2(fmaf(g_own, f.x, 0.f), fmaf(g_own, f.y, 0.f));
              }
              uint4* ydst = reinterpret_cast<uint4*>(yrow + c);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                ydst[i] = make_uint4(yq[4 * i], yq[4 * i + 1], yq[4 * i + 2], yq[4 * i + 3]);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[acc]);
        if (t >= 0 && other >= 0) {
          // both rows of this column tile stored: the later of the two adds them
          __threadfence();
          const int prev = atomicAdd(a.pair_cnt + (static_cast<size_t>(t) * a.n_tiles + n) * 2 + half, 1);
          if (prev == 1) {
            __threadfence();
            const size_t r0 = slot == 0 ? grow : static_cast<size_t>(other);
            const size_t r1 = slot == 0 ? static_cast<size_t>(other) : grow;
            const float g0 = slot == 0 ? g_own : g_other, g1 = slot == 0 ? g_other : g_own;
            const int c0 = half * (kBN / 2);
            const uint4* s0 = reinterpret_cast<const uint4*>(a.D + r0 * a.ldd + n * kBN + c0);
            const uint4* s1 = reinterpret_cast<const uint4*>(a.D + r1 * a.ldd + n * kBN + c0);
            uint4* ydst = reinterpret_cast<uint4*>(yrow + c0);
            const int vcols = max(0, min(kBN / 2, a.out_cols - n * kBN - c0)) / 8;
#pragma unroll 4
            for (int v8 = 0; v8 < vcols; ++v8) {
              const uint4 q0 = __ldcg(s0 + v8), q1 = __ldcg(s1 + v8);
              const __nv_bfloat162* h0 = reinterpret_cast<const __nv_bfloat162*>(&q0);
              const __nv_bfloat162* h1 = reinterpret_cast<const __nv_bfloat162*>(&q1);
              uint32_t o[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float2 f0 = __bfloat1622float2(h0[i]), f1 = __bfloat1622float2(h1[i]);
                o[i] = pack_bf16x2(fmaf(g1, f1.x, fmaf(g0, f0.x, 0.f)), fmaf(g1, f1.y, fmaf(g0, f0.y, 0.f)));
              }
              ydst[v8] = make_uint4(o[0], o[1], o[2], o[3]);
            }
          }
        }
        continue;
      } else {
        __nv_bfloat16* out = a.D + grow * a.ldd + n * kBN;
#pragma unroll 1
        for (int c = half * (kBN / 2); c < (half + 1) * (kBN / 2); c += 32) {
          if (n * kBN + c >= a.out_cols) break;
          uint32_t v[32];
          tmem_ld32(tbase + c, v);
          tmem_ld_wait();
          if (valid) {
            uint32_t p[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) p[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
            if (staged) {
              stage_store(stg, p, lane, &tm_d, n * kBN + c, srow);
            } else {
              uint4* dst = reinterpret_cast<uint4*>(out + c);
#pragma unroll
              for (int i = 0; i < 4; ++i) dst[i] = make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
  }
  __syncwarp();
  if (warp >= 2 && lane == 0) bulk_wait_all();  // the epilogue's staged stores have completed

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (*abort_flag) {
    if (threadIdx.x == 0) report_status(a.status, MOE_STATUS_TIMEOUT);
    if (warp == 0 && lane == 0) {
      // loads issued but never consumed must land before the CTA leaves
      for (int i = *consumed_slot; i < issued; ++i) mbar_wait(&full[i % kStages], (i / kStages) & 1, nullptr);
    }
  }
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// ------------------------------------------------------------------ CTA-pair variant
// Same computation on 256 x 256 tiles shared by a pair of CTAs (a cluster of
// two SMs). Each CTA loads its own 128 rows of A and 128 rows of B per K
// slice into its own shared memory; the pair's leader issues one
// tcgen05.mma.cta_group::2 per 16-deep step, reading both CTAs' operands, and
// each CTA's TMEM receives its own 128 output rows x 256 columns. Per output
// element this halves the B bytes every SM stages and the tile bytes the L2
// serves, compared with the single-CTA 128 x 256 tile.
//   barriers: full[s] lives in the leader and counts both CTAs' bytes; each
//   CTA's empty[s] and tfull[a] are signalled by the leader's commit to both
//   CTAs; tempty[a] lives in the leader and takes one arrival per epilogue
//   warp of both CTAs (16).
// The epilogue is the single-CTA kernel's: eight warps, two per TMEM lane
// quadrant, storing whole 32-row blocks through shared memory with TMA stores.
constexpr int kPairStages = 6;
constexpr int kPairBM = 256;
constexpr uint32_t kPairHalfBytes = 128 * kBK * 2;                 // one CTA's A or B slice
constexpr uint32_t kPairPad = kEpiWarps * kStgBytes;               // store staging; keeps any operand over-read in bounds
static_assert(kPairPad >= 16384, "the region after the operand ring must stay at least 16 KB");

constexpr size_t pair_smem_bytes() {
  return 1024 + 2 * kPairStages * static_cast<size_t>(kPairHalfBytes) + kPairPad + (2 * kPairStages + 5) * 8 + 16 +
         2 * (kMaxE + 1) * 4;
}
static_assert(pair_smem_bytes() <= 227 * 1024, "shared memory");

template <bool kSwiGLU>
__global__ void __launch_bounds__(kPairThreads, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                             const __grid_constant__ CUtensorMap tm_d, const GemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_1024(smem_raw);
  uint8_t* sB = smem;                                           // kPairStages x 16 KB
  uint8_t* sA = smem + kPairStages * kPairHalfBytes;             // kPairStages x 16 KB
  uint8_t* stg_all = smem + 2 * kPairStages * kPairHalfBytes;    // kEpiWarps x kStgBytes, 1024-aligned
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + 2 * kPairStages * kPairHalfBytes + kPairPad);
  uint64_t* empty = full + kPairStages;
  uint64_t* tfull = empty + kPairStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* consumed_slot = reinterpret_cast<int*>(tmem_slot + 2);
  int* s_off = reinterpret_cast<int*>(tmem_slot + 4);
  int* prefix = s_off + (kMaxE + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int E = a.E;
  const int nkb = a.K / kBK;
  const uint32_t peer_abort = mapa_shared(smem_addr(const_cast<int*>(abort_flag)), rank ^ 1u);
  auto raise_abort = [&]() {
    *abort_flag = 1;
    st_shared_cluster_u32(peer_abort, 1u);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 2 * kEpiWarps);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    *consumed_slot = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
    if (a.tma_store) tma_prefetch_desc(&tm_d);
  }
  pdl_wait();  // offsets and the A rows come from the kernels before this one
  for (int e = threadIdx.x; e <= E; e += blockDim.x) s_off[e] = a.offsets[e];
  __syncthreads();
  if (warp == 0) {
    int loc[8];
    int sum = 0;
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      const int e = lane * 8 + v;
      loc[v] = e < E ? (s_off[e + 1] - s_off[e] + kPairBM - 1) / kPairBM : 0;
      sum += loc[v];
    }
    int inc = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int nb = __shfl_up_sync(0xffffffffu, inc, off);
      if (lane >= off) inc += nb;
    }
    int run = inc - sum;
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      const int e = lane * 8 + v;
      if (e < E) prefix[e] = run;
      run += loc[v];
    }
    if (lane == 31) prefix[E] = inc;
  } else if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers initialised before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int m_total = prefix[E];
  const long long total = static_cast<long long>(m_total) * a.n_tiles;
  const int pair_id = blockIdx.x >> 1, n_pairs = gridDim.x >> 1;

  int issued = 0;
  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------------- TMA producer (both CTAs)
      const uint32_t full_leader = mapa_shared(smem_addr(&full[0]), 0);
      int stage = 0;
      uint32_t phase = 0;
      bool stop = false;
      for (long long tile = pair_id; tile < total && !stop; tile += n_pairs) {
        int e, m, n;
        decode_tile(tile, m_total, a.n_tiles, a.band, prefix, E, e, m, n);
        const int a_row = s_off[e] + m * kPairBM + static_cast<int>(rank) * 128;
        const int b_row = e * a.n_per_expert + n * kBN + static_cast<int>(rank) * 128;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) {
            raise_abort();
            stop = true;
            break;
          }
          if (leader) mbar_expect_tx(&full[stage], 4 * kPairHalfBytes);
          tma_load_2d_pair(sA + stage * kPairHalfBytes, &tm_a, full_leader + stage * 8, kb * kBK, a_row);
          tma_load_2d_pair(sB + stage * kPairHalfBytes, &tm_b, full_leader + stage * 8, kb * kBK, b_row);
          ++issued;
          if (++stage == kPairStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------------------------------------------------------- MMA issuer (leader only)
      const uint32_t idesc = idesc_bf16_f32(kPairBM, kBN);
      int stage = 0;
      uint32_t phase = 0;
      int consumed = 0, local = 0;
      bool stop = false;
      if (a.stall && !mbar_wait(drain, 0, abort_flag)) {  // nothing arrives on `drain` before the end
        raise_abort();
        stop = true;
      }
      for (long long tile = pair_id; tile < total && !stop; tile += n_pairs, ++local) {
        const int acc = local & 1;
        const uint32_t acc_phase = (local >> 1) & 1;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1, abort_flag)) {
          raise_abort();
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + acc * kBN;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag)) {
            raise_abort();
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_addr(sA + stage * kPairHalfBytes);
          const uint32_t sb = smem_addr(sB + stage * kPairHalfBytes);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            umma_bf16_pair(d_tmem, sw128_kmajor_desc(sa + kk * 32), sw128_kmajor_desc(sb + kk * 32), idesc,
                           (kb | kk) != 0);
          umma_commit_pair_all(&empty[stage], 0x3);
          ++consumed;
          if (++stage == kPairStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!stop) umma_commit_pair_all(&tfull[acc], 0x3);
      }
      *consumed_slot = consumed;
      umma_commit_pair(drain);
      mbar_wait(drain, 0, nullptr);
    }
  } else {
    // ---------------------------------------------------------------- epilogue (both CTAs)
    const uint32_t tempty_leader = mapa_shared(smem_addr(&tempty[0]), 0);
    const int q = warp & 3;            // TMEM lane quadrant this warp may read
    const int half = (warp - 2) >> 2;  // which half of the tile's columns it drains
    const int row = q * 32 + lane;
    uint8_t* stg = stg_all + (warp - 2) * kStgBytes;
    int local = 0;
    for (long long tile = pair_id; tile < total; tile += n_pairs, ++local) {
      int e, m, n;
      decode_tile(tile, m_total, a.n_tiles, a.band, prefix, E, e, m, n);
      const int acc = local & 1;
      const uint32_t acc_phase = (local >> 1) & 1;
      if (!mbar_wait(&tfull[acc], acc_phase, abort_flag)) {
        raise_abort();
        break;
      }
      tc_fence_after();
      const int row0 = m * kPairBM + static_cast<int>(rank) * 128;  // first row of this CTA within the group
      const int rows_valid = min(128, s_off[e + 1] - s_off[e] - row0);
      const bool valid = row < rows_valid;
      const size_t grow = static_cast<size_t>(s_off[e] + row0 + row);
      const uint32_t tbase = tmem + acc * kBN + (static_cast<uint32_t>(q * 32) << 16);
      // this warp's 32 rows all belong to the expert: stage and TMA-store them
      const bool staged = a.tma_store != 0 && q * 32 + 32 <= rows_valid;
      const int srow = s_off[e] + row0 + q * 32;
      if constexpr (kSwiGLU) {
        // columns [0,128) of the tile are gate, [128,256) the matching up
        __nv_bfloat16* out = a.D + grow * a.ldd + n * (kBN / 2);
#pragma unroll 1
        for (int c = half * (kBN / 4); c < (half + 1) * (kBN / 4); c += 32) {
          uint32_t g[32], u[32];
          tmem_ld32(tbase + c, g);
          tmem_ld32(tbase + kBN / 2 + c, u);
          tmem_ld_wait();
          if (valid) {
            uint32_t p[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float h0 = silu_fast(__uint_as_float(g[2 * i])) * __uint_as_float(u[2 * i]);
              const float h1 = silu_fast(__uint_as_float(g[2 * i + 1])) * __uint_as_float(u[2 * i + 1]);
              p[i] = pack_bf16x2(h0, h1);
            }
            if (staged) {
              stage_store(stg, p, lane, &tm_d, n * (kBN / 2) + c, srow);
            } else {
              uint4* dst = reinterpret_cast<uint4*>(out + c);
#pragma unroll
              for (int i = 0; i < 4; ++i) dst[i] = make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
            }
          }
        }
      } else {
        __nv_bfloat16* out = a.D + grow * a.ldd + n * kBN;
#pragma unroll 1
        for (int c = half * (kBN / 2); c < (half + 1) * (kBN / 2); c += 32) {
          if (n * kBN + c >= a.out_cols) break;
          uint32_t v[32];
          tmem_ld32(tbase + c, v);
          tmem_ld_wait();
          if (valid) {
            uint32_t p[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) p[i] = pack_bf16x2(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
            if (staged) {
              stage_store(stg, p, lane, &tm_d, n * kBN + c, srow);
            } else {
              uint4* dst = reinterpret_cast<uint4*>(out + c);
#pragma unroll
              for (int i = 0; i < 4; ++i) dst[i] = make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader + acc * 8);
    }
  }
  __syncwarp();
  if (warp >= 2 && lane == 0) bulk_wait_all();  // the epilogue's staged stores have completed

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (*abort_flag) {
    if (threadIdx.x == 0) report_status(a.status, MOE_STATUS_TIMEOUT);
    if (warp == 0 && lane == 0 && leader) {
      for (int i = *consumed_slot; i < issued; ++i) mbar_wait(&full[i % kPairStages], (i / kPairStages) & 1, nullptr);
    }
  }
  cluster_sync();  // neither CTA leaves while the pair's MMAs or signals may still touch it
  if (warp == 1) tmem_dealloc_pair(tmem, kTmemCols);
}

// ------------------------------------------------------------------ helpers for the other paths
MOE_DEV int expert_of_row(const int32_t* __restrict__ off, int E, int r) {
  int lo = 0, hi = E;  // off[lo] <= r < off[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (off[mid] <= r)
      lo = mid;
    else
      hi = mid;
  }
  return lo;
}

// Packed row of gate row f (is_up = 0) or up row f (is_up = 1) inside one expert.
MOE_DEV int packed_row(int f, int F, int is_up) {
  const int b = f / MOE_PACK_BLOCK;
  const int w = f - b * MOE_PACK_BLOCK;
  const int pb = min(MOE_PACK_BLOCK, F - b * MOE_PACK_BLOCK);
  return 2 * b * MOE_PACK_BLOCK + (is_up ? pb : 0) + w;
}

// fp32 path, first projection: h_mid[r,f] = silu(x_r . Wg_f) * (x_r . Wu_f)
__global__ void ffn1_f32_kernel(const float* __restrict__ x, const int32_t* __restrict__ off,
                                const float* __restrict__ w13, float* __restrict__ h_mid, int rows_max, int d,
                                int F, int E) {
  const int n = off[E];
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
       i < static_cast<long long>(rows_max) * F; i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int r = static_cast<int>(i / F), f = static_cast<int>(i % F);
    if (r >= n) continue;
    const int e = expert_of_row(off, E, r);
    const float* xr = x + static_cast<size_t>(r) * d;
    const float* wg = w13 + (static_cast<size_t>(e) * 2 * F + packed_row(f, F, 0)) * d;
    const float* wu = w13 + (static_cast<size_t>(e) * 2 * F + packed_row(f, F, 1)) * d;
    float ag = 0.f, au = 0.f;
    for (int c = 0; c < d; ++c) {
      ag = fmaf(xr[c], wg[c], ag);
      au = fmaf(xr[c], wu[c], au);
    }
    h_mid[static_cast<size_t>(r) * F + f] = silu_f(ag) * au;
  }
}

// fp32 path, second projection: y[r,c] = h_mid_r . Wd_c
__global__ void ffn2_f32_kernel(const float* __restrict__ h_mid, const int32_t* __restrict__ off,
                                const float* __restrict__ wd, float* __restrict__ y, int rows_max, int d, int F,
                                int E) {
  const int n = off[E];
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
       i < static_cast<long long>(rows_max) * d; i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int r = static_cast<int>(i / d), c = static_cast<int>(i % d);
    if (r >= n) continue;
    const int e = expert_of_row(off, E, r);
    const float* hr = h_mid + static_cast<size_t>(r) * F;
    const float* wc = wd + (static_cast<size_t>(e) * d + c) * F;
    float acc = 0.f;
    for (int f = 0; f < F; ++f) acc = fmaf(hr[f], wc[f], acc);
    y[static_cast<size_t>(r) * d + c] = acc;
  }
}

// Identity (bit copy) and scale-by-(e+1) test experts, one warp per row.
template <int DT>
__global__ void __launch_bounds__(256) scale_rows_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ off,
                                                         uint4* __restrict__ y, int rows_max, int vpr, int E,
                                                         int scale) {
  const int lane = threadIdx.x & 31;
  const int n = min(off[E], rows_max);
  const int nw = gridDim.x * (blockDim.x >> 5);
  for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < n; r += nw) {
    const float s = scale ? static_cast<float>(expert_of_row(off, E, r) + 1) : 1.f;
    for (int v = lane; v < vpr; v += 32) {
      uint4 q = __ldg(x + static_cast<size_t>(r) * vpr + v);
      if (scale) {
        if (DT == MOE_DTYPE_BF16) {
          __nv_bfloat162* p = reinterpret_cast<__nv_bfloat162*>(&q);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = __bfloat1622float2(p[i]);
            p[i] = __floats2bfloat162_rn(f.x * s, f.y * s);
          }
        } else {
          q.x = __float_as_uint(__uint_as_float(q.x) * s);
          q.y = __float_as_uint(__uint_as_float(q.y) * s);
          q.z = __float_as_uint(__uint_as_float(q.z) * s);
          q.w = __float_as_uint(__uint_as_float(q.w) * s);
        }
      }
      y[static_cast<size_t>(r) * vpr + v] = q;
    }
  }
}

// Packed gate/up layout, one warp per packed row.
__global__ void __launch_bounds__(256) pack_w13_kernel(const uint4* __restrict__ wg, const uint4* __restrict__ wu,
                                                       uint4* __restrict__ w13, int E, int F, int vpr) {
  const int lane = threadIdx.x & 31;
  const long long rows = static_cast<long long>(E) * 2 * F;
  const long long nw = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  for (long long p = blockIdx.x * static_cast<long long>(blockDim.x >> 5) + (threadIdx.x >> 5); p < rows; p += nw) {
    const int e = static_cast<int>(p / (2 * F));
    const int w = static_cast<int>(p - static_cast<long long>(e) * 2 * F);
    const int b = w / (2 * MOE_PACK_BLOCK);
    const int in_blk = w - b * 2 * MOE_PACK_BLOCK;
    const int pb = min(MOE_PACK_BLOCK, F - b * MOE_PACK_BLOCK);
    const bool up = in_blk >= pb;
    const int f = b * MOE_PACK_BLOCK + (up ? in_blk - pb : in_blk);
    const uint4* src = (up ? wu : wg) + (static_cast<size_t>(e) * F + f) * vpr;
    uint4* dst = w13 + static_cast<size_t>(p) * vpr;
    for (int v = lane; v < vpr; v += 32) dst[v] = __ldg(src + v);
  }
}

int blocks_for(long long work, int per_block) {
  long long b = (work + per_block - 1) / per_block;
  const long long cap = static_cast<long long>(device_sm_count()) * 16;
  if (b > cap) b = cap;
  return b < 1 ? 1 : static_cast<int>(b);
}

// Row tiles per band: the largest power of two in [lo, hi] whose A rows
// (tile_rows x K bf16 each) stay within 64 MB, half of the L2.
int band_rows(int tile_rows, int K, int lo, int hi) {
  const long long tile_bytes = static_cast<long long>(tile_rows) * K * 2;
  int b = hi;
  while (b > lo && b * tile_bytes > (64ll << 20)) b >>= 1;
  return b;
}

}  // namespace

namespace {

std::atomic<int> g_stall_gemms{0};

// 1 when this launch takes one of the stalls moe_debug_stall_next_gemms asked for.
int take_stall() {
  int left = g_stall_gemms.load();
  while (left > 0 && !g_stall_gemms.compare_exchange_weak(left, left - 1)) {
  }
  return left > 0 ? 1 : 0;
}

template <int kEpi, int kMode>
cudaError_t launch_gemm_inst(const CUtensorMap& tm_a, const CUtensorMap& tm_b, GemmArgs a, bool pdl,
                             cudaStream_t s, const CUtensorMap* tm_d = nullptr) {
  a.tma_store = tm_d != nullptr ? 1 : 0;
  a.stall = take_stall();
  const size_t smem = gemm_smem_bytes();
  cudaError_t err = cudaFuncSetAttribute(grouped_gemm_kernel<kEpi, kMode>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
  if (err != cudaSuccess) return err;
  err = launch_kernel(grouped_gemm_kernel<kEpi, kMode>, dim3(device_sm_count()), dim3(kGemmThreads), smem, s, pdl, 1,
                      tm_a, tm_b, tm_d != nullptr ? *tm_d : tm_a, a);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_grouped_gemm_tc(const CUtensorMap& tm_a, const CUtensorMap& tm_b, bool swiglu,
                                   const int32_t* offsets, int E, int K, int n_per_expert, int n_tiles,
                                   int out_cols, int ldd, void* D, const int32_t* gather_rows, int32_t* status,
                                   bool pdl, cudaStream_t s, void* preact, const CUtensorMap* tm_d) {
  GemmArgs a{offsets, E, K, n_per_expert, n_tiles, out_cols, ldd, static_cast<__nv_bfloat16*>(D), status,
             band_rows(kBM, K, 8, 32), gather_rows, nullptr, 0, nullptr, 0, nullptr, nullptr, 0};
  a.preact = static_cast<__nv_bfloat16*>(preact);
  a.preact_ld = n_per_expert;
  return swiglu ? launch_gemm_inst<kEpiSwiGLU, kGroupRows>(tm_a, tm_b, a, pdl, s, tm_d)
                : launch_gemm_inst<kEpiStore, kGroupRows>(tm_a, tm_b, a, pdl, s, tm_d);
}

void debug_stall_next_gemms(int n) { g_stall_gemms.store(n > 0 ? n : 0); }

cudaError_t launch_grouped_gemm_combine(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const int32_t* offsets, int E,
                                        int K, int d, void* y_perm, const int32_t* perm_src, const int32_t* dest_row,
                                        const float* gate, int32_t* pair_cnt, void* y, int k, int32_t* status, bool pdl,
                                        cudaStream_t s) {
  GemmArgs a{offsets, E, K, d, (d + kBN - 1) / kBN, d, d, static_cast<__nv_bfloat16*>(y_perm), status,
             band_rows(kBM, K, 8, 32), nullptr, nullptr, 0, nullptr, 0, nullptr, nullptr, 0};
  a.perm_src = perm_src;
  a.dest_row = dest_row;
  a.gate = gate;
  a.pair_cnt = pair_cnt;
  a.Y = static_cast<__nv_bfloat16*>(y);
  a.k = k;
  return launch_gemm_inst<kEpiStoreCombine, kGroupRows>(tm_a, tm_b, a, pdl, s);
}

cudaError_t launch_grouped_gemm_dh_swiglu_bwd(const CUtensorMap& tm_a, const CUtensorMap& tm_b,
                                              const int32_t* offsets, int E, int K, int F, const void* preact,
                                              void* dgu, void* dgu_t, const int32_t* col_off, int ldt, int32_t* status,
                                              bool pdl, cudaStream_t s, const CUtensorMap* tm_d) {
  GemmArgs a{offsets, E, K, F, (F + kBN - 1) / kBN, F, 2 * F, static_cast<__nv_bfloat16*>(dgu), status,
             band_rows(kBM, K, 8, 32), nullptr, nullptr, 0, nullptr, 0, static_cast<__nv_bfloat16*>(dgu_t), col_off,
             ldt};
  a.preact = static_cast<__nv_bfloat16*>(const_cast<void*>(preact));
  a.preact_ld = 2 * F;
  return launch_gemm_inst<kEpiDhSwiGLUBwd, kGroupRows>(tm_a, tm_b, a, pdl, s, tm_d);
}

cudaError_t launch_grouped_gemm_swiglu_bwd(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const int32_t* offsets,
                                           int E, int K, int F, void* dgu, const void* dh_mid, void* dgu_t,
                                           const int32_t* col_off, int ldt, int32_t* status, bool pdl,
                                           cudaStream_t s, const CUtensorMap* tm_d) {
  GemmArgs a{offsets, E, K, 2 * F, 2 * F / kBN, 2 * F, 2 * F, static_cast<__nv_bfloat16*>(dgu), status,
             band_rows(kBM, K, 8, 32), nullptr, static_cast<const __nv_bfloat16*>(dh_mid), F, nullptr, 0,
             static_cast<__nv_bfloat16*>(dgu_t), col_off, ldt};
  return launch_gemm_inst<kEpiSwiGLUBwd, kGroupRows>(tm_a, tm_b, a, pdl, s, tm_d);
}

cudaError_t launch_grouped_gemm_wgrad(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const int32_t* col_offsets,
                                      int E, int M, int N, float* D32, int32_t* status, bool pdl, cudaStream_t s) {
  GemmArgs a{col_offsets, E, 0, 0, (N + kBN - 1) / kBN, N, N, nullptr, status, 0, nullptr, nullptr, 0, D32, M / kBM,
             nullptr, nullptr, 0};
  return launch_gemm_inst<kEpiStoreF32, kGroupReduce>(tm_a, tm_b, a, pdl, s);
}

cudaError_t launch_grouped_gemm_pair(const CUtensorMap& tm_a, const CUtensorMap& tm_b, bool swiglu,
                                     const int32_t* offsets, int E, int K, int n_per_expert, int n_tiles, int out_cols,
                                     int ldd, void* D, int32_t* status, bool pdl, cudaStream_t s,
                                     const CUtensorMap* tm_d) {
  GemmArgs a{offsets, E, K, n_per_expert, n_tiles, out_cols, ldd, static_cast<__nv_bfloat16*>(D), status,
             band_rows(2 * kBM, K, 4, 16), nullptr, nullptr, 0, nullptr, 0, nullptr, nullptr, 0};
  a.tma_store = tm_d != nullptr ? 1 : 0;
  a.stall = take_stall();
  const CUtensorMap& map_d = tm_d != nullptr ? *tm_d : tm_a;
  const size_t smem = pair_smem_bytes();
  const int grid = (device_sm_count() / 2) * 2;
  cudaError_t err;
  if (swiglu) {
    err = cudaFuncSetAttribute(grouped_gemm_pair_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    err = launch_kernel(grouped_gemm_pair_kernel<true>, dim3(grid), dim3(kPairThreads), smem, s, pdl, 2, tm_a, tm_b,
                        map_d, a);
  } else {
    err = cudaFuncSetAttribute(grouped_gemm_pair_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
    if (err != cudaSuccess) return err;
    err = launch_kernel(grouped_gemm_pair_kernel<false>, dim3(grid), dim3(kPairThreads), smem, s, pdl, 2, tm_a, tm_b,
                        map_d, a);
  }
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

cudaError_t launch_ffn_f32(const float* x_perm, const int32_t* offsets, const float* w13, const float* wd,
                           float* h_mid, float* y_perm, int rows_max, int d, int F, int E, cudaStream_t s) {
  if (rows_max == 0) return cudaSuccess;
  ffn1_f32_kernel<<<blocks_for(static_cast<long long>(rows_max) * F, 256), 256, 0, s>>>(x_perm, offsets, w13, h_mid,
                                                                                        rows_max, d, F, E);
  ffn2_f32_kernel<<<blocks_for(static_cast<long long>(rows_max) * d, 256), 256, 0, s>>>(h_mid, offsets, wd, y_perm,
                                                                                        rows_max, d, F, E);
  return cudaGetLastError();
}

cudaError_t launch_scale_rows(int dtype, int kind, const void* x_perm, const int32_t* offsets, void* y_perm,
                              int rows_max, int d, int E, cudaStream_t s) {
  if (rows_max == 0) return cudaSuccess;
  const int elem = dtype == MOE_DTYPE_BF16 ? 2 : 4;
  const int vpr = d * elem / 16;
  const int scale = kind == MOE_EXPERT_SCALE;
  const int grid = blocks_for(rows_max, 8);
  if (dtype == MOE_DTYPE_BF16)
    scale_rows_kernel<MOE_DTYPE_BF16><<<grid, 256, 0, s>>>(static_cast<const uint4*>(x_perm), offsets,
                                                           static_cast<uint4*>(y_perm), rows_max, vpr, E, scale);
  else
    scale_rows_kernel<MOE_DTYPE_F32><<<grid, 256, 0, s>>>(static_cast<const uint4*>(x_perm), offsets,
                                                          static_cast<uint4*>(y_perm), rows_max, vpr, E, scale);
  return cudaGetLastError();
}

cudaError_t launch_pack_w13(const void* w_gate, const void* w_up, void* w13, int E, int F, size_t row_bytes,
                            cudaStream_t s) {
  const long long rows = static_cast<long long>(E) * 2 * F;
  if (rows == 0) return cudaSuccess;
  pack_w13_kernel<<<blocks_for(rows, 8), 256, 0, s>>>(static_cast<const uint4*>(w_gate),
                                                      static_cast<const uint4*>(w_up), static_cast<uint4*>(w13), E, F,
                                                      static_cast<int>(row_bytes / 16));
  return cudaGetLastError();
}

}  // namespace moe
