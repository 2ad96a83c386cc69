// MXFP8 grouped expert FFN: block-scaled 8-bit operands on the tcgen05 tensor
// cores ("Dropless MoE Is a Runtime Problem as Much as a Model Design", the
// MXFP8 paragraph: block-scaled low precision for more arithmetic throughput
// and less data movement, with the scaling checked for overflow and
// underflow).
//
// Format (OCP Microscaling, MXFP8 E4M3): every 32 consecutive elements along
// the reduction axis of a row share one scale 2^E, stored as an E8M0 byte
// E + 127, with E = floor(log2 max|v|) - 8 clamped to [-127, 127]; every
// element is E4M3 of v / 2^E, rounded to nearest even and clamped at 448
// ("saturated"). A non-zero element that becomes 0 has underflowed.
//
// Layouts:
//   * quantised rows: row-major bytes, one byte per element.
//   * scales: in the order the tensor cores read them. For every 128-row block
//     R of a matrix and every 128-element slice kt of its reduction axis there
//     is one 512-byte atom at ((kt * row_blocks) + R) * 512; inside it the
//     scale of row r (0..127 within the block) and 32-element block j (0..3
//     within the slice) is byte (r % 32) * 16 + (r / 32) * 4 + j. One
//     tcgen05.cp 32x128b.warpx4 moves an atom into TMEM in the arrangement the
//     block-scaled MMA reads (the scale of row r, block j at lane r % 32 of
//     every lane quadrant, column r / 32, byte j).
//   * the token rows of the grouped problem are padded so that every expert
//     starts on a 128-row boundary: expert e's rows start at 128 * (the number
//     of 128-row tiles of the experts before it). A tile's rows and its scale
//     atoms are then aligned, and the rows past an expert's count are zero.
//
// Kernels:
//   mx_quantize_rows_kernel   bf16 rows -> E4M3 rows + scale atoms (weights, or
//                             the permuted token rows into the padded layout)
//   mx_dispatch_kernel        the layer's dispatch and quantisation in one pass:
//                             each token row read once, quantised once, written
//                             to each of its kept rows of the padded layout
//   grouped_gemm_mx_kernel    persistent warp-specialised GEMM over the
//                             padded groups: TMA for the operand tiles, bulk
//                             copies for the scale atoms (a warp of their
//                             own), tcgen05.cp of the scales into TMEM (another
//                             warp) and tcgen05.mma
//                             kind::mxf8f6f4.block_scale (128 x 256 x 32) by
//                             one thread. GEMM1 forms silu(gate) * up in its
//                             epilogue and quantises it straight to MXFP8 for
//                             GEMM2; GEMM2 stores bf16 rows in the compact
//                             layout.
// TMEM: the two accumulators overlap. Tile i uses columns [0, 256) when i is
// even and [192, 448) when odd; the epilogue drains the shared columns
// [192, 256) first and signals, so the next tile's MMAs start while it drains
// the rest. Columns [448, 496) hold the scales of the four k-slices in flight
// (12 columns each: 4 for A, 8 for B). A slice's scales are copied into its
// column set by the scale-copy warp, which commits the copies to the slice's
// sf_full barrier; the MMA thread waits for that barrier before the slice's
// MMAs, and a column set is rewritten only after its previous MMAs are done.
#include <cuda_fp8.h>

#include "moe_common.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

constexpr int kMxBM = 128;
constexpr int kMxBN = 256;
constexpr int kMxBK = 128;  // elements (= bytes) of K per stage
constexpr int kMxStages = 4;
// warp 0: TMA producer of the operand tiles, warp 1: TMEM allocation and MMA
// issue, warps 2..9: epilogue, two per TMEM lane quadrant, each draining half
// of a tile, warp 10: copies each stage's scale atoms into TMEM (a ring of
// four column sets) and signals the MMA thread through sf_full, warp 11:
// loads the scale atoms into shared memory (sf_loaded), so the producer
// issues two copies per stage, as in the bf16 kernel
constexpr int kMxThreads = 384;
constexpr int kMxEpiWarps = 8;
constexpr uint32_t kMxABytes = kMxBM * kMxBK;   // 16 KB
constexpr uint32_t kMxBBytes = kMxBN * kMxBK;   // 32 KB
constexpr uint32_t kSfaBytes = 512;
constexpr uint32_t kSfbBytes = 1024;
constexpr uint32_t kMxStageTx = kMxABytes + kMxBBytes;
constexpr uint32_t kMxSfTx = kSfaBytes + kSfbBytes;
constexpr uint32_t kAcc1Col = 192;   // second accumulator; [192, 256) is shared
constexpr uint32_t kSfaCol = 448;    // stage s: SFA at 448 + 12 s, SFB at 452 + 12 s (8 columns)
constexpr uint32_t kMxTmemCols = 512;
static_assert(kSfaCol + 12 * kMxStages <= kMxTmemCols, "scale ring");

// Epilogue store staging: one 2 KB block per epilogue warp (32 rows x 32 bf16
// for GEMM2, 32 rows x 32 E4M3 bytes for GEMM1).
constexpr uint32_t kMxStgBytes = 2048;

constexpr size_t mx_smem_bytes() {
  return 1024 + kMxStages * static_cast<size_t>(kMxABytes + kMxBBytes + kSfaBytes + kSfbBytes) +
         kMxEpiWarps * kMxStgBytes + (4 * kMxStages + 5) * 8 + 16 + 2 * (kMaxE + 1) * 4;
}
static_assert(mx_smem_bytes() <= 227 * 1024, "shared memory");

// ------------------------------------------------------------------ quantisation
// E of the shared scale from the block's largest magnitude: floor(log2 amax) - 8
// from the exponent field (0 or subnormal amax gives the clamp -127).
MOE_DEV int mx_scale_exp(float amax) {
  const int field = static_cast<int>((__float_as_uint(amax) >> 23) & 0xffu);
  return max(field - 127 - 8, -127);
}

// 2^-E for E in [-127, 119], a normal fp32 number.
MOE_DEV float mx_inv_scale(int E) { return __uint_as_float(static_cast<uint32_t>(127 - E) << 23); }

// Quantise 32 values (one block) in place into 32 E4M3 bytes; returns the E8M0
// scale byte and adds the block's saturated and underflowed elements.
// Saturation: |v| inv > 448 for some element exactly when amax inv > 448
// (fp32 rounding is monotonic), so the per-element test runs only then.
// Underflow: a nonzero scaled value whose code has a zero magnitude; the zero
// codes are counted four at a time, and the scaled zeros among them are
// subtracted only when there are any.
MOE_DEV uint32_t mx_quantize_block(const float (&v)[32], uint4 (&out)[2], int& n_sat, int& n_under) {
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const int E = mx_scale_exp(amax);
  const float inv = mx_inv_scale(E);
  float a[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) a[i] = v[i] * inv;
  uint32_t w[8];
  int zero_codes = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a[4 * i], a[4 * i + 1]), __NV_SATFINITE, __NV_E4M3);
    const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(a[4 * i + 2], a[4 * i + 3]), __NV_SATFINITE, __NV_E4M3);
    w[i] = lo | (hi << 16);
    zero_codes += __popc(__vcmpeq4(w[i] & 0x7f7f7f7fu, 0u)) >> 3;
  }
  if (amax * inv > 448.f) {
#pragma unroll
    for (int i = 0; i < 32; ++i) n_sat += fabsf(a[i]) > 448.f;
  }
  if (zero_codes != 0) {
    int zeros = 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) zeros += a[i] == 0.f;
    n_under += zero_codes - zeros;
  }
  out[0] = make_uint4(w[0], w[1], w[2], w[3]);
  out[1] = make_uint4(w[4], w[5], w[6], w[7]);
  return static_cast<uint32_t>(E + 127);
}

// Byte offset of the scale of (row, 32-element block b) in the atom layout.
MOE_DEV size_t mx_sf_offset(long long row, int b, int row_blocks) {
  const int kt = b >> 2, j = b & 3;
  const int r = static_cast<int>(row & 127);
  return (static_cast<size_t>(kt) * row_blocks + static_cast<size_t>(row >> 7)) * 512 + (r & 31) * 16 + (r >> 5) * 4 + j;
}

MOE_DEV void mx_report(int n_sat, int n_under, uint32_t* counts, int32_t* status) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    n_sat += __shfl_xor_sync(0xffffffffu, n_sat, off);
    n_under += __shfl_xor_sync(0xffffffffu, n_under, off);
  }
  if (lane == 0 && (n_sat | n_under)) {
    if (counts != nullptr) {
      if (n_sat) atomicAdd(counts, static_cast<uint32_t>(n_sat));
      if (n_under) atomicAdd(counts + 1, static_cast<uint32_t>(n_under));
    }
    report_status(status, (n_sat ? MOE_STATUS_MX_SATURATED : 0) | (n_under ? MOE_STATUS_MX_UNDERFLOW : 0));
  }
}

// Row tiles per expert, exclusive prefix (warp 0; 8 experts per lane).
MOE_DEV void tile_prefix(const int* s_off, int E, int* prefix) {
  const int lane = threadIdx.x & 31;
  int loc[8];
  int sum = 0;
#pragma unroll
  for (int v = 0; v < 8; ++v) {
    const int e = lane * 8 + v;
    loc[v] = e < E ? (s_off[e + 1] - s_off[e] + kMxBM - 1) / kMxBM : 0;
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
}

// One warp per destination row; lane l quantises the 32-element blocks l,
// l + 32, ... of the row. kGrouped: destination rows are the padded layout of
// the grouped problem (expert e's rows start at 128 * prefix[e]); row p maps to
// source row offsets[e] + (p - 128 prefix[e]) when that is below expert e's
// count, else it is written as zeros. Otherwise row p is source row p.
template <bool kGrouped>
__global__ void __launch_bounds__(256) mx_quantize_rows_kernel(const __nv_bfloat16* __restrict__ src, int cols,
                                                               int rows, const int32_t* __restrict__ offsets, int E,
                                                               uint8_t* __restrict__ q, uint8_t* __restrict__ sf,
                                                               int sf_row_blocks, uint32_t* counts, int32_t* status) {
  __shared__ int s_off[kMaxE + 1];
  __shared__ int prefix[kMaxE + 1];
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  long long n_rows = rows;
  if constexpr (kGrouped) {
    for (int e = threadIdx.x; e <= E; e += blockDim.x) s_off[e] = offsets[e];
    __syncthreads();
    if (warp == 0) tile_prefix(s_off, E, prefix);
    __syncthreads();
    n_rows = static_cast<long long>(prefix[E]) * kMxBM;
  }
  const int nblk = cols / 32;
  int n_sat = 0, n_under = 0;
  const long long nw = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  for (long long p = blockIdx.x * static_cast<long long>(blockDim.x >> 5) + warp; p < n_rows; p += nw) {
    long long s = p;
    if constexpr (kGrouped) {
      const int tile = static_cast<int>(p >> 7);
      int lo = 0, hi = E;  // prefix[lo] <= tile < prefix[hi]
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (prefix[mid] <= tile)
          lo = mid;
        else
          hi = mid;
      }
      const long long local = p - static_cast<long long>(prefix[lo]) * kMxBM;
      s = local < s_off[lo + 1] - s_off[lo] ? s_off[lo] + local : -1;
    }
    const uint4* srow = reinterpret_cast<const uint4*>(src + (s < 0 ? 0 : s) * static_cast<long long>(cols));
    uint4* qrow = reinterpret_cast<uint4*>(q + p * static_cast<long long>(cols));
    for (int b = lane; b < nblk; b += 32) {
      float v[32];
      if (s >= 0) {
        uint4 raw[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) raw[i] = __ldg(srow + 4 * b + i);
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(raw);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 f = __bfloat1622float2(h2[i]);
          v[2 * i] = f.x;
          v[2 * i + 1] = f.y;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f;
      }
      uint4 out[2];
      const uint32_t byte = mx_quantize_block(v, out, n_sat, n_under);
      qrow[2 * b] = out[0];
      qrow[2 * b + 1] = out[1];
      sf[mx_sf_offset(p, b, sf_row_blocks)] = static_cast<uint8_t>(byte);
    }
  }
  mx_report(n_sat, n_under, counts, status);
}

// ------------------------------------------------------------------ block-scaled MMA
// Instruction descriptor of kind::mxf8f6f4 with E4M3 A and B, E8M0 scales,
// both operands K-major; sf_id selects the byte (32-element block) of the
// 32-bit scale words in TMEM.
MOE_DEV uint32_t idesc_mxf8(int M, int N, uint32_t sf_id) {
  return (sf_id << 4)                                // B scale byte
         | (0u << 7) | (0u << 10)                   // A, B: E4M3
         | (static_cast<uint32_t>(N >> 3) << 17)    // N / 8
         | (1u << 23)                               // scales: E8M0
         | (static_cast<uint32_t>(M >> 4) << 24)    // M / 16
         | (sf_id << 29);                           // A scale byte
}

// D[tmem] (+)= (A * 2^SFA) (B * 2^SFB)^T over K = 32, fp32 accumulate.
MOE_DEV void umma_mxf8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t sfa_tmem,
                       uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem));
}

// Shared-memory descriptor of a 32-row x 16-byte block with no swizzle (rows
// 16 bytes apart, groups of 8 rows 128 bytes apart): the source of a
// tcgen05.cp 32x128b copy.
MOE_DEV uint64_t sf_copy_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);  // start address, 16-byte units
  d |= static_cast<uint64_t>(1) << 16;                   // leading-dimension offset (one 16-byte column: unused)
  d |= static_cast<uint64_t>(128 >> 4) << 32;            // stride between 8-row groups
  d |= static_cast<uint64_t>(1) << 46;                   // descriptor version (tcgen05)
  return d;                                              // layout type 0: no swizzle
}

// 32 lanes x 128 bits from shared memory into TMEM columns [taddr, taddr + 4),
// the same 32 lanes written to each of the 4 lane quadrants.
MOE_DEV void tmem_cp_32x128_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

struct MxGemmArgs {
  const int32_t* offsets;  // compact expert offsets [E+1]
  int E;
  int K;                   // reduction length, a multiple of 128
  int n_per_expert;        // rows of B per expert
  int n_tiles;             // 256-column tiles per expert
  int out_cols;            // columns of the output
  const uint8_t* sfa;      // A scale atoms [K/128][ra_blocks]
  int ra_blocks;           // 128-row blocks of the padded A rows
  const uint8_t* sfb;      // B scale atoms [K/128][rb_blocks + 1]
  int rb_blocks;           // 128-row blocks of B (E * n_per_expert / 128)
  int band;                // row tiles per band of the tile walk
  // GEMM1 (SwiGLU, quantised output): h_mid rows in the padded layout
  uint8_t* q_out;          // [padded rows, ldq]
  uint8_t* sf_out;         // atoms [ldq/128][ra_blocks]
  int ldq;
  uint32_t* counts;        // saturated / underflowed elements of h_mid (may be NULL)
  // GEMM2: bf16 rows in the compact layout
  __nv_bfloat16* D;
  int ldd;
  int32_t* status;
  // The output (q_out for GEMM1, D for GEMM2) is also the kernel's tm_d: a
  // warp whose 32 rows of the tile are all to be written stores each
  // 32-column block with one TMA store through its staging buffer.
  int tma_store;
};

// tile -> (expert, row tile within the expert, column tile); bands of row tiles
MOE_DEV void mx_decode_tile(long long tile, int m_total, int n_tiles, int band_rows, const int* prefix, int E, int& e,
                            int& m, int& n) {
  const long long band_size = static_cast<long long>(band_rows) * n_tiles;
  const int band = static_cast<int>(tile / band_size);
  const int within = static_cast<int>(tile - band * band_size);
  const int m0 = band * band_rows;
  const int rows = min(band_rows, m_total - m0);
  n = within / rows;
  const int gm = m0 + within % rows;
  int lo = 0, hi = E;
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

template <bool kSwiGLUQuant>
__global__ void __launch_bounds__(kMxThreads, 1)
    grouped_gemm_mx_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                           const __grid_constant__ CUtensorMap tm_d, const MxGemmArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = sA + kMxStages * kMxABytes;
  uint8_t* stg_all = sB + kMxStages * kMxBBytes;  // kMxEpiWarps x kMxStgBytes, 1024-aligned
  uint8_t* sSFA = stg_all + kMxEpiWarps * kMxStgBytes;
  uint8_t* sSFB = sSFA + kMxStages * kSfaBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sSFB + kMxStages * kSfbBytes);
  uint64_t* empty = full + kMxStages;
  uint64_t* tfull = empty + kMxStages;
  uint64_t* ovl = tfull + 2;
  uint64_t* drain = ovl + 1;
  uint64_t* sf_full = drain + 1;
  uint64_t* cp_drain = sf_full + kMxStages;
  uint64_t* sf_loaded = cp_drain + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sf_loaded + kMxStages);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* consumed_slot = reinterpret_cast<int*>(tmem_slot + 2);
  int* s_off = reinterpret_cast<int*>(tmem_slot + 4);  // [E+1]
  int* prefix = s_off + (kMaxE + 1);                   // [E+1]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = a.E;
  const int nkt = a.K / kMxBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kMxStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&tfull[0], 1);
    mbar_init(&tfull[1], 1);
    mbar_init(ovl, kMxEpiWarps);
    mbar_init(drain, 1);
    for (int s = 0; s < kMxStages; ++s) mbar_init(&sf_full[s], 1);
    mbar_init(cp_drain, 1);
    for (int s = 0; s < kMxStages; ++s) mbar_init(&sf_loaded[s], 1);
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
    tile_prefix(s_off, E, prefix);
  } else if (warp == 1) {
    tmem_alloc(tmem_slot, kMxTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int m_total = prefix[E];
  const long long total = static_cast<long long>(m_total) * a.n_tiles;

  int issued = 0;
  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------------------- TMA producer
      int stage = 0;
      uint32_t phase = 0;
      bool stop = false;
      for (long long tile = blockIdx.x; tile < total && !stop; tile += gridDim.x) {
        int e, m, n;
        mx_decode_tile(tile, m_total, a.n_tiles, a.band, prefix, E, e, m, n);
        const int a_row = (prefix[e] + m) * kMxBM;           // padded rows: 128-aligned per expert
        const int b_row = e * a.n_per_expert + n * kMxBN;
        for (int kt = 0; kt < nkt; ++kt) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) {
            *abort_flag = 1;
            stop = true;
            break;
          }
          mbar_expect_tx(&full[stage], kMxStageTx);
          tma_load_2d(sA + stage * kMxABytes, &tm_a, &full[stage], kt * kMxBK, a_row);
          tma_load_2d(sB + stage * kMxBBytes, &tm_b, &full[stage], kt * kMxBK, b_row);
          ++issued;
          if (++stage == kMxStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------------- MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      int consumed = 0, local = 0;
      bool stop = false;
      for (long long tile = blockIdx.x; tile < total && !stop; tile += gridDim.x, ++local) {
        const int acc = local & 1;
        // the columns this accumulator shares with the previous tile's must
        // have been drained (and with them every column of the tile before)
        if (local > 0 && !mbar_wait(ovl, (local - 1) & 1, abort_flag)) {
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + (acc ? kAcc1Col : 0u);
        for (int kt = 0; kt < nkt; ++kt) {
          if (!mbar_wait(&full[stage], phase, abort_flag)) {
            *abort_flag = 1;
            stop = true;
            break;
          }
          if (!mbar_wait(&sf_full[stage], phase, abort_flag)) {
            *abort_flag = 1;
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t sf_a = tmem + kSfaCol + 12u * stage, sf_b = sf_a + 4;
          const uint32_t sa = smem_addr(sA + stage * kMxABytes);
          const uint32_t sb = smem_addr(sB + stage * kMxBBytes);
#pragma unroll
          for (uint32_t kk = 0; kk < kMxBK / 32; ++kk)
            umma_mxf8(d_tmem, sw128_kmajor_desc(sa + kk * 32), sw128_kmajor_desc(sb + kk * 32),
                      idesc_mxf8(kMxBM, kMxBN, kk), sf_a | (kk << 30), sf_b | (kk << 30),
                      (kt | kk) != 0);
          umma_commit(&empty[stage]);
          ++consumed;
          if (++stage == kMxStages) {
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
  } else if (warp == 2 + kMxEpiWarps) {
    if (lane == 0) {
      // ---------------------------------------------------------------- scale copier
      int stage = 0;
      uint32_t phase = 0;
      bool stop = false;
      for (long long tile = blockIdx.x; tile < total && !stop; tile += gridDim.x) {
        for (int kt = 0; kt < nkt; ++kt) {
          if (!mbar_wait(&sf_loaded[stage], phase, abort_flag)) {
            *abort_flag = 1;
            stop = true;
            break;
          }
          tc_fence_after();
          const uint32_t sf_a = tmem + kSfaCol + 12u * stage, sf_b = sf_a + 4;
          tmem_cp_32x128_x4(sf_a, sf_copy_desc(smem_addr(sSFA + stage * kSfaBytes)));
          tmem_cp_32x128_x4(sf_b, sf_copy_desc(smem_addr(sSFB + stage * kSfbBytes)));
          tmem_cp_32x128_x4(sf_b + 4, sf_copy_desc(smem_addr(sSFB + stage * kSfbBytes + 512)));
          umma_commit(&sf_full[stage]);
          if (++stage == kMxStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      umma_commit(cp_drain);
      mbar_wait(cp_drain, 0, nullptr);
    }
  } else if (warp == 3 + kMxEpiWarps) {
    if (lane == 0) {
      // ---------------------------------------------------------------- scale loader
      int stage = 0;
      uint32_t phase = 0;
      bool stop = false;
      int sf_issued = 0;
      for (long long tile = blockIdx.x; tile < total && !stop; tile += gridDim.x) {
        int e, m, n;
        mx_decode_tile(tile, m_total, a.n_tiles, a.band, prefix, E, e, m, n);
        const int a_row = (prefix[e] + m) * kMxBM;
        const int b_row = e * a.n_per_expert + n * kMxBN;
        for (int kt = 0; kt < nkt; ++kt) {
          // the stage's MMAs of the previous round are done, and with them the
          // copy of its scales into TMEM
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag)) {
            *abort_flag = 1;
            stop = true;
            break;
          }
          mbar_expect_tx(&sf_loaded[stage], kMxSfTx);
          bulk_load(sSFA + stage * kSfaBytes, a.sfa + (static_cast<size_t>(kt) * a.ra_blocks + a_row / 128) * 512,
                    kSfaBytes, &sf_loaded[stage]);
          bulk_load(sSFB + stage * kSfbBytes,
                    a.sfb + (static_cast<size_t>(kt) * (a.rb_blocks + 1) + b_row / 128) * 512, kSfbBytes,
                    &sf_loaded[stage]);
          ++sf_issued;
          if (++stage == kMxStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // each stage holds at most one load that nobody may have waited for:
      // let it land before the CTA leaves
      for (int i = sf_issued > kMxStages ? sf_issued - kMxStages : 0; i < sf_issued; ++i)
        mbar_wait(&sf_loaded[i % kMxStages], (i / kMxStages) & 1, nullptr);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;            // TMEM lane quadrant this warp may read
    const int half = (warp - 2) >> 2;  // chunks half, half + 2, ... of the tile's column order
    const int row = q * 32 + lane;
    uint8_t* stg = stg_all + (warp - 2) * kMxStgBytes;
    int local = 0;
    int n_sat = 0, n_under = 0;
    for (long long tile = blockIdx.x; tile < total; tile += gridDim.x, ++local) {
      int e, m, n;
      mx_decode_tile(tile, m_total, a.n_tiles, a.band, prefix, E, e, m, n);
      const int acc = local & 1;
      if (!mbar_wait(&tfull[acc], (local >> 1) & 1, abort_flag)) {
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem + (acc ? kAcc1Col : 0u) + (static_cast<uint32_t>(q * 32) << 16);
      if constexpr (kSwiGLUQuant) {
        // columns [0,128) of the tile are gate, [128,256) the matching up;
        // the 32-channel chunks in the shared columns go first: channels
        // 64..127 (up columns 192..255) for an even tile, 0..63 (gate columns
        // 0..63) for an odd one
        const long long prow = static_cast<long long>(prefix[e] + m) * kMxBM + row;
        uint8_t* qout = a.q_out + prow * a.ldq + n * (kMxBN / 2);
        // this row's 4 scales for k-slice n of the next GEMM (one per 32 channels)
        uint8_t* sfo = a.sf_out + (static_cast<size_t>(n) * a.ra_blocks + static_cast<size_t>(prow >> 7)) * 512 +
                       (row & 31) * 16 + (row >> 5) * 4;
#pragma unroll 1
        for (int i = half; i < 4; i += 2) {
          const int c = acc ? 32 * i : 32 * ((i + 2) & 3);
          uint32_t g[32], u[32];
          tmem_ld32(tbase + c, g);
          tmem_ld32(tbase + kMxBN / 2 + c, u);
          tmem_ld_wait();
          if (i < 2) {  // this warp's chunk of the shared columns is drained
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(ovl);
          }
          float h[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) h[j] = silu_fast(__uint_as_float(g[j])) * __uint_as_float(u[j]);
          uint4 out[2];
          const uint32_t byte = mx_quantize_block(h, out, n_sat, n_under);
          if (a.tma_store) {
            stage_store_rows<32>(stg, out, lane, &tm_d, n * (kMxBN / 2) + c, static_cast<int>(prow - lane));
          } else {
            uint4* dst = reinterpret_cast<uint4*>(qout + c);
            dst[0] = out[0];
            dst[1] = out[1];
          }
          sfo[c >> 5] = static_cast<uint8_t>(byte);
        }
      } else {
        const int rows_valid = min(kMxBM, s_off[e + 1] - s_off[e] - m * kMxBM);
        const bool valid = row < rows_valid;
        const bool staged = a.tma_store != 0 && q * 32 + 32 <= rows_valid;
        __nv_bfloat16* out = a.D + static_cast<size_t>(s_off[e] + m * kMxBM + row) * a.ldd + n * kMxBN;
#pragma unroll 1
        for (int i = half; i < 8; i += 2) {
          // shared columns first: [192,256) for an even tile, [0,64) for an odd one
          const int c = acc ? 32 * i : 32 * ((i + 6) & 7);
          if (n * kMxBN + c < a.out_cols) {
            uint32_t v[32];
            tmem_ld32(tbase + c, v);
            tmem_ld_wait();
            if (valid) {
              uint32_t p[16];
#pragma unroll
              for (int j = 0; j < 16; ++j)
                p[j] = pack_bf16x2(__uint_as_float(v[2 * j]), __uint_as_float(v[2 * j + 1]));
              const uint4 pv[4] = {make_uint4(p[0], p[1], p[2], p[3]), make_uint4(p[4], p[5], p[6], p[7]),
                                   make_uint4(p[8], p[9], p[10], p[11]), make_uint4(p[12], p[13], p[14], p[15])};
              if (staged) {
                stage_store_rows<64>(stg, pv, lane, &tm_d, n * kMxBN + c, s_off[e] + m * kMxBM + q * 32);
              } else {
                uint4* dst = reinterpret_cast<uint4*>(out + c);
#pragma unroll
                for (int j = 0; j < 4; ++j) dst[j] = pv[j];
              }
            }
          }
          if (i < 2) {  // this warp's chunk of the shared columns is drained
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(ovl);
          }
        }
      }
    }
    if constexpr (kSwiGLUQuant) mx_report(n_sat, n_under, a.counts, a.status);
    if (lane == 0) bulk_wait_all();  // this warp's staged stores have completed
  }
  __syncwarp();

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (*abort_flag) {
    if (threadIdx.x == 0) report_status(a.status, MOE_STATUS_TIMEOUT);
    if (warp == 0 && lane == 0) {
      // loads issued but never consumed must land before the CTA leaves
      for (int i = *consumed_slot; i < issued; ++i) mbar_wait(&full[i % kMxStages], (i / kMxStages) & 1, nullptr);
    }
  }
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, kMxTmemCols);
}

// Dispatch fused with the MXFP8 quantisation of the token rows (the layer's
// path: no bf16 x_perm). Work items w = 0 .. T + 128 E - 1, one warp each:
//   w < T   token t: h[t] is read once and each 32-element block quantised once
//           (lane l takes blocks l, l + 32, ...); the E4M3 bytes and the scale
//           byte go to every kept destination of the token, at its padded row
//           128 prefix[e] + (dest_row - offsets[e]).
//   w >= T  padding: p = w - T, expert e = p / 128, i = p % 128; when expert
//           e's count c is not a multiple of 128, row (c & ~127) + i of its
//           last tile is zeroed if it lies at or past c.
// Saturated and underflowed elements are counted once per destination row,
// as the quantisation of x_perm would count them.
template <int K>
__global__ void __launch_bounds__(256, 4) mx_dispatch_kernel(const __nv_bfloat16* __restrict__ h, int T, int d,
                                                          const int32_t* __restrict__ idx,
                                                          const int32_t* __restrict__ dest_row,
                                                          const int32_t* __restrict__ offsets, int E,
                                                          uint8_t* __restrict__ q, uint8_t* __restrict__ sf,
                                                          int sf_row_blocks, uint32_t* counts, int32_t* status) {
  __shared__ int s_off[kMaxE + 1];
  __shared__ int prefix[kMaxE + 1];
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int e = threadIdx.x; e <= E; e += blockDim.x) s_off[e] = offsets[e];
  __syncthreads();
  if (warp == 0) tile_prefix(s_off, E, prefix);
  __syncthreads();
  const int nblk = d / 32;
  int n_sat = 0, n_under = 0;
  const long long items = static_cast<long long>(T) + 128ll * E;
  const long long nw = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  for (long long w = blockIdx.x * static_cast<long long>(blockDim.x >> 5) + warp; w < items; w += nw) {
    if (w < T) {
      const int t = static_cast<int>(w);
      long long prow[K];
      int nk = 0;
#pragma unroll
      for (int j = 0; j < K; ++j) {
        const int dst = dest_row[static_cast<size_t>(t) * K + j];
        prow[j] = -1;
        if (dst >= 0) {
          const int e = idx[static_cast<size_t>(t) * K + j];
          prow[j] = static_cast<long long>(prefix[e]) * 128 + (dst - s_off[e]);
          ++nk;
        }
      }
      if (nk == 0) continue;
      const uint4* srow = reinterpret_cast<const uint4*>(h + static_cast<size_t>(t) * d);
      for (int b = lane; b < nblk; b += 32) {
        uint4 raw[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) raw[i] = __ldg(srow + 4 * b + i);
        float v[32];
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(raw);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 f = __bfloat1622float2(h2[i]);
          v[2 * i] = f.x;
          v[2 * i + 1] = f.y;
        }
        uint4 out[2];
        int s0 = 0, u0 = 0;
        const uint32_t byte = mx_quantize_block(v, out, s0, u0);
#pragma unroll
        for (int j = 0; j < K; ++j) {
          if (prow[j] < 0) continue;
          uint4* qrow = reinterpret_cast<uint4*>(q + prow[j] * d);
          qrow[2 * b] = out[0];
          qrow[2 * b + 1] = out[1];
          sf[mx_sf_offset(prow[j], b, sf_row_blocks)] = static_cast<uint8_t>(byte);
          n_sat += s0;
          n_under += u0;
        }
      }
    } else {
      const long long pidx = w - T;
      const int e = static_cast<int>(pidx >> 7), i = static_cast<int>(pidx & 127);
      const int c = s_off[e + 1] - s_off[e];
      if ((c & 127) == 0) continue;
      const int local = (c & ~127) + i;
      if (local < c) continue;
      const long long p = static_cast<long long>(prefix[e]) * 128 + local;
      uint4* qrow = reinterpret_cast<uint4*>(q + p * d);
      for (int v = lane; v < d / 16; v += 32) qrow[v] = make_uint4(0, 0, 0, 0);
      for (int b = lane; b < nblk; b += 32) sf[mx_sf_offset(p, b, sf_row_blocks)] = 0;
    }
  }
  mx_report(n_sat, n_under, counts, status);
}

int mx_band_rows(int K) {
  const long long tile_bytes = static_cast<long long>(kMxBM) * K;
  int b = 32;
  while (b > 8 && b * tile_bytes > (64ll << 20)) b >>= 1;
  return b;
}

}  // namespace

size_t mx_smem_size() { return mx_smem_bytes(); }

cudaError_t launch_mx_quantize(const void* src, int rows, int cols, const int32_t* offsets, int E, void* q, void* sf,
                               int sf_row_blocks, uint32_t* counts, int32_t* status, bool pdl, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  const long long want = (static_cast<long long>(rows) + 7) / 8;
  const long long cap = static_cast<long long>(device_sm_count()) * 8;
  const int grid = static_cast<int>(want < cap ? want : cap);
  cudaError_t err;
  if (offsets != nullptr)
    err = launch_kernel(mx_quantize_rows_kernel<true>, dim3(grid), dim3(256), 0, s, pdl, 1,
                        static_cast<const __nv_bfloat16*>(src), cols, rows, offsets, E, static_cast<uint8_t*>(q),
                        static_cast<uint8_t*>(sf), sf_row_blocks, counts, status);
  else
    err = launch_kernel(mx_quantize_rows_kernel<false>, dim3(grid), dim3(256), 0, s, pdl, 1,
                        static_cast<const __nv_bfloat16*>(src), cols, rows, offsets, E, static_cast<uint8_t*>(q),
                        static_cast<uint8_t*>(sf), sf_row_blocks, counts, status);
  return err != cudaSuccess ? err : cudaGetLastError();
}

cudaError_t launch_mx_dispatch(const void* h, int T, int d, int k, const int32_t* idx, const int32_t* dest_row,
                               const int32_t* offsets, int E, void* q, void* sf, int sf_row_blocks, uint32_t* counts,
                               int32_t* status, bool pdl, cudaStream_t s) {
  const long long items = static_cast<long long>(T) + 128ll * E;
  if (items <= 0) return cudaSuccess;
  const long long want = (items + 7) / 8;
  // one wave of 4 CTAs (32 warps) per SM, each warp striding over the items
  // (A/B on B200 against 8-warp CTAs at 3 per SM over 2.7 waves: the
  // dispatch stage 46.5 -> 42.0 us on skewed with capacity, 141.9 -> 137.2
  // us on Mixtral 8x7B)
  const long long cap = static_cast<long long>(device_sm_count()) * 4;
  const int grid = static_cast<int>(want < cap ? want : cap);
  cudaError_t err = cudaErrorInvalidValue;
  switch (k) {
#define MOE_MX_DISPATCH_K(KK)                                                                                      \
  case KK:                                                                                                        \
    err = launch_kernel(mx_dispatch_kernel<KK>, dim3(grid), dim3(256), 0, s, pdl, 1,                               \
                        static_cast<const __nv_bfloat16*>(h), T, d, idx, dest_row, offsets, E,                     \
                        static_cast<uint8_t*>(q), static_cast<uint8_t*>(sf), sf_row_blocks, counts, status);       \
    break;
    MOE_MX_DISPATCH_K(1)
    MOE_MX_DISPATCH_K(2)
    MOE_MX_DISPATCH_K(3)
    MOE_MX_DISPATCH_K(4)
    MOE_MX_DISPATCH_K(5)
    MOE_MX_DISPATCH_K(6)
    MOE_MX_DISPATCH_K(7)
    MOE_MX_DISPATCH_K(8)
#undef MOE_MX_DISPATCH_K
    default:
      break;
  }
  return err != cudaSuccess ? err : cudaGetLastError();
}

cudaError_t launch_grouped_gemm_mx(const CUtensorMap& tm_a, const CUtensorMap& tm_b, bool swiglu_quant,
                                   const int32_t* offsets, int E, int K, int n_per_expert, int out_cols,
                                   const void* sfa, int ra_blocks, const void* sfb, void* q_out, void* sf_out, int ldq,
                                   uint32_t* counts, void* D, int ldd, int32_t* status, bool pdl, cudaStream_t s,
                                   const CUtensorMap* tm_d) {
  MxGemmArgs a{};
  a.tma_store = tm_d != nullptr ? 1 : 0;
  a.offsets = offsets;
  a.E = E;
  a.K = K;
  a.n_per_expert = n_per_expert;
  a.n_tiles = swiglu_quant ? n_per_expert / kMxBN : (n_per_expert + kMxBN - 1) / kMxBN;
  a.out_cols = out_cols;
  a.sfa = static_cast<const uint8_t*>(sfa);
  a.ra_blocks = ra_blocks;
  a.sfb = static_cast<const uint8_t*>(sfb);
  a.rb_blocks = E * n_per_expert / 128;
  a.band = mx_band_rows(K);
  a.q_out = static_cast<uint8_t*>(q_out);
  a.sf_out = static_cast<uint8_t*>(sf_out);
  a.ldq = ldq;
  a.counts = counts;
  a.D = static_cast<__nv_bfloat16*>(D);
  a.ldd = ldd;
  a.status = status;
  const size_t smem = mx_smem_bytes();
  cudaError_t err;
  if (swiglu_quant) {
    err = cudaFuncSetAttribute(grouped_gemm_mx_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
    if (err == cudaSuccess)
      err = launch_kernel(grouped_gemm_mx_kernel<true>, dim3(device_sm_count()), dim3(kMxThreads), smem, s, pdl, 1,
                          tm_a, tm_b, tm_d != nullptr ? *tm_d : tm_a, a);
  } else {
    err = cudaFuncSetAttribute(grouped_gemm_mx_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
    if (err == cudaSuccess)
      err = launch_kernel(grouped_gemm_mx_kernel<false>, dim3(device_sm_count()), dim3(kMxThreads), smem, s, pdl, 1,
                          tm_a, tm_b, tm_d != nullptr ? *tm_d : tm_a, a);
  }
  return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace moe
