// C ABI of the MoE layer: argument checks, workspace carving, TMA descriptor
// encoding and stage launches, for the forward stages, the whole layer and
// its backward. The stage order and the meaning of every argument are
// documented in include/moe.h.
#include <algorithm>
#include <mutex>

#include "moe_common.cuh"

#include "moe_internal.h"

namespace moe {

int device_sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
  if (dev >= 0 && dev < 64 && cached[dev] > 0) return cached[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 1;
  if (dev >= 0 && dev < 64) cached[dev] = n;
  return n;
}

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Row-major bf16 matrix [rows, cols], box of box_rows x 64 columns, 128-byte swizzle.
int make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return MOE_ERR_NO_DEVICE;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t es[2] = {1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

// Row-major bf16 matrix [rows, cols] written by TMA stores: boxes of 32 rows x
// 32 columns (64 bytes), 64-byte swizzle (the GEMM epilogue's staging layout).
int make_map_store(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return MOE_ERR_NO_DEVICE;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {32, 32};
  const cuuint32_t es[2] = {1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                         CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

// Row-major byte matrix [rows, cols] written by TMA stores: boxes of 32 rows x
// 32 bytes, 32-byte swizzle (the MXFP8 GEMM epilogue's staging layout).
int make_map_store_u8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return MOE_ERR_NO_DEVICE;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols};
  const cuuint32_t box[2] = {32, 32};
  const cuuint32_t es[2] = {1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B,
                         CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

// Row-major byte matrix [rows, cols] (E4M3 elements), box of box_rows x 128
// columns, 128-byte swizzle.
int make_map_u8(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return MOE_ERR_NO_DEVICE;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols};
  const cuuint32_t box[2] = {128, box_rows};
  const cuuint32_t es[2] = {1, 1};
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, es,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int elem_bytes(const moe_config& c) { return c.dtype == MOE_DTYPE_BF16 ? 2 : 4; }

// Rows of the permuted buffers: kept rows only (at most T*k), or capacity
// rows per expert in the padded layout.
size_t perm_rows(const moe_config& c) {
  return c.layout == MOE_LAYOUT_PADDED ? static_cast<size_t>(c.E) * c.capacity : static_cast<size_t>(c.T) * c.k;
}


bool is_mx(const moe_config& c) { return c.precision == MOE_PRECISION_MXFP8; }

// The layer's MXFP8 dispatch writes the quantised rows straight from h.
bool mx_dispatch_fused(const moe_config& c) { return is_mx(c) && c.layout == MOE_LAYOUT_COMPACT; }

// Whether the layer's GEMM1 can gather its A rows from h (no x_perm).
bool gather_supported(const moe_config& c) {
  return c.dtype == MOE_DTYPE_BF16 && c.expert_kind == MOE_EXPERT_SWIGLU && c.layout == MOE_LAYOUT_COMPACT &&
         c.gemm_tiles != MOE_GEMM_TILES_PAIR && !is_mx(c);
}

size_t round256(size_t n) { return (n + 255) & ~static_cast<size_t>(255); }

// MXFP8 weight blob: E4M3 bytes [rows, cols], then the scale atoms with one
// extra 128-row block per 128-column slice (a 256-row B tile that ends one
// block past the last expert reads it).
struct MxBlob {
  size_t rows, cols, q_bytes, sf_bytes;
  int row_blocks;  // including the extra one
};

MxBlob mx_blob(const moe_config& c, int which) {
  MxBlob b;
  b.rows = which == 0 ? static_cast<size_t>(c.E) * 2 * c.d_ff : static_cast<size_t>(c.E) * c.d;
  b.cols = which == 0 ? static_cast<size_t>(c.d) : static_cast<size_t>(c.d_ff);
  b.row_blocks = static_cast<int>(b.rows / 128 + 1);
  b.q_bytes = round256(b.rows * b.cols);
  b.sf_bytes = (b.cols / 128) * static_cast<size_t>(b.row_blocks) * 512;
  return b;
}

// Whether the layer's down projection also writes y (the combine fused into
// its epilogue): k <= 2, bf16 SwiGLU experts on single-CTA bf16 tiles.
bool combine_fusable(const moe_config& c) {
  return c.k <= 2 && c.dtype == MOE_DTYPE_BF16 && c.expert_kind == MOE_EXPERT_SWIGLU &&
         c.gemm_tiles != MOE_GEMM_TILES_PAIR && !is_mx(c);
}

// Whether the layer keeps the gate/up pre-activations for the backward.
bool preact_savable(const moe_config& c) {
  return c.dtype == MOE_DTYPE_BF16 && c.expert_kind == MOE_EXPERT_SWIGLU && c.gemm_tiles != MOE_GEMM_TILES_PAIR &&
         !is_mx(c) && c.dispatch != MOE_DISPATCH_GATHER;
}

bool layer_saves_preact(const moe_config& c) { return c.preact == MOE_PREACT_SAVE && preact_savable(c); }

// AUTO keeps the separate combine: fusing it measured 1-3% slower per layer
// on B200 (the down projection's epilogue re-reads both rows of a token and
// competes with the GEMM; the separate kernel streams them at HBM rate).
bool layer_fuses_combine(const moe_config& c) { return c.combine == MOE_COMBINE_FUSED && combine_fusable(c); }

// AUTO copies: gathering costs one four-row TMA gather per 512 bytes of A
// every time a tile reloads its A rows (once per column tile), and measured
// 2.2-2.4x slower per layer on B200 than the row copy plus tiled loads.
bool layer_gathers(const moe_config& c) {
  return c.dispatch == MOE_DISPATCH_GATHER && gather_supported(c);
}

// Tile shape of the bf16 grouped GEMMs. The two shapes give the same bits
// (each output sums its K range in the same order), so this is a speed
// choice only. AUTO takes CTA-pair tiles where they measured faster on B200,
// in 10-step and in 100-2000-step loops under the 1 kW cap: experts of at
// least 1024 rows on average, so that 256-row tiles pad little, with weights
// of at most 128 MiB an expert (3 d F bf16; about the L2 size). Pair tiles
// measured 4-8% faster on the skewed 64-expert layer (d 2048, F 1408) and the
// scaled Mixtral layer (d 1024, F 3584), 2-3% faster with 63 and 88 MB
// experts, even with 132 MB ones, even on the skewed layer with capacity
// 1920, 2% slower with 512-row experts (128 experts, k 8) and 5-8% slower on
// the Mixtral 8x7B layer (352 MB an expert). Options that need single tiles
// keep them.
bool use_pair_tiles(const moe_config& c) {
  if (c.gemm_tiles == MOE_GEMM_TILES_PAIR) return true;
  if (c.gemm_tiles != MOE_GEMM_TILES_AUTO) return false;
  if (c.dtype != MOE_DTYPE_BF16 || c.expert_kind != MOE_EXPERT_SWIGLU || is_mx(c) ||
      c.dispatch == MOE_DISPATCH_GATHER || c.combine == MOE_COMBINE_FUSED || c.preact == MOE_PREACT_SAVE)
    return false;
  long long rows = static_cast<long long>(c.T) * c.k / c.E;
  if (c.capacity >= 0) rows = c.layout == MOE_LAYOUT_PADDED ? c.capacity : std::min<long long>(rows, c.capacity);
  const long long expert_weight_bytes = 3LL * c.d * c.d_ff * 2;
  return rows >= 1024 && expert_weight_bytes <= (128LL << 20);
}

int check_cfg(const moe_config* c) {
  if (c == nullptr) return MOE_ERR_INVALID_ARG;
  if (c->T < 0 || c->d <= 0 || c->E <= 0 || c->k <= 0 || c->capacity < -1) return MOE_ERR_INVALID_ARG;
  if (c->dtype != MOE_DTYPE_BF16 && c->dtype != MOE_DTYPE_F32) return MOE_ERR_INVALID_ARG;
  if (c->expert_kind < MOE_EXPERT_SWIGLU || c->expert_kind > MOE_EXPERT_SCALE) return MOE_ERR_INVALID_ARG;
  if (c->gemm_tiles < MOE_GEMM_TILES_AUTO || c->gemm_tiles > MOE_GEMM_TILES_PAIR) return MOE_ERR_INVALID_ARG;
  if (c->layout != MOE_LAYOUT_COMPACT && c->layout != MOE_LAYOUT_PADDED) return MOE_ERR_INVALID_ARG;
  if (c->layout == MOE_LAYOUT_PADDED && c->capacity < 0) return MOE_ERR_INVALID_ARG;
  if (c->dispatch < MOE_DISPATCH_AUTO || c->dispatch > MOE_DISPATCH_GATHER) return MOE_ERR_INVALID_ARG;
  if (c->dispatch == MOE_DISPATCH_GATHER && !gather_supported(*c)) return MOE_ERR_UNSUPPORTED;
  if (c->expert_kind == MOE_EXPERT_SWIGLU && c->d_ff <= 0) return MOE_ERR_INVALID_ARG;
  if (c->E > MOE_MAX_E || c->k > MOE_MAX_K || c->k > c->E) return MOE_ERR_UNSUPPORTED;
  if (static_cast<long long>(c->T) * c->k >= (1LL << 31)) return MOE_ERR_UNSUPPORTED;
  if (c->layout == MOE_LAYOUT_PADDED && static_cast<long long>(c->E) * c->capacity >= (1LL << 31))
    return MOE_ERR_UNSUPPORTED;
  if (c->precision != MOE_PRECISION_BF16 && c->precision != MOE_PRECISION_MXFP8) return MOE_ERR_INVALID_ARG;
  if (c->combine < MOE_COMBINE_AUTO || c->combine > MOE_COMBINE_FUSED) return MOE_ERR_INVALID_ARG;
  if (c->combine == MOE_COMBINE_FUSED && !combine_fusable(*c)) return MOE_ERR_UNSUPPORTED;
  if (c->preact != MOE_PREACT_RECOMPUTE && c->preact != MOE_PREACT_SAVE) return MOE_ERR_INVALID_ARG;
  if (c->preact == MOE_PREACT_SAVE && !preact_savable(*c)) return MOE_ERR_UNSUPPORTED;
  if (c->precision == MOE_PRECISION_MXFP8 &&
      (c->dtype != MOE_DTYPE_BF16 || c->expert_kind != MOE_EXPERT_SWIGLU || c->gemm_tiles == MOE_GEMM_TILES_PAIR ||
       c->dispatch == MOE_DISPATCH_GATHER))
    return MOE_ERR_UNSUPPORTED;
  if (c->dtype == MOE_DTYPE_BF16) {
    if (c->d % 128 != 0) return MOE_ERR_UNSUPPORTED;
    if (c->expert_kind == MOE_EXPERT_SWIGLU && c->d_ff % 128 != 0) return MOE_ERR_UNSUPPORTED;
  } else if (c->d % 4 != 0) {
    return MOE_ERR_UNSUPPORTED;
  }
  return MOE_OK;
}

// Carves 256-byte aligned pieces off the workspace; with a null base it only
// measures, so sizes and layout come from the same code.
struct Carver {
  uint8_t* base;
  size_t off = 0;
  explicit Carver(void* b) : base(static_cast<uint8_t*>(b)) {}
  template <typename T>
  T* take(size_t bytes) {
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += (bytes + 255) & ~static_cast<size_t>(255);
    return p;
  }
};

struct PermuteScratch {
  int32_t* chunk_counts;
  int32_t* chunk_base;
};

PermuteScratch carve_permute(const moe_config& c, Carver& w) {
  const size_t nc = (static_cast<size_t>(c.T) + kChunkTokens - 1) / kChunkTokens;
  PermuteScratch p;
  p.chunk_counts = w.take<int32_t>(nc * c.E * 4);
  p.chunk_base = w.take<int32_t>(nc * c.E * 4);
  return p;
}

void* carve_ffn(const moe_config& c, Carver& w) {
  if (c.expert_kind != MOE_EXPERT_SWIGLU || is_mx(c)) return nullptr;
  return w.take<void>(perm_rows(c) * c.d_ff * elem_bytes(c));
}

// MXFP8 scratch (first in the workspace of the grouped FFN and the layer):
// the call's four counters, then the quantised token rows and h_mid in the
// padded layout (each expert's rows from a 128-row boundary) with their scale
// atoms. The padded rows are at most P + 127 E.
struct MxBufs {
  uint32_t* counters;  // [4]: x saturated, x underflowed, h_mid saturated, h_mid underflowed
  uint8_t *xq, *xsf, *hq, *hsf;
  int pad_rows, row_blocks;
};

MxBufs carve_mx(const moe_config& c, Carver& w) {
  MxBufs m{};
  m.pad_rows = static_cast<int>((perm_rows(c) + 127) / 128 * 128 + 128 * static_cast<size_t>(c.E));
  m.row_blocks = m.pad_rows / 128;
  const size_t d = c.d, F = c.d_ff, R = m.pad_rows;
  m.counters = w.take<uint32_t>(16);
  m.xq = w.take<uint8_t>(R * d);
  m.xsf = w.take<uint8_t>((d / 128) * m.row_blocks * 512);
  m.hq = w.take<uint8_t>(R * F);
  m.hsf = w.take<uint8_t>((F / 128) * m.row_blocks * 512);
  return m;
}

// Counters of the fused combine per token: one per 256-column tile of the
// down projection and per half of it (two epilogue warps share a tile row).
int pair_entries(const moe_config& c) { return 2 * ((c.d + kGemmTileN - 1) / kGemmTileN); }

struct LayerBufs {
  int32_t *idx, *routed, *kept, *offsets, *dest_row, *perm_src;
  float* gate;
  void *x_perm, *y_perm, *h_mid;
  PermuteScratch perm;
  int32_t* pair_cnt;  // [T][pair_entries(c)] when the combine is fused, else NULL
  void* preact;       // [P, 2F] bf16 gate/up pre-activations when kept for the backward, else NULL
};

LayerBufs carve_layer(const moe_config& c, Carver& w) {
  const size_t A = static_cast<size_t>(c.T) * c.k;
  const size_t P = perm_rows(c);
  const size_t row = static_cast<size_t>(c.d) * elem_bytes(c);
  LayerBufs b;
  b.idx = w.take<int32_t>(A * 4);
  b.gate = w.take<float>(A * 4);
  b.routed = w.take<int32_t>(c.E * 4);
  b.kept = w.take<int32_t>(c.E * 4);
  b.offsets = w.take<int32_t>((c.E + 1) * 4);
  b.dest_row = w.take<int32_t>(A * 4);
  b.perm_src = w.take<int32_t>(P * 4);
  // no x_perm when GEMM1 gathers from h, or when the MXFP8 dispatch quantises h straight into its
  // layout (compact rows; the padded capacity layout keeps the bf16 copy, whose padding rows are zeroed)
  b.x_perm = layer_gathers(c) || mx_dispatch_fused(c) ? nullptr : w.take<void>(P * row);
  b.y_perm = c.expert_kind == MOE_EXPERT_IDENTITY ? nullptr : w.take<void>(P * row);
  b.perm = carve_permute(c, w);
  b.h_mid = carve_ffn(c, w);
  b.pair_cnt = layer_fuses_combine(c) ? w.take<int32_t>(static_cast<size_t>(c.T) * pair_entries(c) * 4) : nullptr;
  b.preact = layer_saves_preact(c) ? w.take<void>(P * 2 * static_cast<size_t>(c.d_ff) * 2) : nullptr;
  return b;
}

// Backward scratch. ppad_max bounds the padded column count of the
// transposed activations: every expert's rows rounded up to 64.
struct BackwardBufs {
  void *dy_perm, *dh_mid, *dgu, *dx_perm;
  float* ds;
  int32_t* col_off;
  void *dy_perm_t, *h_mid_t, *dgu_t, *x_perm_t;
  float* router_scratch;
  int ppad_max;
};

int ppad_max(const moe_config& c) {
  return static_cast<int>((perm_rows(c) + 63) / 64 * 64 + 64 * static_cast<size_t>(c.E));
}

BackwardBufs carve_backward(const moe_config& c, Carver& w) {
  const size_t P = perm_rows(c), A = static_cast<size_t>(c.T) * c.k;
  const size_t d = c.d, F = c.d_ff;
  BackwardBufs b;
  b.ppad_max = ppad_max(c);
  const size_t pp = b.ppad_max;
  b.dy_perm = w.take<void>(P * d * 2);
  b.dh_mid = w.take<void>(P * F * 2);
  b.dgu = w.take<void>(P * 2 * F * 2);
  b.dx_perm = w.take<void>(P * d * 2);
  b.ds = w.take<float>(A * 4);
  b.col_off = w.take<int32_t>((c.E + 1) * 4);
  b.dy_perm_t = w.take<void>(d * pp * 2);
  b.h_mid_t = w.take<void>(F * pp * 2);
  b.dgu_t = w.take<void>(2 * F * pp * 2);
  b.x_perm_t = w.take<void>(d * pp * 2);
  b.router_scratch = w.take<float>(router_wgrad_scratch(c.T, c.E, c.d));
  return b;
}

bool backward_supported(const moe_config& c) {
  return c.dtype == MOE_DTYPE_BF16 && c.expert_kind == MOE_EXPERT_SWIGLU && !layer_gathers(c) && !is_mx(c);
}

size_t ws_size(const moe_config& c, int op) {
  Carver w(nullptr);
  switch (op) {
    case MOE_OP_BACKWARD:
      if (!backward_supported(c)) return 0;
      carve_backward(c, w);
      return w.off;
    case MOE_OP_ROUTE:
      return 0;
    case MOE_OP_PERMUTE:
      carve_permute(c, w);
      return w.off;
    case MOE_OP_GROUPED_FFN:
      if (is_mx(c)) carve_mx(c, w);
      carve_ffn(c, w);
      return w.off;
    case MOE_OP_LAYER:
      if (is_mx(c)) carve_mx(c, w);
      carve_layer(c, w);
      return w.off;
    default:
      return 0;
  }
}

int cuda_rc(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// chunk_counts (may be NULL, bf16 path only): the router also writes the
// expert histogram of every 128-token tile, which the dispatch needs.
int route_impl(const moe_config& c, const void* h, const void* w_router, const float* bias, float* logits,
               int32_t* idx, float* gate, int32_t* chunk_counts, int32_t* status, cudaStream_t s) {
  if (c.T == 0) return MOE_OK;
  if (c.dtype == MOE_DTYPE_F32)
    return cuda_rc(launch_router_f32(static_cast<const float*>(h), static_cast<const float*>(w_router), c.T, c.d, c.E,
                                     c.k, bias, logits, idx, gate, status, s));
  const int npad = router_npad(c.E);
  CUtensorMap tm_h, tm_w;
  int rc = make_map(&tm_h, h, c.T, c.d, kTileM);
  if (rc == MOE_OK) rc = make_map(&tm_w, w_router, c.E, c.d, npad);
  if (rc != MOE_OK) return rc;
  return cuda_rc(
      launch_router_tc(tm_h, tm_w, c.T, c.d, c.E, c.k, npad, bias, logits, idx, gate, chunk_counts, status, s));
}

// pdl (here and in ffn_impl): the first kernel may launch as a programmatic
// dependent of the previous kernel on the stream, which must belong to the
// same library call.
int permute_impl(const moe_config& c, const void* h, const int32_t* idx, int32_t* routed, int32_t* kept,
                 int32_t* offsets, int32_t* dest_row, int32_t* perm_src, void* x_perm, const PermuteScratch& p,
                 bool counts_ready, bool copy_rows, bool pdl, int32_t* status, cudaStream_t s,
                 int32_t* pair_cnt = nullptr, void* y_zero = nullptr) {
  return cuda_rc(launch_permute(h, static_cast<size_t>(c.d) * elem_bytes(c), idx, c.T, c.k, c.E, c.capacity,
                                c.layout == MOE_LAYOUT_PADDED, copy_rows, p.chunk_counts, p.chunk_base, routed, kept,
                                offsets, dest_row, perm_src, x_perm, counts_ready, pdl, status, s, pair_cnt,
                                pair_cnt != nullptr ? pair_entries(c) : 0, y_zero));
}

// The combine done by the down projection (launch_grouped_gemm_combine).
struct FusedCombine {
  const int32_t* perm_src;
  const int32_t* dest_row;
  const float* gate;
  int32_t* pair_cnt;
  void* y;
};

// gather_src / gather_rows (bf16 SwiGLU single tiles only; NULL otherwise):
// GEMM1 reads A row r as gather_src[gather_rows[r]] instead of x_perm[r].
// MXFP8 experts: quantise the permuted rows into the padded layout, GEMM1
// with SwiGLU and the MXFP8 quantisation of h_mid in its epilogue, GEMM2 to
// bf16 y_perm. w13 and w_down are the blobs of moe_pack_weights_mxfp8; the
// counters were zeroed by the caller.
// The layer's MXFP8 dispatch: the token rows go from h straight into the
// padded quantised layout (no bf16 x_perm).
struct MxDispatch {
  const void* h;
  const int32_t* idx;
  const int32_t* dest_row;
};

// The layer's quantising dispatch (part of its dispatch stage).
int mx_dispatch_impl(const moe_config& c, const MxDispatch& md, const int32_t* offsets, const MxBufs& m,
                     int32_t* status, cudaStream_t s) {
  return cuda_rc(launch_mx_dispatch(md.h, c.T, c.d, c.k, md.idx, md.dest_row, offsets, c.E, m.xq, m.xsf,
                                    m.row_blocks, m.counters, status, true, s));
}

// x_quantized: the token rows are already in m.xq (the layer's quantising
// dispatch ran); else x_perm is quantised first.
int ffn_mx_impl(const moe_config& c, const void* x_perm, const int32_t* offsets, const void* w13, const void* w_down,
                void* y_perm, const MxBufs& m, bool pdl, int32_t* status, cudaStream_t s, bool x_quantized) {
  const int F = c.d_ff, d = c.d, E = c.E;
  const MxBlob b13 = mx_blob(c, 0), bd = mx_blob(c, 1);
  const uint8_t* w13q = static_cast<const uint8_t*>(w13);
  const uint8_t* wdq = static_cast<const uint8_t*>(w_down);
  cudaError_t e = cudaSuccess;
  if (!x_quantized)
    e = launch_mx_quantize(x_perm, m.pad_rows, d, offsets, E, m.xq, m.xsf, m.row_blocks, m.counters, status, pdl, s);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  CUtensorMap a1, b1, a2, b2, d1, d2;
  int rc = make_map_u8(&a1, m.xq, m.pad_rows, d, 128);
  if (rc == MOE_OK) rc = make_map_u8(&b1, w13q, b13.rows, d, 256);
  if (rc == MOE_OK) rc = make_map_u8(&a2, m.hq, m.pad_rows, F, 128);
  if (rc == MOE_OK) rc = make_map_u8(&b2, wdq, bd.rows, F, 256);
  if (rc == MOE_OK) rc = make_map_store_u8(&d1, m.hq, m.pad_rows, F);
  if (rc == MOE_OK) rc = make_map_store(&d2, y_perm, perm_rows(c), d);
  if (rc != MOE_OK) return rc;
  e = launch_grouped_gemm_mx(a1, b1, true, offsets, E, d, 2 * F, F, m.xsf, m.row_blocks, w13q + b13.q_bytes, m.hq,
                             m.hsf, F, m.counters + 2, nullptr, 0, status, true, s, &d1);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  e = launch_grouped_gemm_mx(a2, b2, false, offsets, E, F, d, d, m.hsf, m.row_blocks, wdq + bd.q_bytes, nullptr,
                             nullptr, 0, nullptr, y_perm, d, status, true, s, &d2);
  return cuda_rc(e);
}

int ffn_impl(const moe_config& c, const void* x_perm, const int32_t* offsets, const void* w13, const void* w_down,
             void* y_perm, void* h_mid, const void* gather_src, const int32_t* gather_rows, bool pdl,
             int32_t* status, cudaStream_t s, const MxBufs* mx = nullptr, const FusedCombine* fc = nullptr,
             bool mx_x_quantized = false, void* preact = nullptr) {
  const int rows_max = static_cast<int>(perm_rows(c));
  if (rows_max == 0) return MOE_OK;
  if (is_mx(c)) return ffn_mx_impl(c, x_perm, offsets, w13, w_down, y_perm, *mx, pdl, status, s, mx_x_quantized);
  if (c.expert_kind != MOE_EXPERT_SWIGLU)
    return cuda_rc(launch_scale_rows(c.dtype, c.expert_kind, x_perm, offsets, y_perm, rows_max, c.d, c.E, s));
  if (c.dtype == MOE_DTYPE_F32)
    return cuda_rc(launch_ffn_f32(static_cast<const float*>(x_perm), offsets, static_cast<const float*>(w13),
                                  static_cast<const float*>(w_down), static_cast<float*>(h_mid),
                                  static_cast<float*>(y_perm), rows_max, c.d, c.d_ff, c.E, s));
  const int F = c.d_ff, d = c.d, E = c.E;
  // Tile shape: single-CTA 128x256 tiles unless the caller asks for CTA pairs
  // (256x256, each CTA of the pair stages half of the B tile).
  const bool pair = use_pair_tiles(c);
  CUtensorMap a1, b1, a2, b2, d1, d2;
  const bool gather = gather_rows != nullptr && !pair;
  int rc = gather ? make_map(&a1, gather_src, c.T, d, 1) : make_map(&a1, x_perm, rows_max, d, kTileM);
  if (rc == MOE_OK) rc = make_map(&b1, w13, static_cast<uint64_t>(E) * 2 * F, d, pair ? 128 : kGemmTileN);
  if (rc == MOE_OK) rc = make_map(&a2, h_mid, rows_max, F, kTileM);
  if (rc == MOE_OK) rc = make_map(&b2, w_down, static_cast<uint64_t>(E) * d, F, pair ? 128 : kGemmTileN);
  if (rc == MOE_OK) rc = make_map_store(&d1, h_mid, rows_max, F);
  if (rc == MOE_OK) rc = make_map_store(&d2, y_perm, rows_max, d);
  if (rc != MOE_OK) return rc;
  cudaError_t e =
      pair ? launch_grouped_gemm_pair(a1, b1, true, offsets, E, d, 2 * F, F / 128, F, F, h_mid, status, pdl, s, &d1)
           : launch_grouped_gemm_tc(a1, b1, true, offsets, E, d, 2 * F, F / 128, F, F, h_mid,
                                    gather ? gather_rows : nullptr, status, pdl, s, preact, &d1);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  const int n2 = (d + kGemmTileN - 1) / kGemmTileN;
  if (fc != nullptr)
    e = launch_grouped_gemm_combine(a2, b2, offsets, E, F, d, y_perm, fc->perm_src, fc->dest_row, fc->gate,
                                    fc->pair_cnt, fc->y, c.k, status, true, s);
  else
    e = pair ? launch_grouped_gemm_pair(a2, b2, false, offsets, E, F, d, n2, d, d, y_perm, status, true, s, &d2)
             : launch_grouped_gemm_tc(a2, b2, false, offsets, E, F, d, n2, d, d, y_perm, nullptr, status, true, s,
                                      nullptr, &d2);
  return cuda_rc(e);
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

int32_t moe_version(void) { return (1 << 16) | 2; }

int32_t moe_gemm_tiles_used(const moe_config* cfg, int32_t* tiles) {
  if (tiles == nullptr) return MOE_ERR_INVALID_ARG;
  const int rc = check_cfg(cfg);
  if (rc != MOE_OK) return rc;
  *tiles = use_pair_tiles(*cfg) ? MOE_GEMM_TILES_PAIR : MOE_GEMM_TILES_SINGLE;
  return MOE_OK;
}

const char* moe_status_string(int32_t code) {
  switch (code) {
    case MOE_OK:
      return "ok";
    case MOE_ERR_INVALID_ARG:
      return "invalid argument";
    case MOE_ERR_UNSUPPORTED:
      return "unsupported configuration or misaligned pointer";
    case MOE_ERR_WORKSPACE:
      return "workspace too small or misaligned";
    case MOE_ERR_CUDA:
      return "CUDA launch or runtime call failed";
    case MOE_ERR_NO_DEVICE:
      return "no usable sm_100 device or driver entry point";
    default:
      return "unknown status";
  }
}

size_t moe_workspace_size(const moe_config* cfg, int32_t op) {
  if (check_cfg(cfg) != MOE_OK) return 0;
  return ws_size(*cfg, op);
}

int32_t moe_pack_weights(const moe_config* cfg, const void* w_gate, const void* w_up, void* w13_packed,
                         moe_stream_t stream) {
  int rc = check_cfg(cfg);
  if (rc != MOE_OK) return rc;
  if (cfg->expert_kind != MOE_EXPERT_SWIGLU) return MOE_ERR_INVALID_ARG;
  if (!w_gate || !w_up || !w13_packed) return MOE_ERR_INVALID_ARG;
  if (!aligned(w_gate, 16) || !aligned(w_up, 16) || !aligned(w13_packed, 16)) return MOE_ERR_UNSUPPORTED;
  return cuda_rc(launch_pack_w13(w_gate, w_up, w13_packed, cfg->E, cfg->d_ff,
                                 static_cast<size_t>(cfg->d) * elem_bytes(*cfg), static_cast<cudaStream_t>(stream)));
}

int32_t moe_route(const moe_config* cfg, const void* h, const void* w_router, const float* bias, float* logits_out,
                  int32_t* topk_idx, float* topk_gate, void* workspace, size_t ws_bytes, int32_t* status_dev,
                  moe_stream_t stream) {
  (void)workspace;
  (void)ws_bytes;
  int rc = check_cfg(cfg);
  if (rc != MOE_OK) return rc;
  const bool tok = cfg->T > 0;  // token-sized arrays may be NULL when T == 0
  if (!w_router || (tok && (!h || !topk_idx || !topk_gate))) return MOE_ERR_INVALID_ARG;
  if (!aligned(h, 16) || !aligned(w_router, 16) || !aligned(topk_idx, 4) || !aligned(topk_gate, 4) ||
      !aligned(bias, 4) || !aligned(logits_out, 4) || !aligned(status_dev, 4))
    return MOE_ERR_UNSUPPORTED;
  return route_impl(*cfg, h, w_router, bias, logits_out, topk_idx, topk_gate, nullptr, status_dev,
                    static_cast<cudaStream_t>(stream));
}

int32_t moe_permute(const moe_config* cfg, const void* h, const int32_t* topk_idx, int32_t* routed_counts,
                    int32_t* counts, int32_t* offsets, int32_t* dest_row, int32_t* perm_src, void* x_perm,
                    void* workspace, size_t ws_bytes, int32_t* status_dev, moe_stream_t stream) {
  int rc = check_cfg(cfg);
  if (rc != MOE_OK) return rc;
  const bool tok = cfg->T > 0;  // token-sized arrays may be NULL when T == 0
  if (!routed_counts || !counts || !offsets || (tok && (!h || !topk_idx || !dest_row || !perm_src || !x_perm)))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(h, 16) || !aligned(x_perm, 16) || !aligned(topk_idx, 4) || !aligned(routed_counts, 4) ||
      !aligned(counts, 4) || !aligned(offsets, 4) || !aligned(dest_row, 4) || !aligned(perm_src, 4) ||
      !aligned(status_dev, 4))
    return MOE_ERR_UNSUPPORTED;
  const size_t need = ws_size(*cfg, MOE_OP_PERMUTE);
  if (ws_bytes < need || (need > 0 && (!workspace || !aligned(workspace, 16)))) return MOE_ERR_WORKSPACE;
  Carver w(workspace);
  const PermuteScratch p = carve_permute(*cfg, w);
  return permute_impl(*cfg, h, topk_idx, routed_counts, counts, offsets, dest_row, perm_src, x_perm, p, false,
                      true, false, status_dev, static_cast<cudaStream_t>(stream));
}

int32_t moe_grouped_ffn(const moe_config* cfg, const void* x_perm, const int32_t* offsets, const void* w13_packed,
                        const void* w_down, void* y_perm, void* workspace, size_t ws_bytes, int32_t* status_dev,
                        moe_stream_t stream) {
  int rc = check_cfg(cfg);
  if (rc != MOE_OK) return rc;
  const bool swiglu = cfg->expert_kind == MOE_EXPERT_SWIGLU;
  const bool tok = cfg->T > 0;  // token-sized arrays may be NULL when T == 0
  if (!offsets || (tok && (!x_perm || !y_perm)) || (swiglu && (!w13_packed || !w_down))) return MOE_ERR_INVALID_ARG;
  if (!aligned(x_perm, 16) || !aligned(y_perm, 16) || !aligned(offsets, 4) || !aligned(status_dev, 4) ||
      (swiglu && (!aligned(w13_packed, 16) || !aligned(w_down, 16))))
    return MOE_ERR_UNSUPPORTED;
  const size_t need = ws_size(*cfg, MOE_OP_GROUPED_FFN);
  if (ws_bytes < need || (need > 0 && (!workspace || !aligned(workspace, 16)))) return MOE_ERR_WORKSPACE;
  Carver w(workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  MxBufs mx{};
  if (is_mx(*cfg)) {
    mx = carve_mx(*cfg, w);
    if (cudaMemsetAsync(mx.counters, 0, 16, s) != cudaSuccess) return MOE_ERR_CUDA;
  }
  void* h_mid = carve_ffn(*cfg, w);
  return ffn_impl(*cfg, x_perm, offsets, w13_packed, w_down, y_perm, h_mid, nullptr, nullptr, false, status_dev, s,
                  &mx);
}

int32_t moe_unpermute_combine(const moe_config* cfg, const void* y_perm, const int32_t* dest_row,
                              const float* topk_gate, void* y, int32_t* status_dev, moe_stream_t stream) {
  (void)status_dev;
  int rc = check_cfg(cfg);
  if (rc != MOE_OK) return rc;
  if (cfg->T > 0 && (!y_perm || !dest_row || !topk_gate || !y)) return MOE_ERR_INVALID_ARG;
  if (!aligned(y_perm, 16) || !aligned(y, 16) || !aligned(dest_row, 4) || !aligned(topk_gate, 4) ||
      !aligned(status_dev, 4))
    return MOE_ERR_UNSUPPORTED;
  return cuda_rc(
      launch_combine(cfg->dtype, y_perm, dest_row, topk_gate, y, cfg->T, cfg->k, cfg->d, false,
                     static_cast<cudaStream_t>(stream), status_dev));
}

int32_t moe_layer_forward(const moe_config* cfg, const void* h, const void* w_router, const float* bias,
                          const void* w13_packed, const void* w_down, void* y, int32_t* topk_idx, float* topk_gate,
                          int32_t* routed_counts, int32_t* counts, void* workspace, size_t ws_bytes,
                          int32_t* status_dev, moe_stream_t stream) {
  return moe_layer_forward_timed(cfg, h, w_router, bias, w13_packed, w_down, y, topk_idx, topk_gate, routed_counts,
                                 counts, workspace, ws_bytes, status_dev, stream, nullptr);
}

int32_t moe_layer_forward_timed(const moe_config* cfg, const void* h, const void* w_router, const float* bias,
                                const void* w13_packed, const void* w_down, void* y, int32_t* topk_idx,
                                float* topk_gate, int32_t* routed_counts, int32_t* counts, void* workspace,
                                size_t ws_bytes, int32_t* status_dev, moe_stream_t stream,
                                void* const* stage_events) {
  int rc = check_cfg(cfg);
  if (rc != MOE_OK) return rc;
  const moe_config& c = *cfg;
  const bool swiglu = c.expert_kind == MOE_EXPERT_SWIGLU;
  if (!w_router || (c.T > 0 && (!h || !y)) || (swiglu && (!w13_packed || !w_down))) return MOE_ERR_INVALID_ARG;
  if (!aligned(h, 16) || !aligned(w_router, 16) || !aligned(y, 16) || !aligned(bias, 4) || !aligned(topk_idx, 4) ||
      !aligned(topk_gate, 4) || !aligned(routed_counts, 4) || !aligned(counts, 4) || !aligned(status_dev, 4) ||
      (swiglu && (!aligned(w13_packed, 16) || !aligned(w_down, 16))))
    return MOE_ERR_UNSUPPORTED;
  const size_t need = ws_size(c, MOE_OP_LAYER);
  if (ws_bytes < need || (need > 0 && (!workspace || !aligned(workspace, 16)))) return MOE_ERR_WORKSPACE;
  Carver w(workspace);
  MxBufs mx{};
  if (is_mx(c)) mx = carve_mx(c, w);
  LayerBufs b = carve_layer(c, w);
  if (topk_idx) b.idx = topk_idx;
  if (topk_gate) b.gate = topk_gate;
  if (routed_counts) b.routed = routed_counts;
  if (counts) b.kept = counts;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  auto mark = [&](int i) {
    if (stage_events == nullptr || stage_events[i] == nullptr) return MOE_OK;
    return cuda_rc(cudaEventRecord(static_cast<cudaEvent_t>(stage_events[i]), s));
  };
  if (is_mx(c) && cudaMemsetAsync(mx.counters, 0, 16, s) != cudaSuccess) return MOE_ERR_CUDA;
  if ((rc = mark(0)) != MOE_OK) return rc;
  // the bf16 router also writes the per-tile expert histogram the dispatch needs
  const bool router_counts = c.dtype == MOE_DTYPE_BF16;
  rc = route_impl(c, h, w_router, bias, nullptr, b.idx, b.gate, router_counts ? b.perm.chunk_counts : nullptr,
                  status_dev, s);
  if (rc != MOE_OK || (rc = mark(1)) != MOE_OK) return rc;
  // after the router, every kernel of the layer launches as a programmatic
  // dependent of the one before it, so its launch and prologue overlap the
  // previous kernel's tail
  const bool gather = layer_gathers(c);
  const bool fused = b.pair_cnt != nullptr;
  rc = permute_impl(c, h, b.idx, b.routed, b.kept, b.offsets, b.dest_row, b.perm_src, b.x_perm, b.perm,
                    router_counts, b.x_perm != nullptr, true, status_dev, s, b.pair_cnt, fused ? y : nullptr);
  // MXFP8 (compact): the rows go from h straight into the quantised layout, as part of the dispatch
  const bool mx_disp = mx_dispatch_fused(c) && perm_rows(c) > 0;
  if (rc == MOE_OK && mx_disp) rc = mx_dispatch_impl(c, MxDispatch{h, b.idx, b.dest_row}, b.offsets, mx, status_dev, s);
  if (rc != MOE_OK || (rc = mark(2)) != MOE_OK) return rc;
  const void* y_src = b.x_perm;
  const FusedCombine fc{b.perm_src, b.dest_row, b.gate, b.pair_cnt, y};
  if (c.expert_kind != MOE_EXPERT_IDENTITY) {
    rc = ffn_impl(c, b.x_perm, b.offsets, w13_packed, w_down, b.y_perm, b.h_mid, gather ? h : nullptr,
                  gather ? b.perm_src : nullptr, true, status_dev, s, &mx, fused ? &fc : nullptr, mx_disp,
                  b.preact);
    if (rc != MOE_OK) return rc;
    y_src = b.y_perm;
  }
  if ((rc = mark(3)) != MOE_OK) return rc;
  if (!fused) {
    rc = cuda_rc(launch_combine(c.dtype, y_src, b.dest_row, b.gate, y, c.T, c.k, c.d, true, s, status_dev));
    if (rc != MOE_OK) return rc;
  }
  return mark(4);
}

int32_t moe_debug_stall_next_gemms(int32_t n) {
  if (n < 0) return MOE_ERR_INVALID_ARG;
  debug_stall_next_gemms(n);
  return MOE_OK;
}

int32_t moe_mxfp8_quantize(const void* x, int32_t rows, int32_t cols, void* q, void* sf, uint32_t* counts,
                           int32_t* status_dev, moe_stream_t stream) {
  if (rows < 0 || cols <= 0) return MOE_ERR_INVALID_ARG;
  if (cols % 128 != 0) return MOE_ERR_UNSUPPORTED;
  if (rows > 0 && (!x || !q || !sf)) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(q, 16) || !aligned(counts, 4) || !aligned(status_dev, 4))
    return MOE_ERR_UNSUPPORTED;
  return cuda_rc(launch_mx_quantize(x, rows, cols, nullptr, 0, q, sf, (rows + 127) / 128, counts, status_dev, false,
                                    static_cast<cudaStream_t>(stream)));
}

size_t moe_mxfp8_weights_size(const moe_config* cfg, int32_t which) {
  if (check_cfg(cfg) != MOE_OK || cfg->dtype != MOE_DTYPE_BF16 || cfg->expert_kind != MOE_EXPERT_SWIGLU ||
      (which != 0 && which != 1))
    return 0;
  const MxBlob b = mx_blob(*cfg, which);
  return b.q_bytes + b.sf_bytes;
}

int32_t moe_pack_weights_mxfp8(const moe_config* cfg, const void* w13_packed, const void* w_down, void* w13_mx,
                               void* w_down_mx, uint32_t* counts, moe_stream_t stream) {
  int rc = check_cfg(cfg);
  if (rc != MOE_OK) return rc;
  const moe_config& c = *cfg;
  if (c.dtype != MOE_DTYPE_BF16 || c.expert_kind != MOE_EXPERT_SWIGLU) return MOE_ERR_UNSUPPORTED;
  if (!w13_packed || !w_down || !w13_mx || !w_down_mx) return MOE_ERR_INVALID_ARG;
  if (!aligned(w13_packed, 16) || !aligned(w_down, 16) || !aligned(w13_mx, 256) || !aligned(w_down_mx, 256) ||
      !aligned(counts, 4))
    return MOE_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const void* src[2] = {w13_packed, w_down};
  void* dst[2] = {w13_mx, w_down_mx};
  for (int which = 0; which < 2; ++which) {
    const MxBlob b = mx_blob(c, which);
    uint8_t* q = static_cast<uint8_t*>(dst[which]);
    if (cudaMemsetAsync(q + b.q_bytes, 0, b.sf_bytes, s) != cudaSuccess) return MOE_ERR_CUDA;
    const cudaError_t e = launch_mx_quantize(src[which], static_cast<int>(b.rows), static_cast<int>(b.cols), nullptr,
                                             0, q, q + b.q_bytes, b.row_blocks, counts, nullptr, false, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

int32_t moe_pack_weights_backward(const moe_config* cfg, const void* w13_packed, const void* w_down, void* w13_t,
                                  void* w_down_t, moe_stream_t stream) {
  int rc = check_cfg(cfg);
  if (rc != MOE_OK) return rc;
  const moe_config& c = *cfg;
  if (c.dtype != MOE_DTYPE_BF16 || c.expert_kind != MOE_EXPERT_SWIGLU) return MOE_ERR_UNSUPPORTED;
  if (!w13_packed || !w_down || !w13_t || !w_down_t) return MOE_ERR_INVALID_ARG;
  if (!aligned(w13_packed, 16) || !aligned(w_down, 16) || !aligned(w13_t, 16) || !aligned(w_down_t, 16))
    return MOE_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_transpose_batched(w13_packed, c.E, 2 * c.d_ff, c.d, w13_t, s);
  if (e == cudaSuccess) e = launch_transpose_batched(w_down, c.E, c.d, c.d_ff, w_down_t, s);
  return cuda_rc(e);
}

int32_t moe_layer_backward(const moe_config* cfg, const void* h, const void* w_router, const void* w13_packed,
                           const void* w13_t, const void* w_down_t, const void* dy, void* dh, float* dw_router,
                           float* dbias, float* dw13, float* dw_down, const void* fwd_workspace, size_t fwd_ws_bytes,
                           void* workspace, size_t ws_bytes, int32_t* status_dev, moe_stream_t stream) {
  int rc = check_cfg(cfg);
  if (rc != MOE_OK) return rc;
  const moe_config& c = *cfg;
  if (!backward_supported(c)) return MOE_ERR_UNSUPPORTED;
  if (!w_router || !w13_packed || !w13_t || !w_down_t || !dw_router || !dw13 || !dw_down || !fwd_workspace ||
      (c.T > 0 && (!h || !dy || !dh)))
    return MOE_ERR_INVALID_ARG;
  if (!aligned(h, 16) || !aligned(w_router, 16) || !aligned(w13_packed, 16) || !aligned(w13_t, 16) ||
      !aligned(w_down_t, 16) || !aligned(dy, 16) || !aligned(dh, 16) || !aligned(dw_router, 16) ||
      !aligned(dbias, 4) || !aligned(dw13, 16) || !aligned(dw_down, 16) || !aligned(status_dev, 4))
    return MOE_ERR_UNSUPPORTED;
  if (fwd_ws_bytes < ws_size(c, MOE_OP_LAYER) || !aligned(fwd_workspace, 16)) return MOE_ERR_WORKSPACE;
  const size_t need = ws_size(c, MOE_OP_BACKWARD);
  if (ws_bytes < need || !workspace || !aligned(workspace, 16)) return MOE_ERR_WORKSPACE;
  Carver fw(const_cast<void*>(fwd_workspace));
  const LayerBufs f = carve_layer(c, fw);
  Carver bw(workspace);
  const BackwardBufs b = carve_backward(c, bw);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int E = c.E, d = c.d, F = c.d_ff, T = c.T, k = c.k;
  const int P = static_cast<int>(perm_rows(c));
  cudaError_t e = cudaSuccess;
  // 1. combine: dy_perm rows and the gate gradient through the softmax over the picks.
  //    In the padded layout the padding rows take part in every expert GEMM
  //    below (their x_perm and h_mid rows are zero), so their dy_perm rows are
  //    zeroed first.
  if (c.layout == MOE_LAYOUT_PADDED && P > 0) {
    e = cudaMemsetAsync(b.dy_perm, 0, static_cast<size_t>(P) * d * 2, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
  }
  e = launch_combine_bwd(dy, f.y_perm, f.dest_row, f.gate, b.dy_perm, b.ds, T, k, d, s);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  if (P > 0) {
    CUtensorMap ta, tb;
    e = launch_col_offsets(f.offsets, E, b.col_off, s);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    rc = make_map(&ta, b.dy_perm, P, d, kTileM);
    if (rc == MOE_OK) rc = make_map(&tb, w_down_t, static_cast<uint64_t>(E) * F, d, kGemmTileN);
    if (rc != MOE_OK) return rc;
    if (f.preact != nullptr) {
      // 2+3. dL/dh_mid = dy_perm W_down (per expert) with the SwiGLU backward in
      //      the epilogue, from the pre-activations the forward kept: writes
      //      dgu and its transposed copy; no recompute of the gate/up GEMM
      CUtensorMap tdg;
      rc = make_map_store(&tdg, b.dgu, P, 2 * F);
      if (rc != MOE_OK) return rc;
      e = launch_grouped_gemm_dh_swiglu_bwd(ta, tb, f.offsets, E, d, F, f.preact, b.dgu, b.dgu_t, b.col_off,
                                            b.ppad_max, status_dev, false, s, &tdg);
      if (e != cudaSuccess) return MOE_ERR_CUDA;
    } else {
      // 2. dh_mid = dy_perm W_down (per expert), B = W_down^T rows
      CUtensorMap td;
      rc = make_map_store(&td, b.dh_mid, P, F);
      if (rc != MOE_OK) return rc;
      e = launch_grouped_gemm_tc(ta, tb, false, f.offsets, E, d, F, (F + kGemmTileN - 1) / kGemmTileN, F, F,
                                 b.dh_mid, nullptr, status_dev, false, s, nullptr, &td);
      if (e != cudaSuccess) return MOE_ERR_CUDA;
      // 3. gate/up pre-activations recomputed from x_perm; SwiGLU backward in the
      //    epilogue, which also writes dgu transposed for the weight gradient
      rc = make_map(&ta, f.x_perm, P, d, kTileM);
      if (rc == MOE_OK) rc = make_map(&tb, w13_packed, static_cast<uint64_t>(E) * 2 * F, d, kGemmTileN);
      if (rc != MOE_OK) return rc;
      CUtensorMap tdg;
      if (rc == MOE_OK) rc = make_map_store(&tdg, b.dgu, P, 2 * F);
      if (rc != MOE_OK) return rc;
      e = launch_grouped_gemm_swiglu_bwd(ta, tb, f.offsets, E, d, F, b.dgu, b.dh_mid, b.dgu_t, b.col_off,
                                         b.ppad_max, status_dev, false, s, &tdg);
      if (e != cudaSuccess) return MOE_ERR_CUDA;
    }
    // 4. dx_perm = dgu w13 (per expert), B = w13^T rows
    CUtensorMap tdx;
    rc = make_map(&ta, b.dgu, P, 2 * F, kTileM);
    if (rc == MOE_OK) rc = make_map(&tb, w13_t, static_cast<uint64_t>(E) * d, 2 * F, kGemmTileN);
    if (rc == MOE_OK) rc = make_map_store(&tdx, b.dx_perm, P, d);
    if (rc != MOE_OK) return rc;
    e = launch_grouped_gemm_tc(ta, tb, false, f.offsets, E, 2 * F, d, (d + kGemmTileN - 1) / kGemmTileN, d, d,
                               b.dx_perm, nullptr, status_dev, false, s, nullptr, &tdx);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
  }
  // 5. dh: expert rows back to their tokens plus the router-score term
  e = launch_token_grad(b.dx_perm, f.dest_row, f.idx, b.ds, w_router, dh, T, k, d, s);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  // 6. router weights and bias
  e = launch_router_wgrad(h, f.idx, b.ds, T, k, d, E, dw_router, dbias, b.router_scratch, s);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  // 7. expert weight gradients: operands transposed to [channels, rows], each
  //    expert's rows at a 64-aligned column offset, reduced per expert
  if (P == 0) e = launch_col_offsets(f.offsets, E, b.col_off, s);  // else done before step 3
  if (e == cudaSuccess) e = launch_transpose_grouped(b.dy_perm, d, f.offsets, b.col_off, E, b.ppad_max, b.dy_perm_t, s);
  if (e == cudaSuccess) e = launch_transpose_grouped(f.h_mid, F, f.offsets, b.col_off, E, b.ppad_max, b.h_mid_t, s);
  if (e == cudaSuccess) e = launch_transpose_grouped(f.x_perm, d, f.offsets, b.col_off, E, b.ppad_max, b.x_perm_t, s);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  CUtensorMap ta, tb;
  rc = make_map(&ta, b.dy_perm_t, d, b.ppad_max, kTileM);
  if (rc == MOE_OK) rc = make_map(&tb, b.h_mid_t, F, b.ppad_max, kGemmTileN);
  if (rc != MOE_OK) return rc;
  e = launch_grouped_gemm_wgrad(ta, tb, b.col_off, E, d, F, dw_down, status_dev, false, s);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  rc = make_map(&ta, b.dgu_t, 2 * F, b.ppad_max, kTileM);
  if (rc == MOE_OK) rc = make_map(&tb, b.x_perm_t, d, b.ppad_max, kGemmTileN);
  if (rc != MOE_OK) return rc;
  e = launch_grouped_gemm_wgrad(ta, tb, b.col_off, E, 2 * F, d, dw13, status_dev, false, s);
  return cuda_rc(e);
}

}  // extern "C"
