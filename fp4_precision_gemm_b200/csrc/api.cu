// The C ABI (include/fp8q.h): argument validation, the per-device scratch pool, TMA
// descriptor encoding and kernel launches.  Every entry point validates on the host and
// either enqueues its kernels on the caller's stream or returns an error without launching.
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/fp8q.h"
#include "kernels.h"

using namespace fp8q;

namespace {

constexpr int kMaxDevices = 64;
constexpr int kAmaxSlots = 1024;  // rotating 8-byte slots for global amax words

struct DeviceScratch {
  // [0] status word, [64 + 2*i] amax slot i.  Published with release order after num_sms
  // is set, read with acquire order, so a thread that sees the pointer sees the pool whole.
  std::atomic<uint32_t*> base{nullptr};
  std::atomic<uint32_t> next{0};
  int num_sms = 0;
};

DeviceScratch g_scratch[kMaxDevices];
std::mutex g_mutex;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

fp8q_status from_cuda(cudaError_t e) { return e == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA; }

// Returns the current device's scratch pool, allocating it on first use.
fp8q_status scratch(DeviceScratch** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FP8Q_ERR_CUDA;
  DeviceScratch& d = g_scratch[dev];
  if (d.base.load(std::memory_order_acquire) == nullptr) {
    std::lock_guard<std::mutex> lock(g_mutex);
    if (d.base.load(std::memory_order_relaxed) == nullptr) {
      int sms = 0;
      if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return FP8Q_ERR_CUDA;
      void* p = nullptr;
      const size_t bytes = (64 + 2 * kAmaxSlots) * sizeof(uint32_t);
      if (cudaMalloc(&p, bytes) != cudaSuccess) return FP8Q_ERR_CUDA;
      if (cudaMemset(p, 0, bytes) != cudaSuccess) return FP8Q_ERR_CUDA;
      d.num_sms = sms;
      d.base.store(static_cast<uint32_t*>(p), std::memory_order_release);
    }
  }
  *out = &d;
  return FP8Q_OK;
}

// Next pair of amax words, zeroed on `stream` before use.
fp8q_status amax_slot(DeviceScratch* d, cudaStream_t s, uint32_t** out) {
  const uint32_t i = d->next.fetch_add(1) % kAmaxSlots;
  uint32_t* p = d->base.load(std::memory_order_acquire) + 64 + 2 * i;
  if (cudaMemsetAsync(p, 0, 2 * sizeof(uint32_t), s) != cudaSuccess) return FP8Q_ERR_CUDA;
  *out = p;
  return FP8Q_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// 2-D tensor map: `inner` x `outer` elements, row stride `stride_bytes`, box inner x outer.
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t inner, uint64_t outer,
              uint64_t stride_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {stride_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t sf_bytes(int64_t outer, int64_t sf_cols, fp8q_sf_layout layout) {
  if (layout == FP8Q_SF_MMA_TILED) return (size_t)((outer + 127) / 128 * 128) * (size_t)((sf_cols + 3) / 4 * 4);
  return (size_t)outer * (size_t)sf_cols;
}

}  // namespace

extern "C" {

const char* fp8q_status_string(fp8q_status s) {
  switch (s) {
    case FP8Q_OK: return "ok";
    case FP8Q_ERR_NULL: return "required pointer is NULL";
    case FP8Q_ERR_SHAPE: return "size, stride or block-multiple requirement not met";
    case FP8Q_ERR_ALIGN: return "pointer or leading dimension not 16-byte aligned";
    case FP8Q_ERR_UNSUPPORTED: return "unsupported combination";
    case FP8Q_ERR_CUDA: return "CUDA runtime/driver error";
    case FP8Q_ERR_TIMEOUT: return "a kernel's bounded wait ran out";
    case FP8Q_ERR_DEVICE_ARG: return "an argument read on the device was out of range (clamped)";
  }
  return "unknown status";
}

const char* fp8q_version(void) { return "fp8q 0.1.0 sm_100a"; }

size_t fp8q_sf_bytes(fp8q_recipe recipe, int64_t outer, int64_t inner, fp8q_sf_layout layout) {
  if (outer < 0 || inner < 0) return 0;
  if (recipe == FP8Q_MXFP8) return sf_bytes(outer, inner / 32, layout);
  if (recipe == FP8Q_NVFP4) return sf_bytes(outer, inner / 16, layout);
  return 0;
}

fp8q_status fp8q_get_device_status(void* stream) {
  DeviceScratch* d = nullptr;
  fp8q_status st = scratch(&d);
  if (st != FP8Q_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t word = 0;
  uint32_t* base = d->base.load(std::memory_order_acquire);
  if (cudaMemcpyAsync(&word, base, sizeof(word), cudaMemcpyDeviceToHost, s) != cudaSuccess) return FP8Q_ERR_CUDA;
  if (cudaMemsetAsync(base, 0, sizeof(uint32_t), s) != cudaSuccess) return FP8Q_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return FP8Q_ERR_CUDA;
  return word == 0 ? FP8Q_OK : static_cast<fp8q_status>(word);
}

fp8q_status fp8q_selftest_bounded_wait(uint64_t limit_ns, void* stream) {
  if (limit_ns < 1000ull || limit_ns > 1000000000ull) return FP8Q_ERR_SHAPE;
  DeviceScratch* d = nullptr;
  fp8q_status st = scratch(&d);
  if (st != FP8Q_OK) return st;
  return from_cuda(launch_selftest_wait(d->base.load(std::memory_order_acquire), limit_ns,
                                       static_cast<cudaStream_t>(stream)));
}

fp8q_status fp8q_release_scratch(void) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return FP8Q_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceScratch& d = g_scratch[dev];
  uint32_t* base = d.base.load(std::memory_order_acquire);
  if (base) {
    if (cudaDeviceSynchronize() != cudaSuccess) return FP8Q_ERR_CUDA;
    d.base.store(nullptr, std::memory_order_release);
    if (cudaFree(base) != cudaSuccess) return FP8Q_ERR_CUDA;
  }
  return FP8Q_OK;
}

// ------------------------------------------------------------------ quantization
static fp8q_status check_input(const void* x, int64_t rows, int64_t cols, int64_t ld_x) {
  if (rows < 0 || cols < 0) return FP8Q_ERR_SHAPE;
  if (rows > 0 && cols > 0) {
    if (!x) return FP8Q_ERR_NULL;
    if (ld_x < cols || ld_x % 8 != 0) return FP8Q_ERR_SHAPE;
    if (!aligned16(x)) return FP8Q_ERR_ALIGN;
  }
  if (rows >= (1ll << 31) || cols >= (1ll << 31)) return FP8Q_ERR_SHAPE;
  return FP8Q_OK;
}

static int64_t tiles_of(int64_t rows, int64_t cols) { return ((rows + 127) / 128) * ((cols + 127) / 128); }

}  // extern "C"

namespace {

// Validation and launch parameters of one 1x128 quantization (the rules of
// fp8q_quantize_1x128); `tiles` is 0 when there is nothing to do.
fp8q_status plan_1x128(const void* x, int64_t rows, int64_t cols, int64_t ld_x, uint8_t* q_row, float* s_row,
                       int64_t ld_s_row, uint8_t* q_col, float* s_col, int64_t ld_s_col, TileQuantParams& p,
                       bool& row, bool& col, int64_t& tiles) {
  fp8q_status st = check_input(x, rows, cols, ld_x);
  if (st != FP8Q_OK) return st;
  row = q_row || s_row;
  col = q_col || s_col;
  if (!row && !col) return FP8Q_ERR_NULL;
  if ((row && (!q_row || !s_row)) || (col && (!q_col || !s_col))) return FP8Q_ERR_NULL;
  if (row && (cols % 128 != 0 || ld_s_row < rows || ld_s_row % 4 != 0)) return FP8Q_ERR_SHAPE;
  if (col && (rows % 128 != 0 || cols % 16 != 0 || ld_s_col < cols || ld_s_col % 4 != 0)) return FP8Q_ERR_SHAPE;
  if ((row && !aligned16(q_row)) || (col && !aligned16(q_col))) return FP8Q_ERR_ALIGN;
  p = TileQuantParams{static_cast<const uint16_t*>(x), rows, cols, ld_x, q_row, s_row, ld_s_row,
                      q_col, s_col, ld_s_col, (int)((cols + 127) / 128), 0};
  tiles = (rows == 0 || cols == 0) ? 0 : tiles_of(rows, cols);
  return FP8Q_OK;
}

// The same for one 128x128 quantization (the rules of fp8q_quantize_128x128).
fp8q_status plan_128x128(const void* w, int64_t K, int64_t N, int64_t ld_w, uint8_t* q_t, uint8_t* q, float* s,
                         TileQuantParams& p, int64_t& tiles) {
  fp8q_status st = check_input(w, K, N, ld_w);
  if (st != FP8Q_OK) return st;
  if (!s) return FP8Q_ERR_NULL;
  if (K % 128 != 0 || N % 128 != 0) return FP8Q_ERR_SHAPE;
  if ((q && !aligned16(q)) || (q_t && !aligned16(q_t))) return FP8Q_ERR_ALIGN;
  p = TileQuantParams{static_cast<const uint16_t*>(w), K, N, ld_w, q, s, K / 128, q_t, nullptr, 0,
                      (int)(N / 128), 0};
  tiles = (K == 0 || N == 0) ? 0 : tiles_of(K, N);
  return FP8Q_OK;
}

}  // namespace

extern "C" {

fp8q_status fp8q_quantize_1x128(const void* x, int64_t rows, int64_t cols, int64_t ld_x, uint8_t* q_row,
                                float* s_row, int64_t ld_s_row, uint8_t* q_col, float* s_col, int64_t ld_s_col,
                                void* stream) {
  TileQuantParams p{};
  bool row = false, col = false;
  int64_t tiles = 0;
  fp8q_status st = plan_1x128(x, rows, cols, ld_x, q_row, s_row, ld_s_row, q_col, s_col, ld_s_col, p, row, col, tiles);
  if (st != FP8Q_OK || tiles == 0) return st;
  return from_cuda(launch_tile_quant(kTile1x128, row, col, p, tiles, static_cast<cudaStream_t>(stream)));
}

fp8q_status fp8q_quantize_128x128(const void* w, int64_t K, int64_t N, int64_t ld_w, uint8_t* q_t, uint8_t* q,
                                  float* s, void* stream) {
  TileQuantParams p{};
  int64_t tiles = 0;
  fp8q_status st = plan_128x128(w, K, N, ld_w, q_t, q, s, p, tiles);
  if (st != FP8Q_OK || tiles == 0) return st;
  return from_cuda(launch_tile_quant(kTile128, q != nullptr, q_t != nullptr, p, tiles,
                                     static_cast<cudaStream_t>(stream)));
}

fp8q_status fp8q_quantize_multi(const fp8q_quant_item* items, int32_t n_items, void* stream) {
  if (n_items < 0 || n_items > FP8Q_MAX_QUANT_ITEMS) return FP8Q_ERR_SHAPE;
  if (n_items > 0 && !items) return FP8Q_ERR_NULL;
  TileQuantMulti m{};
  int64_t tiles = 0;
  for (int i = 0; i < n_items; ++i) {   // every item is checked before anything is launched
    const fp8q_quant_item& it = items[i];
    TileQuantParams p{};
    int64_t t = 0;
    int kind;
    fp8q_status st;
    if (it.kind == FP8Q_ITEM_1X128) {
      bool row = false, col = false;
      st = plan_1x128(it.x, it.rows, it.cols, it.ld_x, it.q_row, it.s_row, it.ld_s_row, it.q_col, it.s_col,
                      it.ld_s_col, p, row, col, t);
      kind = row && col ? kMulti1x128Both : row ? kMulti1x128Row : kMulti1x128Col;
    } else if (it.kind == FP8Q_ITEM_128X128) {
      st = plan_128x128(it.x, it.rows, it.cols, it.ld_x, it.q_t, it.q, it.s, p, t);
      kind = it.q && it.q_t ? kMulti128Both : it.q ? kMulti128Row : kMulti128Col;
      if (st == FP8Q_OK && !it.q && !it.q_t) st = FP8Q_ERR_NULL;
    } else {
      return FP8Q_ERR_UNSUPPORTED;
    }
    if (st != FP8Q_OK) return st;
    if (t == 0) continue;
    m.kind[m.n] = kind;
    m.item[m.n] = p;
    m.tile_begin[m.n] = tiles;
    ++m.n;
    tiles += t;
  }
  if (tiles == 0) return FP8Q_OK;
  if (tiles >= (1ll << 31)) return FP8Q_ERR_SHAPE;
  m.tile_begin[m.n] = tiles;
  return from_cuda(launch_tile_quant_multi(m, tiles, static_cast<cudaStream_t>(stream)));
}

fp8q_status fp8q_quantize_128x128_grouped(const void* w, int64_t groups, int64_t K, int64_t N, int64_t ld_w,
                                          uint8_t* q_t, uint8_t* q, float* s, void* stream) {
  if (groups < 0) return FP8Q_ERR_SHAPE;
  fp8q_status st = check_input(w, K, N, ld_w);
  if (st != FP8Q_OK) return st;
  if (!s) return FP8Q_ERR_NULL;
  if (K % 128 != 0 || N % 128 != 0) return FP8Q_ERR_SHAPE;
  if ((q && !aligned16(q)) || (q_t && !aligned16(q_t))) return FP8Q_ERR_ALIGN;
  if (groups == 0 || K == 0 || N == 0) return FP8Q_OK;
  const int64_t per = tiles_of(K, N);
  if (groups * per >= (1ll << 31)) return FP8Q_ERR_SHAPE;
  TileQuantParams p{static_cast<const uint16_t*>(w), K, N, ld_w, q, s, K / 128, q_t, nullptr, 0,
                    (int)(N / 128), 0};
  p.batch_tiles = per;
  p.x_bstride = K * ld_w;
  p.q_row_bstride = K * N;
  p.q_col_bstride = N * K;
  p.s_row_bstride = (N / 128) * (K / 128) * (int64_t)sizeof(float);
  return from_cuda(launch_tile_quant(kTile128, q != nullptr, q_t != nullptr, p, groups * per,
                                     static_cast<cudaStream_t>(stream)));
}

fp8q_status fp8q_quantize_mx32(const void* x, int64_t rows, int64_t cols, int64_t ld_x, uint8_t* q_row,
                               uint8_t* e8m0_row, uint8_t* q_col, uint8_t* e8m0_col, fp8q_sf_layout sf_layout,
                               void* stream) {
  fp8q_status st = check_input(x, rows, cols, ld_x);
  if (st != FP8Q_OK) return st;
  const bool row = q_row || e8m0_row, col = q_col || e8m0_col;
  if (!row && !col) return FP8Q_ERR_NULL;
  if ((row && (!q_row || !e8m0_row)) || (col && (!q_col || !e8m0_col))) return FP8Q_ERR_NULL;
  if (sf_layout != FP8Q_SF_ROWMAJOR && sf_layout != FP8Q_SF_MMA_TILED) return FP8Q_ERR_UNSUPPORTED;
  if (row && cols % 32 != 0) return FP8Q_ERR_SHAPE;
  if (col && (rows % 32 != 0 || cols % 16 != 0)) return FP8Q_ERR_SHAPE;
  if ((row && !aligned16(q_row)) || (col && !aligned16(q_col))) return FP8Q_ERR_ALIGN;
  if (sf_layout == FP8Q_SF_MMA_TILED && ((row && !aligned16(e8m0_row)) || (col && !aligned16(e8m0_col))))
    return FP8Q_ERR_ALIGN;
  if (rows == 0 || cols == 0) return FP8Q_OK;
  TileQuantParams p{static_cast<const uint16_t*>(x), rows, cols, ld_x, q_row, e8m0_row, 0,
                    q_col, e8m0_col, 0, (int)((cols + 127) / 128), sf_layout == FP8Q_SF_MMA_TILED};
  return from_cuda(launch_tile_quant(kTileMX, row, col, p, tiles_of(rows, cols), static_cast<cudaStream_t>(stream)));
}

fp8q_status fp8q_quantize_tensor(const void* x, int64_t rows, int64_t cols, int64_t ld_x, uint8_t* q, float* s_dec,
                                 void* stream) {
  fp8q_status st = check_input(x, rows, cols, ld_x);
  if (st != FP8Q_OK) return st;
  if (!q || !s_dec) return FP8Q_ERR_NULL;
  if (cols % 8 != 0) return FP8Q_ERR_SHAPE;
  if (!aligned16(q)) return FP8Q_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DeviceScratch* d = nullptr;
  if ((st = scratch(&d)) != FP8Q_OK) return st;
  uint32_t* amax = nullptr;
  if ((st = amax_slot(d, s, &amax)) != FP8Q_OK) return st;
  if (rows == 0 || cols == 0)   // empty tensor: amax 0 -> sf 1 -> decode scale 1, written on `stream`
    return from_cuda(launch_fill_f32(s_dec, 1.0f, s));
  cudaError_t e = launch_tensor_amax(static_cast<const uint16_t*>(x), rows, cols, ld_x, amax, s);
  if (e == cudaSuccess) e = launch_tensor_cast(static_cast<const uint16_t*>(x), rows, cols, ld_x, amax, q, s_dec, s);
  return from_cuda(e);
}

fp8q_status fp8q_quantize_tensor_delayed(const void* x, int64_t rows, int64_t cols, int64_t ld_x,
                                         float* amax_history, int32_t history_len, int32_t history_pos,
                                         fp8q_fp8_format fmt, uint8_t* q, float* s_dec, void* stream) {
  fp8q_status st = check_input(x, rows, cols, ld_x);
  if (st != FP8Q_OK) return st;
  if (!q || !s_dec || !amax_history) return FP8Q_ERR_NULL;
  if (fmt != FP8Q_E4M3 && fmt != FP8Q_E5M2) return FP8Q_ERR_UNSUPPORTED;
  if (history_len < 1 || history_len > 1024 || history_pos < 0 || history_pos >= history_len) return FP8Q_ERR_SHAPE;
  if (cols % 8 != 0) return FP8Q_ERR_SHAPE;
  if (!aligned16(q)) return FP8Q_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DeviceScratch* d = nullptr;
  if ((st = scratch(&d)) != FP8Q_OK) return st;
  uint32_t* amax = nullptr;
  if ((st = amax_slot(d, s, &amax)) != FP8Q_OK) return st;
  return from_cuda(launch_tensor_delayed(static_cast<const uint16_t*>(x), rows, cols, ld_x, amax_history,
                                         history_len, history_pos, fmt == FP8Q_E5M2, q, s_dec, amax, s));
}

fp8q_status fp4q_rht16_quantize_sr(const void* x, int64_t rows, int64_t cols, int64_t ld_x, int rht,
                                   uint64_t rht_seed, int sr, uint64_t sr_seed, uint8_t* q_row, uint8_t* sf_row,
                                   float* g_dec_row, uint8_t* q_col, uint8_t* sf_col, float* g_dec_col,
                                   fp8q_sf_layout sf_layout, void* stream) {
  fp8q_status st = check_input(x, rows, cols, ld_x);
  if (st != FP8Q_OK) return st;
  const bool row = q_row || sf_row || g_dec_row, col = q_col || sf_col || g_dec_col;
  if (!row && !col) return FP8Q_ERR_NULL;
  if ((row && (!q_row || !sf_row || !g_dec_row)) || (col && (!q_col || !sf_col || !g_dec_col))) return FP8Q_ERR_NULL;
  if ((rht & ~3) || (sr & ~3)) return FP8Q_ERR_UNSUPPORTED;
  if (sf_layout != FP8Q_SF_ROWMAJOR && sf_layout != FP8Q_SF_MMA_TILED) return FP8Q_ERR_UNSUPPORTED;
  if (cols % 16 != 0) return FP8Q_ERR_SHAPE;
  if (col && rows % 16 != 0) return FP8Q_ERR_SHAPE;
  if ((row && !aligned16(q_row)) || (col && !aligned16(q_col))) return FP8Q_ERR_ALIGN;
  if (rows == 0 || cols == 0) return FP8Q_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DeviceScratch* d = nullptr;
  if ((st = scratch(&d)) != FP8Q_OK) return st;
  uint32_t* amax = nullptr;
  if ((st = amax_slot(d, s, &amax)) != FP8Q_OK) return st;
  Fp4QuantParams p;
  p.x = static_cast<const uint16_t*>(x);
  p.rows = rows;
  p.cols = cols;
  p.ld_x = ld_x;
  p.rht_row = (rht & FP4Q_ROW) != 0;
  p.rht_col = (rht & FP4Q_COL) != 0;
  p.sr_row = (sr & FP4Q_ROW) != 0;
  p.sr_col = (sr & FP4Q_COL) != 0;
  p.rht_k0 = (uint32_t)rht_seed;
  p.rht_k1 = (uint32_t)(rht_seed >> 32);
  p.sr_k0 = (uint32_t)sr_seed;
  p.sr_k1 = (uint32_t)(sr_seed >> 32);
  for (int r = 0; r < 10; ++r) {   // Philox4x32-10 key schedule (Weyl sequence of the key)
    p.sr_rk[2 * r] = p.sr_k0 + (uint32_t)r * 0x9E3779B9u;
    p.sr_rk[2 * r + 1] = p.sr_k1 + (uint32_t)r * 0xBB67AE85u;
  }
  p.q_row = row ? q_row : nullptr;
  p.sf_row = sf_row;
  p.g_row = g_dec_row;
  p.q_col = col ? q_col : nullptr;
  p.sf_col = sf_col;
  p.g_col = g_dec_col;
  p.sf_tiled = sf_layout == FP8Q_SF_MMA_TILED;
  p.tiles_c = (int)((cols + 127) / 128);
  p.amax_bits = amax;
  const int64_t tiles = tiles_of(rows, cols);
  cudaError_t e = launch_fp4_amax(p, tiles, s);
  if (e == cudaSuccess) e = launch_fp4_quant(p, tiles, s);
  return from_cuda(e);
}

fp8q_status fp4q_quantize_2d16(const void* x, int64_t rows, int64_t cols, int64_t ld_x, uint8_t* q_row,
                               uint8_t* sf_row, uint8_t* q_col, uint8_t* sf_col, float* g_dec,
                               fp8q_sf_layout sf_layout, void* stream) {
  fp8q_status st = check_input(x, rows, cols, ld_x);
  if (st != FP8Q_OK) return st;
  const bool row = q_row || sf_row, col = q_col || sf_col;
  if ((!row && !col) || !g_dec) return FP8Q_ERR_NULL;
  if ((row && (!q_row || !sf_row)) || (col && (!q_col || !sf_col))) return FP8Q_ERR_NULL;
  if (sf_layout != FP8Q_SF_ROWMAJOR && sf_layout != FP8Q_SF_MMA_TILED) return FP8Q_ERR_UNSUPPORTED;
  if (rows % 16 != 0 || cols % 16 != 0) return FP8Q_ERR_SHAPE;
  if ((row && !aligned16(q_row)) || (col && !aligned16(q_col))) return FP8Q_ERR_ALIGN;
  if (rows == 0 || cols == 0) return FP8Q_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  DeviceScratch* d = nullptr;
  if ((st = scratch(&d)) != FP8Q_OK) return st;
  uint32_t* amax = nullptr;
  if ((st = amax_slot(d, s, &amax)) != FP8Q_OK) return st;
  Fp4QuantParams p;
  p.x = static_cast<const uint16_t*>(x);
  p.rows = rows;
  p.cols = cols;
  p.ld_x = ld_x;
  p.rht_row = p.rht_col = p.sr_row = p.sr_col = 0;
  p.rht_k0 = p.rht_k1 = p.sr_k0 = p.sr_k1 = 0;
  for (int r = 0; r < 20; ++r) p.sr_rk[r] = 0;
  p.q_row = row ? q_row : nullptr;
  p.sf_row = sf_row;
  p.g_row = g_dec;
  p.q_col = col ? q_col : nullptr;
  p.sf_col = sf_col;
  p.g_col = nullptr;
  p.sf_tiled = sf_layout == FP8Q_SF_MMA_TILED;
  p.tiles_c = (int)((cols + 127) / 128);
  p.amax_bits = amax;
  return from_cuda(launch_fp4_quant_2d(p, tiles_of(rows, cols), s));
}

// ------------------------------------------------------------------ GEMM
fp8q_status fp8q_gemm_blockscaled(const fp8q_gemm_args* a, void* stream) {
  if (!a) return FP8Q_ERR_NULL;
  if (a->recipe < FP8Q_BLOCKWISE || a->recipe > FP8Q_NVFP4) return FP8Q_ERR_UNSUPPORTED;
  if (a->layout < FP8Q_FPROP || a->layout > FP8Q_WGRAD) return FP8Q_ERR_UNSUPPORTED;
  if (a->M < 0 || a->N < 0 || a->K < 0) return FP8Q_ERR_SHAPE;
  if (a->M >= (1ll << 31) || a->N >= (1ll << 31) || a->K >= (1ll << 31)) return FP8Q_ERR_SHAPE;
  const bool acc32 = a->c_fp32_accumulate != 0;
  if (acc32 && a->recipe != FP8Q_BLOCKWISE) return FP8Q_ERR_UNSUPPORTED;
  if (a->a_format < 0 || a->a_format > 1 || a->b_format < 0 || a->b_format > 1) return FP8Q_ERR_UNSUPPORTED;
  if ((a->a_format || a->b_format) && a->recipe != FP8Q_PERTENSOR) return FP8Q_ERR_UNSUPPORTED;
  const bool qout = a->q_out != nullptr || a->s_out != nullptr;
  if (qout) {
    if (a->recipe != FP8Q_BLOCKWISE || acc32 || a->num_groups != 0) return FP8Q_ERR_UNSUPPORTED;
    if (!a->q_out || !a->s_out) return FP8Q_ERR_NULL;
    if (a->N % 128 != 0 || a->K < 384 || a->ld_q_out < a->N || a->ld_q_out % 16 != 0 || a->ld_s_out < a->M)
      return FP8Q_ERR_SHAPE;
    if (!aligned16(a->q_out)) return FP8Q_ERR_ALIGN;
  }
  if (a->M == 0 || a->N == 0) return FP8Q_OK;
  if (!a->c) return FP8Q_ERR_NULL;
  if (a->ldc < a->N || a->ldc % (acc32 ? 4 : 8) != 0) return FP8Q_ERR_SHAPE;
  if (!aligned16(a->c)) return FP8Q_ERR_ALIGN;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (a->K == 0) {  // empty sum: C = 0, or C unchanged when accumulating
    if (acc32) return FP8Q_OK;
    return from_cuda(cudaMemset2DAsync(a->c, (size_t)a->ldc * 2, 0, (size_t)a->N * 2, (size_t)a->M, s));
  }
  const bool fp4 = a->recipe == FP8Q_NVFP4;
  const int64_t kbytes = fp4 ? a->K / 2 : a->K;
  if (a->K % (fp4 ? 256 : 128) != 0) return FP8Q_ERR_SHAPE;
  if (!a->a || !a->b) return FP8Q_ERR_NULL;
  if (a->lda < kbytes || a->ldb < kbytes || a->lda % 16 != 0 || a->ldb % 16 != 0) return FP8Q_ERR_SHAPE;
  if (!aligned16(a->a) || !aligned16(a->b)) return FP8Q_ERR_ALIGN;
  const bool grouped = a->num_groups > 0;
  if (a->num_groups < 0) return FP8Q_ERR_SHAPE;
  if (grouped) {
    if (a->recipe != FP8Q_BLOCKWISE || a->layout != FP8Q_FPROP) return FP8Q_ERR_UNSUPPORTED;
    if (a->num_groups > 256) return FP8Q_ERR_UNSUPPORTED;
    if (!a->m_offsets) return FP8Q_ERR_NULL;
  }
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  p.recipe = a->recipe;
  p.layout = a->layout;
  p.M = (int)a->M;
  p.N = (int)a->N;
  p.K = (int)a->K;
  p.c = acc32 ? nullptr : static_cast<uint16_t*>(a->c);
  p.c32 = acc32 ? static_cast<float*>(a->c) : nullptr;
  p.a_fmt = a->a_format;
  p.b_fmt = a->b_format;
  p.q_out = qout ? a->q_out : nullptr;
  p.s_out = qout ? a->s_out : nullptr;
  p.ld_q_out = a->ld_q_out;
  p.ld_s_out = a->ld_s_out;
  if (a->workspace != nullptr && a->workspace_bytes >= 1024 && a->recipe == FP8Q_BLOCKWISE && !qout && !grouped) {
    if (!aligned16(a->workspace)) return FP8Q_ERR_ALIGN;
    p.ws = static_cast<float*>(a->workspace);
    p.ws_bytes = a->workspace_bytes;
  }
  p.ldc = a->ldc;
  p.m_offsets = a->m_offsets;
  p.num_groups = a->num_groups;
  p.tiles_n = (int)((a->N + 255) / 256);
  p.tiles_m = (int)((a->M + 127) / 128) + (grouped ? a->num_groups : 0);
  const int64_t nb128 = (a->N + 127) / 128;
  if (a->recipe == FP8Q_BLOCKWISE) {
    if (!a->a_scale || !a->b_scale) return FP8Q_ERR_NULL;
    if (a->ld_sa < a->M) return FP8Q_ERR_SHAPE;
    if (a->layout == FP8Q_FPROP && a->ld_sb < a->K / 128) return FP8Q_ERR_SHAPE;
    if (a->layout == FP8Q_DGRAD && a->ld_sb < nb128) return FP8Q_ERR_SHAPE;
    if (a->layout == FP8Q_WGRAD) {
      if (a->ld_sb < a->N || a->ld_sb % 4 != 0) return FP8Q_ERR_SHAPE;
      if (!aligned16(a->b_scale)) return FP8Q_ERR_ALIGN;
    }
    p.sa = static_cast<const float*>(a->a_scale);
    p.ld_sa = a->ld_sa;
    p.sb = static_cast<const float*>(a->b_scale);
    p.ld_sb = a->ld_sb;
  } else if (a->recipe == FP8Q_MXFP8 || fp4) {
    if (!a->a_scale || !a->b_scale) return FP8Q_ERR_NULL;
    if (!aligned16(a->a_scale) || !aligned16(a->b_scale)) return FP8Q_ERR_ALIGN;
    p.sfa = static_cast<const uint8_t*>(a->a_scale);
    p.sfb = static_cast<const uint8_t*>(a->b_scale);
    const int64_t sf_cols = fp4 ? a->K / 16 : a->K / 32;
    p.sfa_s4 = p.sfb_s4 = (sf_cols + 3) / 4;
  }
  if (a->recipe == FP8Q_PERTENSOR || fp4) {
    if (!a->a_global || !a->b_global) return FP8Q_ERR_NULL;
    p.a_global = a->a_global;
    p.b_global = a->b_global;
  }
  DeviceScratch* d = nullptr;
  fp8q_status st = scratch(&d);
  if (st != FP8Q_OK) return st;
  p.status = d->base.load(std::memory_order_acquire);

  CUtensorMap ma, mb, msb;
  const int64_t b_rows = grouped ? (int64_t)a->num_groups * a->N : a->N;
  if (!make_map(&ma, a->a, CU_TENSOR_MAP_DATA_TYPE_UINT8, kbytes, a->M, a->lda, 128, 128,
                CU_TENSOR_MAP_SWIZZLE_128B))
    return FP8Q_ERR_CUDA;
  // B box rows: each CTA of a blockwise pair loads half of its 256-column tile; the other
  // kernel loads its whole 256-column tile.  The wgrad scale box spans the full tile width.
  const uint32_t bn = (a->recipe == FP8Q_BLOCKWISE) ? kBlockwiseTileN : 256;
  const uint32_t b_box = (a->recipe == FP8Q_BLOCKWISE) ? bn / 2 : 256;
  if (!make_map(&mb, a->b, CU_TENSOR_MAP_DATA_TYPE_UINT8, kbytes, b_rows, a->ldb, 128, b_box,
                CU_TENSOR_MAP_SWIZZLE_128B))
    return FP8Q_ERR_CUDA;
  if (a->recipe == FP8Q_BLOCKWISE && a->layout == FP8Q_WGRAD) {
    if (!make_map(&msb, a->b_scale, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a->N, a->K / 128, a->ld_sb * 4, bn, 1,
                  CU_TENSOR_MAP_SWIZZLE_NONE))
      return FP8Q_ERR_CUDA;
  } else {
    msb = ma;
  }
  // the blockwise epilogues send their staged boxes by TMA: BF16 32 x 32 boxes (and the fused
  // quantization's 32 x 64 code boxes) stored, FP32 boxes added
  CUtensorMap mc = ma, mq = ma;
  if (a->recipe == FP8Q_BLOCKWISE && acc32 && a->M > 0 && a->N > 0) {
    // FP32 accumulation: 32 x 16 FP32 boxes added into C by TMA reduction
    if (!make_map(&mc, a->c, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, a->N, a->M, a->ldc * 4, 16, 32,
                  CU_TENSOR_MAP_SWIZZLE_64B))
      return FP8Q_ERR_CUDA;
  } else if (a->recipe == FP8Q_BLOCKWISE && a->M > 0 && a->N > 0) {
    if (!make_map(&mc, a->c, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a->N, a->M, a->ldc * 2, 32, 32,
                  CU_TENSOR_MAP_SWIZZLE_64B))
      return FP8Q_ERR_CUDA;
    if (qout && !make_map(&mq, a->q_out, CU_TENSOR_MAP_DATA_TYPE_UINT8, a->N, a->M, a->ld_q_out, 64, 32,
                          CU_TENSOR_MAP_SWIZZLE_64B))
      return FP8Q_ERR_CUDA;
  }
  // the split tail's workspace: FP32 rows of 256 columns, stored in 16 x 32 boxes
  CUtensorMap mws = ma;
  if (p.ws != nullptr && !make_map(&mws, p.ws, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, kBlockwiseTileN,
                                   (uint64_t)p.ws_bytes / (kBlockwiseTileN * 4), kBlockwiseTileN * 4, 16, 32,
                                   CU_TENSOR_MAP_SWIZZLE_64B))
    return FP8Q_ERR_CUDA;
  return from_cuda(launch_gemm(p, ma, mb, msb, mc, mq, mws, d->num_sms, s));
}

size_t fp8q_gemm_workspace_bytes(const fp8q_gemm_args* a) {
  if (!a || a->recipe != FP8Q_BLOCKWISE || a->layout < FP8Q_FPROP || a->layout > FP8Q_WGRAD) return 0;
  if (a->q_out || a->s_out || a->num_groups != 0) return 0;
  if (a->M <= 0 || a->N <= 0 || a->K <= 0 || a->K % 128 != 0) return 0;
  if (a->M >= (1ll << 31) || a->N >= (1ll << 31) || a->K >= (1ll << 31)) return 0;
  DeviceScratch* d = nullptr;
  if (scratch(&d) != FP8Q_OK) return 0;
  GemmParams p;
  std::memset(&p, 0, sizeof(p));
  p.recipe = a->recipe;
  p.layout = a->layout;
  p.M = (int)a->M;
  p.N = (int)a->N;
  p.K = (int)a->K;
  return blockwise_workspace_bytes(p, d->num_sms);
}

}  // extern "C"
