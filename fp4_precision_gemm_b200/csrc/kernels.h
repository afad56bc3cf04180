// Host-side launch interfaces of the kernels (internal to the library).
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace fp8q {

enum { kTile1x128 = 0, kTile128 = 1, kTileMX = 2 };

struct TileQuantParams {
  const uint16_t* x;
  int64_t rows, cols, ld_x;
  uint8_t* q_row;
  void* s_row;      // float* (1x128, 128x128) or uint8_t* (MX)
  int64_t ld_s_row;  // 1x128: scale row stride; 128x128: K/128
  uint8_t* q_col;
  void* s_col;
  int64_t ld_s_col;
  int tiles_c;      // 128-column tiles per 128-row band
  int sf_tiled;     // MX scale bytes in the MMA-tiled layout
  // grouped calls (0 = one matrix): tiles per matrix, and each operand's stride between
  // consecutive matrices (x in elements, outputs and scales in bytes)
  int64_t batch_tiles;
  int64_t x_bstride, q_row_bstride, q_col_bstride, s_row_bstride, s_col_bstride;
};

cudaError_t launch_tile_quant(int mode, bool row, bool col, const TileQuantParams& p,
                              int64_t tiles, cudaStream_t s);

// Multi-tensor launch: up to kMaxMultiItems tensors, each a 1x128 (rowwise, colwise or both)
// or a 128x128 (either or both layouts) quantization; item i owns the launch's tiles
// [tile_begin[i], tile_begin[i + 1]).
constexpr int kMaxMultiItems = 8;
enum { kMulti1x128Row = 0, kMulti1x128Col = 1, kMulti1x128Both = 2, kMulti128Row = 3, kMulti128Col = 4,
       kMulti128Both = 5 };
struct TileQuantMulti {
  int n;
  int kind[kMaxMultiItems];
  int64_t tile_begin[kMaxMultiItems + 1];
  TileQuantParams item[kMaxMultiItems];
};
cudaError_t launch_tile_quant_multi(const TileQuantMulti& m, int64_t tiles, cudaStream_t s);

// Per-tensor current scaling: amax pass into *amax_bits (zeroed by the caller), then cast.
cudaError_t launch_tensor_amax(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld_x,
                               uint32_t* amax_bits, cudaStream_t s);
cudaError_t launch_tensor_cast(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld_x,
                               const uint32_t* amax_bits, uint8_t* q, float* s_dec,
                               cudaStream_t s);

struct Fp4QuantParams {
  const uint16_t* x;
  int64_t rows, cols, ld_x;
  int rht_row, rht_col, sr_row, sr_col;
  uint32_t rht_k0, rht_k1, sr_k0, sr_k1;
  uint8_t* q_row;
  uint8_t* sf_row;
  float* g_row;
  uint8_t* q_col;
  uint8_t* sf_col;
  float* g_col;
  int sf_tiled;
  int tiles_c;
  uint32_t* amax_bits;  // [0]: rowwise output's global amax, [1]: colwise output's
  uint32_t sr_rk[20];   // Philox key schedule of the stochastic-rounding key (sr_k0, sr_k1)
};

// One float written on the stream (the decode scale of an empty tensor), no host sync.
cudaError_t launch_fill_f32(float* dst, float v, cudaStream_t s);

cudaError_t launch_tensor_delayed(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld_x, float* hist,
                                  int hlen, int pos, bool e5m2, uint8_t* q, float* s_dec, uint32_t* amax_bits,
                                  cudaStream_t s);

cudaError_t launch_fp4_amax(const Fp4QuantParams& p, int64_t tiles, cudaStream_t s);
cudaError_t launch_fp4_quant(const Fp4QuantParams& p, int64_t tiles, cudaStream_t s);
// 16x16-block weight quantizer: global amax into amax_bits[0], then codes in the layouts
// whose q pointer is set; g_row receives the decode scale.
cudaError_t launch_fp4_quant_2d(const Fp4QuantParams& p, int64_t tiles, cudaStream_t s);

// ------------------------------------------------------------------ GEMM
// Output tile width of the blockwise (FP32-promotion) kernel; the B and wgrad-scale TMA boxes
// are built with it.
constexpr uint32_t kBlockwiseTileN = 256;

struct GemmParams {
  int recipe;       // fp8q_recipe
  int layout;       // fp8q_layout
  int M, N, K;
  const float* sa;  // BLOCKWISE: A decode scales, sa[kb * ld_sa + m]
  int64_t ld_sa;
  const float* sb;  // BLOCKWISE: B scales (indexed per layout)
  int64_t ld_sb;
  const float* a_global;
  const float* b_global;
  uint16_t* c;      // BF16 row-major (nullptr when accumulating into c32)
  float* c32;       // BLOCKWISE FP32 accumulate target (C += A.B^T), else nullptr
  int64_t ldc;
  const uint8_t* sfa;  // MX / NVFP4: MMA-tiled scale images
  const uint8_t* sfb;
  int64_t sfa_s4, sfb_s4;  // atoms per 128-row band (ceil(scale columns / 4))
  const int32_t* m_offsets;
  int num_groups;
  int tiles_m, tiles_n;    // output tile grid (non-grouped)
  int group_m;             // raster: row tiles per column sweep (set by the launcher)
  int group_n;             // raster: > 0 -> column tiles per row sweep instead (set by the launcher)
  int a_fmt, b_fmt;        // PERTENSOR: element format of A / B (0 E4M3, 1 E5M2)
  uint8_t* q_out;          // BLOCKWISE, optional: 1x128 E4M3 codes of the BF16 output (along N)
  float* s_out;            //   and their decode scales, s_out[(n / 128) * ld_s_out + m]
  int64_t ld_q_out, ld_s_out;
  uint32_t* status;        // device status word
  // BLOCKWISE, not grouped (set by the launcher): units [0, main_tiles) are the
  // whole raster tiles; with tail_splits > 0 the remaining tiles (the last, partial wave)
  // follow as tail_splits K ranges each, whose FP32 partial sums go to ws (256 x 256 floats
  // per range) and are then added by a second kernel.
  int main_tiles;
  int tail_splits;
  float* ws;
  int64_t ws_bytes;
};

cudaError_t launch_selftest_wait(uint32_t* status, uint64_t limit_ns, cudaStream_t s);

// tma_c: C for the blockwise kernel's epilogues, N inner, M outer, 64-byte swizzle: BF16 with
// 32 x 32 boxes (stored), or FP32 with 16 x 32 boxes (added, FP32 accumulation); tma_q: the
// fused quantization's E4M3 codes (64 x 32 boxes, stored); tma_ws: p.ws as FP32 rows of 256
// (16 x 32 boxes, the same swizzle), used only when the last wave is split (in place of
// tma_q, which the BF16 and FP32-accumulate epilogues do not use).
cudaError_t launch_gemm(const GemmParams& p, const CUtensorMap& tma_a, const CUtensorMap& tma_b,
                        const CUtensorMap& tma_sb, const CUtensorMap& tma_c, const CUtensorMap& tma_q,
                        const CUtensorMap& tma_ws, int num_sms, cudaStream_t s);

// Workspace bytes that a blockwise BF16 GEMM with these parameters uses to split its last,
// partial wave into K ranges on the current device (0: it would not split).
size_t blockwise_workspace_bytes(const GemmParams& p, int num_sms);

}  // namespace fp8q
