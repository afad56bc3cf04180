// Tile quantize kernels: 1x128 tiles (rowwise and fused transposed colwise), 128x128
// weight blocks (both K-major layouts) and MX 1x32 blocks with E8M0 scales.
//
// "Can you explain the role of FP8 precision in DeepSeek-V3 training", sections
// "Fine-grained quantization" and "Online quantization": each 1x128 activation tile and
// each 128x128 weight block gets its own scale from its live amax and is cast to E4M3.
// "Accelerating FP8 training performance with the NVIDIA NeMo framework": MXFP8 scales
// blocks of 32 values.
//
// One CTA (256 threads) quantizes one 128x128 tile of the BF16 input, read once with
// coalesced 16-byte loads.  Thread t owns the 8x8 sub-block rows 8*(t/16)..+7, columns
// 8*(t%16)..+7 of the tile, so
//   * a row's 128 values sit in 16 lanes (1x128 row amax: 4 xor-shuffles),
//   * a row's 32-value MX block sits in 4 lanes (2 xor-shuffles),
//   * a column's 8-row pieces sit in lanes t and t^16 and across the 8 warps.
// Magnitudes are reduced as packed 15-bit BF16 patterns (vmaxu2), which is exact.
// Transposed outputs are staged in shared memory with an XOR swizzle on 8-byte chunks so
// both the scattered writes and the row-contiguous reads are bank-conflict free, then
// stored as full 128-byte row segments.
#include "common.cuh"
#include "kernels.h"

namespace fp8q {

namespace {

__device__ __forceinline__ uint32_t row_word_max(const uint4& v) {
  return hmax(max2(max2(abs2(v.x), abs2(v.y)), max2(abs2(v.z), abs2(v.w))));
}

__device__ __forceinline__ float elem(const uint4& v, int j) {
  uint32_t w = (j < 2) ? v.x : (j < 4) ? v.y : (j < 6) ? v.z : v.w;
  return (j & 1) ? bf16_hi(w) : bf16_lo(w);
}

__device__ __forceinline__ uint32_t word(const uint4& v, int jw) {
  return (jw == 0) ? v.x : (jw == 1) ? v.y : (jw == 2) ? v.z : v.w;
}

// Physical 8-byte chunk of logical row-chunk k in transposed row c of the staging tile.
__device__ __forceinline__ int tq_chunk(int c, int k) { return k ^ ((c >> 3) ^ (c & 1)); }

// Shared memory of one tile: reduction slots, column scales / exponents and the transposed
// staging tile.
struct TileSmem {
  uint32_t red[8][64];
  float colsf[128];
  uint8_t colexp[128 * 4];
  __align__(16) uint8_t tq[128 * 128];
};

}  // namespace

// Resident CTAs per SM: the kernel is latency bound on its loads, so the register budget is
// set for 4 CTAs (64 registers); the rowwise-only variants need a few more and get 3.
template <bool ROW, bool COL>
constexpr int kTileQuantCtas = (ROW && !COL) ? 3 : 4;

// One 128x128 tile (index `tile` of the call, grouped calls counting every matrix's tiles)
// quantized by the CTA's 256 threads.
template <int MODE, bool ROW, bool COL>
__device__ __forceinline__ void tile_quant_tile(const TileQuantParams& P, int64_t tile, TileSmem& sm) {
  auto& red = sm.red;
  auto& colsf = sm.colsf;
  auto& colexp = sm.colexp;
  auto& tq = sm.tq;

  const int t = threadIdx.x, warp = t >> 5;
  const int cs = t & 15, rb = t >> 4;
  // grouped calls: CTA -> (matrix b, tile within it); every operand pointer moves by b strides
  const int64_t bidx = P.batch_tiles ? tile / P.batch_tiles : 0;
  tile -= bidx * P.batch_tiles;
  const uint16_t* X = P.x + bidx * P.x_bstride;
  uint8_t* QR = P.q_row ? P.q_row + bidx * P.q_row_bstride : nullptr;
  uint8_t* QC = P.q_col ? P.q_col + bidx * P.q_col_bstride : nullptr;
  uint8_t* SR = P.s_row ? (uint8_t*)P.s_row + bidx * P.s_row_bstride : nullptr;
  uint8_t* SC = P.s_col ? (uint8_t*)P.s_col + bidx * P.s_col_bstride : nullptr;
  const int64_t r0 = (tile / P.tiles_c) * 128;
  const int64_t c0 = (tile % P.tiles_c) * 128;
  const int64_t col = c0 + cs * 8;
  const bool cok = col < P.cols;

  uint4 v[8];
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    const int64_t row = r0 + rb * 8 + p;
    v[p] = (cok && row < P.rows) ? ldg_nc_v4(X + row * P.ld_x + col) : make_uint4(0, 0, 0, 0);
  }

  // ---------------------------------------------------------------- amax reductions
  uint32_t rp[4];  // row maxima, two rows per word (row 2i low, 2i+1 high)
#pragma unroll
  for (int i = 0; i < 4; ++i) rp[i] = row_word_max(v[2 * i]) | (row_word_max(v[2 * i + 1]) << 16);

  float blk_sf = 1.0f;
  if (MODE == kTile128) {
    uint32_t m = max(hmax(max2(rp[0], rp[1])), hmax(max2(rp[2], rp[3])));
#pragma unroll
    for (int s = 1; s < 32; s <<= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, s));
    if ((t & 31) == 0) red[warp][0] = m;
    __syncthreads();
    uint32_t bm = red[0][0];
#pragma unroll
    for (int w = 1; w < 8; ++w) bm = max(bm, red[w][0]);
    blk_sf = e4m3_sf(bf16_bits_to_float(bm));
    if (t == 0 && SR != nullptr)
      ((float*)SR)[(c0 >> 7) * P.ld_s_row + (r0 >> 7)] = __frcp_rn(blk_sf);
  } else if (ROW) {
    const int lanes = (MODE == kTile1x128) ? 16 : 4;
#pragma unroll
    for (int s = 1; s < lanes; s <<= 1) {
#pragma unroll
      for (int i = 0; i < 4; ++i) rp[i] = max2(rp[i], __shfl_xor_sync(0xFFFFFFFFu, rp[i], s));
    }
  }

  uint32_t cm[4];  // column maxima over the thread's 8 rows, two columns per word
  int ecol[8];     // MX colwise exponents of the thread's 8 columns
  if (COL && MODE != kTile128) {
#pragma unroll
    for (int jw = 0; jw < 4; ++jw) {
      uint32_t m = 0;
#pragma unroll
      for (int p = 0; p < 8; ++p) m = max2(m, abs2(word(v[p], jw)));
      cm[jw] = max2(m, __shfl_xor_sync(0xFFFFFFFFu, m, 16));
    }
    if ((t & 31) < 16) {
#pragma unroll
      for (int jw = 0; jw < 4; ++jw) red[warp][cs * 4 + jw] = cm[jw];
    }
    __syncthreads();
    if (MODE == kTile1x128) {
      if (t < 128) {   // one column per thread: word t/2 holds columns cc and cc + 1
        const int wd = t >> 1, h = t & 1;
        uint32_t m = red[0][wd];
#pragma unroll
        for (int w = 1; w < 8; ++w) m = max2(m, red[w][wd]);
        const int cc = (wd >> 2) * 8 + (wd & 3) * 2 + h;
        const float sf = e4m3_sf(bf16_bits_to_float(h ? (m >> 16) : (m & 0xFFFFu)));
        colsf[cc] = sf;
        if (c0 + cc < P.cols) ((float*)SC)[(r0 >> 7) * P.ld_s_col + c0 + cc] = __frcp_rn(sf);
      }
      __syncthreads();
    } else {  // MX: 32-row block b = warp / 2 spans warps 2b and 2b+1
      const int b = warp >> 1;
#pragma unroll
      for (int jw = 0; jw < 4; ++jw) {
        const uint32_t m = max2(red[warp][cs * 4 + jw], red[warp ^ 1][cs * 4 + jw]);
        ecol[2 * jw] = mx_exponent(bf16_bits_to_float(m & 0xFFFFu));
        ecol[2 * jw + 1] = mx_exponent(bf16_bits_to_float(m >> 16));
      }
      if ((warp & 1) == 0 && (t & 31) < 16) {
#pragma unroll
        for (int j = 0; j < 8; ++j) colexp[(cs * 8 + j) * 4 + b] = (uint8_t)(ecol[j] + 127);
      }
      __syncthreads();
      if (t < 128) {
        const int64_t cg = c0 + t;
        const uint32_t e4 = *(const uint32_t*)&colexp[t * 4];
        uint8_t* dst = SC;
        const int64_t nsf = P.rows >> 5;
        if (P.sf_tiled) {  // padding rows of the tiled image get code 0 (their amax is 0)
          const int64_t s4 = (nsf + 3) >> 2;
          *(uint32_t*)(dst + sf_tiled_offset(cg, r0 >> 5, s4)) = e4;
        } else if (cg < P.cols) {
#pragma unroll
          for (int b2 = 0; b2 < 4; ++b2)
            if ((r0 >> 5) + b2 < nsf) dst[cg * nsf + (r0 >> 5) + b2] = (uint8_t)(e4 >> (8 * b2));
        }
      }
    }
  }

  // ---------------------------------------------------------------- rowwise output
  if (ROW) {
    // 1x128: the 16 lanes of a row group hold the same 8 row maxima; lane cs divides for row
    // cs % 8 and the scales are shuffled out (one IEEE division per thread instead of 8)
    float sf_own = 1.0f;
    if (MODE == kTile1x128) {
      const int pr = cs & 7;
      const uint32_t w = pr < 2 ? rp[0] : pr < 4 ? rp[1] : pr < 6 ? rp[2] : rp[3];
      sf_own = e4m3_sf(bf16_bits_to_float((pr & 1) ? (w >> 16) : (w & 0xFFFFu)));
      // lane cs < 8 of the row group also writes row cs's decode scale (one reciprocal per
      // lane instead of one per row with a single lane active)
      const int64_t row = r0 + rb * 8 + cs;
      if (cs < 8 && row < P.rows) ((float*)SR)[(c0 >> 7) * P.ld_s_row + row] = __frcp_rn(sf_own);
    }
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      const int64_t row = r0 + rb * 8 + p;
      const uint32_t abits = (rp[p >> 1] >> ((p & 1) * 16)) & 0xFFFFu;
      float sf;
      int e = 0;
      if (MODE == kTile128) {
        sf = blk_sf;
      } else if (MODE == kTile1x128) {
        sf = __shfl_sync(0xFFFFFFFFu, sf_own, (t & 16) | p);
      } else {
        e = mx_exponent(bf16_bits_to_float(abits));
        sf = pow2_neg(e);
      }
      if (row < P.rows && cok) {
        const float2 s2 = make_float2(sf, sf);
        uint32_t c[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 y = __fmul2_rn(make_float2(elem(v[p], 2 * q), elem(v[p], 2 * q + 1)), s2);
          c[q] = cvt_e4m3x2(y.x, y.y);
        }
        *(uint2*)(QR + row * P.cols + col) = make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
      }
      if (MODE == kTileMX && (cs & 3) == 0) {
        const int64_t kc = (col >> 5);
        uint8_t* dst = SR;
        const int64_t nsf = P.cols >> 5;
        if (P.sf_tiled) {
          const int64_t s4 = (nsf + 3) >> 2;
          if (kc < s4 * 4) dst[sf_tiled_offset(row, kc, s4)] = (uint8_t)(e + 127);
        } else if (row < P.rows && kc < nsf) {
          dst[row * nsf + kc] = (uint8_t)(e + 127);
        }
      }
    }
  }

  // ---------------------------------------------------------------- colwise output
  if (COL) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float sf;
      if (MODE == kTile128) sf = blk_sf;
      else if (MODE == kTile1x128) sf = colsf[cs * 8 + j];
      else sf = pow2_neg(ecol[j]);
      const float2 s2 = make_float2(sf, sf);
      uint32_t lo = 0, hi = 0;
#pragma unroll
      for (int p = 0; p < 8; p += 2) {
        const float2 y = __fmul2_rn(make_float2(elem(v[p], j), elem(v[p + 1], j)), s2);
        const uint32_t c = cvt_e4m3x2(y.x, y.y);
        if (p < 4) lo |= c << (8 * p);
        else hi |= c << (8 * (p - 4));
      }
      const int c = cs * 8 + j;
      *(uint2*)&tq[c * 128 + tq_chunk(c, rb) * 8] = make_uint2(lo, hi);
    }
    __syncthreads();
#pragma unroll
    for (int pass = 0; pass < 4; ++pass) {
      const int c = pass * 32 + (t >> 3), h = t & 7;
      const int64_t cg = c0 + c, rg = r0 + 16 * h;
      const uint2 a = *(const uint2*)&tq[c * 128 + tq_chunk(c, 2 * h) * 8];
      const uint2 b = *(const uint2*)&tq[c * 128 + tq_chunk(c, 2 * h + 1) * 8];
      if (cg < P.cols && rg < P.rows)
        *(uint4*)(QC + cg * P.rows + rg) = make_uint4(a.x, a.y, b.x, b.y);
    }
  }
}

template <int MODE, bool ROW, bool COL>
__global__ void __launch_bounds__(256, kTileQuantCtas<ROW, COL>) tile_quant_kernel(const __grid_constant__ TileQuantParams P) {
  __shared__ TileSmem sm;
  tile_quant_tile<MODE, ROW, COL>(P, blockIdx.x, sm);
}

// Several tensors in one launch (each its own mode and outputs): CTA b takes tile
// b - tile_begin[i] of the item i whose range holds b, so the launch pays one ramp and one
// partial last wave for all of them.  The rowwise-only forms need more registers (3 CTAs
// per SM); a launch without them is compiled for 4.
template <bool ROWONLY>
__global__ void __launch_bounds__(256, ROWONLY ? 3 : 4) tile_quant_multi_kernel(const __grid_constant__ TileQuantMulti M) {
  __shared__ TileSmem sm;
  const int64_t b = blockIdx.x;
  int i = 0;
  while (i + 1 < M.n && b >= M.tile_begin[i + 1]) ++i;
  const TileQuantParams P = M.item[i];   // by value: registers, not indexed parameter loads
  const int64_t tile = b - M.tile_begin[i];
  switch (M.kind[i]) {
    case kMulti1x128Col: tile_quant_tile<kTile1x128, false, true>(P, tile, sm); break;
    case kMulti1x128Both: tile_quant_tile<kTile1x128, true, true>(P, tile, sm); break;
    case kMulti128Col: tile_quant_tile<kTile128, false, true>(P, tile, sm); break;
    case kMulti128Both: tile_quant_tile<kTile128, true, true>(P, tile, sm); break;
    default:
      if constexpr (ROWONLY) {
        if (M.kind[i] == kMulti1x128Row) tile_quant_tile<kTile1x128, true, false>(P, tile, sm);
        else tile_quant_tile<kTile128, true, false>(P, tile, sm);
      }
      break;
  }
}

cudaError_t launch_tile_quant_multi(const TileQuantMulti& m, int64_t tiles, cudaStream_t s) {
  bool rowonly = false;
  for (int i = 0; i < m.n; ++i) rowonly |= (m.kind[i] == kMulti1x128Row || m.kind[i] == kMulti128Row);
  if (rowonly) tile_quant_multi_kernel<true><<<dim3((unsigned)tiles), dim3(256), 0, s>>>(m);
  else tile_quant_multi_kernel<false><<<dim3((unsigned)tiles), dim3(256), 0, s>>>(m);
  return cudaGetLastError();
}

cudaError_t launch_tile_quant(int mode, bool row, bool col, const TileQuantParams& p,
                              int64_t tiles, cudaStream_t s) {
  dim3 grid((unsigned)tiles), block(256);
#define FP8Q_TQ(M, R, C) \
  if (mode == M && row == R && col == C) { tile_quant_kernel<M, R, C><<<grid, block, 0, s>>>(p); return cudaGetLastError(); }
  FP8Q_TQ(kTile1x128, true, false) FP8Q_TQ(kTile1x128, false, true) FP8Q_TQ(kTile1x128, true, true)
  FP8Q_TQ(kTile128, true, false) FP8Q_TQ(kTile128, false, true) FP8Q_TQ(kTile128, true, true)
  FP8Q_TQ(kTileMX, true, false) FP8Q_TQ(kTileMX, false, true) FP8Q_TQ(kTileMX, true, true)
#undef FP8Q_TQ
  return cudaErrorInvalidValue;
}

}  // namespace fp8q
