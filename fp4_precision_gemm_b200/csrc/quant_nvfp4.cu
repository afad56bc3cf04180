// NVFP4 quantization with the 16x16 random Hadamard transform and stochastic rounding.
//
// "NVIDIA developed a method to train neural networks in 4-bit precision", section "How it
// works": 4-bit (E2M1) values, 16x16 random Hadamard transforms applied to gradient
// inputs, stochastic rounding.  The two-level scale (E4M3 per 16 elements, FP32 per
// tensor) keeps every block scale inside the E4M3 range: S_g = 2688 / G maps the tensor
// amax G to 448 * 6.
//
// Two passes over the BF16 input: (1) the global amax of each requested output (after its
// transform), one atomicMax per CTA into the library's scratch words; (2) recompute the
// transform, per-16 block amax, E4M3 block scale, encode scale, and E2M1 codes by
// round-to-nearest-even or by Philox4x32-10 stochastic rounding.
//
// Rowwise output: one thread per 16-element group of a row (two 16-byte loads); the group's
// transform, amax and codes stay in-thread.
// Colwise output and the two-output amax pass: one CTA (256 threads) per 128x128 tile, warp w
// owns rows 16w..16w+15, lane l owns columns 4l..4l+3, so a thread holds a 16x4 sub-block:
//   * colwise (along rows) 16-element groups and blocks are entirely in-thread, so the
//     transform's butterflies and the block amax need no shuffles;
//   * rowwise 16-element groups span 4 lanes (2 xor-shuffles for the amax, and for the
//     two upper butterfly stages when the rowwise transform is on);
//   * one Philox call yields the 4 words of 4 consecutive output elements.
// The transposed colwise codes are staged in shared memory and stored as 64-byte rows.
// With both outputs requested one kernel makes both from a single read of each tile.
#include "common.cuh"
#include "kernels.h"

namespace fp8q {

namespace {

constexpr uint32_t kRhtCounterTag = 0x52485431u;

__device__ __forceinline__ uint2 ldg_nc_v2(const void* p) {
  uint2 r;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(r.x), "=r"(r.y) : "l"(p));
  return r;
}

__device__ __forceinline__ float flip(float v, uint32_t signs, int i) {
  return __uint_as_float(__float_as_uint(v) ^ (((signs >> i) & 1u) << 31));
}

// Butterflies h = 1, 2, 4, 8 over 16 in-thread values, then the 1/4 normalisation.
__device__ __forceinline__ void fwht16(float (&e)[16]) {
#pragma unroll
  for (int h = 1; h < 16; h <<= 1) {
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      if ((k & h) == 0) {
        const float a = e[k], b = e[k + h];
        e[k] = __fadd_rn(a, b);
        e[k + h] = __fsub_rn(a, b);
      }
    }
  }
#pragma unroll
  for (int k = 0; k < 16; ++k) e[k] = __fmul_rn(e[k], 0.25f);
}

// Rowwise transform of one row's 4 values held by this lane (positions 4*(lane&3)..+3 of
// the 16-element group); the partner lanes supply the other 12.
__device__ __forceinline__ void rht_row4(float (&e)[4], uint32_t signs, int lane) {
  const int base = (lane & 3) * 4;
#pragma unroll
  for (int j = 0; j < 4; ++j) e[j] = flip(e[j], signs, base + j);
#pragma unroll
  for (int h = 1; h < 4; h <<= 1) {
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      if ((k & h) == 0) {
        const float a = e[k], b = e[k + h];
        e[k] = __fadd_rn(a, b);
        e[k + h] = __fsub_rn(a, b);
      }
    }
  }
#pragma unroll
  for (int s = 1; s <= 2; s <<= 1) {          // h = 4 (lane ^ 1), h = 8 (lane ^ 2)
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float o = __shfl_xor_sync(0xFFFFFFFFu, e[k], s);
      e[k] = upper ? __fsub_rn(o, e[k]) : __fadd_rn(e[k], o);
    }
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) e[k] = __fmul_rn(e[k], 0.25f);
}

__device__ __forceinline__ float global_scale(uint32_t amax_bits) {
  const float G = __uint_as_float(amax_bits);
  if (G == 0.0f) return 1.0f;
  const float s = __fdiv_rn(2688.0f, G);
  return (s > FLT_MAX) ? FLT_MAX : s;
}

// fp32(m / 6), correctly rounded.  For m in [2^-125, FLT_MAX] one FMA correction of
// m * fp32(1/6) gives the correctly rounded quotient (checked on the CPU for every FP32
// significand over the binades where an intermediate can be subnormal, and on whole binades
// above, where all steps scale exactly); zero, tiny and non-finite m take the IEEE division.
__device__ __forceinline__ float div6_rn(float m) {
  constexpr float kSixth = 0.16666667163372039794921875f;   // fp32(1/6) = 0x3E2AAAAB
  if (m >= 0x1p-125f && m <= FLT_MAX) {
    const float q0 = __fmul_rn(m, kSixth);
    return __fmaf_rn(__fmaf_rn(-6.0f, q0, m), kSixth, q0);
  }
  return __fdiv_rn(m, 6.0f);
}

// E4M3 block scale and the matching encode scale S_g / decode(sb) for block amax `m`; the
// encode scales of all 128 non-negative codes are tabulated once per CTA (enc_tab).
__device__ __forceinline__ void block_scale(float m, float S_g, const float* enc_tab, uint32_t& sb, float& enc) {
  const float t = __fmul_rn(div6_rn(m), S_g);
  sb = cvt_e4m3x2(t, 0.0f) & 0xFFu;
  enc = enc_tab[sb & 0x7Fu];
}

// enc_tab[c] = S_g / decode(c) for codes 1..126 (code 0: 0, no value is encoded).
__device__ __forceinline__ void fill_enc_tab(float* enc_tab, float S_g) {
  const int c = threadIdx.x & 127;
  enc_tab[c] = (c == 0 || c == 0x7F) ? 0.0f : __fdiv_rn(S_g, e4m3_to_float((uint32_t)c));
}

__device__ __forceinline__ uint32_t rht_signs(const Fp4QuantParams& P) {
  return philox4x32_10(make_uint4(0, 0, 0, kRhtCounterTag), P.rht_k0, P.rht_k1).x & 0xFFFFu;
}

struct Tile {
  int64_t r0, c0, col;
  bool cok;
  int lane, w;
};

__device__ __forceinline__ Tile tile_coords(const Fp4QuantParams& P, int64_t tile) {
  Tile T;
  T.lane = threadIdx.x & 31;
  T.w = threadIdx.x >> 5;
  T.r0 = (tile / P.tiles_c) * 128;
  T.c0 = (tile % P.tiles_c) * 128;
  T.col = T.c0 + T.lane * 4;
  T.cok = T.col < P.cols;
  return T;
}

__device__ __forceinline__ void load16x4(const Fp4QuantParams& P, const Tile& T, float (&x)[16][4]) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int64_t row = T.r0 + T.w * 16 + i;
    const uint2 v = (T.cok && row < P.rows) ? ldg_nc_v2(P.x + row * P.ld_x + T.col) : make_uint2(0, 0);
    x[i][0] = bf16_lo(v.x);
    x[i][1] = bf16_hi(v.x);
    x[i][2] = bf16_lo(v.y);
    x[i][3] = bf16_hi(v.y);
  }
}

__device__ __forceinline__ void block_max_atomic(float m, uint32_t* dst) {
  __shared__ float red[8];
  uint32_t b = __float_as_uint(m);
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) b = max(b, __shfl_xor_sync(0xFFFFFFFFu, b, s));
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = __uint_as_float(b);
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t r = __float_as_uint(red[0]);
    for (int k = 1; k < 8; ++k) r = max(r, __float_as_uint(red[k]));
    if (r) atomicMax(dst, r);
  }
}

}  // namespace

// Grid-stride over 128x128 tiles with a bounded grid: one atomicMax per output per CTA.
template <bool ROW, bool COL>
__global__ void __launch_bounds__(256, 3) fp4_amax_kernel(const __grid_constant__ Fp4QuantParams P, int64_t tiles) {
  const uint32_t signs = (P.rht_row || P.rht_col) ? rht_signs(P) : 0u;
  float m_row = 0.0f, m_col = 0.0f;
  for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
    const Tile T = tile_coords(P, tile);
    float x[16][4];
    load16x4(P, T, x);
    float m_plain = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) m_plain = fmaxf(m_plain, fabsf(x[i][j]));
    if (ROW) {
      float m = m_plain;
      if (P.rht_row) {
        m = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float e[4] = {x[i][0], x[i][1], x[i][2], x[i][3]};
          rht_row4(e, signs, T.lane);
#pragma unroll
          for (int j = 0; j < 4; ++j) m = fmaxf(m, fabsf(e[j]));
        }
      }
      m_row = fmaxf(m_row, m);
    }
    if (COL) {
      float m = m_plain;
      if (P.rht_col) {
        m = 0.0f;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          float e[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) e[i] = flip(x[i][j], signs, i);
          fwht16(e);
#pragma unroll
          for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(e[i]));
        }
      }
      m_col = fmaxf(m_col, m);
    }
  }
  if (ROW) block_max_atomic(m_row, P.amax_bits);
  if (COL) block_max_atomic(m_col, P.amax_bits + 1);
}

// Colwise output of one 128x128 tile (16-element groups along rows), from the thread's 16x4
// sub-block: each column's group, its transform and its block amax are in-thread.  The
// transposed codes are staged in `tq` (128 x 64 bytes, 8-byte chunks XOR-swizzled) and
// stored as 64-byte rows; the caller synchronizes the CTA between the two halves.
template <bool SR>
__device__ __forceinline__ void col_codes_to_stage(const Fp4QuantParams& P, const Tile& T, const float (&x)[16][4],
                                                   uint32_t signs, const float* enc_tab, float S_g, uint8_t* tq) {
  const int64_t nsf = P.rows >> 4, s4 = (nsf + 3) >> 2;
  const int64_t kr = (T.r0 >> 4) + T.w;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int64_t cg = T.col + j;
    float e[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) e[i] = P.rht_col ? flip(x[i][j], signs, i) : x[i][j];
    if (P.rht_col) fwht16(e);
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(e[i]));
    uint32_t sb;
    float enc;
    block_scale(m, S_g, enc_tab, sb, enc);
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t c4;
      if (SR) {
        const uint64_t blk = (uint64_t)(cg * P.rows + T.r0 + T.w * 16 + 4 * q) >> 2;
        const uint4 r = philox4x32_10_rk(make_uint4((uint32_t)blk, (uint32_t)(blk >> 32), 0u, 1u), P.sr_rk);
        c4 = e2m1_sr(__fmul_rn(e[4 * q], enc), r.x) | (e2m1_sr(__fmul_rn(e[4 * q + 1], enc), r.y) << 4) |
             (e2m1_sr(__fmul_rn(e[4 * q + 2], enc), r.z) << 8) | (e2m1_sr(__fmul_rn(e[4 * q + 3], enc), r.w) << 12);
      } else {
        c4 = e2m1x2_rne(__fmul_rn(e[4 * q + 1], enc), __fmul_rn(e[4 * q], enc)) |
             (e2m1x2_rne(__fmul_rn(e[4 * q + 3], enc), __fmul_rn(e[4 * q + 2], enc)) << 8);
      }
      if (q < 2) lo |= c4 << (16 * q);
      else hi |= c4 << (16 * (q - 2));
    }
    const int c = T.lane * 4 + j;
    *(uint2*)&tq[c * 64 + ((T.w ^ ((c >> 2) & 7)) * 8)] = make_uint2(lo, hi);
    if (P.sf_tiled) {
      if (kr < s4 * 4) P.sf_col[sf_tiled_offset(cg, kr, s4)] = (uint8_t)sb;
    } else if (cg < P.cols && kr < nsf) {
      P.sf_col[cg * nsf + kr] = (uint8_t)sb;
    }
  }
}

// Stores the staged transposed codes of one tile (after a CTA barrier): 64-byte rows,
// 16-byte stores when the transposed row stride (rows / 2 bytes) allows.
__device__ __forceinline__ void col_stage_store(const Fp4QuantParams& P, const Tile& T, const uint8_t* tq) {
#pragma unroll
  for (int pass = 0; pass < 2; ++pass) {
    const int c = pass * 64 + (threadIdx.x >> 2), h = threadIdx.x & 3;
    const int64_t cg = T.c0 + c, rg = T.r0 + 32 * h;
    const uint2 a = *(const uint2*)&tq[c * 64 + (((2 * h) ^ ((c >> 2) & 7)) * 8)];
    const uint2 b = *(const uint2*)&tq[c * 64 + (((2 * h + 1) ^ ((c >> 2) & 7)) * 8)];
    uint8_t* dst = P.q_col + cg * (P.rows >> 1) + (rg >> 1);
    // the transposed row stride is rows/2 bytes: 16-byte aligned only when rows % 32 == 0
    if (cg < P.cols) {
      if (rg + 32 <= P.rows) {
        if (((P.rows >> 1) & 15) == 0) {
          *(uint4*)dst = make_uint4(a.x, a.y, b.x, b.y);
        } else {
          *(uint2*)dst = a;
          *(uint2*)(dst + 8) = b;
        }
      } else if (rg + 16 <= P.rows) {
        *(uint2*)dst = a;
      }
    }
  }
}

// Colwise output alone.
template <bool SR>
__global__ void __launch_bounds__(256, 3) fp4_quant_col_kernel(const __grid_constant__ Fp4QuantParams P) {
  __shared__ __align__(16) uint8_t tq[128 * 64];
  __shared__ float enc_tab[128];
  const Tile T = tile_coords(P, blockIdx.x);
  float x[16][4];
  load16x4(P, T, x);
  const uint32_t signs = P.rht_col ? rht_signs(P) : 0u;
  const float S_g = global_scale(P.amax_bits[1]);
  if (threadIdx.x < 128) fill_enc_tab(enc_tab, S_g);
  if (blockIdx.x == 0 && threadIdx.x == 0) *P.g_col = __frcp_rn(S_g);
  __syncthreads();
  col_codes_to_stage<SR>(P, T, x, signs, enc_tab, S_g, tq);
  __syncthreads();
  col_stage_store(P, T, tq);
}

// Both outputs from one read of the tile.  The colwise half is the kernel above; the
// rowwise 16-element groups are the 16x4 sub-blocks of 4 consecutive lanes: the group amax
// (and, with the rowwise transform, its two upper butterfly stages) takes two xor-shuffles,
// and each lane's 4 values of a row are 4 consecutive output elements, i.e. one Philox call.
// A warp stores 64 contiguous bytes of each of its 16 rows.  With the MMA-tiled scale layout
// the tiles also cover the image's padding rows and scale columns (their data reads as zero,
// so their scale code is 0).
template <bool SR_ROW, bool SR_COL>
__global__ void __launch_bounds__(256, 2) fp4_quant_rowcol_kernel(const __grid_constant__ Fp4QuantParams P) {
  __shared__ __align__(16) uint8_t tq[128 * 64];
  __shared__ float enc_tab[2][128];
  const Tile T = tile_coords(P, blockIdx.x);
  float x[16][4];
  load16x4(P, T, x);
  const uint32_t signs = (P.rht_row || P.rht_col) ? rht_signs(P) : 0u;
  const float S_row = global_scale(P.amax_bits[0]), S_col = global_scale(P.amax_bits[1]);
  fill_enc_tab(enc_tab[threadIdx.x >> 7], threadIdx.x < 128 ? S_row : S_col);
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    *P.g_row = __frcp_rn(S_row);
    *P.g_col = __frcp_rn(S_col);
  }
  __syncthreads();

  // rowwise output, four rows at a time: lane l & 3 of each 4-lane group makes the block
  // scale (and writes the scale byte) of row i0 + (l & 3); the encode scales are shuffled out
  {
    const int64_t nsf = P.cols >> 4, s4 = (nsf + 3) >> 2;
    const int64_t kc = (T.c0 >> 4) + (T.lane >> 2);
    const int jj = T.lane & 3, grp = T.lane & ~3;
    const bool kc_ok = P.sf_tiled ? kc < s4 * 4 : kc < nsf;
#pragma unroll
    for (int i0 = 0; i0 < 16; i0 += 4) {
      float e[4][4], m[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
#pragma unroll
        for (int k = 0; k < 4; ++k) e[j][k] = x[i0 + j][k];
        if (P.rht_row) rht_row4(e[j], signs, T.lane);
        m[j] = fmaxf(fmaxf(fabsf(e[j][0]), fabsf(e[j][1])), fmaxf(fabsf(e[j][2]), fabsf(e[j][3])));
        m[j] = fmaxf(m[j], __shfl_xor_sync(0xFFFFFFFFu, m[j], 1));
        m[j] = fmaxf(m[j], __shfl_xor_sync(0xFFFFFFFFu, m[j], 2));
      }
      uint32_t sb;
      float enc_own;
      block_scale(jj == 0 ? m[0] : jj == 1 ? m[1] : jj == 2 ? m[2] : m[3], S_row, enc_tab[0], sb, enc_own);
      {
        const int64_t row = T.r0 + T.w * 16 + i0 + jj;
        if (kc_ok) {
          if (P.sf_tiled) P.sf_row[sf_tiled_offset(row, kc, s4)] = (uint8_t)sb;
          else if (row < P.rows) P.sf_row[row * nsf + kc] = (uint8_t)sb;
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t row = T.r0 + T.w * 16 + i0 + j;
        const float enc = __shfl_sync(0xFFFFFFFFu, enc_own, grp | j);
        uint32_t c4;
        if (SR_ROW) {
          const uint64_t blk = (uint64_t)(row * P.cols + T.col) >> 2;
          const uint4 r = philox4x32_10_rk(make_uint4((uint32_t)blk, (uint32_t)(blk >> 32), 0u, 0u), P.sr_rk);
          c4 = e2m1_sr(__fmul_rn(e[j][0], enc), r.x) | (e2m1_sr(__fmul_rn(e[j][1], enc), r.y) << 4) |
               (e2m1_sr(__fmul_rn(e[j][2], enc), r.z) << 8) | (e2m1_sr(__fmul_rn(e[j][3], enc), r.w) << 12);
        } else {
          c4 = e2m1x2_rne(__fmul_rn(e[j][1], enc), __fmul_rn(e[j][0], enc)) |
               (e2m1x2_rne(__fmul_rn(e[j][3], enc), __fmul_rn(e[j][2], enc)) << 8);
        }
        if (T.cok && row < P.rows) *(uint16_t*)(P.q_row + row * (P.cols >> 1) + (T.col >> 1)) = (uint16_t)c4;
      }
    }
  }

  col_codes_to_stage<SR_COL>(P, T, x, signs, enc_tab[1], S_col, tq);
  __syncthreads();
  col_stage_store(P, T, tq);
}

// ------------------------------------------------------------------ 16x16 weight blocks
// One scale per 16x16 block, codes emitted in both layouts (the forward GEMM reads the
// weights along one axis, the backward-data GEMM along the other, and both must see one
// quantized matrix).  Same tile mapping as the colwise kernel: a block is the 16x4
// sub-blocks of 4 consecutive lanes, so its amax is an in-thread max plus two xor-shuffles.
// Codes are computed once, row-paired (2 bytes per row per lane, a warp stores 64 contiguous
// bytes of each row); the colwise words are the same nibbles regrouped along the rows and go
// out through the shared staging tile like the colwise kernel's.
__global__ void __launch_bounds__(256, 3) fp4_quant_2d_kernel(const __grid_constant__ Fp4QuantParams P) {
  __shared__ __align__(16) uint8_t tq[128 * 64];
  __shared__ float enc_tab[128];
  const Tile T = tile_coords(P, blockIdx.x);
  float x[16][4];
  load16x4(P, T, x);
  const float S_g = global_scale(P.amax_bits[0]);
  if (threadIdx.x < 128) fill_enc_tab(enc_tab, S_g);
  if (blockIdx.x == 0 && threadIdx.x == 0) *P.g_row = __frcp_rn(S_g);
  __syncthreads();

  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) m = fmaxf(m, fabsf(x[i][j]));
  m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
  m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
  uint32_t sb;
  float enc;
  block_scale(m, S_g, enc_tab, sb, enc);

  // rc[k]: the 4 codes of row 2k (low half) and of row 2k+1 (high half), column 4*lane + j in
  // nibble j of each half
  uint32_t rc[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    uint32_t v = 0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int i = 2 * k + h;
      v |= (e2m1x2_rne(__fmul_rn(x[i][1], enc), __fmul_rn(x[i][0], enc)) |
            (e2m1x2_rne(__fmul_rn(x[i][3], enc), __fmul_rn(x[i][2], enc)) << 8)) << (16 * h);
    }
    rc[k] = v;
  }

  const int64_t row0 = T.r0 + T.w * 16;
  const int64_t kc = (T.c0 >> 4) + (T.lane >> 2);      // this block's scale column (rowwise)
  const int64_t kr = (T.r0 >> 4) + T.w;                 // its scale column in the colwise output
  if (P.q_row) {
    const int64_t nsf = P.cols >> 4, s4 = (nsf + 3) >> 2;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int64_t row = row0 + i;
      if (T.cok && row < P.rows)
        *(uint16_t*)(P.q_row + row * (P.cols >> 1) + (T.col >> 1)) = (uint16_t)(rc[i >> 1] >> (16 * (i & 1)));
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {                        // lane & 3 == q writes rows 4q..4q+3
      const int64_t row = row0 + 4 * (T.lane & 3) + i;
      if (P.sf_tiled) {
        if (kc < s4 * 4) P.sf_row[sf_tiled_offset(row, kc, s4)] = (uint8_t)sb;
      } else if (row < P.rows && kc < nsf) {
        P.sf_row[row * nsf + kc] = (uint8_t)sb;
      }
    }
  }
  if (P.q_col) {
    const int64_t nsf = P.rows >> 4, s4 = (nsf + 3) >> 2;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t lo = 0, hi = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {           // row i: half i & 1 of rc[i >> 1]
        lo |= ((rc[i >> 1] >> (16 * (i & 1) + 4 * j)) & 0xFu) << (4 * i);
        hi |= ((rc[4 + (i >> 1)] >> (16 * (i & 1) + 4 * j)) & 0xFu) << (4 * i);
      }
      const int c = T.lane * 4 + j;
      const int64_t cg = T.col + j;
      *(uint2*)&tq[c * 64 + ((T.w ^ ((c >> 2) & 7)) * 8)] = make_uint2(lo, hi);
      if (P.sf_tiled) {
        if (kr < s4 * 4) P.sf_col[sf_tiled_offset(cg, kr, s4)] = (uint8_t)sb;
      } else if (cg < P.cols && kr < nsf) {
        P.sf_col[cg * nsf + kr] = (uint8_t)sb;
      }
    }
    __syncthreads();
#pragma unroll
    for (int pass = 0; pass < 2; ++pass) {
      const int c = pass * 64 + (threadIdx.x >> 2), h = threadIdx.x & 3;
      const int64_t cg = T.c0 + c, rg = T.r0 + 32 * h;
      const uint2 a = *(const uint2*)&tq[c * 64 + (((2 * h) ^ ((c >> 2) & 7)) * 8)];
      const uint2 b = *(const uint2*)&tq[c * 64 + (((2 * h + 1) ^ ((c >> 2) & 7)) * 8)];
      uint8_t* dst = P.q_col + cg * (P.rows >> 1) + (rg >> 1);
      if (cg < P.cols) {
        if (rg + 32 <= P.rows) {
          if (((P.rows >> 1) & 15) == 0) {
            *(uint4*)dst = make_uint4(a.x, a.y, b.x, b.y);
          } else {
            *(uint2*)dst = a;
            *(uint2*)(dst + 8) = b;
          }
        } else if (rg + 16 <= P.rows) {
          *(uint2*)dst = a;
        }
      }
    }
  }
}

// ------------------------------------------------------------------ rowwise-only path
// When only the rowwise output is requested, one thread owns one 16-element group of a row
// (two 16-byte loads): the group's transform, amax, scale and codes stay in-thread and a warp
// reads 1 KB of a row per instruction pair.  The butterflies run in the same stage order as
// the tiled kernels, so every value is identical.  With the MMA-tiled scale layout the
// threads also cover the image's padding (rows up to a multiple of 128, scale columns up to
// a multiple of 4), writing scale code 0 there.
__device__ __forceinline__ void load_group16(const Fp4QuantParams& P, int64_t row, int64_t c, float (&e)[16]) {
  const uint16_t* src = P.x + row * P.ld_x + c;
  const uint4 a = ldg_nc_v4(src), b = ldg_nc_v4(src + 8);
  const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    e[2 * i] = bf16_lo(w[i]);
    e[2 * i + 1] = bf16_hi(w[i]);
  }
}

__device__ __forceinline__ void rht16_inthread(float (&e)[16], uint32_t signs) {
#pragma unroll
  for (int i = 0; i < 16; ++i) e[i] = flip(e[i], signs, i);
  fwht16(e);
}

// Grid-stride over the groups with a bounded grid, so the per-CTA atomicMax on the single
// amax word stays rare (one launch per group of 256 would serialize on it).
__global__ void __launch_bounds__(256) fp4_amax_row_kernel(const __grid_constant__ Fp4QuantParams P) {
  const int64_t ng = P.cols >> 4, total = P.rows * ng;
  const uint32_t signs = P.rht_row ? rht_signs(P) : 0u;
  float m = 0.0f;
  for (int64_t g = (int64_t)blockIdx.x * 256 + threadIdx.x; g < total; g += (int64_t)gridDim.x * 256) {
    float e[16];
    load_group16(P, g / ng, (g % ng) * 16, e);
    if (P.rht_row) rht16_inthread(e, signs);
#pragma unroll
    for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(e[i]));
  }
  block_max_atomic(m, P.amax_bits);
}

__global__ void __launch_bounds__(256) fp4_quant_row_kernel(const __grid_constant__ Fp4QuantParams P) {
  __shared__ float enc_tab[128];
  const float S_g = global_scale(P.amax_bits[0]);
  if (threadIdx.x < 128) fill_enc_tab(enc_tab, S_g);
  if (blockIdx.x == 0 && threadIdx.x == 0) *P.g_row = __frcp_rn(S_g);
  __syncthreads();
  const int64_t nsf = P.cols >> 4, s4 = (nsf + 3) >> 2;
  const int64_t kdom = P.sf_tiled ? s4 * 4 : nsf;
  const int64_t rdom = P.sf_tiled ? (P.rows + 127) / 128 * 128 : P.rows;
  const uint32_t signs = P.rht_row ? rht_signs(P) : 0u;
  for (int64_t g = (int64_t)blockIdx.x * 256 + threadIdx.x; g < rdom * kdom; g += (int64_t)gridDim.x * 256) {
    const int64_t row = g / kdom, kc = g % kdom;
    uint32_t sb = 0;
    if (row < P.rows && kc < nsf) {
      const int64_t c = kc * 16;
      float e[16];
      load_group16(P, row, c, e);
      if (P.rht_row) rht16_inthread(e, signs);
      float m = 0.0f;
#pragma unroll
      for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(e[i]));
      float enc;
      block_scale(m, S_g, enc_tab, sb, enc);
      uint32_t w[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t codes = 0;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int j = 8 * h + 4 * q;
          uint32_t c4;
          if (P.sr_row) {
            const uint64_t blk = (uint64_t)(row * P.cols + c + j) >> 2;
            const uint4 r = philox4x32_10_rk(make_uint4((uint32_t)blk, (uint32_t)(blk >> 32), 0u, 0u), P.sr_rk);
            c4 = e2m1_sr(__fmul_rn(e[j], enc), r.x) | (e2m1_sr(__fmul_rn(e[j + 1], enc), r.y) << 4) |
                 (e2m1_sr(__fmul_rn(e[j + 2], enc), r.z) << 8) | (e2m1_sr(__fmul_rn(e[j + 3], enc), r.w) << 12);
          } else {
            c4 = e2m1x2_rne(__fmul_rn(e[j + 1], enc), __fmul_rn(e[j], enc)) |
                 (e2m1x2_rne(__fmul_rn(e[j + 3], enc), __fmul_rn(e[j + 2], enc)) << 8);
          }
          codes |= c4 << (16 * q);
        }
        w[h] = codes;
      }
      *(uint2*)(P.q_row + row * (P.cols >> 1) + (c >> 1)) = make_uint2(w[0], w[1]);
    }
    if (P.sf_tiled) P.sf_row[sf_tiled_offset(row, kc, s4)] = (uint8_t)sb;
    else P.sf_row[row * nsf + kc] = (uint8_t)sb;
  }
}

// Grid of the group-per-thread kernels: enough CTAs to fill the GPU, at most 8192.
static unsigned blocks_for(int64_t threads) {
  const int64_t b = (threads + 255) / 256;
  return (unsigned)(b < 8192 ? b : 8192);
}

cudaError_t launch_fp4_amax(const Fp4QuantParams& p, int64_t tiles, cudaStream_t s) {
  const bool row = p.q_row != nullptr, col = p.q_col != nullptr;
  const unsigned tile_grid = (unsigned)(tiles < 2048 ? tiles : 2048);
  if (row && col) fp4_amax_kernel<true, true><<<tile_grid, 256, 0, s>>>(p, tiles);
  else if (row) fp4_amax_row_kernel<<<blocks_for(p.rows * (p.cols >> 4)), 256, 0, s>>>(p);
  else fp4_amax_kernel<false, true><<<tile_grid, 256, 0, s>>>(p, tiles);
  return cudaGetLastError();
}

cudaError_t launch_fp4_quant_2d(const Fp4QuantParams& p, int64_t tiles, cudaStream_t s) {
  fp4_amax_row_kernel<<<blocks_for(p.rows * (p.cols >> 4)), 256, 0, s>>>(p);
  fp4_quant_2d_kernel<<<(unsigned)tiles, 256, 0, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_fp4_quant(const Fp4QuantParams& p, int64_t tiles, cudaStream_t s) {
  const bool row = p.q_row != nullptr, col = p.q_col != nullptr;
  const unsigned grid = (unsigned)tiles;
  if (row && col) {   // both outputs from one read of each tile
    if (p.sr_row && p.sr_col) fp4_quant_rowcol_kernel<true, true><<<grid, 256, 0, s>>>(p);
    else if (p.sr_row) fp4_quant_rowcol_kernel<true, false><<<grid, 256, 0, s>>>(p);
    else if (p.sr_col) fp4_quant_rowcol_kernel<false, true><<<grid, 256, 0, s>>>(p);
    else fp4_quant_rowcol_kernel<false, false><<<grid, 256, 0, s>>>(p);
    return cudaGetLastError();
  }
  if (row) {
    const int64_t nsf = p.cols >> 4, kdom = p.sf_tiled ? (nsf + 3) / 4 * 4 : nsf;
    const int64_t rdom = p.sf_tiled ? (p.rows + 127) / 128 * 128 : p.rows;
    fp4_quant_row_kernel<<<blocks_for(rdom * kdom), 256, 0, s>>>(p);
  }
  if (col) {
    if (p.sr_col) fp4_quant_col_kernel<true><<<grid, 256, 0, s>>>(p);
    else fp4_quant_col_kernel<false><<<grid, 256, 0, s>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace fp8q
