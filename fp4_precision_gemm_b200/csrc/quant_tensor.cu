// Per-tensor current scaling (the coarse NeMo recipe): "Accelerating FP8 training
// performance with the NVIDIA NeMo framework" compares it with the fine-grained recipes.
// Current scaling needs the tensor's amax before any code can be written, so it takes two
// passes: an amax reduction (packed BF16 magnitudes, warp shuffles, one atomicMax per CTA
// on the FP32 bit pattern, which orders like the value for non-negative floats) and a cast.
// Both are 2-D grids over (16-byte column chunks, rows) so no thread divides by the row
// length; the row loop strides by gridDim.y.
#include "common.cuh"
#include "kernels.h"

namespace fp8q {

__global__ void __launch_bounds__(256) tensor_amax_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                          int64_t cols, int64_t ld_x, uint32_t* amax_bits) {
  __shared__ uint32_t red[8];
  const int64_t c8 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  uint32_t m = 0;
  if (c8 * 8 < cols) {
    for (int64_t r = blockIdx.y; r < rows; r += gridDim.y) {
      const uint4 v = ldg_nc_v4(x + r * ld_x + c8 * 8);
      m = max2(m, max2(max2(abs2(v.x), abs2(v.y)), max2(abs2(v.z), abs2(v.w))));
    }
  }
  m = hmax(m);
#pragma unroll
  for (int s = 16; s > 0; s >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, s));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t b = red[0];
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) b = max(b, red[w]);
    if (b) atomicMax(amax_bits, b << 16);
  }
}

__global__ void __launch_bounds__(256) tensor_cast_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                          int64_t cols, int64_t ld_x,
                                                          const uint32_t* amax_bits, uint8_t* q,
                                                          float* s_dec) {
  const float sf = e4m3_sf(__uint_as_float(*amax_bits));
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *s_dec = __frcp_rn(sf);
  const int64_t c8 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (c8 * 8 >= cols) return;
  for (int64_t r = blockIdx.y; r < rows; r += gridDim.y) {
    const uint4 v = ldg_nc_v4(x + r * ld_x + c8 * 8);
    uint2 o;
    o.x = cvt_e4m3x2(__fmul_rn(bf16_lo(v.x), sf), __fmul_rn(bf16_hi(v.x), sf)) |
          (cvt_e4m3x2(__fmul_rn(bf16_lo(v.y), sf), __fmul_rn(bf16_hi(v.y), sf)) << 16);
    o.y = cvt_e4m3x2(__fmul_rn(bf16_lo(v.z), sf), __fmul_rn(bf16_hi(v.z), sf)) |
          (cvt_e4m3x2(__fmul_rn(bf16_lo(v.w), sf), __fmul_rn(bf16_hi(v.w), sf)) << 16);
    *(uint2*)(q + r * cols + c8 * 8) = o;
  }
}

static dim3 tensor_grid(int64_t rows, int64_t cols) {
  const int64_t gx = (cols / 8 + 255) / 256;
  int64_t gy = (148 * 16 + gx - 1) / gx;  // about 16 CTAs per SM in total
  if (gy > rows) gy = rows;
  if (gy > 65535) gy = 65535;
  if (gy < 1) gy = 1;
  return dim3((unsigned)gx, (unsigned)gy);
}

cudaError_t launch_tensor_amax(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld_x,
                               uint32_t* amax_bits, cudaStream_t s) {
  tensor_amax_kernel<<<tensor_grid(rows, cols), 256, 0, s>>>(x, rows, cols, ld_x, amax_bits);
  return cudaGetLastError();
}

cudaError_t launch_tensor_cast(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld_x,
                               const uint32_t* amax_bits, uint8_t* q, float* s_dec,
                               cudaStream_t s) {
  tensor_cast_kernel<<<tensor_grid(rows, cols), 256, 0, s>>>(x, rows, cols, ld_x, amax_bits, q, s_dec);
  return cudaGetLastError();
}

}  // namespace fp8q
