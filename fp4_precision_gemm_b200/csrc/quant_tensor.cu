// Per-tensor current scaling (the coarse NeMo recipe): "Accelerating FP8 training
// performance with the NVIDIA NeMo framework" compares it with the fine-grained recipes.
// Current scaling needs the tensor's amax before any code can be written, so it takes two
// passes: an amax reduction (packed BF16 magnitudes, warp shuffles, one atomicMax per CTA
// on the FP32 bit pattern, which orders like the value for non-negative floats) and a cast.
// Both are 2-D grids over (16-byte column chunks, rows) so no thread divides by the row
// length; the row loop strides by gridDim.y.
#include <cfloat>
#include <mutex>

#include "../../include/fp8q.h"
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

// Eight BF16 values times sf, to E4M3 (or E5M2), as two words.
template <bool E5M2>
__device__ __forceinline__ uint2 cast8(const uint4& v, float sf) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t c[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float a = __fmul_rn(bf16_lo(w[i]), sf), b = __fmul_rn(bf16_hi(w[i]), sf);
    c[i] = E5M2 ? cvt_e5m2x2(a, b) : cvt_e4m3x2(a, b);
  }
  return make_uint2(c[0] | (c[1] << 16), c[2] | (c[3] << 16));
}

__global__ void __launch_bounds__(256) tensor_cast_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                          int64_t cols, int64_t ld_x,
                                                          const uint32_t* amax_bits, uint8_t* q,
                                                          float* s_dec) {
  const float sf = e4m3_sf(__uint_as_float(*amax_bits));
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *s_dec = __frcp_rn(sf);
  const int64_t c8 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (c8 * 8 >= cols) return;
  for (int64_t r = blockIdx.y; r < rows; r += gridDim.y)
    *(uint2*)(q + r * cols + c8 * 8) = cast8<false>(ldg_nc_v4(x + r * ld_x + c8 * 8), sf);
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

__global__ void fill_f32_kernel(float* dst, float v) { *dst = v; }

cudaError_t launch_fill_f32(float* dst, float v, cudaStream_t s) {
  fill_f32_kernel<<<1, 1, 0, s>>>(dst, v);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ delayed scaling
// One pass: the scale comes from the largest amax of earlier iterations (the history), so
// every CTA can cast as it reads (four rows' loads in flight per thread: 8-11% faster than
// one; the same unrolling made the two-pass current-scaling kernels slower on the smaller
// tensors, so they keep one); the tensor's own amax is reduced on the way (one
// atomicMax per CTA into a scratch word) and recorded into the history by a one-thread
// kernel afterwards, so no CTA reads a history slot while it is being replaced.
template <bool E5M2>
__global__ void __launch_bounds__(256) tensor_delayed_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                             int64_t cols, int64_t ld_x, const float* hist, int hlen,
                                                             uint8_t* q, float* s_dec, uint32_t* amax_bits) {
  __shared__ float sf_sh;
  __shared__ uint32_t red[8];
  if (threadIdx.x < 32) {
    float hm = 0.0f;
    for (int i = threadIdx.x; i < hlen; i += 32) hm = fmaxf(hm, hist[i]);
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) hm = fmaxf(hm, __shfl_xor_sync(0xFFFFFFFFu, hm, s));
    if (threadIdx.x == 0) {
      float sf = 1.0f;
      if (hm > 0.0f) {
        sf = __fdiv_rn(E5M2 ? 57344.0f : 448.0f, hm);
        if (sf > FLT_MAX) sf = FLT_MAX;
      }
      sf_sh = sf;
    }
  }
  __syncthreads();
  const float sf = sf_sh;
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *s_dec = __frcp_rn(sf);
  const int64_t c8 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  uint32_t m = 0;
  if (c8 * 8 < cols) {
    const int64_t g = gridDim.y;
    int64_t r = blockIdx.y;
    for (; r + 3 * g < rows; r += 4 * g) {
      uint4 v[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) v[k] = ldg_nc_v4(x + (r + k * g) * ld_x + c8 * 8);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        m = max2(m, max2(max2(abs2(v[k].x), abs2(v[k].y)), max2(abs2(v[k].z), abs2(v[k].w))));
        *(uint2*)(q + (r + k * g) * cols + c8 * 8) = cast8<E5M2>(v[k], sf);
      }
    }
    for (; r < rows; r += g) {
      const uint4 v = ldg_nc_v4(x + r * ld_x + c8 * 8);
      m = max2(m, max2(max2(abs2(v.x), abs2(v.y)), max2(abs2(v.z), abs2(v.w))));
      *(uint2*)(q + r * cols + c8 * 8) = cast8<E5M2>(v, sf);
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

__global__ void tensor_delayed_record(const uint32_t* amax_bits, float* hist, int pos) {
  hist[pos] = __uint_as_float(*amax_bits);
}

cudaError_t launch_tensor_delayed(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld_x, float* hist,
                                  int hlen, int pos, bool e5m2, uint8_t* q, float* s_dec, uint32_t* amax_bits,
                                  cudaStream_t s) {
  const dim3 grid = (rows > 0 && cols > 0) ? tensor_grid(rows, cols) : dim3(1, 1);
  if (e5m2) tensor_delayed_kernel<true><<<grid, 256, 0, s>>>(x, rows, cols, ld_x, hist, hlen, q, s_dec, amax_bits);
  else tensor_delayed_kernel<false><<<grid, 256, 0, s>>>(x, rows, cols, ld_x, hist, hlen, q, s_dec, amax_bits);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  tensor_delayed_record<<<1, 1, 0, s>>>(amax_bits, hist, pos);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ allocation-free variant
// Scratch of fp8q_quantize_tensor_noalloc: a fixed array in the library's own device
// globals, so the call never allocates.  Word 0 holds the running amax of the current call.
namespace {
constexpr int kNoAllocWords = 64;  // 256 bytes on every device that loads the library
constexpr int kNoAllocMaxDevices = 64;
static __device__ __align__(256) uint32_t g_noalloc_scratch[kNoAllocWords];
uint32_t* g_noalloc_addr[kNoAllocMaxDevices] = {};
std::mutex g_noalloc_mutex;

// Device address of g_noalloc_scratch on the current device (the host-side symbol is only
// a stand-in); looked up once per device, with that device current.
cudaError_t noalloc_scratch(uint32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_addr[dev] = static_cast<uint32_t*>(p);
  }
  *out = g_noalloc_addr[dev];
  return cudaSuccess;
}
}  // namespace

}  // namespace fp8q

extern "C" fp8q_status fp8q_quantize_tensor_noalloc(const void* x, int64_t rows, int64_t cols, int64_t ld_x,
                                                    uint8_t* q, float* s_dec, void* stream) {
  using namespace fp8q;
  if (rows < 0 || cols < 0 || rows >= (1ll << 31) || cols >= (1ll << 31)) return FP8Q_ERR_SHAPE;
  if (!q || !s_dec) return FP8Q_ERR_NULL;
  if (rows > 0 && cols > 0) {
    if (!x) return FP8Q_ERR_NULL;
    if (ld_x < cols || ld_x % 8 != 0) return FP8Q_ERR_SHAPE;
    if ((reinterpret_cast<uintptr_t>(x) & 15u) != 0) return FP8Q_ERR_ALIGN;
  }
  if (cols % 8 != 0) return FP8Q_ERR_SHAPE;
  if ((reinterpret_cast<uintptr_t>(q) & 15u) != 0) return FP8Q_ERR_ALIGN;
  constexpr int kWordsNeeded = 1;  // one amax word per call
  static_assert(kWordsNeeded <= kNoAllocWords, "scratch array too small");
  if (kWordsNeeded > kNoAllocWords) return FP8Q_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t* amax = nullptr;
  if (noalloc_scratch(&amax) != cudaSuccess) return FP8Q_ERR_CUDA;
  if (rows == 0 || cols == 0)   // empty tensor: amax 0 -> sf 1 -> decode scale 1, written on `stream`
    return launch_fill_f32(s_dec, 1.0f, s) == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
  // the array keeps the previous call's amax: clear the word before this call's reduction
  if (cudaMemsetAsync(amax, 0, kWordsNeeded * sizeof(uint32_t), s) != cudaSuccess) return FP8Q_ERR_CUDA;
  cudaError_t e = launch_tensor_amax(static_cast<const uint16_t*>(x), rows, cols, ld_x, amax, s);
  if (e == cudaSuccess) e = launch_tensor_cast(static_cast<const uint16_t*>(x), rows, cols, ld_x, amax, q, s_dec, s);
  return e == cudaSuccess ? FP8Q_OK : FP8Q_ERR_CUDA;
}

