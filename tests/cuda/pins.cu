// Test-only kernels that pin the CPU oracle to CUDA itself (not part of the library):
//   * cuRAND's Philox4x32-10 (curand_Philox4x32_10) on given counters and keys, so the
//     oracle's Philox can be checked word for word against CUDA's outputs;
//   * the conversion instructions the quantize kernels rely on, on arbitrary FP32 inputs,
//     so the oracle's E4M3 / E5M2 / E2M1 encoders can be checked against the hardware.
#include <cstdint>
#include <cuda_runtime.h>
#include <curand_kernel.h>

__global__ void curand_philox_kernel(const uint4* ctr, const uint2* key, uint4* out, int n) {
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = curand_Philox4x32_10(ctr[i], key[i]);
}

__global__ void cvt_e4m3_kernel(const float* x, uint8_t* out, int n) {
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x[i]));
    out[i] = (uint8_t)(r & 0xFF);
  }
}

__global__ void cvt_e5m2_kernel(const float* x, uint8_t* out, int n) {
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    uint16_t r;
    asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x[i]));
    out[i] = (uint8_t)(r & 0xFF);
  }
}

__global__ void cvt_e2m1_kernel(const float* x, uint8_t* out, int n) {
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
        : "=r"(r) : "f"(0.0f), "f"(x[i]));
    out[i] = (uint8_t)(r & 0xF);
  }
}

extern "C" {
int pins_curand_philox(const void* ctr, const void* key, void* out, int n, void* stream) {
  curand_philox_kernel<<<(n + 255) / 256, 256, 0, (cudaStream_t)stream>>>((const uint4*)ctr, (const uint2*)key,
                                                                         (uint4*)out, n);
  return (int)cudaGetLastError();
}
int pins_cvt_e4m3(const void* x, void* out, int n, void* stream) {
  cvt_e4m3_kernel<<<(n + 255) / 256, 256, 0, (cudaStream_t)stream>>>((const float*)x, (uint8_t*)out, n);
  return (int)cudaGetLastError();
}
int pins_cvt_e5m2(const void* x, void* out, int n, void* stream) {
  cvt_e5m2_kernel<<<(n + 255) / 256, 256, 0, (cudaStream_t)stream>>>((const float*)x, (uint8_t*)out, n);
  return (int)cudaGetLastError();
}
int pins_cvt_e2m1(const void* x, void* out, int n, void* stream) {
  cvt_e2m1_kernel<<<(n + 255) / 256, 256, 0, (cudaStream_t)stream>>>((const float*)x, (uint8_t*)out, n);
  return (int)cudaGetLastError();
}
}
