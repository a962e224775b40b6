// synth_cuda.cu - device-side fill of the seeded synthetic inputs (moe_synth.h).
// Produces bit-identical values to synth_host.c for the same (seed, tensor id,
// index, sigma, mean). Exported with a plain C ABI.
#include <cuda_runtime.h>
#include <stdint.h>

#include "moe_synth.h"

namespace {

__global__ void fill_kernel(uint64_t key, uint64_t start, uint64_t n, float sigma, float mean,
                            uint16_t* __restrict__ out) {
  const uint64_t stride = (uint64_t)gridDim.x * blockDim.x * 2;
  for (uint64_t i = ((uint64_t)blockIdx.x * blockDim.x + threadIdx.x) * 2; i < n; i += stride) {
    const uint16_t a = ms_value_bf16(key, start + i, sigma, mean);
    if (i + 1 < n && ((reinterpret_cast<uintptr_t>(out + i) & 3u) == 0)) {
      const uint16_t b = ms_value_bf16(key, start + i + 1, sigma, mean);
      *reinterpret_cast<uint32_t*>(out + i) = (uint32_t)a | ((uint32_t)b << 16);
    } else {
      out[i] = a;
      if (i + 1 < n) out[i + 1] = ms_value_bf16(key, start + i + 1, sigma, mean);
    }
  }
}

__global__ void fill_e4m3_kernel(uint64_t key, uint64_t start, uint64_t n, uint8_t* __restrict__ out) {
  const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
    out[i] = ms_code_e4m3(key, start + i);
}

__global__ void fill_e4m3_cover_kernel(uint64_t key, uint64_t start, uint64_t n, uint64_t rows, uint64_t cols,
                                       uint32_t phase, uint8_t* __restrict__ out) {
  const uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
    out[i] = ms_code_e4m3_cover(key, start + i, rows, cols, phase);
}

}  // namespace

extern "C" {

// Fills out[0..n) (device memory) with the coverage codes ms_code_e4m3_cover of elements
// start .. start + n - 1 of an expert stack [E][rows][cols]. Asynchronous on `stream`;
// returns a cudaError_t value (0 on success).
int ms_fill_e4m3_cover_device(uint64_t seed, uint64_t tensor_id, uint64_t start, uint64_t n, uint64_t rows,
                              uint64_t cols, uint32_t phase, void* out, void* stream) {
  if (n == 0) return 0;
  if (out == nullptr || rows == 0 || cols == 0) return (int)cudaErrorInvalidValue;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return (int)e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return (int)e;
  uint64_t blocks = (n + 255) / 256;
  const uint64_t cap = (uint64_t)sms * 16;
  if (blocks > cap) blocks = cap;
  fill_e4m3_cover_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(ms_key(seed, tensor_id), start, n,
                                                                             rows, cols, phase, (uint8_t*)out);
  return (int)cudaGetLastError();
}

// Fills out[0..n) (device memory) with the E4M3 codes ms_code_e4m3(key(seed, tid), start + i).
// Asynchronous on `stream`; returns a cudaError_t value (0 on success).
int ms_fill_e4m3_device(uint64_t seed, uint64_t tensor_id, uint64_t start, uint64_t n, void* out, void* stream) {
  if (n == 0) return 0;
  if (out == nullptr) return (int)cudaErrorInvalidValue;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return (int)e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return (int)e;
  uint64_t blocks = (n + 255) / 256;
  const uint64_t cap = (uint64_t)sms * 16;
  if (blocks > cap) blocks = cap;
  fill_e4m3_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(ms_key(seed, tensor_id), start, n,
                                                                       (uint8_t*)out);
  return (int)cudaGetLastError();
}


// Fills out[0..n) (device memory) with bf16(mean + sigma * z(key(seed, tid), start + i)).
// Asynchronous on `stream`; returns a cudaError_t value (0 on success).
int ms_fill_device(uint64_t seed, uint64_t tensor_id, uint64_t start, uint64_t n, float sigma,
                   float mean, void* out, void* stream) {
  if (n == 0) return 0;
  if (out == nullptr) return (int)cudaErrorInvalidValue;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return (int)e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return (int)e;
  const uint64_t pairs = (n + 1) / 2;
  uint64_t blocks = (pairs + 255) / 256;
  const uint64_t cap = (uint64_t)sms * 16;
  if (blocks > cap) blocks = cap;
  fill_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(ms_key(seed, tensor_id), start, n,
                                                                  sigma, mean, (uint16_t*)out);
  return (int)cudaGetLastError();
}

}  // extern "C"
