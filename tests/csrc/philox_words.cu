// Test-only export of the library's device Philox4x32-10 (uno_device.cuh):
// evaluates it at caller-given counters and keys so that a test can compare
// the device's words with the generator's published known-answer vectors.
// Built by tests/test_gpu_philox.py; not part of libuno.so.
#include <cstdint>

#include <cuda_runtime.h>

#include "uno_device.cuh"

namespace {

__global__ void philox_words_kernel(const uint32_t* in, uint32_t* out, int n) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= n) return;
  const uint32_t* c = in + 6 * j;  // counter words 0..3, then key words 0..1
  const uint4 w = uno::philox4x32_10(make_uint4(c[0], c[1], c[2], c[3]), make_uint2(c[4], c[5]));
  out[4 * j + 0] = w.x;
  out[4 * j + 1] = w.y;
  out[4 * j + 2] = w.z;
  out[4 * j + 3] = w.w;
}

}  // namespace

// host_in: n x 6 words (counter, key); host_out: n x 4 words. Returns 0 on
// success, otherwise the CUDA error code.
extern "C" int philox_words(const uint32_t* host_in, uint32_t* host_out, int n) {
  if (n <= 0) return 0;
  uint32_t *d_in = nullptr, *d_out = nullptr;
  cudaError_t e = cudaMalloc(&d_in, sizeof(uint32_t) * 6 * n);
  if (e == cudaSuccess) e = cudaMalloc(&d_out, sizeof(uint32_t) * 4 * n);
  if (e == cudaSuccess)
    e = cudaMemcpy(d_in, host_in, sizeof(uint32_t) * 6 * n, cudaMemcpyHostToDevice);
  if (e == cudaSuccess) {
    philox_words_kernel<<<(n + 127) / 128, 128>>>(d_in, d_out, n);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess)
    e = cudaMemcpy(host_out, d_out, sizeof(uint32_t) * 4 * n, cudaMemcpyDeviceToHost);
  cudaFree(d_in);
  cudaFree(d_out);
  return static_cast<int>(e);
}
