// Test helper: Philox4x32-10 words from cuRAND's own implementation, used to pin the
// CPU oracle's generator to an implementation other than itself.
#include <cuda_runtime.h>
#include <curand_philox4x32_x.h>

__global__ void philox_curand_kernel(const unsigned* in, unsigned* out, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const uint4 c = make_uint4(in[6 * i], in[6 * i + 1], in[6 * i + 2], in[6 * i + 3]);
  const uint2 k = make_uint2(in[6 * i + 4], in[6 * i + 5]);
  const uint4 r = curand_Philox4x32_10(c, k);
  out[4 * i] = r.x;
  out[4 * i + 1] = r.y;
  out[4 * i + 2] = r.z;
  out[4 * i + 3] = r.w;
}

// ctr_key: n rows of (c0, c1, c2, c3, k0, k1); out: n rows of 4 words.  Returns 0 on success.
extern "C" int philox_curand(const unsigned* ctr_key, unsigned* out, int n) {
  unsigned *d_in = nullptr, *d_out = nullptr;
  if (cudaMalloc(&d_in, sizeof(unsigned) * 6 * n) != cudaSuccess) return 1;
  if (cudaMalloc(&d_out, sizeof(unsigned) * 4 * n) != cudaSuccess) return 1;
  cudaMemcpy(d_in, ctr_key, sizeof(unsigned) * 6 * n, cudaMemcpyHostToDevice);
  philox_curand_kernel<<<(n + 127) / 128, 128>>>(d_in, d_out, n);
  const cudaError_t e = cudaMemcpy(out, d_out, sizeof(unsigned) * 4 * n, cudaMemcpyDeviceToHost);
  cudaFree(d_in);
  cudaFree(d_out);
  return e == cudaSuccess ? 0 : 2;
}
