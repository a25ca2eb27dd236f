// Test-only probe: evaluates the library's FMA-pipe exp2 polynomial and
// CUDA's exp2f on the same inputs so the test can check the error bound.
#include <cuda_runtime.h>

#include "../../swa_hybrid_attention_b200/csrc/exp2_poly.cuh"

__global__ void probe(const float* x, float* y_poly, float* y_pack, float* y_ref, int n) {
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) {
    y_poly[i] = rtp::exp2_poly(x[i]);
    y_ref[i] = exp2f(x[i]);
    const int j = ((i ^ 1) < n) ? (i ^ 1) : i;  // pair each input with a neighbour
    y_pack[i] = rtp::lo2(rtp::exp2_poly2(x[i], x[j]));
  }
}

extern "C" int exp2_probe(const float* x_host, float* poly_host, float* pack_host, float* ref_host, int n) {
  float *x, *yp, *yk, *yr;
  if (cudaMalloc(&x, n * sizeof(float)) != cudaSuccess) return 1;
  cudaMalloc(&yp, n * sizeof(float));
  cudaMalloc(&yk, n * sizeof(float));
  cudaMalloc(&yr, n * sizeof(float));
  cudaMemcpy(x, x_host, n * sizeof(float), cudaMemcpyHostToDevice);
  probe<<<(n + 255) / 256, 256>>>(x, yp, yk, yr, n);
  cudaError_t e = cudaDeviceSynchronize();
  cudaMemcpy(poly_host, yp, n * sizeof(float), cudaMemcpyDeviceToHost);
  cudaMemcpy(pack_host, yk, n * sizeof(float), cudaMemcpyDeviceToHost);
  cudaMemcpy(ref_host, yr, n * sizeof(float), cudaMemcpyDeviceToHost);
  cudaFree(x);
  cudaFree(yp);
  cudaFree(yk);
  cudaFree(yr);
  return e == cudaSuccess ? 0 : 2;
}
