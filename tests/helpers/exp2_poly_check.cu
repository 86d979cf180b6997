// Test helper: compares the library's FMA-pipe 2^x (exp2_poly2) with CUDA's
// exp2f over x in [-125, 8] and reports the maximum relative error, plus the
// values at the clamp (x = -126, -200, -inf).
#include <cstdio>
#include <cmath>
#include "dd_device.cuh"

__global__ void check(int n, float lo, float hi, double* maxrel, float* clamp_out) {
  __shared__ double red[256];
  double worst = 0.0;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const float x0 = lo + (hi - lo) * (float)i / (float)(n - 1);
    const float x1 = -x0 * 0.5f;  // also exercise the second lane
    const float2 r = dd::exp2_poly2(make_float2(x0, x1));
    const double e0 = fabs((double)r.x / (double)exp2f(x0) - 1.0);
    const double e1 = fabs((double)r.y / (double)exp2f(x1) - 1.0);
    worst = fmax(worst, fmax(e0, e1));
  }
  red[threadIdx.x] = worst;
  __syncthreads();
  for (int s = 128; s > 0; s >>= 1) {
    if (threadIdx.x < s) red[threadIdx.x] = fmax(red[threadIdx.x], red[threadIdx.x + s]);
    __syncthreads();
  }
  if (threadIdx.x == 0) maxrel[blockIdx.x] = red[0];
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    const float2 a = dd::exp2_poly2(make_float2(-126.0f, -200.0f));
    const float2 b = dd::exp2_poly2(make_float2(-INFINITY, 0.0f));
    clamp_out[0] = a.x; clamp_out[1] = a.y; clamp_out[2] = b.x; clamp_out[3] = b.y;
  }
}

int main() {
  const int blocks = 256, n = 1 << 24;
  double* d; float* c;
  cudaMalloc(&d, blocks * sizeof(double));
  cudaMalloc(&c, 4 * sizeof(float));
  check<<<blocks, 256>>>(n, -125.0f, 8.0f, d, c);
  double h[blocks]; float hc[4];
  if (cudaMemcpy(h, d, sizeof h, cudaMemcpyDeviceToHost) != cudaSuccess) return 2;
  cudaMemcpy(hc, c, sizeof hc, cudaMemcpyDeviceToHost);
  double m = 0; for (double v : h) m = v > m ? v : m;
  printf("maxrel %.6e\nclamp %.9e %.9e %.9e %.9e\n", m, hc[0], hc[1], hc[2], hc[3]);
  return 0;
}
