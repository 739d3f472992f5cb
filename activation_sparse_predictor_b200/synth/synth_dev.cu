/*
 * Device side of the seeded synthetic-input generator (see rng.h): fills
 * device buffers in place with exactly the bits the host generator
 * produces, so multi-gigabyte layer stacks never cross PCIe.  Compiled with
 * -fmad=false so no multiply-add contraction can change a rounding.
 */
#include <stdint.h>
#include <cuda_runtime.h>
#include "rng.h"

namespace {

__global__ void fill_f32(uint64_t key, double sigma, int64_t n, float* out) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n;
       e += (int64_t)gridDim.x * blockDim.x)
    out[e] = (float)(sigma * sy_gauss(key, (uint64_t)e));
}

__global__ void fill_f16(uint64_t key, double sigma, int64_t n, uint16_t* out) {
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < n;
       e += (int64_t)gridDim.x * blockDim.x)
    out[e] = sy_half_bits(sigma * sy_gauss(key, (uint64_t)e));
}

__global__ void fill_q4_0(uint64_t key, double sigma, int64_t rows, int64_t cols,
                          uint8_t* qs, uint16_t* scales) {
  int64_t nb = cols / 32;
  for (int64_t blk = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; blk < rows * nb;
       blk += (int64_t)gridDim.x * blockDim.x) {
    int64_t i = blk / nb, b = blk % nb;
    double w[32];
    for (int k = 0; k < 32; ++k)
      w[k] = sigma * sy_gauss(key, (uint64_t)(i * cols + b * 32 + k));
    uint8_t q[16];
    uint16_t s;
    sy_q4_0_encode(w, q, &s);
    uint4 v;
    v.x = q[0] | (q[1] << 8) | (q[2] << 16) | ((uint32_t)q[3] << 24);
    v.y = q[4] | (q[5] << 8) | (q[6] << 16) | ((uint32_t)q[7] << 24);
    v.z = q[8] | (q[9] << 8) | (q[10] << 16) | ((uint32_t)q[11] << 24);
    v.w = q[12] | (q[13] << 8) | (q[14] << 16) | ((uint32_t)q[15] << 24);
    *reinterpret_cast<uint4*>(qs + blk * 16) = v;
    scales[blk] = s;
  }
}

int grid_for(int64_t n) {
  int64_t g = (n + 255) / 256;
  if (g > 148 * 64) g = 148 * 64;
  if (g < 1) g = 1;
  return (int)g;
}

}  // namespace

extern "C" {

/* All return 0 on success, else the cudaError_t of the launch. */
int sy_dev_fill_f32(uint64_t key, double sigma, int64_t n, float* out, void* stream) {
  if (n <= 0) return 0;
  fill_f32<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(key, sigma, n, out);
  return (int)cudaGetLastError();
}

int sy_dev_fill_f16(uint64_t key, double sigma, int64_t n, uint16_t* out, void* stream) {
  if (n <= 0) return 0;
  fill_f16<<<grid_for(n), 256, 0, (cudaStream_t)stream>>>(key, sigma, n, out);
  return (int)cudaGetLastError();
}

int sy_dev_fill_q4_0(uint64_t key, double sigma, int64_t rows, int64_t cols, uint8_t* qs,
                     uint16_t* scales, void* stream) {
  if (rows <= 0 || cols <= 0 || (cols % 32) != 0) return rows <= 0 ? 0 : 1;
  fill_q4_0<<<grid_for(rows * (cols / 32)), 256, 0, (cudaStream_t)stream>>>(key, sigma, rows,
                                                                         cols, qs, scales);
  return (int)cudaGetLastError();
}

}  // extern "C"
