// Float32 CUDA-core GEMM for the SAMBAY_F32 mode (true fp32 FFMA, no TF32),
// with the same fused epilogues as the tensor-core path.
//
//   D[m, n] = sum_k A[m, k] * B[k, n],  A(m, k) = A[m * sam + k * sak],
//                                       B(k, n) = B[k * sbk + n * sbn]
// Tile 64 x 64 x 16, 256 threads, 4 x 4 outputs per thread.
#pragma once

#include "common.cuh"

namespace sambay {
namespace simt {

enum Kind : int { F32_STORE = 0, GATE = 1, RESID = 2, SOFTPLUS = 3 };

struct Args {
  const float* A;
  long long sam, sak;
  const float* B;
  long long sbk, sbn;
  int M, N, K;
  float* out;          // [M, N] row-major, leading dimension ldo
  long long ldo;
  const float* aux;    // GATE: memory readout [M, N]; RESID: residual or NULL
  const float* vec;    // SOFTPLUS: per-column bias
  int trans;           // store out[n * ldo + m] (and read aux the same way)
};

template <int KIND>
__global__ void __launch_bounds__(256) simt_gemm_kernel(const Args g) {
  pdl_wait();
  pdl_launch_dependents();
  __shared__ float sa[16][64 + 4];
  __shared__ float sb[16][64 + 4];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < g.K; k0 += 16) {
    for (int i = threadIdx.x; i < 16 * 64; i += 256) {
      const int kk = i / 64, mm = i % 64;
      const int m = m0 + mm, k = k0 + kk;
      sa[kk][mm] = (m < g.M && k < g.K) ? g.A[m * g.sam + k * g.sak] : 0.0f;
      const int n = n0 + mm;
      sb[kk][mm] = (n < g.N && k < g.K) ? g.B[k * g.sbk + n * g.sbn] : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = sa[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = sb[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= g.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n >= g.N) continue;
      const long long o = g.trans ? static_cast<long long>(n) * g.ldo + m
                                  : static_cast<long long>(m) * g.ldo + n;
      const float v = acc[i][j];
      if (KIND == F32_STORE) g.out[o] = v;
      else if (KIND == GATE) g.out[o] = silu(v) * g.aux[o];
      else if (KIND == RESID) g.out[o] = v + (g.aux ? g.aux[o] : 0.0f);
      else g.out[o] = softplus(v + g.vec[n]);
    }
  }
}

}  // namespace simt
}  // namespace sambay
