// Host-side launchers of the straight-through backward and of the fp16 contraction it runs on.
// Internal to libmmf.so.
#pragma once

#include "kernels.cuh"

namespace mmf {

// fp16 x fp16 -> fp32 contraction on the CTA-pair tensor-core pipeline:
//   y[m][n] = scale * sum_k A[m][k] * B[n][k],   m < M, n < rows, k < Kc.
// A [M x Kc] and B [rows x Kc] row-major with row strides lda/ldb elements (multiples of 8);
// rows % 32 == 0.  With ksplit > 1 the contraction is split over ksplit work items per output
// tile, whose partial tiles go to `part` (f16_gemm_part_bytes) and are summed into y.
struct F16GemmCall {
  const void* A;
  int64_t M;
  int64_t lda;
  const void* B;
  int rows;
  int64_t ldb;
  int64_t Kc;
  const float* scale;     // device scalar, or nullptr for 1
  float* y;               // [M x rows]
  float* part;            // partial tiles when ksplit > 1
  int ksplit;
  unsigned* status;
  uint64_t wait_limit_ns;
};
int f16_gemm_split(int64_t M, int rows, int64_t Kc);
size_t f16_gemm_part_bytes(int64_t M, int rows, int ksplit);
cudaError_t launch_f16_gemm(const F16GemmCall& c, cudaStream_t s);

// Straight-through backward of the projection (see backward.cu for the arithmetic).
struct BwdCall {
  const void* x;
  int xdt;
  int64_t T;
  int K;
  const float* norm_w;
  float eps;
  const int8_t* A;        // forward codes [T x K]
  const float* gamma;     // forward scales [T]
  const uint8_t* Wp;
  const float* beta;
  int N;
  const void* dy;         // fp16 [T x N]
  void* dx;               // [T x K] or nullptr
  int dxdt;
  float* dW;              // [N x K] or nullptr
  float* dnorm_w;         // [K] or nullptr
  unsigned* status;
  uint64_t wait_limit_ns;
};
struct BwdWs {
  int8_t* A;
  float* gamma;
  void* cT;
  void* dyT;
  void* qT;
  float* dxh;
  float* rinv;
  float* dg_part;
  float* part;
};
size_t bwd_ws_bytes(int64_t T, int64_t K, int64_t N);
BwdWs bwd_ws(void* ws, int64_t T, int64_t K, int64_t N);
cudaError_t launch_bitlinear_backward(const BwdCall& c, const BwdWs& w, cudaStream_t s);

}  // namespace mmf
