// Straight-through backward of the FusedBitLinear projection.
//
// The pages print no backward pass.  "MatMul-freie LLMs: Zentrale Konzepte erklärt", section
// "MatMul durch ternäre Operationen ersetzen": the weights are trained in full precision and
// mapped to {-1, 0, 1} by absmean quantisation during training, so both quantisers sit inside
// the training forward pass.  Reading (straight-through): their rounding and clamping pass the
// gradient unchanged; the layer is differentiated as the bilinear map of its dequantised
// operands, xq = q * gamma / 127 and wq = c * beta, after the RMSNorm xhat = x / r * g:
//   dW   = dy^T xq                       (the latent weight takes wq's gradient)
//   dxh  = dy wq                          (the quantiser's input takes xq's gradient)
//   dx   = g dxh / r - x (sum_k g_k dxh_k x_k) / (K r^3)     per token
//   dg   = sum_t dxh x / r
//
// Both contractions are dense over fp16 operands with fp32 accumulators, on the tensor cores
// (the CTA-pair pipeline of the prefill contraction, kind::f16):
//   dxh [T x K] = beta * dy [T x N] . cT [K x N]^T       (contraction over N)
//   dW  [N x K] = dyT [N x T] . qT [K x T]^T             (contraction over the tokens)
// Both operands of a contraction must have the contraction index innermost, so the call first
// writes the weight codes transposed (cT[k][n] = c[n][k], exact in fp16), the gradient scaled by
// each token's gamma/127 and transposed (dyT[n][t], rounded once to fp16), and the activation
// codes transposed (qT[k][t], exact).  The per-token norm step and the norm-weight gradient are
// memory-bound passes over dxh.
#include <cuda_fp16.h>

#include <algorithm>

#include "backward.cuh"

namespace mmf {
namespace {

constexpr int kDgChunks = 64;   // token blocks of the norm-weight gradient's partial sums

size_t up256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }
int64_t up64(int64_t v) { return (v + 63) / 64 * 64; }

// A 64 x 64 fp16 transpose tile in shared memory, rows of 128 bytes whose 16-byte chunks are
// permuted by XOR with (row / 8): the column-wise scatter of a transpose (eight rows 8 apart
// per warp) then falls on eight different bank groups, and every chunk stays 16-byte aligned
// for the row-wise vector reads.
__device__ __forceinline__ int tsw(int row, int col) {
  return row * 64 + ((((col >> 3) ^ (row >> 3)) & 7) << 3) + (col & 7);
}

// cT[k][n] = c[n][k] as fp16, from the packed codes (layout L1: code 16G + 4i + j of a row at
// bits 8j + 2i of its 32-bit word G, stored as e = c + 1).  One block per 64 x 64 tile.
__global__ void __launch_bounds__(256) codes_t_f16_kernel(const uint32_t* __restrict__ wp, int N,
                                                          int K, __half* __restrict__ cT) {
  __shared__ __align__(16) __half s[64 * 64];   // [k][n], swizzled
  const int n0 = blockIdx.x * 64, k0 = blockIdx.y * 64;
  {
    const int rr = threadIdx.x >> 2, ww = threadIdx.x & 3;
    const uint32_t w = __ldg(wp + static_cast<int64_t>(n0 + rr) * (K / 16) + k0 / 16 + ww);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j)
        s[tsw(16 * ww + 4 * i + j, rr)] =
            __int2half_rn(static_cast<int>((w >> (8 * j + 2 * i)) & 3u) - 1);
  }
  __syncthreads();
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int idx = threadIdx.x + 256 * h;
    const int row = idx >> 3, ch = idx & 7;
    *reinterpret_cast<uint4*>(cT + static_cast<int64_t>(k0 + row) * N + n0 + ch * 8) =
        *reinterpret_cast<const uint4*>(&s[tsw(row, ch * 8)]);
  }
}

// dyT[n][t] = fp16(dy[t][n] * (gamma_t / 127)); columns t >= T of the padded rows are zero.
__global__ void __launch_bounds__(256) grad_scale_t_kernel(const __half* __restrict__ dy, int64_t T,
                                                           int N, const float* __restrict__ gamma,
                                                           __half* __restrict__ dyT, int64_t ldT) {
  __shared__ __align__(16) __half s[64 * 64];   // [n][t], swizzled
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * 64;
  const int n0 = blockIdx.y * 64;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int idx = threadIdx.x + 256 * h;
    const int tt = idx >> 3, ch = idx & 7;
    const int64_t t = t0 + tt;
    __half v[8];
    if (t < T) {
      const uint4 raw = __ldcs(reinterpret_cast<const uint4*>(dy + t * N + n0 + ch * 8));
      const float a = __fdiv_rn(__ldg(gamma + t), 127.0f);
      const __half2* hv = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(hv[e]);
        v[2 * e] = __float2half_rn(f.x * a);
        v[2 * e + 1] = __float2half_rn(f.y * a);
      }
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] = __float2half_rn(0.0f);
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) s[tsw(ch * 8 + e, tt)] = v[e];
  }
  __syncthreads();
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int idx = threadIdx.x + 256 * h;
    const int row = idx >> 3, ch = idx & 7;
    *reinterpret_cast<uint4*>(dyT + static_cast<int64_t>(n0 + row) * ldT + t0 + ch * 8) =
        *reinterpret_cast<const uint4*>(&s[tsw(row, ch * 8)]);
  }
}

// qT[k][t] = q[t][k] as fp16 (exact); columns t >= T of the padded rows are zero.
__global__ void __launch_bounds__(256) codes_tt_kernel(const int8_t* __restrict__ A, int64_t T,
                                                       int K, __half* __restrict__ qT, int64_t ldT) {
  __shared__ __align__(16) __half s[64 * 64];   // [k][t], swizzled
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * 64;
  const int k0 = blockIdx.y * 64;
  {
    const int tt = threadIdx.x >> 2, ch = threadIdx.x & 3;
    const int64_t t = t0 + tt;
    uint4 raw = make_uint4(0u, 0u, 0u, 0u);
    if (t < T) raw = __ldcs(reinterpret_cast<const uint4*>(A + t * K + k0 + ch * 16));
    const int8_t* b = reinterpret_cast<const int8_t*>(&raw);
#pragma unroll
    for (int e = 0; e < 16; ++e) s[tsw(ch * 16 + e, tt)] = __int2half_rn(b[e]);
  }
  __syncthreads();
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int idx = threadIdx.x + 256 * h;
    const int row = idx >> 3, ch = idx & 7;
    *reinterpret_cast<uint4*>(qT + static_cast<int64_t>(k0 + row) * ldT + t0 + ch * 8) =
        *reinterpret_cast<const uint4*>(&s[tsw(row, ch * 8)]);
  }
}

template <typename TX>
__device__ __forceinline__ void load4(const TX* p, float (&v)[4]);
template <>
__device__ __forceinline__ void load4<float>(const float* p, float (&v)[4]) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
}
template <>
__device__ __forceinline__ void load4<__half>(const __half* p, float (&v)[4]) {
  const uint2 a = *reinterpret_cast<const uint2*>(p);
  const float2 lo = __half22float2(*reinterpret_cast<const __half2*>(&a.x));
  const float2 hi = __half22float2(*reinterpret_cast<const __half2*>(&a.y));
  v[0] = lo.x; v[1] = lo.y; v[2] = hi.x; v[3] = hi.y;
}

template <typename TO>
__device__ __forceinline__ void store4(TO* p, const float (&v)[4]);
template <>
__device__ __forceinline__ void store4<float>(float* p, const float (&v)[4]) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
template <>
__device__ __forceinline__ void store4<__half>(__half* p, const float (&v)[4]) {
  const __half2 lo = __floats2half2_rn(v[0], v[1]);
  const __half2 hi = __floats2half2_rn(v[2], v[3]);
  uint2 a;
  a.x = *reinterpret_cast<const uint32_t*>(&lo);
  a.y = *reinterpret_cast<const uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(p) = a;
}

// Through the RMSNorm, one token per block:
//   dx_k = g_k dxh_k / r - x_k * (sum_j g_j dxh_j x_j) / (K r^3),  r = sqrt(mean x^2 + eps).
// Writes dx (when not null) and 1/r (for the norm-weight gradient).
template <typename TX, typename TO>
__global__ void __launch_bounds__(256) norm_bwd_kernel(const TX* __restrict__ x,
                                                       const float* __restrict__ dxh, int K,
                                                       const float* __restrict__ g, float eps,
                                                       TO* __restrict__ dx, float* __restrict__ rinv) {
  __shared__ float sh[2][8];
  const int64_t t = blockIdx.x;
  const TX* xr = x + t * K;
  const float* dr = dxh + t * K;
  float ss = 0.0f, dot = 0.0f;
  for (int k = threadIdx.x * 4; k < K; k += 1024) {
    float xv[4];
    load4<TX>(xr + k, xv);
    const float4 d = *reinterpret_cast<const float4*>(dr + k);
    const float4 gv = g ? *reinterpret_cast<const float4*>(g + k) : make_float4(1.f, 1.f, 1.f, 1.f);
    ss += xv[0] * xv[0] + xv[1] * xv[1] + xv[2] * xv[2] + xv[3] * xv[3];
    dot += gv.x * d.x * xv[0] + gv.y * d.y * xv[1] + gv.z * d.z * xv[2] + gv.w * d.w * xv[3];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ss += __shfl_xor_sync(0xffffffffu, ss, o);
    dot += __shfl_xor_sync(0xffffffffu, dot, o);
  }
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) {
    sh[0][w] = ss;
    sh[1][w] = dot;
  }
  __syncthreads();
  ss = 0.0f;
  dot = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    ss += sh[0][i];
    dot += sh[1][i];
  }
  const float r = sqrtf(ss / static_cast<float>(K) + eps);
  const float inv = 1.0f / r;
  const float c2 = dot * inv * inv * inv / static_cast<float>(K);
  if (threadIdx.x == 0 && rinv) rinv[t] = inv;
  if (!dx) return;
  for (int k = threadIdx.x * 4; k < K; k += 1024) {
    float xv[4];
    load4<TX>(xr + k, xv);
    const float4 d = *reinterpret_cast<const float4*>(dr + k);
    const float4 gv = g ? *reinterpret_cast<const float4*>(g + k) : make_float4(1.f, 1.f, 1.f, 1.f);
    float o[4];
    o[0] = gv.x * d.x * inv - xv[0] * c2;
    o[1] = gv.y * d.y * inv - xv[1] * c2;
    o[2] = gv.z * d.z * inv - xv[2] * c2;
    o[3] = gv.w * d.w * inv - xv[3] * c2;
    store4<TO>(dx + t * K + k, o);
  }
}

template <typename TX>
__device__ __forceinline__ float to_f(TX v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<__half>(__half v) { return __half2float(v); }

// part[chunk][k] = sum over the chunk's tokens of dxh[t][k] * x[t][k] / r_t.
template <typename TX>
__global__ void __launch_bounds__(128) dg_part_kernel(const TX* __restrict__ x,
                                                      const float* __restrict__ dxh,
                                                      const float* __restrict__ rinv, int64_t T,
                                                      int K, int64_t rows_per,
                                                      float* __restrict__ part) {
  const int k = blockIdx.x * 128 + threadIdx.x;
  const int64_t ta = blockIdx.y * rows_per;
  const int64_t tb = ta + rows_per < T ? ta + rows_per : T;
  float acc = 0.0f;
#pragma unroll 4
  for (int64_t t = ta; t < tb; ++t)
    acc += dxh[t * K + k] * to_f<TX>(x[t * K + k]) * __ldg(rinv + t);
  part[static_cast<int64_t>(blockIdx.y) * K + k] = acc;
}

__global__ void __launch_bounds__(128) dg_sum_kernel(const float* __restrict__ part, int nch, int K,
                                                     float* __restrict__ dg) {
  const int k = blockIdx.x * 128 + threadIdx.x;
  float acc = 0.0f;
  for (int c = 0; c < nch; ++c) acc += part[static_cast<int64_t>(c) * K + k];
  dg[k] = acc;
}

template <typename TX, typename TO>
cudaError_t launch_norm_bwd(const BwdCall& c, const float* dxh, float* rinv, cudaStream_t s) {
  norm_bwd_kernel<TX, TO><<<static_cast<unsigned>(c.T), 256, 0, s>>>(
      static_cast<const TX*>(c.x), dxh, c.K, c.norm_w, c.eps, static_cast<TO*>(c.dx), rinv);
  return cudaGetLastError();
}

}  // namespace

size_t bwd_ws_bytes(int64_t T, int64_t K, int64_t N) {
  const size_t t = static_cast<size_t>(T), k = static_cast<size_t>(K), n = static_cast<size_t>(N);
  const size_t ldT = static_cast<size_t>(up64(T));
  const size_t part = std::max(
      f16_gemm_part_bytes(T, static_cast<int>(K), f16_gemm_split(T, static_cast<int>(K), N)),
      f16_gemm_part_bytes(N, static_cast<int>(K), f16_gemm_split(N, static_cast<int>(K), T)));
  return up256(t * k) + up256(4 * t) + up256(2 * k * n) + up256(2 * n * ldT) +
         up256(2 * k * ldT) + up256(4 * t * k) + up256(4 * t) + up256(4 * kDgChunks * k) +
         up256(part);
}

BwdWs bwd_ws(void* ws, int64_t T, int64_t K, int64_t N) {
  const size_t t = static_cast<size_t>(T), k = static_cast<size_t>(K), n = static_cast<size_t>(N);
  const size_t ldT = static_cast<size_t>(up64(T));
  uint8_t* b = static_cast<uint8_t*>(ws);
  BwdWs w;
  w.A = reinterpret_cast<int8_t*>(b);
  b += up256(t * k);
  w.gamma = reinterpret_cast<float*>(b);
  b += up256(4 * t);
  w.cT = b;
  b += up256(2 * k * n);
  w.dyT = b;
  b += up256(2 * n * ldT);
  w.qT = b;
  b += up256(2 * k * ldT);
  w.dxh = reinterpret_cast<float*>(b);
  b += up256(4 * t * k);
  w.rinv = reinterpret_cast<float*>(b);
  b += up256(4 * t);
  w.dg_part = reinterpret_cast<float*>(b);
  b += up256(4 * kDgChunks * k);
  w.part = reinterpret_cast<float*>(b);
  return w;
}

cudaError_t launch_bitlinear_backward(const BwdCall& c, const BwdWs& w, cudaStream_t s) {
  cudaError_t e;
  const int8_t* q = c.A;
  const float* gamma = c.gamma;
  if (q == nullptr) {
    // the forward's codes and scales again (same kernel, same arithmetic as the forward)
    e = launch_act_quant(c.x, c.xdt, c.T, c.K, c.norm_w, c.eps, w.A, w.gamma, nullptr, s);
    if (e != cudaSuccess) return e;
    q = w.A;
    gamma = w.gamma;
  }
  const int64_t ldT = up64(c.T);
  if (c.dx != nullptr || c.dnorm_w != nullptr) {
    // dxh = beta * dy . C   (the gradient through the activation quantiser)
    codes_t_f16_kernel<<<dim3(static_cast<unsigned>(c.N / 64), static_cast<unsigned>(c.K / 64)),
                         256, 0, s>>>(reinterpret_cast<const uint32_t*>(c.Wp), c.N, c.K,
                                      static_cast<__half*>(w.cT));
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    F16GemmCall g;
    g.A = c.dy;
    g.M = c.T;
    g.lda = c.N;
    g.B = w.cT;
    g.rows = c.K;
    g.ldb = c.N;
    g.Kc = c.N;
    g.scale = c.beta;
    g.y = w.dxh;
    g.part = w.part;
    g.ksplit = f16_gemm_split(c.T, c.K, c.N);
    g.status = c.status;
    g.wait_limit_ns = c.wait_limit_ns;
    if ((e = launch_f16_gemm(g, s)) != cudaSuccess) return e;
    // through the RMSNorm
    const bool xh = c.xdt == kInF16, oh = c.dxdt == kInF16;
    if (xh && oh) e = launch_norm_bwd<__half, __half>(c, w.dxh, w.rinv, s);
    else if (xh) e = launch_norm_bwd<__half, float>(c, w.dxh, w.rinv, s);
    else if (oh) e = launch_norm_bwd<float, __half>(c, w.dxh, w.rinv, s);
    else e = launch_norm_bwd<float, float>(c, w.dxh, w.rinv, s);
    if (e != cudaSuccess) return e;
    if (c.dnorm_w != nullptr) {
      const int64_t rows_per = (c.T + kDgChunks - 1) / kDgChunks;
      const dim3 grid(static_cast<unsigned>(c.K / 128), kDgChunks);
      if (xh)
        dg_part_kernel<__half><<<grid, 128, 0, s>>>(static_cast<const __half*>(c.x), w.dxh, w.rinv,
                                                    c.T, c.K, rows_per, w.dg_part);
      else
        dg_part_kernel<float><<<grid, 128, 0, s>>>(static_cast<const float*>(c.x), w.dxh, w.rinv,
                                                   c.T, c.K, rows_per, w.dg_part);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
      dg_sum_kernel<<<static_cast<unsigned>(c.K / 128), 128, 0, s>>>(w.dg_part, kDgChunks, c.K,
                                                                     c.dnorm_w);
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
  }
  if (c.dW != nullptr) {
    // dW = (dy gamma / 127)^T . q   (the latent weight's gradient)
    const dim3 gy(static_cast<unsigned>(ldT / 64), static_cast<unsigned>(c.N / 64));
    grad_scale_t_kernel<<<gy, 256, 0, s>>>(static_cast<const __half*>(c.dy), c.T, c.N, gamma,
                                           static_cast<__half*>(w.dyT), ldT);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const dim3 gq(static_cast<unsigned>(ldT / 64), static_cast<unsigned>(c.K / 64));
    codes_tt_kernel<<<gq, 256, 0, s>>>(q, c.T, c.K, static_cast<__half*>(w.qT), ldT);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    F16GemmCall g;
    g.A = w.dyT;
    g.M = c.N;
    g.lda = ldT;
    g.B = w.qT;
    g.rows = c.K;
    g.ldb = ldT;
    g.Kc = c.T;
    g.scale = nullptr;
    g.y = c.dW;
    g.part = w.part;
    g.ksplit = f16_gemm_split(c.N, c.K, c.T);
    g.status = c.status;
    g.wait_limit_ns = c.wait_limit_ns;
    if ((e = launch_f16_gemm(g, s)) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace mmf
