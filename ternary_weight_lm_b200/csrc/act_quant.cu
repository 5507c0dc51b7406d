// RMSNorm inside the projection + per-token absmax int8 activation quantisation.
//
// "MatMul-freie LLMs: Zentrale Konzepte erklärt", section "Kernkomponenten: MLGRU und GLU",
// figure item 5: RMSNorm normalises the activations before they are quantised; the
// FusedBitLinear layers of the HGRNBit tree carry RMSNorm(eps=1e-08) inside the projection
// ("matmulfreellm 評価 ...", section "HGRNBit という層構成を読む").
//
// One CTA of 128 threads per token row.  The row is read once from HBM with 16-byte loads and
// kept in registers across the three block reductions it needs: sum of squares (double),
// max |xhat| (float) and the sum of the int8 codes (int, used by the contraction to undo the
// +1 offset of the packed weight codes).  Every rounding decision uses the same single-
// precision operation sequence as the definition: ms = float(sum/K), r = sqrt(ms + eps),
// inv = 1/r, xhat = (x * inv) * g, s = 127/gamma, q = round_half_even(xhat * s).
#include <cuda_fp16.h>

#include "kernels.cuh"

namespace mmf {
namespace {

constexpr int kAqThreads = 128;
constexpr int kAqWarps = kAqThreads / 32;

// A 16-byte vector of the input row, kept raw in registers (4 registers whatever the dtype)
// and widened to float where it is used, so a thread holds twice as many fp16 elements.
template <typename TIn>
struct Vec;
template <>
struct Vec<float> {
  static constexpr int E = 4;
  __device__ static void widen(const uint4& a, float (&v)[E]) {
    v[0] = __uint_as_float(a.x); v[1] = __uint_as_float(a.y);
    v[2] = __uint_as_float(a.z); v[3] = __uint_as_float(a.w);
  }
};
template <>
struct Vec<__half> {
  static constexpr int E = 8;
  __device__ static void widen(const uint4& a, float (&v)[E]) {
    const __half2* h = reinterpret_cast<const __half2*>(&a);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __half22float2(h[i]);
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
  }
};

__device__ __forceinline__ double block_sum_d(double v, double* sh) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) sh[w] = v;
  __syncthreads();
  double t = 0.0;
#pragma unroll
  for (int i = 0; i < kAqWarps; ++i) t += sh[i];
  __syncthreads();
  return t;
}

__device__ __forceinline__ float block_max_f(float v, float* sh) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) sh[w] = v;
  __syncthreads();
  float t = 0.0f;
#pragma unroll
  for (int i = 0; i < kAqWarps; ++i) t = fmaxf(t, sh[i]);
  __syncthreads();
  return t;
}

__device__ __forceinline__ int block_sum_i(int v, int* sh) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) sh[w] = v;
  __syncthreads();
  int t = 0;
#pragma unroll
  for (int i = 0; i < kAqWarps; ++i) t += sh[i];
  __syncthreads();
  return t;
}

__device__ __forceinline__ uint32_t code_byte(float xh, float s) {
  int q = __float2int_rn(__fmul_rn(xh, s));
  q = max(-128, min(127, q));
  return static_cast<uint32_t>(q) & 0xFFu;
}

// MAXV = most 16-byte vectors one thread holds: K <= kAqThreads * MAXV * E.
template <typename TIn, int MAXV, int MINB>
__global__ void __launch_bounds__(kAqThreads, MINB)
act_quant_kernel(const TIn* __restrict__ x, int K, const float* __restrict__ g, float eps,
                 int8_t* __restrict__ A, float* __restrict__ gamma,
                 int32_t* __restrict__ rowsum) {
  using V = Vec<TIn>;
  constexpr int E = V::E;
  __shared__ double sh_d[kAqWarps];
  __shared__ float sh_f[kAqWarps];
  __shared__ int sh_i[kAqWarps];

  const int64_t row = blockIdx.x;
  const int nvec = K / E;
  const uint4* xr = reinterpret_cast<const uint4*>(x + row * static_cast<int64_t>(K));
  // The next launch may begin its set-up; this grid waits for its own producers before it
  // reads x (which the previous launch may have written).
  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");

  uint4 raw[MAXV];
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int vi = threadIdx.x + i * kAqThreads;
    if (vi < nvec) raw[i] = __ldcs(xr + vi);   // streamed once: do not keep in L1
  }
  double ss = 0.0;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int vi = threadIdx.x + i * kAqThreads;
    if (vi < nvec) {
      float v[E];
      V::widen(raw[i], v);
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const double d = static_cast<double>(v[e]);
        ss = __fma_rn(d, d, ss);   // d*d is exact in double: same as an add of the square
      }
    }
  }
  ss = block_sum_d(ss, sh_d);
  const float ms = __double2float_rn(__ddiv_rn(ss, static_cast<double>(K)));
  const float inv_r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));

  auto norm_weight = [&](int vi, float (&gk)[E]) {
    if (g != nullptr) {
#pragma unroll
      for (int e = 0; e < E; e += 4) {
        const float4 t = __ldg(reinterpret_cast<const float4*>(g + vi * E + e));
        gk[e] = t.x; gk[e + 1] = t.y; gk[e + 2] = t.z; gk[e + 3] = t.w;
      }
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) gk[e] = 1.0f;
    }
  };

  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int vi = threadIdx.x + i * kAqThreads;
    if (vi < nvec) {
      float v[E], gk[E];
      V::widen(raw[i], v);
      norm_weight(vi, gk);
#pragma unroll
      for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(__fmul_rn(__fmul_rn(v[e], inv_r), gk[e])));
    }
  }
  amax = block_max_f(amax, sh_f);
  const float gm = fmaxf(amax, 1e-5f);
  const float s = __fdiv_rn(127.0f, gm);

  int rs = 0;
  int8_t* ar = A + row * static_cast<int64_t>(K);
#pragma unroll
  for (int i = 0; i < MAXV; ++i) {
    const int vi = threadIdx.x + i * kAqThreads;
    if (vi < nvec) {
      float v[E], gk[E];
      V::widen(raw[i], v);
      norm_weight(vi, gk);
      uint32_t w[E / 4];
#pragma unroll
      for (int c = 0; c < E / 4; ++c) {
        uint32_t word = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const float xh = __fmul_rn(__fmul_rn(v[4 * c + b], inv_r), gk[4 * c + b]);
          const uint32_t cb = code_byte(xh, s);
          rs += static_cast<int>(static_cast<int8_t>(cb));
          word |= cb << (8 * b);
        }
        w[c] = word;
      }
      if constexpr (E == 8) {
        *reinterpret_cast<uint2*>(ar + vi * E) = make_uint2(w[0], w[1]);
      } else {
        *reinterpret_cast<uint32_t*>(ar + vi * E) = w[0];
      }
    }
  }
  rs = block_sum_i(rs, sh_i);
  if (threadIdx.x == 0) {
    gamma[row] = gm;
    if (rowsum != nullptr) rowsum[row] = rs;
  }
}

// Warp-per-row variant for short rows (K <= 32 * VPL * E): eight rows per 256-thread CTA,
// every reduction a warp shuffle, no block barriers.  Same arithmetic, same op order.
constexpr int kWarpRowsPerCta = 8;

template <typename TIn, int VPL>
__global__ void __launch_bounds__(32 * kWarpRowsPerCta)
act_quant_warp_kernel(const TIn* __restrict__ x, int64_t T, int K, const float* __restrict__ g,
                      float eps, int8_t* __restrict__ A, float* __restrict__ gamma,
                      int32_t* __restrict__ rowsum) {
  using V = Vec<TIn>;
  constexpr int E = V::E;
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kWarpRowsPerCta + (threadIdx.x >> 5);
  if (threadIdx.x == 0) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (row >= T) return;
  const int nvec = K / E;
  const uint4* xr = reinterpret_cast<const uint4*>(x + row * static_cast<int64_t>(K));

  uint4 raw[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int vi = lane + 32 * i;
    if (vi < nvec) raw[i] = __ldcs(xr + vi);
  }
  double ss = 0.0;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    if (lane + 32 * i < nvec) {
      float v[E];
      V::widen(raw[i], v);
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const double d = static_cast<double>(v[e]);
        ss = __fma_rn(d, d, ss);
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float ms = __double2float_rn(__ddiv_rn(ss, static_cast<double>(K)));
  const float inv_r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));

  auto norm_weight = [&](int vi, float (&gk)[E]) {
    if (g != nullptr) {
#pragma unroll
      for (int e = 0; e < E; e += 4) {
        const float4 t = __ldg(reinterpret_cast<const float4*>(g + vi * E + e));
        gk[e] = t.x; gk[e + 1] = t.y; gk[e + 2] = t.z; gk[e + 3] = t.w;
      }
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) gk[e] = 1.0f;
    }
  };
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int vi = lane + 32 * i;
    if (vi < nvec) {
      float v[E], gk[E];
      V::widen(raw[i], v);
      norm_weight(vi, gk);
#pragma unroll
      for (int e = 0; e < E; ++e) amax = fmaxf(amax, fabsf(__fmul_rn(__fmul_rn(v[e], inv_r), gk[e])));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float gm = fmaxf(amax, 1e-5f);
  const float s = __fdiv_rn(127.0f, gm);

  int rs = 0;
  int8_t* ar = A + row * static_cast<int64_t>(K);
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int vi = lane + 32 * i;
    if (vi < nvec) {
      float v[E], gk[E];
      V::widen(raw[i], v);
      norm_weight(vi, gk);
      uint32_t w[E / 4];
#pragma unroll
      for (int c = 0; c < E / 4; ++c) {
        uint32_t word = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const float xh = __fmul_rn(__fmul_rn(v[4 * c + b], inv_r), gk[4 * c + b]);
          const uint32_t cb = code_byte(xh, s);
          rs += static_cast<int>(static_cast<int8_t>(cb));
          word |= cb << (8 * b);
        }
        w[c] = word;
      }
      if constexpr (E == 8) {
        *reinterpret_cast<uint2*>(ar + vi * E) = make_uint2(w[0], w[1]);
      } else {
        *reinterpret_cast<uint32_t*>(ar + vi * E) = w[0];
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) rs += __shfl_xor_sync(0xffffffffu, rs, o);
  if (lane == 0) {
    gamma[row] = gm;
    if (rowsum != nullptr) rowsum[row] = rs;
  }
}

__global__ void __launch_bounds__(kAqThreads)
rowsum_kernel(const int8_t* __restrict__ A, int K, int32_t* __restrict__ rowsum) {
  __shared__ int sh_i[kAqWarps];
  const int64_t row = blockIdx.x;
  const int8_t* ar = A + row * static_cast<int64_t>(K);
  int s = 0;
  for (int i = threadIdx.x * 16; i < K; i += kAqThreads * 16) {
    int4 q = *reinterpret_cast<const int4*>(ar + i);
    const int w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
#pragma unroll
      for (int b = 0; b < 4; ++b) s += static_cast<int8_t>((w[j] >> (8 * b)) & 0xFF);
    }
  }
  s = block_sum_i(s, sh_i);
  if (threadIdx.x == 0) rowsum[row] = s;
}

}  // namespace

cudaError_t launch_act_quant(const void* x, int xdt, int64_t T, int K, const float* g, float eps,
                             int8_t* A, float* gamma, int32_t* rowsum, cudaStream_t s) {
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.stream = s;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  const int e = xdt == kInF16 ? 8 : 4;          // elements per 16-byte vector
  const int nvec = K / e;
  if (nvec <= 32 * 16 && T >= 256) {
    // many short rows (prefill): one warp per row; few rows (decode) keep a CTA per row so
    // each row's loads and reductions spread over more threads
    cfg.gridDim = dim3(static_cast<unsigned>((T + kWarpRowsPerCta - 1) / kWarpRowsPerCta));
    cfg.blockDim = dim3(32 * kWarpRowsPerCta);
    if (xdt == kInF16) {
      if (nvec <= 32 * 8)
        return cudaLaunchKernelEx(&cfg, act_quant_warp_kernel<__half, 8>,
                                  reinterpret_cast<const __half*>(x), T, K, g, eps, A, gamma, rowsum);
      return cudaLaunchKernelEx(&cfg, act_quant_warp_kernel<__half, 16>,
                                reinterpret_cast<const __half*>(x), T, K, g, eps, A, gamma, rowsum);
    }
    if (nvec <= 32 * 8)
      return cudaLaunchKernelEx(&cfg, act_quant_warp_kernel<float, 8>,
                                reinterpret_cast<const float*>(x), T, K, g, eps, A, gamma, rowsum);
    return cudaLaunchKernelEx(&cfg, act_quant_warp_kernel<float, 16>,
                              reinterpret_cast<const float*>(x), T, K, g, eps, A, gamma, rowsum);
  }
  // long rows: one 128-thread CTA per row
  cfg.gridDim = dim3(static_cast<unsigned>(T));
  cfg.blockDim = dim3(kAqThreads);
  if (xdt == kInF16) {
    // 8 halves per vector: K <= 128 * 8 * 8 = 8192
    return cudaLaunchKernelEx(&cfg, act_quant_kernel<__half, 8, 8>,
                              reinterpret_cast<const __half*>(x), K, g, eps, A, gamma, rowsum);
  }
  // 4 floats per vector: K <= 128 * 16 * 4 = 8192
  return cudaLaunchKernelEx(&cfg, act_quant_kernel<float, 16, 4>,
                            reinterpret_cast<const float*>(x), K, g, eps, A, gamma, rowsum);
}

cudaError_t launch_rowsum(const int8_t* A, int64_t T, int K, int32_t* rowsum, cudaStream_t s) {
  rowsum_kernel<<<static_cast<unsigned>(T), kAqThreads, 0, s>>>(A, K, rowsum);
  return cudaGetLastError();
}

}  // namespace mmf
