// RMSNorm inside the projection + per-token absmax int8 activation quantisation.
//
// "MatMul-freie LLMs: Zentrale Konzepte erklärt", section "Kernkomponenten: MLGRU und GLU",
// figure item 5: RMSNorm normalises the activations before they are quantised; the
// FusedBitLinear layers of the HGRNBit tree carry RMSNorm(eps=1e-08) inside the projection
// ("matmulfreellm 評価 ...", section "HGRNBit という層構成を読む").
//
// Many rows (prefill): one warp per row; few or very long rows: one 128-thread CTA per row.
// The row is read once from HBM with 16-byte loads and kept in registers for the reductions it
// needs: the sum of squares (double) together with max|x|, then (only with a norm weight)
// max |xhat|, then the sum of the int8 codes (used by the contraction to undo the +1 offset of
// the packed weight codes).  Every rounding decision uses the same single-precision operation
// sequence as the definition: ms = float(sum/K), r = sqrt(ms + eps), inv = 1/r,
// xhat = (x * inv) * g, s = 127/gamma, q = round_half_even(xhat * s).
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

// q = round_half_even(y) saturated to [-128, 127], in one conversion; the low byte is the code.
__device__ __forceinline__ int code_s8(float y) {
  int q;
  asm("cvt.rni.sat.s8.f32 %0, %1;" : "=r"(q) : "f"(y));
  return q;
}

// Four codes packed little-endian into one word (byte b = code b).
__device__ __forceinline__ uint32_t pack4(int q0, int q1, int q2, int q3) {
  const uint32_t lo = __byte_perm(static_cast<uint32_t>(q0), static_cast<uint32_t>(q1), 0x0040);
  const uint32_t hi = __byte_perm(static_cast<uint32_t>(q2), static_cast<uint32_t>(q3), 0x0040);
  return __byte_perm(lo, hi, 0x5410);
}

// Codes of one 16-byte input vector: E/4 packed words; rs += the sum of the E signed codes.
template <int E, bool kG>
__device__ __forceinline__ void quantise_vec(const float (&v)[E], const float* gk, float inv_r,
                                             float s, uint32_t (&w)[E / 4], int& rs) {
#pragma unroll
  for (int c = 0; c < E / 4; ++c) {
    int q[4];
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      // without a norm weight (x*inv)*1 is x*inv exactly
      float xh = __fmul_rn(v[4 * c + b], inv_r);
      if constexpr (kG) xh = __fmul_rn(xh, gk[4 * c + b]);
      q[b] = code_s8(__fmul_rn(xh, s));
    }
    w[c] = pack4(q[0], q[1], q[2], q[3]);
    rs = __dp4a(static_cast<int>(w[c]), 0x01010101, rs);
  }
}

template <int E>
__device__ __forceinline__ void load_norm_weight(const float* g, int vi, float (&gk)[E]) {
#pragma unroll
  for (int e = 0; e < E; e += 4) {
    const float4 t = __ldg(reinterpret_cast<const float4*>(g + vi * E + e));
    gk[e] = t.x; gk[e + 1] = t.y; gk[e + 2] = t.z; gk[e + 3] = t.w;
  }
}

// The row passes over the register-resident input:
//   1. sum of squares (double) and, without a norm weight, max|x|;
//   2. only with a norm weight (kG): gamma = max |(x*inv)*g| element by element;
//   3. the codes and their sum.
// Without a norm weight gamma = (max|x|)*inv exactly: round-to-nearest is monotone and odd, so
// the largest |x*inv| is the rounded product of the largest |x| with inv.

// MAXV = most 16-byte vectors one thread holds: K <= kAqThreads * MAXV * E.
template <typename TIn, int MAXV, int MINB, bool kG>
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
  float mx = 0.0f;
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
        if constexpr (!kG) mx = fmaxf(mx, fabsf(v[e]));
      }
    }
  }
  // one barrier pair reduces both the sum of squares and max|x|
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if constexpr (!kG) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  {
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    if (l == 0) { sh_d[w] = ss; sh_f[w] = mx; }
    __syncthreads();
    ss = 0.0;
    mx = 0.0f;
#pragma unroll
    for (int i = 0; i < kAqWarps; ++i) { ss += sh_d[i]; mx = fmaxf(mx, sh_f[i]); }
    __syncthreads();
  }
  const float ms = __double2float_rn(__ddiv_rn(ss, static_cast<double>(K)));
  const float inv_r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));

  float amax;
  if constexpr (kG) {
    amax = 0.0f;
#pragma unroll
    for (int i = 0; i < MAXV; ++i) {
      const int vi = threadIdx.x + i * kAqThreads;
      if (vi < nvec) {
        float v[E], gk[E];
        V::widen(raw[i], v);
        load_norm_weight(g, vi, gk);
#pragma unroll
        for (int e = 0; e < E; ++e)
          amax = fmaxf(amax, fabsf(__fmul_rn(__fmul_rn(v[e], inv_r), gk[e])));
      }
    }
    amax = block_max_f(amax, sh_f);
  } else {
    amax = __fmul_rn(mx, inv_r);
  }
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
      if constexpr (kG) load_norm_weight(g, vi, gk);
      uint32_t w[E / 4];
      quantise_vec<E, kG>(v, gk, inv_r, s, w, rs);
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

template <typename TIn, int VPL, bool kG>
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
  float mx = 0.0f;
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    if (lane + 32 * i < nvec) {
      float v[E];
      V::widen(raw[i], v);
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const double d = static_cast<double>(v[e]);
        ss = __fma_rn(d, d, ss);
        if constexpr (!kG) mx = fmaxf(mx, fabsf(v[e]));
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if constexpr (!kG) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  const float ms = __double2float_rn(__ddiv_rn(ss, static_cast<double>(K)));
  const float inv_r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));

  float amax;
  if constexpr (kG) {
    amax = 0.0f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int vi = lane + 32 * i;
      if (vi < nvec) {
        float v[E], gk[E];
        V::widen(raw[i], v);
        load_norm_weight(g, vi, gk);
#pragma unroll
        for (int e = 0; e < E; ++e)
          amax = fmaxf(amax, fabsf(__fmul_rn(__fmul_rn(v[e], inv_r), gk[e])));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  } else {
    amax = __fmul_rn(mx, inv_r);
  }
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
      if constexpr (kG) load_norm_weight(g, vi, gk);
      uint32_t w[E / 4];
      quantise_vec<E, kG>(v, gk, inv_r, s, w, rs);
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

template <bool kG>
cudaError_t launch_act_quant_t(const cudaLaunchConfig_t& base, const void* x, int xdt, int64_t T,
                               int K, const float* g, float eps, int8_t* A, float* gamma,
                               int32_t* rowsum) {
  cudaLaunchConfig_t cfg = base;
  const int e = xdt == kInF16 ? 8 : 4;          // elements per 16-byte vector
  const int nvec = K / e;
  const __half* xh = reinterpret_cast<const __half*>(x);
  const float* xf = reinterpret_cast<const float*>(x);
  if (nvec <= 32 * 24 && T >= 256) {
    // many rows (prefill): one warp per row; few rows (decode) keep a CTA per row so each
    // row's loads and reductions spread over more threads
    cfg.gridDim = dim3(static_cast<unsigned>((T + kWarpRowsPerCta - 1) / kWarpRowsPerCta));
    cfg.blockDim = dim3(32 * kWarpRowsPerCta);
    if (xdt == kInF16) {
      if (nvec <= 32 * 8)
        return cudaLaunchKernelEx(&cfg, act_quant_warp_kernel<__half, 8, kG>, xh, T, K, g, eps,
                                  A, gamma, rowsum);
      if (nvec <= 32 * 16)
        return cudaLaunchKernelEx(&cfg, act_quant_warp_kernel<__half, 16, kG>, xh, T, K, g, eps,
                                  A, gamma, rowsum);
      return cudaLaunchKernelEx(&cfg, act_quant_warp_kernel<__half, 24, kG>, xh, T, K, g, eps,
                                A, gamma, rowsum);
    }
    if (nvec <= 32 * 8)
      return cudaLaunchKernelEx(&cfg, act_quant_warp_kernel<float, 8, kG>, xf, T, K, g, eps, A,
                                gamma, rowsum);
    if (nvec <= 32 * 16)
      return cudaLaunchKernelEx(&cfg, act_quant_warp_kernel<float, 16, kG>, xf, T, K, g, eps, A,
                                gamma, rowsum);
    return cudaLaunchKernelEx(&cfg, act_quant_warp_kernel<float, 24, kG>, xf, T, K, g, eps, A,
                              gamma, rowsum);
  }
  // few or long rows: one 128-thread CTA per row
  cfg.gridDim = dim3(static_cast<unsigned>(T));
  cfg.blockDim = dim3(kAqThreads);
  if (xdt == kInF16) {
    // 8 halves per vector: K <= 128 * 8 * 8 = 8192
    return cudaLaunchKernelEx(&cfg, act_quant_kernel<__half, 8, 8, kG>, xh, K, g, eps, A, gamma,
                              rowsum);
  }
  // 4 floats per vector: K <= 128 * 16 * 4 = 8192
  return cudaLaunchKernelEx(&cfg, act_quant_kernel<float, 16, 4, kG>, xf, K, g, eps, A, gamma,
                            rowsum);
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
  if (g != nullptr) return launch_act_quant_t<true>(cfg, x, xdt, T, K, g, eps, A, gamma, rowsum);
  return launch_act_quant_t<false>(cfg, x, xdt, T, K, g, eps, A, gamma, rowsum);
}

cudaError_t launch_rowsum(const int8_t* A, int64_t T, int K, int32_t* rowsum, cudaStream_t s) {
  rowsum_kernel<<<static_cast<unsigned>(T), kAqThreads, 0, s>>>(A, K, rowsum);
  return cudaGetLastError();
}

}  // namespace mmf
