// Absmean ternary weight quantisation and 2-bit packing.
//
// "MatMul-freie LLMs: Zentrale Konzepte erklärt", section "MatMul durch ternäre Operationen
// ersetzen": the weight matrix is scaled by its mean absolute value and every element is
// rounded to the nearest of -1, 0, 1.
//
// beta is made independent of summation order: every finite float magnitude is m * 2^s in
// units of 2^-149 (m < 2^24, s = exponent field - 1, or m = fraction and s = 0 for
// subnormals).  Pass 1 adds m into 256 per-exponent 64-bit bins (warp-aggregated with
// __match_any_sync / __reduce_add_sync, then shared-memory and global atomics): integer adds,
// so the result is exact whatever the order.  Pass 2 (one thread) carries the bins into a
// 384-bit integer, rounds it to the nearest double (ties to even), divides by N*K in double
// and rounds to float.  Pass 3 writes the codes c = clamp(rint(W / beta), -1, 1) packed four
// to a byte in the library's layout: for each group of 16 codes, code 4i + j goes to bits
// 8j + 2i of a 32-bit word as c + 1.
#include <cuda_fp16.h>

#include "kernels.cuh"

namespace mmf {
namespace {

constexpr int kBins = 256;

struct QuantWs {
  unsigned long long bins[kBins];
  unsigned nonfinite;
};

template <typename TIn>
__device__ __forceinline__ float load_f(const TIn* p, int64_t i);
template <>
__device__ __forceinline__ float load_f<float>(const float* p, int64_t i) {
  return __ldg(p + i);
}
template <>
__device__ __forceinline__ float load_f<__half>(const __half* p, int64_t i) {
  return __half2float(p[i]);
}

template <typename TIn>
__global__ void __launch_bounds__(256)
absum_bins_kernel(const TIn* __restrict__ W, int64_t n, QuantWs* ws) {
  __shared__ unsigned long long sb[kBins];
  for (int i = threadIdx.x; i < kBins; i += blockDim.x) sb[i] = 0ull;
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int64_t warp_global = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t warp_stride = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  bool bad = false;
  for (int64_t base = warp_global * 32; base < n; base += warp_stride * 32) {
    const int64_t i = base + lane;
    uint32_t m = 0, bin = kBins - 1;   // bin 255 never holds a finite value: used as "none"
    if (i < n) {
      const uint32_t bits = __float_as_uint(load_f(W, i)) & 0x7FFFFFFFu;
      const uint32_t e = bits >> 23, f = bits & 0x7FFFFFu;
      if (e == 255u) {
        bad = true;
      } else if (e == 0u) {
        m = f;
        bin = 0;
      } else {
        m = f | 0x800000u;
        bin = e - 1u;
      }
    }
    const unsigned grp = __match_any_sync(0xFFFFFFFFu, bin);
    const unsigned tot = __reduce_add_sync(grp, m);   // <= 32 * 2^24
    if (lane == __ffs(grp) - 1 && bin != kBins - 1 && tot != 0u)
      atomicAdd(&sb[bin], static_cast<unsigned long long>(tot));
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kBins; i += blockDim.x)
    if (sb[i] != 0ull) atomicAdd(&ws->bins[i], sb[i]);
  if (bad) atomicOr(&ws->nonfinite, 1u);
}

// Bits [lo, lo + 64) of the 384-bit integer L (bits past the top read as zero, below 0 as 0).
__device__ __forceinline__ unsigned long long window64(const unsigned long long (&L)[6], int lo) {
  unsigned long long r = 0;
  const int li = lo >> 6, sh = lo & 63;
  if (li >= 0 && li < 6) r = L[li] >> sh;
  if (sh != 0 && li + 1 < 6 && li + 1 >= 0) r |= L[li + 1] << (64 - sh);
  return r;
}

__global__ void beta_finalize_kernel(const QuantWs* ws, int64_t n, float* beta) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  unsigned long long L[6] = {0, 0, 0, 0, 0, 0};
  for (int s = 0; s < kBins - 1; ++s) {
    const unsigned long long v = ws->bins[s];
    if (v == 0ull) continue;
    const int li = s >> 6, sh = s & 63;
    unsigned long long add[6] = {0, 0, 0, 0, 0, 0};
    add[li] = v << sh;
    if (sh != 0) add[li + 1] = v >> (64 - sh);
    unsigned long long carry = 0;
    for (int k = 0; k < 6; ++k) {
      const unsigned long long a = L[k] + add[k];
      const unsigned long long c1 = a < add[k] ? 1ull : 0ull;
      const unsigned long long b = a + carry;
      const unsigned long long c2 = b < carry ? 1ull : 0ull;
      L[k] = b;
      carry = c1 | c2;
    }
  }
  int top = -1;
  for (int k = 5; k >= 0 && top < 0; --k)
    if (L[k] != 0ull) top = 64 * k + 63 - __clzll(static_cast<long long>(L[k]));

  double sum;
  if (top < 0) {
    sum = 0.0;
  } else if (top < 53) {
    sum = static_cast<double>(L[0]) * 0x1p-149;   // exact: below 2^53, scaled by a power of 2
  } else {
    // 64-bit window whose top bit is `top`: 53 kept bits, 11 rounding bits, then sticky.
    const unsigned long long win = window64(L, top - 63);
    unsigned long long mant = win >> 11;
    const unsigned long long rem = win & 0x7FFull;
    bool sticky = false;
    const int below = top - 63;            // bits under the window
    for (int b = 0; b < below && !sticky; b += 64) {
      const int len = min(64, below - b);
      const unsigned long long w = window64(L, b);
      const unsigned long long mask = len == 64 ? ~0ull : ((1ull << len) - 1ull);
      sticky = (w & mask) != 0ull;
    }
    const bool up = rem > 0x400ull || (rem == 0x400ull && (sticky || (mant & 1ull)));
    int e2 = top;
    if (up) {
      mant += 1ull;
      if (mant == (1ull << 53)) {
        mant >>= 1;
        e2 += 1;
      }
    }
    // value = mant * 2^(e2 - 52) * 2^-149, mant in [2^52, 2^53): biased exponent e2 - 149 + 1023
    const unsigned long long bits =
        (static_cast<unsigned long long>(e2 - 149 + 1023) << 52) | (mant & ((1ull << 52) - 1ull));
    sum = __longlong_as_double(static_cast<long long>(bits));
  }
  float b = __double2float_rn(__ddiv_rn(sum, static_cast<double>(n)));
  if (ws->nonfinite != 0u) {
    b = __int_as_float(0x7FC00000);
  } else if (!(b >= 1e-5f)) {
    b = 1e-5f;
  }
  *beta = b;
}

template <typename TIn>
__global__ void __launch_bounds__(256)
ternary_pack_kernel(const TIn* __restrict__ W, int64_t nwords, const float* __restrict__ beta_p,
                    uint32_t* __restrict__ Wp) {
  const float beta = *beta_p;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t w = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; w < nwords;
       w += stride) {
    float v[16];
    if constexpr (sizeof(TIn) == 4) {
      const float4* p = reinterpret_cast<const float4*>(W) + w * 4;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float4 a = __ldg(p + i);
        v[4 * i] = a.x; v[4 * i + 1] = a.y; v[4 * i + 2] = a.z; v[4 * i + 3] = a.w;
      }
    } else {
      const uint4* p = reinterpret_cast<const uint4*>(W) + w * 2;
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const uint4 a = __ldg(p + i);
        const __half2* h = reinterpret_cast<const __half2*>(&a);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = __half22float2(h[j]);
          v[8 * i + 2 * j] = f.x;
          v[8 * i + 2 * j + 1] = f.y;
        }
      }
    }
    uint32_t word = 0;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      int c = __float2int_rn(__fdiv_rn(v[k], beta));
      c = max(-1, min(1, c));
      word |= static_cast<uint32_t>(c + 1) << (8 * (k & 3) + 2 * (k >> 2));
    }
    Wp[w] = word;
  }
}

unsigned grid_for(int64_t work, int per_block, int cap) {
  int64_t b = (work + per_block - 1) / per_block;
  if (b < 1) b = 1;
  if (b > cap) b = cap;
  return static_cast<unsigned>(b);
}

}  // namespace

cudaError_t launch_absmean(const void* W, int wdt, int64_t n, void* ws_raw, float* beta,
                           cudaStream_t s) {
  QuantWs* ws = reinterpret_cast<QuantWs*>(ws_raw);
  cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(QuantWs), s);
  if (e != cudaSuccess) return e;
  const unsigned grid = grid_for(n, 256 * 8, 148 * 8);
  if (wdt == kInF16)
    absum_bins_kernel<__half><<<grid, 256, 0, s>>>(reinterpret_cast<const __half*>(W), n, ws);
  else
    absum_bins_kernel<float><<<grid, 256, 0, s>>>(reinterpret_cast<const float*>(W), n, ws);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  beta_finalize_kernel<<<1, 32, 0, s>>>(ws, n, beta);
  return cudaGetLastError();
}

cudaError_t launch_ternary_pack(const void* W, int wdt, int64_t n, const float* beta,
                                uint8_t* Wp, cudaStream_t s) {
  const int64_t nwords = n / 16;
  const unsigned grid = grid_for(nwords, 256, 148 * 16);
  if (wdt == kInF16)
    ternary_pack_kernel<__half><<<grid, 256, 0, s>>>(reinterpret_cast<const __half*>(W), nwords,
                                                     beta, reinterpret_cast<uint32_t*>(Wp));
  else
    ternary_pack_kernel<float><<<grid, 256, 0, s>>>(reinterpret_cast<const float*>(W), nwords,
                                                    beta, reinterpret_cast<uint32_t*>(Wp));
  return cudaGetLastError();
}

}  // namespace mmf
