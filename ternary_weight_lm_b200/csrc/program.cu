// A program of FusedBitLinear projections (a decode step) in one persistent launch.
//
// The projections are the ones of an HGRNBit block ("matmulfreellm 評価 ...", section "HGRNBit
// という層構成を読む"): i/f/g/o, gate_proj with the SiLU-GLU epilogue, down_proj reading the GLU
// output.  Each one computes what mmf_bitlinear_forward computes ("MatMul-freie LLMs: Zentrale
// Konzepte erklärt", sections "MatMul durch ternäre Operationen ersetzen" and "Kernkomponenten:
// MLGRU und GLU", figure items 4 and 5), with the same operation order, so the results match
// the single-projection entry points.
//
// Why one launch: at decode sizes (T <= 64 tokens) a projection streams a few hundred KB to a
// few MB of packed weights, well under a microsecond of HBM time, while every separate launch
// costs microseconds of latency.  Here one CTA per SM runs the whole program:
//   for each dependency level L
//     1. the four epilogue warps of every CTA quantise a share of the level's input rows
//        (RMSNorm + per-token absmax int8), then arrive on grid barrier Q[L];
//     2. each CTA runs its planned units (a 128-row weight tile and a range of k-blocks): a
//        producer thread streams the unit's packed weights (re-tiled at init into 16 KB
//        blocks, one contiguous bulk copy per stage; ahead of time, across levels) and, once
//        Q[L] has passed, the stage's activation codes (written tiled by step 1, one copy);
//        two sets of four warps unpack the 2-bit codes of alternate stages into TMEM; one or
//        two warps issue tcgen05 kind::i8 MMAs into one of two TMEM accumulators; the four
//        epilogue warps dequantise (and apply the GLU) or, for a tile split over several CTAs,
//        add the int32 partial sums into the tile's accumulator, the last split finishing the
//        tile;
//     3. every CTA arrives on grid barrier O[L]; the next level may read this level's outputs.
// Grid barriers are counters in the workspace with bounded waits; a timeout anywhere sets a
// poison flag that makes every other wait give up too, and is reported as MMF_ERR_TIMEOUT.
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>
#include <mutex>
#include <unordered_map>
#include <vector>

#include "../../include/mmf.h"
#include "kernels.cuh"
#include "ptx.cuh"

#define MMF_EXPORT extern "C" __attribute__((visibility("default")))

namespace mmf {
namespace {

// Warp roles: 0 and 14 TMA producers (weights, activation codes), 1 and 15 MMA issuers (even
// and odd stages; warp 1 alone for 64-token tiles), 2-5 and 10-13 unpack (even and odd
// stages), 6-9 quantise + epilogue.
constexpr int kPThreads = 512;
constexpr int kPEpi = 128;
constexpr int kPEpiT0 = 192;               // first epilogue thread
constexpr int kPKB = 128;                  // K per TMEM slot (one sub-block)
constexpr int kPSub = 4;                   // sub-blocks per shared-memory stage
constexpr int kPKS = kPKB * kPSub;         // K per stage (512)
constexpr int kPWRow = kPKS / 4;           // packed bytes per weight row per stage: 128
constexpr int kPWStage = 128 * kPWRow;     // 16 KB: one 128-byte line of each of 128 rows
// TMEM: two accumulators (the next unit's MMAs run while the epilogue reads the other), then
// A slots of one sub-block (32 columns) each.  Stage counter c writes slot group c % groups.
// With 16-token tiles the accumulators take 64 columns.  (Stages of two sub-blocks, for a
// deeper ring of seven slot groups, measured slower: a stage has a fixed cost.)
template <int BN>
constexpr int kPACol0 = BN <= 16 ? 64 : 128;
template <int BN>
constexpr int kPSlots = (512 - kPACol0<BN>) / 32;
template <int BN>
constexpr int kPGroups = kPSlots<BN> / kPSub;
template <int BN>
constexpr int kAccStride = BN <= 16 ? 32 : 64;    // TMEM columns per accumulator
template <int BN>
constexpr int kPartStride = BN <= 16 ? 16 : 32;   // second partial sum within an accumulator
constexpr int kMaxLevels = 128;
constexpr int kMaxProj = 1024;
constexpr int kMaxSplit = 16;
constexpr int kMinSplitKb = 32;            // a split tile costs a few microseconds of reduction
constexpr uint64_t kPDrainNs = 2000000000ull;
constexpr uint32_t kPlanMagic = 0x4d4d4650u;   // "PFMM"

static_assert(kPACol0<16> + kPSlots<16> * 32 == 512 && kPACol0<64> + kPSlots<64> * 32 == 512,
              "TMEM columns");
static_assert(2 * kAccStride<16> <= kPACol0<16> && 2 * kAccStride<64> <= kPACol0<64>,
              "accumulators below the A slots");
// Two partial accumulators per unit (even / odd sub-blocks) when they fit in the unit's 64
// accumulator columns.
template <int BN>
constexpr bool kSplitAcc = BN <= 32;

// nst: stages of K = 512 per row (the last one may be partial).  Wt: the projection's packed
// weights re-tiled in the workspace, [tile][stage][128 rows x 128 B], each 16 KB block stored as
// the shared-memory image the unpack warps read (128-byte swizzle: 16-byte chunk c of row r at
// position c ^ (r mod 8)); bytes past the end of a row are zero.
struct PProj {
  const uint8_t* Wp;
  const uint8_t* Wt;
  const float* beta;
  void* y;
  int32_t K, N, glu, ydt, in, level, nst, pad;
};

// A: the input's int8 codes, tiled as [stage][sub-block][BN token rows][128 B] with the same
// 128-byte swizzle (chunk c of token row t at position c ^ (t mod 8)), so that the activation
// sub-tiles of a stage are one contiguous block in the layout the MMA reads.  Token rows T..BN-1
// are never written: they only feed accumulator columns that are not stored.
struct PIn {
  const void* x;
  const float* g;
  int8_t* A;
  float* gamma;
  int32_t* rowsum;
  int32_t K, xdt, level, nst;
};

struct PUnit {
  int32_t proj, tile, kb0, nkb, split, nsplit, tile_id, part_off;
};

// What the epilogue needs of a unit, flattened at plan time and staged in shared memory by
// the epilogue threads (kERecMax units at a time, one load each), so that starting a unit
// costs no chain of dependent L2 round trips (unit -> projection -> input -> scales).
struct PERec {
  void* y;
  const float* beta;
  const float* gamma;
  const int32_t* rowsum;
  int32_t tile, nsplit, part_off, tile_id;
  int32_t nkb, N, level, flags;   // flags: glu | ydt << 1
};
static_assert(sizeof(PERec) == 64, "four 16-byte words");
constexpr int kERecMax = 128;

// What the producer, the unpack warps and the MMA warps need of a unit, flattened at plan time
// and copied into shared memory at the start of a run (the first kSRecMax units of the CTA;
// any further ones are read from the workspace).  A unit change then costs no dependent global
// loads: with records read from the workspace, the producer stalled about a microsecond at
// every unit boundary, which bounded the whole decode stream.
struct PSRec {
  const uint8_t* w;     // the unit's first 16 KB block of re-tiled weights
  const int8_t* a;      // its input's tiled codes
  int32_t nkb, kb0, level, pad;
};
static_assert(sizeof(PSRec) == 32, "two 16-byte words");
template <int BN>
constexpr int kSRecMax = BN <= 32 ? 256 : 64;

struct PHeader {
  int32_t n_proj, n_in, n_levels, n_ctas, n_units, T, BN, n_tiles;
  float eps;
  uint32_t magic;       // kPlanMagic once a plan is written
  uint32_t gen;         // init generation: every run passes the generation it was planned with
  int32_t pad;
  int64_t off_in, off_proj, off_units, off_ctaoff, off_wt, off_tilectr, off_levelctr, off_part;
  int64_t off_erec, off_srec;
  int32_t in_begin[kMaxLevels + 1];
  int32_t qgroup[kMaxLevels];   // epilogue threads per input row in level L's quantisation
};

template <int BN>
struct PCfg {
  static constexpr int kActSub = BN * kPKB;       // activation codes of one sub-block
  static constexpr int kAct = kPSub * kActSub;
  static constexpr int kStage = kAct + kPWStage;
  static constexpr int kCh = 16;                  // epilogue chunk: tokens per TMEM load
  static constexpr int kXbuf = kCh * 64 * 4;      // GLU exchange: multiplier half, fp32
  static constexpr int kTok = 8 * 64;             // per-token scale and code sum
  static constexpr int kOst = BN * 128 * 2;       // fp16 output staging [token][column]
  static constexpr int kERec = kERecMax * 64;     // staged epilogue records
  static constexpr int kSRec = kSRecMax<BN> * 32; // staged stream records
  static constexpr int kFixed = 1024 + 1024 + kXbuf + kTok + kOst + kERec + kSRec + 64;
  static constexpr int kStagesFit = (227 * 1024 - 512 - kFixed) / kStage;
  static constexpr int kStages = kStagesFit < 16 ? kStagesFit : 16;
  static constexpr int kBar = (8 * (2 * kStages + kPGroups<BN> + 5) + 127) / 128 * 128;
  static constexpr int kSmem =
      1024 + kStages * kStage + kBar + kXbuf + kTok + kOst + kERec + kSRec + 64;
  static_assert(kStages >= (BN <= 32 ? 6 : 4), "pipeline depth");
  static_assert(kBar <= 1024, "barrier area");
  static_assert(kSmem <= 227 * 1024 - 512, "shared memory");
  static_assert(kSmem >= 118 * 1024, "one CTA per SM");
};

// ------------------------------------------------------------------------------ device helpers
__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Arrive on a grid barrier: one fire-and-forget reduction with release semantics (orders this
// thread's earlier writes, and those of the CTA published to it by a preceding bar.sync).
__device__ __forceinline__ void grid_arrive(unsigned* ctr) {
  asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(ctr) : "memory");
}

// Waits until *ctr >= target.  Bounded: gives up after limit_ns, or at once when the poison
// flag is set (another CTA timed out); a timeout sets the poison flag and the status word.
__device__ __forceinline__ bool grid_wait(const unsigned* ctr, unsigned target, unsigned* poison,
                                          uint64_t limit_ns, unsigned* status) {
  if (ld_acquire_u32(ctr) >= target) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    __nanosleep(64);
    if (ld_acquire_u32(ctr) >= target) return true;
    if (ld_acquire_u32(poison) != 0u) return false;
    if (globaltimer_ns() - t0 > limit_ns) {
      atomicExch(poison, 1u);
      atomicOr(status, kStatusTimeout);
      return false;
    }
  }
}

template <typename P>
__device__ __forceinline__ P* u64ptr(uint32_t lo, uint32_t hi) {
  return reinterpret_cast<P*>((static_cast<uint64_t>(hi) << 32) | lo);
}

// Byte offset of code k of token t in an input's tiled codes (k a multiple of 4).
__device__ __forceinline__ int64_t a_tiled(int t, int k, int bn) {
  const int sub = k >> 7;                       // global sub-block index = 4 * stage + i
  const int c = (k >> 4) & 7;
  return (static_cast<int64_t>(sub) * bn + t) * 128 + ((c ^ (t & 7)) << 4) + (k & 15);
}

__device__ __forceinline__ void widen16(const uint4& a, int xdt, float (&v)[8], int& n) {
  if (xdt == kInF16) {
    const __half2* h = reinterpret_cast<const __half2*>(&a);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __half22float2(h[i]);
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
    n = 8;
  } else {
    v[0] = __uint_as_float(a.x); v[1] = __uint_as_float(a.y);
    v[2] = __uint_as_float(a.z); v[3] = __uint_as_float(a.w);
    n = 4;
  }
}

// A group of G epilogue threads (G = 32, 64 or 128: one, two or all four warps) quantises row
// t of input `in` with the same operations per element as the activation pre-pass kernel
// (mean of squares in double, rounded once; inv = 1/sqrt(ms+eps); xhat = (x*inv)*g;
// gamma = max|xhat| floored at 1e-5; q = rne(xhat * (127/gamma)), saturated to int8).  The
// row is read once (ld.global.cg: this launch may have written it) into registers, at most 8
// vectors of 16 bytes per thread, so nvec <= 8*G; thread gt holds vectors gt, gt+G, ...
// Without a norm weight gamma = (max|x|)*inv exactly: round-to-nearest is monotone and odd, so
// the largest |x*inv| is the rounded product of the largest |x| with inv.
// Partials cross warps through red_d/red_f/red_i (indexed by the epilogue warp 0-3) under
// named barrier `bar` of G threads; only the order in which the per-thread sums of squares
// are added depends on G, which can move the double sum by an ulp, far below the float
// rounding of the mean.
__device__ __forceinline__ int code_s8(float y) {
  int q;
  asm("cvt.rni.sat.s8.f32 %0, %1;" : "=r"(q) : "f"(y));
  return q;
}

__device__ __forceinline__ uint32_t pack4(int q0, int q1, int q2, int q3) {
  const uint32_t lo = __byte_perm(static_cast<uint32_t>(q0), static_cast<uint32_t>(q1), 0x0040);
  const uint32_t hi = __byte_perm(static_cast<uint32_t>(q2), static_cast<uint32_t>(q3), 0x0040);
  return __byte_perm(lo, hi, 0x5410);
}

__device__ void quant_row_g(const PIn in, int t, float eps, int gt, int G, int bar, int w,
                            int bn, double* red_d, float* red_f, int* red_i) {
  constexpr int kVmax = 8;
  const int K = in.K;
  const int E = in.xdt == kInF16 ? 8 : 4;
  const int nvec = K / E;
  const int lane = gt & 31;
  const int w0 = w - (gt >> 5);                 // first epilogue warp of the group
  const int nw = G >> 5;
  const uint4* xr = reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(in.x) +
                                                   static_cast<int64_t>(t) * K * (E == 8 ? 2 : 4));
  uint4 raw[kVmax];
#pragma unroll
  for (int i = 0; i < kVmax; ++i) {
    const int vi = gt + G * i;
    if (vi < nvec) raw[i] = __ldcg(xr + vi);
  }
  const bool has_g = in.g != nullptr;
  double ss = 0.0;
  float mx = 0.0f;
#pragma unroll
  for (int i = 0; i < kVmax; ++i) {
    if (gt + G * i < nvec) {
      float v[8];
      int n;
      widen16(raw[i], in.xdt, v, n);
      for (int e = 0; e < n; ++e) {
        const double d = static_cast<double>(v[e]);
        ss = __fma_rn(d, d, ss);
        mx = fmaxf(mx, fabsf(v[e]));
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    ss += __shfl_xor_sync(0xffffffffu, ss, o);
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  if (nw > 1) {
    if (lane == 0) {
      red_d[w] = ss;
      red_f[w] = mx;
    }
    named_bar_sync(bar, G);
    ss = red_d[w0];
    mx = red_f[w0];
    for (int j = 1; j < nw; ++j) {
      ss += red_d[w0 + j];
      mx = fmaxf(mx, red_f[w0 + j]);
    }
  }
  const float ms = __double2float_rn(__ddiv_rn(ss, static_cast<double>(K)));
  const float inv_r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, eps)));
  float amax = 0.0f;
  if (!has_g) {
    amax = __fmul_rn(mx, inv_r);
  } else {
#pragma unroll
    for (int i = 0; i < kVmax; ++i) {
      const int vi = gt + G * i;
      if (vi < nvec) {
        float v[8];
        int n;
        widen16(raw[i], in.xdt, v, n);
        for (int e = 0; e < n; ++e)
          amax = fmaxf(amax, fabsf(__fmul_rn(__fmul_rn(v[e], inv_r), __ldg(in.g + vi * E + e))));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (nw > 1) {
      if (lane == 0) red_f[4 + w] = amax;
      named_bar_sync(bar, G);
      amax = red_f[4 + w0];
      for (int j = 1; j < nw; ++j) amax = fmaxf(amax, red_f[4 + w0 + j]);
    }
  }
  const float gm = fmaxf(amax, 1e-5f);
  const float s = __fdiv_rn(127.0f, gm);
  int rs = 0;
#pragma unroll
  for (int i = 0; i < kVmax; ++i) {
    const int vi = gt + G * i;
    if (vi < nvec) {
      float v[8];
      int n;
      widen16(raw[i], in.xdt, v, n);
      uint32_t wd[2];
      for (int c = 0; c < n / 4; ++c) {
        int q[4];
        for (int b = 0; b < 4; ++b) {
          const int e = 4 * c + b;
          float xh = __fmul_rn(v[e], inv_r);    // (x*inv)*1 is x*inv exactly
          if (has_g) xh = __fmul_rn(xh, __ldg(in.g + vi * E + e));
          q[b] = code_s8(__fmul_rn(xh, s));
        }
        wd[c] = pack4(q[0], q[1], q[2], q[3]);
        rs = __dp4a(static_cast<int>(wd[c]), 0x01010101, rs);
      }
      if (E == 8)
        *reinterpret_cast<uint2*>(in.A + a_tiled(t, vi * 8, bn)) = make_uint2(wd[0], wd[1]);
      else
        *reinterpret_cast<uint32_t*>(in.A + a_tiled(t, vi * 4, bn)) = wd[0];
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) rs += __shfl_xor_sync(0xffffffffu, rs, o);
  if (nw > 1) {
    if (lane == 0) red_i[w] = rs;
    named_bar_sync(bar, G);
    if (gt == 0)
      for (int j = 1; j < nw; ++j) rs += red_i[w0 + j];
  }
  if (gt == 0) {
    in.gamma[t] = gm;
    in.rowsum[t] = rs;
  }
  // red_* are written again only after the next row's first barrier, which every thread of
  // the group reaches after its reads above
}

__device__ __forceinline__ void unpack_word4(uint32_t w, uint32_t* out) {
  out[0] = w & 0x03030303u;
  out[1] = (w >> 2) & 0x03030303u;
  out[2] = (w >> 4) & 0x03030303u;
  out[3] = (w >> 6) & 0x03030303u;
}

// Dequantise (and GLU) tokens c0 .. c0+CH-1 of a finished tile, held as int32 sums v[jj]
// (token c0+jj, tile row r).  tsc/trs: per-token scale (gamma/127 * beta) and code sum, staged
// in shared memory.  fp16 results go to ostage ([token][column] fp16, written out by
// store_tile); fp32 results are stored directly.  The GLU pairs row r < 64 (gated half) with
// row r + 64 (multiplier) through xbuf.
template <int CH>
__device__ __forceinline__ void finalize_chunk(const PProj& pj, int tile, int T, int c0,
                                               const int32_t (&v)[CH], int r,
                                               const float* __restrict__ tsc,
                                               const int32_t* __restrict__ trs,
                                               float* __restrict__ xbuf,
                                               __half* __restrict__ ostage) {
  // every shared-memory operand is read into registers before the first store: the compiler
  // cannot tell these buffers apart, and loads interleaved with stores would run one by one
  float f[CH];
  {
    float sc[CH];
    int32_t rs[CH];
#pragma unroll
    for (int jj = 0; jj < CH; ++jj) {
      sc[jj] = tsc[c0 + jj];
      rs[jj] = trs[c0 + jj];
    }
#pragma unroll
    for (int jj = 0; jj < CH; ++jj) f[jj] = static_cast<float>(v[jj] - rs[jj]) * sc[jj];
  }
  if (!pj.glu) {
    if (pj.ydt == MMF_F16) {
#pragma unroll
      for (int jj = 0; jj < CH; ++jj)
        if (c0 + jj < T) ostage[(c0 + jj) * 128 + r] = __float2half_rn(f[jj]);
    } else {
      float* y = reinterpret_cast<float*>(pj.y) + static_cast<int64_t>(tile) * 128 + r;
#pragma unroll
      for (int jj = 0; jj < CH; ++jj)
        if (c0 + jj < T) y[static_cast<int64_t>(c0 + jj) * pj.N] = f[jj];
    }
    return;
  }
  if (r >= 64) {
#pragma unroll
    for (int jj = 0; jj < CH; ++jj) xbuf[jj * 64 + (r - 64)] = f[jj];
  }
  named_bar_sync(1, kPEpi);
  if (r < 64) {
    float u[CH];
#pragma unroll
    for (int jj = 0; jj < CH; ++jj) u[jj] = xbuf[jj * 64 + r];
#pragma unroll
    for (int jj = 0; jj < CH; ++jj) f[jj] = __fdividef(f[jj], 1.0f + expf(-f[jj])) * u[jj];
    if (pj.ydt == MMF_F16) {
#pragma unroll
      for (int jj = 0; jj < CH; ++jj)
        if (c0 + jj < T) ostage[(c0 + jj) * 64 + r] = __float2half_rn(f[jj]);
    } else {
      float* y = reinterpret_cast<float*>(pj.y) + static_cast<int64_t>(tile) * 64 + r;
      const int64_t I = pj.N / 2;
#pragma unroll
      for (int jj = 0; jj < CH; ++jj)
        if (c0 + jj < T) y[static_cast<int64_t>(c0 + jj) * I] = f[jj];
    }
  }
  named_bar_sync(1, kPEpi);   // xbuf is reused by the next chunk
}

// fp16 outputs leave ostage as 16-byte stores: T rows of 128 (or 64 for the GLU) columns.
__device__ __forceinline__ void store_tile(const PProj& pj, int tile, int T, int et,
                                           const __half* __restrict__ ostage) {
  if (pj.ydt != MMF_F16) return;
  named_bar_sync(1, kPEpi);
  if (!pj.glu) {
    for (int c = et; c < T * 16; c += kPEpi) {
      const int j = c >> 4, k8 = (c & 15) * 8;
      *reinterpret_cast<uint4*>(reinterpret_cast<__half*>(pj.y) + static_cast<int64_t>(j) * pj.N +
                                static_cast<int64_t>(tile) * 128 + k8) =
          *reinterpret_cast<const uint4*>(ostage + j * 128 + k8);
    }
  } else {
    const int64_t I = pj.N / 2;
    for (int c = et; c < T * 8; c += kPEpi) {
      const int j = c >> 3, k8 = (c & 7) * 8;
      *reinterpret_cast<uint4*>(reinterpret_cast<__half*>(pj.y) + static_cast<int64_t>(j) * I +
                                static_cast<int64_t>(tile) * 64 + k8) =
          *reinterpret_cast<const uint4*>(ostage + j * 64 + k8);
    }
  }
}

// Loads CH accumulator columns of the partial sums selected by `mask` (bit 0: at taddr, bit 1:
// 32 columns further on) and adds them.
template <int CH>
__device__ __forceinline__ void load_acc(uint32_t taddr, int32_t (&v)[CH]) {
  uint32_t u[32];
  if constexpr (CH == 16) {
    tc_ld_32x32b_x16(taddr, u);
  } else {
    static_assert(CH == 32, "chunk");
    tc_ld_32x32b_x32(taddr, u);
  }
  tc_wait_ld();
#pragma unroll
  for (int j = 0; j < CH; ++j) v[j] = static_cast<int32_t>(u[j]);
}

template <int CH, int PS>
__device__ __forceinline__ void load_acc_sum(uint32_t taddr, int mask, int32_t (&v)[CH]) {
  load_acc<CH>(mask == 2 ? taddr + PS : taddr, v);
  if (mask == 3) {
    int32_t w[CH];
    load_acc<CH>(taddr + PS, w);
#pragma unroll
    for (int j = 0; j < CH; ++j) v[j] += w[j];
  }
}

template <int BN>
__global__ void __launch_bounds__(kPThreads, 1)
program_kernel(const uint8_t* __restrict__ ws, uint32_t gen, unsigned* status, uint64_t limit_ns) {
  using C = PCfg<BN>;
  constexpr int S = C::kStages;
  // With BN <= 32 two MMA warps on different SM sub-partitions take alternate stages, each into
  // its own partial accumulator (32 columns of the unit's 64); the epilogue adds the two.
  constexpr bool kTwoMma = kSplitAcc<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* s_act = smem;                              // S stages of kAct (1024-aligned)
  uint8_t* s_w = smem + S * C::kAct;                  // S stages of 16 KB (1024-aligned)
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_w + S * kPWStage);
  float* xbuf = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + C::kBar);
  float* tsc = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(xbuf) + C::kXbuf);
  int32_t* trs = reinterpret_cast<int32_t*>(tsc + 64);
  __half* ostage = reinterpret_cast<__half*>(trs + 64);
  uint4* s_erec = reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(ostage) + C::kOst);
  PSRec* s_srec = reinterpret_cast<PSRec*>(reinterpret_cast<uint8_t*>(s_erec) + C::kERec);
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ int s_flag;
  __shared__ int s_qflag;
  __shared__ double s_red_d[4];
  __shared__ float s_red_f[8];
  __shared__ int s_red_i[4];

  // Stage counter c (per CTA, over all its units) uses shared-memory stage c % S and TMEM slot
  // group c % 3 (four slots, one per sub-block).  full(s): stage s's weight line and activation
  // sub-tiles landed.  empty(s): the unpack warps read its weights and the MMAs of that stage
  // completed -- one commit per stage, which also tells the unpack warps that the stage's slot
  // group is free again (so there is no per-slot barrier to wait on).
  // afull(g): the unpack warps wrote slot group g.  accfull/accempty(b): accumulator b finished /
  // read by the epilogue.
  auto full = [&](int st) { return smem_u32(bars + st); };
  auto empty = [&](int st) { return smem_u32(bars + S + st); };
  auto afull = [&](int gi) { return smem_u32(bars + 2 * S + gi); };
  auto accfull = [&](int b) { return smem_u32(bars + 2 * S + kPGroups<BN> + b); };
  auto accempty = [&](int b) { return smem_u32(bars + 2 * S + kPGroups<BN> + 2 + b); };
  const uint32_t drainbar = smem_u32(bars + 2 * S + kPGroups<BN> + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int st = 0; st < S; ++st) {
      mbar_init(full(st), 1);
      mbar_init(empty(st), 1 + 4);
    }
    for (int gi = 0; gi < kPGroups<BN>; ++gi) mbar_init(afull(gi), 4);
    for (int b = 0; b < 2; ++b) {
      mbar_init(accfull(b), kTwoMma ? 2 : 1);   // one commit per MMA warp
      mbar_init(accempty(b), 4);
    }
    mbar_init(drainbar, kTwoMma ? 2 : 1);
    s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&s_tmem), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  volatile int* abort_flag = &s_abort;
  if (threadIdx.x == 0) pdl_launch_dependents();
  pdl_wait();
  // the plan in the workspace is read only after the wait
  const PHeader& H = *reinterpret_cast<const PHeader*>(ws);
  // A workspace that does not hold the plan this launch was made for (never planned, planned
  // again for another program, or overwritten) is refused by every CTA alike: nothing is
  // read or written beyond the header, and the status word records it.
  if (H.magic != kPlanMagic || H.gen != gen || H.BN != BN || H.n_ctas != static_cast<int>(gridDim.x)) {
    if (threadIdx.x == 0 && blockIdx.x == 0) atomicOr(status, kStatusBadPlan);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc(tmem, 512);
    }
    return;
  }
  const PIn* ins = reinterpret_cast<const PIn*>(ws + H.off_in);
  const int32_t* ctaoff = reinterpret_cast<const int32_t*>(ws + H.off_ctaoff);
  unsigned* tilectr = reinterpret_cast<unsigned*>(const_cast<uint8_t*>(ws) + H.off_tilectr);
  unsigned* lvl = reinterpret_cast<unsigned*>(const_cast<uint8_t*>(ws) + H.off_levelctr);
  unsigned* poison = lvl + 2 * kMaxLevels;
  unsigned* exitctr = lvl + 2 * kMaxLevels + 1;
  int32_t* parts = reinterpret_cast<int32_t*>(const_cast<uint8_t*>(ws) + H.off_part);

  const int nct = H.n_ctas;
  const int u_begin = ctaoff[blockIdx.x], u_end = ctaoff[blockIdx.x + 1];
  const int T = H.T;
  const PSRec* g_srec = reinterpret_cast<const PSRec*>(ws + H.off_srec);
  {
    const int n4 = 2 * min(kSRecMax<BN>, u_end - u_begin);
    const uint4* src = reinterpret_cast<const uint4*>(g_srec + u_begin);
    for (int i = threadIdx.x; i < n4; i += kPThreads)
      reinterpret_cast<uint4*>(s_srec)[i] = __ldg(src + i);
  }
  __syncthreads();
  // unit ui of this CTA (u_begin <= ui < u_end)
  auto srec = [&](int ui) -> PSRec {
    const int j = ui - u_begin;
    return j < kSRecMax<BN> ? s_srec[j] : g_srec[ui];
  };

  if (warp == 0 || warp == 14) {
    // ------------------------------------------------------------------ TMA producers
    // A stage is up to four k-blocks of one unit: the unit's 16 KB block of re-tiled weights
    // (one 128-byte line of each of the tile's 128 rows) and the stage's activation sub-tiles,
    // each one contiguous bulk copy.  Two threads issue them: warp 0 the weights, warp 14 the
    // activation codes.  Each waits for the stage to be free (empty) on its own, so the
    // weights keep streaming, up to a full ring, while a level is being quantised, and the
    // activation copies wait for their level's codes without holding the weights back.  (One
    // thread issuing both took about 0.6 us per stage and bounded the decode stream.)  The
    // weight thread sets the stage's expected bytes, both copies complete on full(s).
    if (lane == 0) {
      const bool wts = warp == 0;
      const uint64_t pol = wts ? l2_policy_evict_first() : l2_policy_evict_last();
      int ui = u_begin, k = 0, q_level = -1;
      PSRec r = {};
      if (ui < u_end) r = srec(ui);
      uint32_t i = 0;                      // stage counter (32-bit: cheap % and /)
      while (ui < u_end) {
        const int st = static_cast<int>(i % S);
        if (i >= static_cast<uint32_t>(S) &&
            !mbar_wait_bounded(empty(st), static_cast<uint32_t>(((i / S) - 1) & 1), limit_ns,
                               abort_flag, status))
          break;
        const int nsub = min(kPSub, r.nkb - k);
        if (wts) {
          mbar_arrive_expect_tx(full(st), kPWStage + nsub * C::kActSub);
          bulk_load(smem_u32(s_w + st * kPWStage), r.w + static_cast<int64_t>(k / kPSub) * kPWStage,
                    kPWStage, full(st), pol);
        } else {
          if (r.level > q_level) {   // the level's codes exist once every CTA arrived
            if (!grid_wait(lvl + 2 * r.level, static_cast<unsigned>(nct), poison, limit_ns,
                           status)) {
              *abort_flag = 1;
              break;
            }
            fence_proxy_async_global();
            q_level = r.level;
          }
          // sub-blocks (kb0 + k) .. +nsub of the input, contiguous in its tiled codes
          bulk_load(smem_u32(s_act + st * C::kAct), r.a + static_cast<int64_t>(r.kb0 + k) * C::kActSub,
                    static_cast<uint32_t>(nsub * C::kActSub), full(st), pol);
        }
        ++i;
        k += kPSub;
        if (k >= r.nkb) {
          k = 0;
          if (++ui < u_end) r = srec(ui);
        }
      }
      // Every copy this thread started lands before the block may exit (on the abort path a
      // stage missing its other copy never completes; the bounded wait gives up on it).
      for (uint32_t j = i > static_cast<uint32_t>(S) ? i - S : 0; j < i; ++j)
        mbar_wait_bounded(full(static_cast<int>(j % S)), static_cast<uint32_t>((j / S) & 1),
                          kPDrainNs, nullptr, status);
    }
  } else if (kTwoMma && (warp == 1 || warp == 15)) {
    // ------------------------------------------------------------------ MMA issuers (BN <= 32)
    // Warp 1 takes the even stages and warp 15 the odd ones; each adds its stages' MMAs into
    // its own partial accumulator, columns 64b + 32 * mset.  A warp with no stage in a unit
    // still commits to accfull(b) (after the accumulator is free), so that the epilogue always
    // sees two arrivals per unit.
    const int mset = warp == 1 ? 0 : 1;
    constexpr uint32_t idesc = idesc_i8_u8s8(128, BN);
    const uint64_t bdesc0 = smem_desc_kmajor_sw128(smem_u32(s_act));
    uint32_t c = 0;                      // stage counter (32-bit: cheap % and /)
    bool ok = true;
    int n = 0;
    for (int ui = u_begin; ui < u_end && ok; ++ui, ++n) {
      const int nkb = srec(ui).nkb;
      const int b = n & 1;
      const int ns = (nkb + kPSub - 1) / kPSub;
      // this warp's stages of the unit are s = first_s, first_s + 2, ... <= last_s
      const int first_s = static_cast<int>((c & 1) != static_cast<uint32_t>(mset));
      const int last_s = ns - 1 - static_cast<int>(((c + ns - 1) & 1) != static_cast<uint32_t>(mset));
      const uint32_t d = tmem + static_cast<uint32_t>(b * kAccStride<BN> + mset * kPartStride<BN>);
      if (n >= 2) {   // every MMA warp, even one with no stage here (see above)
        const bool w = mbar_wait_bounded(accempty(b), static_cast<uint32_t>(((n >> 1) - 1) & 1),
                                         limit_ns, abort_flag, status);
        if (!__all_sync(0xFFFFFFFFu, w)) break;
      }
      if (first_s >= ns) {               // no stage of this warp in the unit
        tc_fence_after();
        tc_commit_warp(accfull(b));
        c += static_cast<uint32_t>(ns);
        continue;
      }
      for (int k = 0; k < nkb; k += kPSub, ++c) {
        if ((c & 1) != static_cast<uint32_t>(mset)) continue;
        const int nsub = min(kPSub, nkb - k);
        const int st = static_cast<int>(c % S);
        const int gi = static_cast<int>(c % kPGroups<BN>);
        const bool w = mbar_wait_bounded(afull(gi), static_cast<uint32_t>((c / kPGroups<BN>) & 1),
                                         limit_ns, abort_flag, status);
        if (!__all_sync(0xFFFFFFFFu, w)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int s_idx = k / kPSub;
        const uint64_t bst = bdesc0 + static_cast<uint64_t>((st * C::kAct) >> 4);
        const uint32_t ast = tmem + kPACol0<BN> + gi * kPSub * 32;
        auto sub = [&](int i) {
          const uint64_t bd = bst + static_cast<uint64_t>((i * C::kActSub) >> 4);
          const uint32_t ad = ast + i * 32;
          tc_mma_i8_ts_warp(d, ad, bd, idesc, (s_idx == first_s && i == 0) ? 0u : 1u);
          tc_mma_i8_ts_warp(d, ad + 8, bd + 2, idesc, 1u);
          tc_mma_i8_ts_warp(d, ad + 16, bd + 4, idesc, 1u);
          tc_mma_i8_ts_warp(d, ad + 24, bd + 6, idesc, 1u);
        };
        if (nsub == kPSub) {
#pragma unroll
          for (int i = 0; i < kPSub; ++i) sub(i);
        } else {
          for (int i = 0; i < nsub; ++i) sub(i);
        }
        tc_commit_warp(empty(st));
        if (s_idx == last_s) tc_commit_warp(accfull(b));
      }
    }
    // Drain: nothing this warp issued may still be running when TMEM is freed.
    tc_commit_warp(drainbar);
    mbar_wait_bounded(drainbar, 0u, kPDrainNs, nullptr, status);
    __syncwarp();
  } else if (!kTwoMma && warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (BN = 64)
    // The whole warp runs the loop (waits and their outcomes are warp-uniform) and one elected
    // lane issues each MMA and commit.
    constexpr uint32_t idesc = idesc_i8_u8s8(128, BN);
    const uint64_t bdesc0 = smem_desc_kmajor_sw128(smem_u32(s_act));
    uint32_t c = 0;                      // stage counter (32-bit: cheap % and /)
    bool ok = true;
    int n = 0;
    for (int ui = u_begin; ui < u_end && ok; ++ui, ++n) {
      const int nkb = srec(ui).nkb;
      const int b = n & 1;
      if (n >= 2) {
        const bool w = mbar_wait_bounded(accempty(b), static_cast<uint32_t>(((n >> 1) - 1) & 1),
                                         limit_ns, abort_flag, status);
        if (!__all_sync(0xFFFFFFFFu, w)) break;
      }
      tc_fence_after();
      // accumulator b spans TMEM columns [64b, 64b + 64).  With BN <= 32 it holds two partial
      // sums, even sub-blocks at column 64b and odd ones at 64b + 32: consecutive MMAs into
      // different accumulators keep the tensor pipe busier than a chain on one (the epilogue
      // adds the two, exactly, in int32).
      const uint32_t d = tmem + static_cast<uint32_t>(b * kAccStride<BN>);
      for (int k = 0; k < nkb; k += kPSub, ++c) {
        const int nsub = min(kPSub, nkb - k);
        const int st = static_cast<int>(c % S);
        const int gi = static_cast<int>(c % kPGroups<BN>);
        const bool w = mbar_wait_bounded(afull(gi), static_cast<uint32_t>((c / kPGroups<BN>) & 1),
                                         limit_ns, abort_flag, status);
        if (!__all_sync(0xFFFFFFFFu, w)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // descriptor start address is in 16-byte units: a sub-tile is kActSub bytes, a 32-deep
        // k step is 32 bytes within the 128-byte swizzled rows
        const uint64_t bst = bdesc0 + static_cast<uint64_t>((st * C::kAct) >> 4);
        const uint32_t ast = tmem + kPACol0<BN> + gi * kPSub * 32;
        auto sub = [&](int i) {
          const uint64_t bd = bst + static_cast<uint64_t>((i * C::kActSub) >> 4);
          const uint32_t ad = ast + i * 32;
          const int j = k + i;                       // sub-block index within the unit
          const uint32_t dj = kSplitAcc<BN> ? d + static_cast<uint32_t>((j & 1) * 32) : d;
          const bool first = kSplitAcc<BN> ? (j < 2) : (j == 0);
          tc_mma_i8_ts_warp(dj, ad, bd, idesc, first ? 0u : 1u);
          tc_mma_i8_ts_warp(dj, ad + 8, bd + 2, idesc, 1u);
          tc_mma_i8_ts_warp(dj, ad + 16, bd + 4, idesc, 1u);
          tc_mma_i8_ts_warp(dj, ad + 24, bd + 6, idesc, 1u);
        };
        if (nsub == kPSub) {
          // a full stage as straight-line code: a runtime loop here costs the tensor pipe
          // about 40 % of its issue rate
#pragma unroll
          for (int i = 0; i < kPSub; ++i) sub(i);
        } else {
          for (int i = 0; i < nsub; ++i) sub(i);
        }
        tc_commit_warp(empty(st));
      }
      if (ok) tc_commit_warp(accfull(b));
    }
    // Drain: nothing this warp issued may still be running when TMEM is freed.
    tc_commit_warp(drainbar);
    mbar_wait_bounded(drainbar, 0u, kPDrainNs, nullptr, status);
    __syncwarp();
  } else if (warp < 6 || (warp >= 10 && warp < 14)) {
    // ------------------------------------------------------------------ unpack
    // Each lane owns one tile row (= TMEM lane): per stage it reads its row's 128-byte weight
    // line once and unpacks its sub-blocks (32 bytes, 128 codes each) into TMEM slots.  Two
    // sets of four warps take alternate stages, so that one set's store and barrier latencies
    // overlap the other's unpacking.
    const int set = warp >= 10 ? 1 : 0;
    const int q = warp & 3;              // TMEM lane quarter this warp may access
    const int r = q * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    uint32_t c = 0;                      // stage counter (32-bit: cheap % and /)
    bool ok = true;
    for (int ui = u_begin; ui < u_end && ok; ++ui) {
      const int nkb = srec(ui).nkb;
      for (int k = 0; k < nkb; k += kPSub, ++c) {
        if (static_cast<int>(c & 1) != set) continue;
        const int nsub = min(kPSub, nkb - k);
        const int st = static_cast<int>(c % S);
        const int gi = static_cast<int>(c % kPGroups<BN>);
        // Both conditions of this stage (its data landed; its slot group is free, see below)
        // are tested in one statement first; the bounded waits run only if one is not met.
        const uint32_t cp = c - kPGroups<BN>;   // valid when c >= kPGroups
        const bool both = c >= kPGroups<BN> && mbar_try_wait2(full(st), static_cast<uint32_t>((c / S) & 1),
                                                     empty(static_cast<int>(cp % S)),
                                                     static_cast<uint32_t>((cp / S) & 1));
        bool w = both || mbar_wait_bounded(full(st), static_cast<uint32_t>((c / S) & 1),
                                           limit_ns, abort_flag, status);
        if (!__all_sync(0xFFFFFFFFu, w)) {
          ok = false;
          break;
        }
        // 128-byte swizzle: 16-byte chunk c of row r sits at chunk position c ^ (r mod 8), so
        // the eight rows a quarter-warp reads hit eight bank groups
        const uint8_t* wrow = s_w + st * kPWStage + r * kPWRow;
        uint4 ch[2 * kPSub];
#pragma unroll
        for (int cc = 0; cc < 2 * kPSub; ++cc)
          ch[cc] = *reinterpret_cast<const uint4*>(wrow + ((cc ^ (r & 7)) << 4));
        __syncwarp();
        if (lane == 0) mbar_arrive(empty(st));
        // slot group gi was last read by the MMAs of stage c - 3: their commit completed
        // empty((c - 3) % S).  (That barrier cannot have moved a further phase on: it needs
        // the arrivals for stage c - 3 + S, which come after this stage's.)
        if (c >= kPGroups<BN> && !both) {
          w = mbar_wait_bounded(empty(static_cast<int>(cp % S)), static_cast<uint32_t>((cp / S) & 1),
                                limit_ns, abort_flag, status);
          if (!__all_sync(0xFFFFFFFFu, w)) {
            ok = false;
            break;
          }
        }
        // all sub-blocks of the stage are stored before one wait: the store latency is paid
        // once per stage, not once per sub-block
#pragma unroll
        for (int i = 0; i < kPSub; ++i) {
          if (i < nsub) {
            uint32_t uu[32];
            const uint4 lo = ch[2 * i], hi = ch[2 * i + 1];
            unpack_word4(lo.x, uu + 0);
            unpack_word4(lo.y, uu + 4);
            unpack_word4(lo.z, uu + 8);
            unpack_word4(lo.w, uu + 12);
            unpack_word4(hi.x, uu + 16);
            unpack_word4(hi.y, uu + 20);
            unpack_word4(hi.z, uu + 24);
            unpack_word4(hi.w, uu + 28);
            tc_st_32x32b_x32(tmem + lane_addr + kPACol0<BN> + (gi * kPSub + i) * 32, uu);
          }
        }
        tc_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(afull(gi));
      }
    }
  } else if (warp < 10) {
    // ------------------------------------------------------------------ quantise + epilogue
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const int et = threadIdx.x - kPEpiT0;
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    constexpr int CH = C::kCh;
    bool ok = true;
    int n = 0;
    uint32_t cs = 0;                     // stage counter (the MMA warps' c)
    int ui = u_begin;
    // epilogue records of units [rec0, rec0 + kERecMax) staged in shared memory
    const uint4* erecs = reinterpret_cast<const uint4*>(ws + H.off_erec);
    int rec0 = u_begin;
    auto stage_recs = [&](int u0) {
      named_bar_sync(1, kPEpi);                // the previous records are no longer read
      const int nq = 4 * min(kERecMax, u_end - u0);
      for (int i = et; i < nq; i += kPEpi) s_erec[i] = __ldg(erecs + 4 * u0 + i);
      named_bar_sync(1, kPEpi);
      rec0 = u0;
    };
    if (u_begin < u_end) stage_recs(u_begin);
    bool have_next = false;
    float g_next = 0.0f, b_next = 0.0f;
    int32_t rs_next = 0;
    for (int L = 0; L < H.n_levels; ++L) {
      // 1. quantise a share of this level's input rows (the 128 threads take one row at a time)
      const int ib = H.in_begin[L], ie = H.in_begin[L + 1];
      const int rows = (ie - ib) * T;
      // a group of G threads per row, G fixed per level at plan time: the largest group that
      // still finishes the level's rows in the fewest rounds, each row read in one pass
      const int G = H.qgroup[L];
      const int R = kPEpi / G;                    // rows in flight per CTA
      const int gid = et / G, gt = et % G;
      // first every row this group will quantise is requested into L2 at once
      if (gt == 0)
        for (int rho = blockIdx.x * R + gid; rho < rows; rho += nct * R) {
          const PIn& in = ins[ib + rho / T];
          const int rb = in.K * (in.xdt == kInF16 ? 2 : 4);
          bulk_prefetch_l2(reinterpret_cast<const uint8_t*>(in.x) + static_cast<int64_t>(rho % T) * rb,
                           static_cast<uint32_t>(rb));
        }
      for (int rho = blockIdx.x * R + gid; rho < rows && ok; rho += nct * R)
        quant_row_g(ins[ib + rho / T], rho % T, H.eps, gt, G, G == kPEpi ? 1 : 2 + gid, et >> 5,
                    H.BN, s_red_d, s_red_f, s_red_i);
      fence_proxy_async_global();   // the codes are read by TMA (async proxy) in other CTAs
      named_bar_sync(1, kPEpi);
      if (et == 0) {
        grid_arrive(lvl + 2 * L);
        // gamma and the code sums of this level are read below (staged per unit): wait until
        // every CTA has quantised its rows
        s_qflag = grid_wait(lvl + 2 * L, static_cast<unsigned>(nct), poison, limit_ns, status) ? 1 : 0;
        if (!s_qflag) *abort_flag = 1;
      }
      named_bar_sync(1, kPEpi);
      if (!s_qflag) ok = false;
      // 2. this CTA's units of level L
      while (ok && ui < u_end) {
        if (ui >= rec0 + kERecMax) stage_recs(ui);
        const uint4* rq = s_erec + 4 * (ui - rec0);
        const uint4 q0 = rq[0], q1 = rq[1], q2 = rq[2], q3 = rq[3];
        if (static_cast<int>(q3.z) != L) break;
        // the unit's record, in registers (output stores cannot alias them)
        struct {
          int tile, nsplit, part_off, tile_id, nkb;
        } u = {static_cast<int>(q2.x), static_cast<int>(q2.y), static_cast<int>(q2.z),
               static_cast<int>(q2.w), static_cast<int>(q3.x)};
        PProj pj = {};
        pj.y = u64ptr<void>(q0.x, q0.y);
        pj.N = static_cast<int32_t>(q3.y);
        pj.glu = static_cast<int32_t>(q3.w & 1u);
        pj.ydt = static_cast<int32_t>(q3.w >> 1);
        // this unit's per-token scale and code sum (requested while the previous unit was
        // finished, when that one was of the same level), then the next unit's
        float gv = 0.0f, bv = 0.0f;
        int32_t rv = 0;
        if (have_next) {
          gv = g_next;
          rv = rs_next;
          bv = b_next;
        } else if (et < T) {
          gv = __ldcg(u64ptr<const float>(q1.x, q1.y) + et);
          rv = __ldcg(u64ptr<const int32_t>(q1.z, q1.w) + et);
          bv = __ldg(u64ptr<const float>(q0.z, q0.w));
        }
        have_next = false;
        if (ui + 1 < u_end && ui + 1 < rec0 + kERecMax) {
          const uint4* rn = s_erec + 4 * (ui + 1 - rec0);
          const uint4 n0 = rn[0], n1 = rn[1], n3 = rn[3];
          if (static_cast<int>(n3.z) == L) {   // its codes exist (this level's barrier passed)
            if (et < T) {
              g_next = __ldcg(u64ptr<const float>(n1.x, n1.y) + et);
              rs_next = __ldcg(u64ptr<const int32_t>(n1.z, n1.w) + et);
              b_next = __ldg(u64ptr<const float>(n0.z, n0.w));
            }
            have_next = true;
          }
        }
        if (et < T) {
          tsc[et] = __fmul_rn(__fdiv_rn(gv, 127.0f), bv);
          trs[et] = rv;
        } else if (et < 64) {
          tsc[et] = 0.0f;   // padding tokens of the last chunk
          trs[et] = 0;
        }
        const int b = n & 1;
        const bool w = mbar_wait_bounded(accfull(b), static_cast<uint32_t>((n >> 1) & 1),
                                         limit_ns, abort_flag, status);
        ok = named_bar_and(1, kPEpi, __all_sync(0xFFFFFFFFu, w));   // also publishes tsc/trs
        if (!ok) break;
        tc_fence_after();
        const uint32_t dcol = tmem + lane_addr + static_cast<uint32_t>(b * kAccStride<BN>);
        // partial accumulators written for this unit: one per MMA warp (stage parity), both
        // when the unit has two or more stages
        const int ns_u = (u.nkb + kPSub - 1) / kPSub;
        const int pmask = !kTwoMma ? 1 : (ns_u >= 2 ? 3 : 1 << static_cast<int>(cs & 1));
        cs += static_cast<uint32_t>(ns_u);
        if (u.nsplit == 1) {
#pragma unroll 1
          for (int c0 = 0; c0 < BN && c0 < T; c0 += CH) {
            int32_t v[CH];
            load_acc_sum<CH, kPartStride<BN>>(dcol + static_cast<uint32_t>(c0), pmask, v);
            finalize_chunk<CH>(pj, u.tile, T, c0, v, r, tsc, trs, xbuf, ostage);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(accempty(b));
          store_tile(pj, u.tile, T, et, ostage);
        } else {
          // every split adds its partial sums into the tile's int32 accumulator in the
          // workspace (fire-and-forget reductions; integer addition is exact in any order);
          // the split that finishes last reads the total once, finalises the tile and zeroes
          // the accumulator for the next run
          int32_t* tacc = parts + static_cast<int64_t>(u.part_off) * BN * 128;
#pragma unroll 1
          for (int c0 = 0; c0 < BN && c0 < T; c0 += CH) {
            int32_t v[CH];
            load_acc_sum<CH, kPartStride<BN>>(dcol + static_cast<uint32_t>(c0), pmask, v);
#pragma unroll
            for (int jj = 0; jj < CH; ++jj) atomicAdd(tacc + (c0 + jj) * 128 + r, v[jj]);
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(accempty(b));
          __threadfence();
          named_bar_sync(1, kPEpi);
          if (et == 0) s_flag = (atomicAdd(tilectr + u.tile_id, 1u) == static_cast<unsigned>(u.nsplit - 1));
          named_bar_sync(1, kPEpi);
          if (s_flag) {
            __threadfence();
#pragma unroll 1
            for (int c0 = 0; c0 < BN && c0 < T; c0 += CH) {
              int32_t v[CH];
#pragma unroll
              for (int jj = 0; jj < CH; ++jj) v[jj] = __ldcg(tacc + (c0 + jj) * 128 + r);
#pragma unroll
              for (int jj = 0; jj < CH; ++jj) __stcg(tacc + (c0 + jj) * 128 + r, 0);
              finalize_chunk<CH>(pj, u.tile, T, c0, v, r, tsc, trs, xbuf, ostage);
            }
            store_tile(pj, u.tile, T, et, ostage);
            if (et == 0) tilectr[u.tile_id] = 0u;   // ready for the next run
          }
        }
        named_bar_sync(1, kPEpi);   // ostage, tsc and trs are reused by the next unit
        ++n;
        ++ui;
      }
      // 3. this level's outputs are written once every CTA arrives
      named_bar_sync(1, kPEpi);
      if (et == 0) {
        grid_arrive(lvl + 2 * L + 1);
        s_flag = grid_wait(lvl + 2 * L + 1, static_cast<unsigned>(nct), poison, limit_ns, status) ? 1 : 0;
        if (!s_flag) *abort_flag = 1;
      }
      named_bar_sync(1, kPEpi);
      if (!s_flag || !ok) {
        ok = false;
        // keep arriving on the remaining levels so that no other CTA waits for this one
        for (int L2 = L + 1; L2 < H.n_levels; ++L2)
          if (et == 0) {
            grid_arrive(lvl + 2 * L2);
            grid_arrive(lvl + 2 * L2 + 1);
          }
        break;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(exitctr, 1u) == static_cast<unsigned>(nct - 1)) {
      // last CTA out: every other CTA is done with the counters, reset them for the next run
      // (the poison flag stays set after a timeout until the program is planned again)
      for (int L = 0; L < H.n_levels; ++L) {
        lvl[2 * L] = 0u;
        lvl[2 * L + 1] = 0u;
      }
      *exitctr = 0u;
      __threadfence();
    }
  }
}

// Re-tiles one projection's packed weights (canonical layout: [N x K/4] row-major) into
// [tile][stage][128 rows x 128 B] blocks stored as the kernel's shared-memory image.  One CTA
// per block; thread r copies row r of the block (a GLU tile takes 64 gated rows, then the 64
// multiplier rows I apart).  Bytes past the end of a row are written as zeros.
__global__ void __launch_bounds__(128) retile_weights_kernel(const uint8_t* __restrict__ Wp, int K,
                                                             int N, int glu,
                                                             uint8_t* __restrict__ Wt) {
  const int row_bytes = K / 4;
  const int nst = (row_bytes + kPWRow - 1) / kPWRow;
  const int tile = static_cast<int>(blockIdx.x) / nst, st = static_cast<int>(blockIdx.x) % nst;
  const int r = threadIdx.x;
  const int row = glu ? (r < 64 ? tile * 64 + r : N / 2 + tile * 64 + (r - 64)) : tile * 128 + r;
  const uint8_t* src = Wp + static_cast<int64_t>(row) * row_bytes + st * kPWRow;
  uint8_t* dst = Wt + static_cast<int64_t>(blockIdx.x) * kPWStage + r * kPWRow;
#pragma unroll
  for (int c = 0; c < kPWRow / 16; ++c) {
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (st * kPWRow + c * 16 < row_bytes) v = *reinterpret_cast<const uint4*>(src + c * 16);
    *reinterpret_cast<uint4*>(dst + ((c ^ (r & 7)) << 4)) = v;
  }
}

// ------------------------------------------------------------------------------ host planning
struct Plan {
  std::vector<PIn> ins;
  std::vector<PProj> projs;
  std::vector<PUnit> units;
  std::vector<PERec> erec;
  std::vector<PSRec> srec;
  std::vector<int32_t> ctaoff;
  PHeader h;
  size_t bytes = 0;
  std::vector<std::pair<size_t, size_t>> in_buf;   // offset of A, and of gamma/rowsum, per input
  int BN = 0;
};

size_t al(size_t v, size_t a) { return (v + a - 1) / a * a; }

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    return 148;
  return n;
}

mmf_status validate(const mmf_projection* p, int n, int64_t T) {
  if (!p || n < 1 || n > kMaxProj) return MMF_ERR_INVALID_ARG;
  if (T < 1 || T > 64) return MMF_ERR_UNSUPPORTED_SHAPE;
  for (int i = 0; i < n; ++i) {
    const mmf_projection& q = p[i];
    if (!q.x || !q.Wp || !q.beta || !q.y) return MMF_ERR_INVALID_ARG;
    if ((q.xdt != MMF_F16 && q.xdt != MMF_F32) || (q.ydt != MMF_F16 && q.ydt != MMF_F32))
      return MMF_ERR_INVALID_ARG;
    if (q.glu != 0 && q.glu != 1) return MMF_ERR_INVALID_ARG;
    if (q.level < 0 || q.level >= kMaxLevels) return MMF_ERR_INVALID_ARG;
    const int64_t kmax = q.xdt == MMF_F16 ? 8192 : 4096;
    if (q.K < 128 || q.K > kmax || q.K % 128 != 0) return MMF_ERR_UNSUPPORTED_SHAPE;
    if (q.N < 128 || q.N > (1 << 20) || q.N % 128 != 0) return MMF_ERR_UNSUPPORTED_SHAPE;
    const uintptr_t a = reinterpret_cast<uintptr_t>(q.x) | reinterpret_cast<uintptr_t>(q.Wp) |
                        reinterpret_cast<uintptr_t>(q.y) |
                        reinterpret_cast<uintptr_t>(q.norm_w ? q.norm_w : q.x);
    if ((a & 15u) != 0 || (reinterpret_cast<uintptr_t>(q.beta) & 3u) != 0) return MMF_ERR_ALIGNMENT;
  }
  return MMF_OK;
}

// Builds the plan (without device addresses of the workspace regions, which `base` supplies).
mmf_status build_plan(const mmf_projection* p, int n, int64_t T, float eps, uintptr_t base,
                      int nct, Plan& P) {
  mmf_status st = validate(p, n, T);
  if (st != MMF_OK) return st;
  P = Plan();
  P.BN = T <= 16 ? 16 : (T <= 32 ? 32 : 64);
  int n_levels = 0;
  for (int i = 0; i < n; ++i) n_levels = std::max(n_levels, p[i].level + 1);
  // inputs: one per distinct (x, norm_w, K, dtype, level), ordered by level
  std::vector<int> order(n);
  for (int i = 0; i < n; ++i) order[i] = i;
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return p[a].level < p[b].level; });
  std::vector<int> proj_in(n, -1);
  for (int oi = 0; oi < n; ++oi) {
    const int i = order[oi];
    int found = -1;
    for (size_t k = 0; k < P.ins.size(); ++k) {
      const PIn& in = P.ins[k];
      if (in.x == p[i].x && in.g == p[i].norm_w && in.K == p[i].K && in.level == p[i].level &&
          in.xdt == (p[i].xdt == MMF_F16 ? kInF16 : kInF32)) {
        found = static_cast<int>(k);
        break;
      }
    }
    if (found < 0) {
      PIn in = {};
      in.x = p[i].x;
      in.g = p[i].norm_w;
      in.K = static_cast<int32_t>(p[i].K);
      in.xdt = p[i].xdt == MMF_F16 ? kInF16 : kInF32;
      in.level = p[i].level;
      found = static_cast<int>(P.ins.size());
      P.ins.push_back(in);
    }
    proj_in[i] = found;
  }
  // projections: kept in caller order, weight map index = projection index
  int tiles = 0;
  std::vector<int> tile_base(n);
  for (int i = 0; i < n; ++i) {
    PProj q = {};
    q.Wp = p[i].Wp;
    q.beta = p[i].beta;
    q.y = p[i].y;
    q.K = static_cast<int32_t>(p[i].K);
    q.N = static_cast<int32_t>(p[i].N);
    q.glu = p[i].glu;
    q.ydt = p[i].ydt;
    q.in = proj_in[i];
    q.level = p[i].level;
    q.nst = static_cast<int32_t>((p[i].K / kPKB + kPSub - 1) / kPSub);
    P.projs.push_back(q);
    tile_base[i] = tiles;
    tiles += static_cast<int>(p[i].N / 128);
  }
  // units: per level, split every tile's k-blocks so the level's work spreads over all SMs,
  // then assign longest-first to the least loaded CTA
  std::vector<std::vector<PUnit>> per_cta(nct);
  int part_slots = 0;
  for (int L = 0; L < n_levels; ++L) {
    int64_t work = 0;
    for (int i = 0; i < n; ++i)
      if (p[i].level == L) work += (p[i].N / 128) * (p[i].K / kPKB);
    if (work == 0) continue;
    const int64_t target = std::max<int64_t>(kMinSplitKb, (work + nct - 1) / nct);
    std::vector<PUnit> lu;
    for (int i = 0; i < n; ++i) {
      if (p[i].level != L) continue;
      // splits fall on stage boundaries (kPSub k-blocks), so that only the last stage of a
      // row can be partial
      const int nkb = static_cast<int>(p[i].K / kPKB);
      const int nst = (nkb + kPSub - 1) / kPSub;
      const int ns = static_cast<int>(std::min<int64_t>(
          {static_cast<int64_t>(kMaxSplit), static_cast<int64_t>(nst), (nkb + target - 1) / target}));
      for (int t = 0; t < p[i].N / 128; ++t) {
        const int part_off = ns > 1 ? part_slots : 0;   // one int32 accumulator tile per split tile
        if (ns > 1) part_slots += 1;
        for (int sp = 0; sp < ns; ++sp) {
          PUnit u;
          u.proj = i;
          u.tile = t;
          u.kb0 = kPSub * (sp * nst / ns);
          u.nkb = std::min(nkb, kPSub * ((sp + 1) * nst / ns)) - u.kb0;
          u.split = sp;
          u.nsplit = ns;
          u.tile_id = tile_base[i] + t;
          u.part_off = part_off;
          lu.push_back(u);
        }
      }
    }
    std::stable_sort(lu.begin(), lu.end(), [](const PUnit& a, const PUnit& b) { return a.nkb > b.nkb; });
    std::vector<int64_t> load(nct, 0);
    for (const PUnit& u : lu) {
      const int c = static_cast<int>(std::min_element(load.begin(), load.end()) - load.begin());
      load[c] += u.nkb + 2;   // +2: per-unit set-up and epilogue cost, in k-block units
      per_cta[c].push_back(u);
    }
  }
  P.ctaoff.push_back(0);
  for (int c = 0; c < nct; ++c) {
    for (const PUnit& u : per_cta[c]) P.units.push_back(u);
    P.ctaoff.push_back(static_cast<int32_t>(P.units.size()));
  }
  // workspace layout
  PHeader& h = P.h;
  std::memset(&h, 0, sizeof(h));
  h.n_proj = n;
  h.n_in = static_cast<int32_t>(P.ins.size());
  h.n_levels = n_levels;
  h.n_ctas = nct;
  h.n_units = static_cast<int32_t>(P.units.size());
  h.T = static_cast<int32_t>(T);
  h.BN = P.BN;
  h.n_tiles = tiles;
  h.eps = eps;
  size_t off = al(sizeof(PHeader), 256);
  h.off_in = static_cast<int64_t>(off);
  off = al(off + P.ins.size() * sizeof(PIn), 256);
  h.off_proj = static_cast<int64_t>(off);
  off = al(off + P.projs.size() * sizeof(PProj), 256);
  h.off_units = static_cast<int64_t>(off);
  off = al(off + P.units.size() * sizeof(PUnit), 256);
  h.off_erec = static_cast<int64_t>(off);
  off = al(off + P.units.size() * sizeof(PERec), 256);
  h.off_srec = static_cast<int64_t>(off);
  off = al(off + P.units.size() * sizeof(PSRec), 256);
  h.off_ctaoff = static_cast<int64_t>(off);
  off = al(off + P.ctaoff.size() * sizeof(int32_t), 256);
  h.off_tilectr = static_cast<int64_t>(off);
  off = al(off + static_cast<size_t>(tiles) * 4, 256);
  h.off_levelctr = static_cast<int64_t>(off);
  off = al(off + (2 * kMaxLevels + 2) * 4, 256);
  // per input: its codes tiled for BN token rows (K x BN bytes), then gamma and the code sums
  for (size_t k = 0; k < P.ins.size(); ++k) {
    const size_t a_off = off;
    off = al(off + static_cast<size_t>(P.BN) * P.ins[k].K, 256);
    const size_t v_off = off;
    off = al(off + static_cast<size_t>(T) * 8, 256);
    P.in_buf.push_back({a_off, v_off});
    P.ins[k].A = reinterpret_cast<int8_t*>(base + a_off);
    P.ins[k].gamma = reinterpret_cast<float*>(base + v_off);
    P.ins[k].rowsum = reinterpret_cast<int32_t*>(base + v_off + static_cast<size_t>(T) * 4);
    P.ins[k].nst = static_cast<int32_t>((P.ins[k].K / kPKB + kPSub - 1) / kPSub);
  }
  h.off_part = static_cast<int64_t>(off);
  off = al(off + static_cast<size_t>(part_slots) * P.BN * 128 * 4, 256);
  // the re-tiled packed weights of every projection: (N/128) tiles x nst stages x 16 KB
  h.off_wt = static_cast<int64_t>(off);
  for (size_t i = 0; i < P.projs.size(); ++i) {
    PProj& q = P.projs[i];
    q.Wt = reinterpret_cast<const uint8_t*>(base + off);
    off = al(off + static_cast<size_t>(q.N / 128) * q.nst * kPWStage, 256);
  }
  P.bytes = off;
  P.srec.resize(P.units.size());
  for (size_t i = 0; i < P.units.size(); ++i) {
    const PUnit& u = P.units[i];
    const PProj& q = P.projs[u.proj];
    PSRec& r = P.srec[i];
    r.w = q.Wt + (static_cast<int64_t>(u.tile) * q.nst + u.kb0 / kPSub) * kPWStage;
    r.a = P.ins[q.in].A;
    r.nkb = u.nkb;
    r.kb0 = u.kb0;
    r.level = q.level;
    r.pad = 0;
  }
  P.erec.resize(P.units.size());
  for (size_t i = 0; i < P.units.size(); ++i) {
    const PUnit& u = P.units[i];
    const PProj& q = P.projs[u.proj];
    const PIn& in = P.ins[q.in];
    PERec& e = P.erec[i];
    e.y = q.y;
    e.beta = q.beta;
    e.gamma = in.gamma;
    e.rowsum = in.rowsum;
    e.tile = u.tile;
    e.nsplit = u.nsplit;
    e.part_off = u.part_off;
    e.tile_id = u.tile_id;
    e.nkb = u.nkb;
    e.N = q.N;
    e.level = q.level;
    e.flags = (q.glu ? 1 : 0) | (q.ydt << 1);
  }
  int k = 0;
  for (int L = 0; L <= n_levels; ++L) {
    while (k < static_cast<int>(P.ins.size()) && P.ins[k].level < L) ++k;
    h.in_begin[L] = k;
  }
  h.in_begin[n_levels] = static_cast<int32_t>(P.ins.size());
  // quantisation group per level: at most 8 vectors of 16 bytes per thread, then the fewest
  // rounds of rows over the CTAs, then the most threads per row (shortest row latency)
  for (int L = 0; L < n_levels; ++L) {
    int nvec = 0;
    for (int i = h.in_begin[L]; i < h.in_begin[L + 1]; ++i)
      nvec = std::max(nvec, P.ins[i].K / (P.ins[i].xdt == kInF16 ? 8 : 4));
    const int64_t rows = static_cast<int64_t>(h.in_begin[L + 1] - h.in_begin[L]) * T;
    int best = kPEpi;
    int64_t best_rounds = -1;
    for (int G = kPEpi; G >= 32; G >>= 1) {
      if (nvec > 8 * G) break;
      const int64_t slots = static_cast<int64_t>(nct) * (kPEpi / G);
      const int64_t rounds = (rows + slots - 1) / slots;
      if (best_rounds < 0 || rounds < best_rounds) {
        best = G;
        best_rounds = rounds;
      }
    }
    h.qgroup[L] = best;
  }
  return MMF_OK;
}

struct RunInfo {
  int BN;
  int nct;
  uint32_t gen;   // the plan's generation, also written into the workspace header
  int mode;       // launch attributes (see launch_mode)
};
std::mutex g_runs_mu;
std::unordered_map<const void*, RunInfo> g_runs;
uint32_t g_next_gen = 1;

template <int BN>
cudaError_t set_program_attr() {
  using C = PCfg<BN>;
  static std::once_flag once[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  cudaError_t ae = cudaSuccess;
  std::call_once(once[dev], [&] {
    ae = cudaFuncSetAttribute(program_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              C::kSmem);
  });
  return ae;
}

// CTAs of program_kernel<BN> one device can hold at once (0 on failure).
template <int BN>
int resident_ctas() {
  using C = PCfg<BN>;
  if (set_program_attr<BN>() != cudaSuccess) return 0;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, program_kernel<BN>, kPThreads,
                                                    C::kSmem) != cudaSuccess)
    return 0;
  return per_sm * sm_count();
}

int resident_ctas_for(int BN) {
  return BN == 16 ? resident_ctas<16>() : (BN == 32 ? resident_ctas<32>() : resident_ctas<64>());
}

__global__ void launch_mode_probe_kernel() {}

// Launch attributes every program run uses on this device, found once (outside any stream
// capture: mmf_program_init is never captured) by launching an empty kernel with them.  A
// cooperative launch makes the driver place every CTA of the grid at once, which the grid
// barriers need; programmatic serialisation lets the launch's set-up overlap the tail of the
// previous kernel on the stream.  Bit 0: cooperative, bit 1: programmatic serialisation.
int launch_mode(cudaStream_t s) {
  static int modes[kMaxDevices];
  static std::once_flag once[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  std::call_once(once[dev], [&] {
    const int tries[3] = {3, 1, 2};
    modes[dev] = 0;
    for (int m : tries) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(1);
      cfg.blockDim = dim3(32);
      cfg.stream = s;
      cudaLaunchAttribute attr[2];
      int na = 0;
      if (m & 1) {
        attr[na].id = cudaLaunchAttributeCooperative;
        attr[na++].val.cooperative = 1;
      }
      if (m & 2) {
        attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[na++].val.programmaticStreamSerializationAllowed = 1;
      }
      cfg.attrs = attr;
      cfg.numAttrs = na;
      if (cudaLaunchKernelEx(&cfg, launch_mode_probe_kernel) == cudaSuccess) {
        modes[dev] = m;
        break;
      }
      (void)cudaGetLastError();   // a refused configuration is not sticky
    }
  });
  return modes[dev];
}

template <int BN>
cudaError_t launch_program(const void* ws, int nct, uint32_t gen, int mode, unsigned* status,
                           cudaStream_t s) {
  using C = PCfg<BN>;
  cudaError_t ae = set_program_attr<BN>();
  if (ae != cudaSuccess) return ae;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(nct));
  cfg.blockDim = dim3(kPThreads);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (mode & 1) {
    attr[na].id = cudaLaunchAttributeCooperative;
    attr[na++].val.cooperative = 1;
  }
  if (mode & 2) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na++].val.programmaticStreamSerializationAllowed = 1;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, program_kernel<BN>, reinterpret_cast<const uint8_t*>(ws), gen,
                            status, kWaitLimitNs);
}

}  // namespace
}  // namespace mmf

using namespace mmf;

MMF_EXPORT size_t mmf_program_workspace_bytes(const mmf_projection* p, int n, int64_t T) {
  Plan P;
  if (build_plan(p, n, T, 1e-8f, 0, sm_count(), P) != MMF_OK) return 0;
  return P.bytes;
}

MMF_EXPORT mmf_status mmf_program_init(const mmf_projection* p, int n, int64_t T, float eps,
                                       void* ws, size_t ws_bytes, void* stream) {
  if (!(eps > 0.0f) || eps != eps || eps > 1.0f) return MMF_ERR_INVALID_ARG;
  mmf_status st = validate(p, n, T);
  if (st != MMF_OK) return st;
  if (!ws) return MMF_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return MMF_ERR_ALIGNMENT;
  const int nct = sm_count();
  Plan P;
  st = build_plan(p, n, T, eps, reinterpret_cast<uintptr_t>(ws), nct, P);
  if (st != MMF_OK) return st;
  if (ws_bytes < P.bytes) return MMF_ERR_WORKSPACE;
  // Every CTA of a run waits for all the others at the level barriers: the device must be able
  // to hold the whole grid at once.
  if (resident_ctas_for(P.BN) < nct) return MMF_ERR_RESOURCES;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int mode = launch_mode(s);
  uint32_t gen;
  {
    std::lock_guard<std::mutex> lk(g_runs_mu);
    gen = g_next_gen++;
    if (g_next_gen == 0) g_next_gen = 1;
  }
  P.h.magic = kPlanMagic;
  P.h.gen = gen;
  // host image of the plan region, copied in one stream-ordered copy; counters zeroed
  const size_t plan_end = static_cast<size_t>(P.h.off_levelctr) + (2 * kMaxLevels + 2) * 4;
  std::vector<uint8_t> img(plan_end, 0);
  std::memcpy(img.data(), &P.h, sizeof(PHeader));
  std::memcpy(img.data() + P.h.off_in, P.ins.data(), P.ins.size() * sizeof(PIn));
  std::memcpy(img.data() + P.h.off_proj, P.projs.data(), P.projs.size() * sizeof(PProj));
  std::memcpy(img.data() + P.h.off_units, P.units.data(), P.units.size() * sizeof(PUnit));
  std::memcpy(img.data() + P.h.off_erec, P.erec.data(), P.erec.size() * sizeof(PERec));
  std::memcpy(img.data() + P.h.off_srec, P.srec.data(), P.srec.size() * sizeof(PSRec));
  std::memcpy(img.data() + P.h.off_ctaoff, P.ctaoff.data(), P.ctaoff.size() * sizeof(int32_t));
  // pageable source: the copy has consumed the host buffer when cudaMemcpyAsync returns
  if (cudaMemcpyAsync(ws, img.data(), img.size(), cudaMemcpyHostToDevice, s) != cudaSuccess)
    return MMF_ERR_CUDA;
  // the packed weights, re-tiled into the workspace once (they must not change afterwards)
  for (size_t i = 0; i < P.projs.size(); ++i) {
    const PProj& q = P.projs[i];
    retile_weights_kernel<<<static_cast<unsigned>((q.N / 128) * q.nst), 128, 0, s>>>(
        q.Wp, q.K, q.N, q.glu, const_cast<uint8_t*>(q.Wt));
    if (cudaGetLastError() != cudaSuccess) return MMF_ERR_CUDA;
  }
  // split tiles accumulate into zeroed int32 tiles (each run leaves them zeroed again)
  if (P.h.off_wt > P.h.off_part &&
      cudaMemsetAsync(static_cast<uint8_t*>(ws) + P.h.off_part, 0,
                      static_cast<size_t>(P.h.off_wt - P.h.off_part), s) != cudaSuccess)
    return MMF_ERR_CUDA;
  {
    std::lock_guard<std::mutex> lk(g_runs_mu);
    g_runs[ws] = RunInfo{P.BN, nct, gen, mode};
  }
  return MMF_OK;
}

MMF_EXPORT mmf_status mmf_program_run(void* ws, void* stream) {
  if (!ws) return MMF_ERR_INVALID_ARG;
  RunInfo ri;
  {
    std::lock_guard<std::mutex> lk(g_runs_mu);
    auto it = g_runs.find(ws);
    if (it == g_runs.end()) return MMF_ERR_INVALID_ARG;
    ri = it->second;
  }
  unsigned* status = device_status_word();
  if (!status) return MMF_ERR_CUDA;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (ri.BN == 16)
    e = launch_program<16>(ws, ri.nct, ri.gen, ri.mode, status, s);
  else if (ri.BN == 32)
    e = launch_program<32>(ws, ri.nct, ri.gen, ri.mode, status, s);
  else
    e = launch_program<64>(ws, ri.nct, ri.gen, ri.mode, status, s);
  if (e == cudaErrorCooperativeLaunchTooLarge) {
    (void)cudaGetLastError();
    return MMF_ERR_RESOURCES;
  }
  return e == cudaSuccess ? MMF_OK : MMF_ERR_CUDA;
}
