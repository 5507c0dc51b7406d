// Ternary contraction on the 5th-generation tensor cores (tcgen05, kind::i8) with the
// dequantisation and SiLU-GLU epilogues.
//
// "MatMul-freie LLMs: Zentrale Konzepte erklärt": section "MatMul durch ternäre Operationen
// ersetzen" (weights in {-1,0,1}: products become adds and subtracts) and figure item 4
// (scaled ternary accumulation); the GLU paragraph (one branch through SiLU times the other).
//
// Orientation ("swap AB"): the MMA's M side is 128 weight rows and its N side is BN tokens,
// so one kernel serves a single decode token (N = 16) up to prefill tiles (N = 256).
//   A (u8, TMEM)  : unpacked weight codes e = c + 1 in {0,1,2}, one TMEM lane per weight row
//   B (s8, SMEM)  : int8 activation codes, loaded by TMA with the 128-byte swizzle
//   D (s32, TMEM) : sum_k e_nk q_tk; the epilogue subtracts sum_k q_tk (computed by the
//                   activation pre-pass), giving exactly sum_k c_nk q_tk.
// The packed weights reach shared memory by TMA at 2 bits per weight (32-byte swizzle); four
// "unpack" warps, one thread per weight row, turn each 32-bit word of 16 codes into four
// 32-bit words of int8 codes with one shift and one mask each (the packing puts code 4i + j
// at bits 8j + 2i), and store them straight into TMEM with tcgen05.st.  Unpacked weights
// never touch shared memory, so shared-memory traffic stays at the packed 2 bits per weight.
//
// Warp roles (192 threads): warp 0 issues TMA, warp 1 owns TMEM and issues the MMAs (one
// thread), warps 2-5 unpack and then run the epilogue (TMEM lane quarter = warp % 4).
// Every mbarrier wait is bounded (mbar_wait_bounded): on a timeout the block records
// kStatusTimeout, stops, drains the copies and MMAs it issued, frees TMEM and returns.
#include <cuda_fp16.h>

#include <mutex>

#include "kernels.cuh"
#include "ptx.cuh"

namespace mmf {
namespace {

constexpr int kKB = 128;                       // K elements per pipeline stage
constexpr int kWRowBytes = kKB / 4;            // packed bytes of one weight row per stage
constexpr int kWHalfBytes = 64 * kWRowBytes;   // one TMA box: 64 rows x 32 bytes
constexpr int kWStageBytes = 2 * kWHalfBytes;  // 128 rows
constexpr int kThreads = 192;
constexpr int kEpiThreads = 128;
constexpr uint64_t kDrainNs = 2000000000ull;
constexpr int64_t kSplitTargetCtas = 148;       // SMs of a B200

// TC: TMEM columns a CTA allocates.  512: one CTA owns the SM.  256: two CTAs share an SM
// (half the shared memory each), so one CTA's epilogue overlaps the other's main loop.
// The shared-memory ring (activation tile + packed weights per k-block) and the TMEM ring of
// unpacked weight slots are separate: a stage is held from its copy's issue until its MMAs
// complete, a slot only from its unpack until then.  The copies of a stage are L2 hits with
// microseconds of latency under the prefill load, so the shared-memory ring is made as deep
// as shared memory allows, whatever the number of TMEM slots.
template <int BN, int TC = 512>
struct Cfg {
  static constexpr int kActStage = BN * kKB;               // int8 activation tile
  static constexpr int kStage = kActStage + kWStageBytes;
  static constexpr int kTmemCols = TC;
  static constexpr int kACol0 = ((BN + 31) / 32) * 32;     // first TMEM column of A slots
  static constexpr int kSlotsMax = (kTmemCols - kACol0) / 32;
  static constexpr int kSlots = kSlotsMax > 16 ? 16 : kSlotsMax;
  static constexpr int kSmemBudget = TC == 512 ? 214 * 1024 : 108 * 1024;
  static constexpr int kStagesSmem = kSmemBudget / kStage;
  static constexpr int kStages = kStagesSmem > 16 ? 16 : kStagesSmem;
  static constexpr int kChunk = BN < 32 ? BN : 32;         // epilogue token columns per pass
  static constexpr int kBarBytes = 8 * (2 * kStages + 2 * kSlots + 1);
  static constexpr int kTokBytes = 8 * BN;                 // per-token scale and code sum
  static constexpr int kSmemUsed = 1024 + kStages * kStage + kBarBytes + kTokBytes;
  // TC == 512: at least ~116 KB, so only one CTA lives on an SM (its TMEM allocation never
  // waits).  TC == 256: at most ~112 KB, so exactly two fit, and their TMEM halves fit too.
  static constexpr int kSmem =
      TC == 512 ? (kSmemUsed < 118 * 1024 ? 118 * 1024 : kSmemUsed) : kSmemUsed;
  static_assert(kStages >= 4 && kSlots >= 4, "pipeline needs four stages");
  static_assert(kSmem <= 227 * 1024, "shared memory per block");
  static_assert(TC == 512 || kSmem <= 112 * 1024, "two CTAs per SM");
  static_assert(kChunk * 128 * 4 <= kStages * kActStage, "epilogue staging must fit");
};

struct Params {
  int64_t T;
  int K;
  int rows;       // weight rows addressed by the tensor map
  int glu;
  int half;       // GLU: I (row offset of the multiplier half)
  int out_mode;
  int ldy;        // output row stride in elements
  const float* gamma;
  const int32_t* rowsum;
  const float* beta;
  void* y;
  unsigned* status;
  uint64_t wait_limit_ns;
};

// One 32-bit word of 16 packed codes -> four words of four int8 codes e = c + 1 in K order.
__device__ __forceinline__ void unpack_word(uint32_t w, uint32_t* out) {
  out[0] = w & 0x03030303u;
  out[1] = (w >> 2) & 0x03030303u;
  out[2] = (w >> 4) & 0x03030303u;
  out[3] = (w >> 6) & 0x03030303u;
}

__device__ __forceinline__ float sigmoid_mul(float g, float u) {
  return __fdividef(g, 1.0f + expf(-g)) * u;
}

// Split-K epilogue: CTA z of the cluster finalises tokens [z*BN/C, (z+1)*BN/C) of the tile,
// adding the C partial sums (exact int32) read from each CTA's shared memory.  Thread et is
// tile row et (non-GLU) or output column et < 64 (GLU: row et is the gated half, row et + 64
// the multiplier).
template <int BN, int TC>
__device__ __forceinline__ void split_k_reduce(const Params& p, int csize, int64_t t0, int r0,
                                               const uint8_t* s_act, const float* s_scale,
                                               const int32_t* s_rsum) {
  const int et = threadIdx.x - 64;
  const uint32_t crank = cluster_ctarank();
  const int per = BN / csize;
  const uint32_t part0 = smem_u32(s_act);
  for (int j = static_cast<int>(crank) * per; j < (static_cast<int>(crank) + 1) * per; ++j) {
    const int64_t t = t0 + j;
    if (t >= p.T) break;
    if (!p.glu) {
      int32_t v = 0;
      for (int c = 0; c < csize; ++c)
        v += ld_cluster_s32(map_peer(part0 + 4u * static_cast<uint32_t>(j * 128 + et), c));
      v -= s_rsum[j];
      const int64_t off = t * p.ldy + r0 + et;
      if (p.out_mode == kOutI32) {
        reinterpret_cast<int32_t*>(p.y)[off] = v;
      } else {
        const float f = static_cast<float>(v) * s_scale[j];
        if (p.out_mode == kOutF16)
          reinterpret_cast<__half*>(p.y)[off] = __float2half_rn(f);
        else
          reinterpret_cast<float*>(p.y)[off] = f;
      }
    } else if (et < 64) {
      int32_t g = 0, u = 0;
      for (int c = 0; c < csize; ++c) {
        g += ld_cluster_s32(map_peer(part0 + 4u * static_cast<uint32_t>(j * 128 + et), c));
        u += ld_cluster_s32(map_peer(part0 + 4u * static_cast<uint32_t>(j * 128 + 64 + et), c));
      }
      const float yg = static_cast<float>(g - s_rsum[j]) * s_scale[j];
      const float yu = static_cast<float>(u - s_rsum[j]) * s_scale[j];
      const float h = sigmoid_mul(yg, yu);
      const int64_t off = t * p.ldy + static_cast<int64_t>(blockIdx.x) * 64 + et;
      if (p.out_mode == kOutF16)
        reinterpret_cast<__half*>(p.y)[off] = __float2half_rn(h);
      else
        reinterpret_cast<float*>(p.y)[off] = h;
    }
  }
}

template <int BN, int TC>
__global__ void __launch_bounds__(kThreads, TC == 512 ? 1 : 2)
ternary_gemm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_a,
                    const Params p) {
  using C = Cfg<BN, TC>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* s_act = smem;
  uint8_t* s_w = smem + C::kStages * C::kActStage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_w + C::kStages * kWStageBytes);
  float* s_scale = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + C::kBarBytes);
  int32_t* s_rsum = reinterpret_cast<int32_t*>(s_scale + BN);
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Split K: the gridDim.z CTAs of a cluster share one output tile and each sums a contiguous
  // range of k-blocks; their int32 partial sums are added through distributed shared memory.
  const int csize = static_cast<int>(gridDim.z);
  const int nkb_all = p.K / kKB;
  const int kb0 = static_cast<int>(blockIdx.z) * nkb_all / csize;
  const int nkb = (static_cast<int>(blockIdx.z) + 1) * nkb_all / csize - kb0;
  const int64_t t0 = static_cast<int64_t>(blockIdx.y) * BN;
  int r0, r1;  // first weight row of each 64-row half of the tile
  if (p.glu) {
    r0 = blockIdx.x * 64;
    r1 = p.half + blockIdx.x * 64;
  } else {
    r0 = blockIdx.x * 128;
    r1 = r0 + 64;
  }

  // full(s): stage s's TMA bytes landed.  empty(s): the MMAs that read stage s's activation
  // tile completed and the unpack warps read its packed weights.  afull(a): the four unpack
  // warps wrote TMEM slot a (after seeing full of the same k-block, so it also implies that
  // k-block's activation tile is in).  afree(a): the MMAs that read slot a completed.
  auto full = [&](int s) { return smem_u32(bars + s); };
  auto empty = [&](int s) { return smem_u32(bars + C::kStages + s); };
  auto afull = [&](int a) { return smem_u32(bars + 2 * C::kStages + a); };
  auto afree = [&](int a) { return smem_u32(bars + 2 * C::kStages + C::kSlots + a); };
  const uint32_t accfull = smem_u32(bars + 2 * C::kStages + 2 * C::kSlots);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1 + 4);   // the MMA commit + the four unpack warps
    }
    for (int a = 0; a < C::kSlots; ++a) {
      mbar_init(afull(a), 4);       // the four unpack warps
      mbar_init(afree(a), 1);       // the MMA commit
    }
    mbar_init(accfull, 1);
    s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_a);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&s_tmem), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  volatile int* abort_flag = &s_abort;
  // Everything above is private set-up.  From here on the kernel reads and writes global
  // memory, so it first waits for the launches it depends on; the next launch may begin its
  // own set-up now.
  if (threadIdx.x == 0) pdl_launch_dependents();
  pdl_wait();

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      // One token tile (decode): each weight byte is used once, the activation tile by every
      // CTA.  Several token tiles (prefill): every token tile re-reads the whole weight
      // matrix, so the weights stay in L2; an activation tile is read by the row tiles that run
      // at about the same time.
      const bool many_tok = gridDim.y > 1;
      const uint64_t pol_w = many_tok ? l2_policy_evict_last() : l2_policy_evict_first();
      const uint64_t pol_a = many_tok ? l2_policy_evict_normal() : l2_policy_evict_last();
      int issued = 0;
      for (int kb = 0; kb < nkb; ++kb) {
        const int s = kb % C::kStages;
        if (kb >= C::kStages &&
            !mbar_wait_bounded(empty(s), ((kb / C::kStages) - 1) & 1, p.wait_limit_ns,
                               abort_flag, p.status))
          break;
        const int kg = kb0 + kb;   // k-block index within the whole K
        mbar_arrive_expect_tx(full(s), C::kStage);
        tma_load_2d(smem_u32(s_act + s * C::kActStage), &tm_a, full(s), kg * kKB,
                    static_cast<int32_t>(t0), pol_a);
        uint8_t* wdst = s_w + s * kWStageBytes;
        tma_load_2d(smem_u32(wdst), &tm_w, full(s), kg * kWRowBytes, r0, pol_w);
        tma_load_2d(smem_u32(wdst + kWHalfBytes), &tm_w, full(s), kg * kWRowBytes, r1, pol_w);
        issued = kb + 1;
      }
      // Every copy this thread started must land before the block may exit.
      for (int kb = issued > C::kStages ? issued - C::kStages : 0; kb < issued; ++kb)
        mbar_wait_bounded(full(kb % C::kStages), (kb / C::kStages) & 1, kDrainNs, nullptr,
                          p.status);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop (waits and their outcomes are warp-uniform) and one elected
    // lane issues each MMA and commit.
    constexpr uint32_t idesc = idesc_i8_u8s8(128, BN);
    const uint64_t bdesc0 = smem_desc_kmajor_sw128(smem_u32(s_act));
    for (int kb = 0; kb < nkb; ++kb) {
      const int s = kb % C::kStages, a = kb % C::kSlots;
      const bool w = mbar_wait_bounded(afull(a), (kb / C::kSlots) & 1, p.wait_limit_ns,
                                       abort_flag, p.status);
      if (!__all_sync(0xFFFFFFFFu, w)) break;
      tc_fence_after();
      // descriptor start address is in 16-byte units: a stage is kActStage bytes, a 32-deep
      // k step is 32 bytes within the 128-byte swizzled rows
      const uint64_t bd = bdesc0 + static_cast<uint64_t>((s * C::kActStage) >> 4);
      const uint32_t ad = tmem + C::kACol0 + a * 32;
      tc_mma_i8_ts_warp(tmem, ad, bd, idesc, kb > 0 ? 1u : 0u);   // kb counts this CTA's range
      tc_mma_i8_ts_warp(tmem, ad + 8, bd + 2, idesc, 1u);
      tc_mma_i8_ts_warp(tmem, ad + 16, bd + 4, idesc, 1u);
      tc_mma_i8_ts_warp(tmem, ad + 24, bd + 6, idesc, 1u);
      tc_commit_warp(empty(s));
      tc_commit_warp(afree(a));
    }
    // Signals the epilogue; in the abort path it also tells this warp when the MMAs it issued
    // have finished, so TMEM is not freed under them.
    tc_commit_warp(accfull);
    mbar_wait_bounded(accfull, 0, kDrainNs, nullptr, p.status);
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ unpack + epilogue
    const int q = warp & 3;              // TMEM lane quarter this warp may access
    const int r = q * 32 + lane;         // tile row = TMEM lane
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    // Wait outcomes are made warp-uniform (__all_sync) before the .sync.aligned tcgen05
    // instructions, and the epilogue is entered by all four warps or by none.
    // Per-token dequantisation scale (gamma/127 * beta) and code sum for this tile, staged
    // once so the epilogue does no dependent global loads.
    if (p.out_mode != kOutI32) {
      const float beta = *p.beta;
      for (int i = threadIdx.x - 64; i < BN; i += kEpiThreads) {
        const int64_t t = t0 + i;
        s_scale[i] = t < p.T ? __fmul_rn(__fdiv_rn(p.gamma[t], 127.0f), beta) : 0.0f;
        s_rsum[i] = t < p.T ? p.rowsum[t] : 0;
      }
    } else {
      for (int i = threadIdx.x - 64; i < BN; i += kEpiThreads) {
        const int64_t t = t0 + i;
        s_scale[i] = 0.0f;
        s_rsum[i] = t < p.T ? p.rowsum[t] : 0;
      }
    }
    bool ok = true;
    for (int kb = 0; kb < nkb; ++kb) {
      const int s = kb % C::kStages, a = kb % C::kSlots;
      bool w = mbar_wait_bounded(full(s), (kb / C::kStages) & 1, p.wait_limit_ns, abort_flag,
                                 p.status);
      if (!__all_sync(0xFFFFFFFFu, w)) {
        ok = false;
        break;
      }
      // Row r of the 32-byte-swizzled tile: 16-byte chunk c sits at c ^ ((r >> 2) & 1).
      const uint8_t* wrow = s_w + s * kWStageBytes + r * kWRowBytes;
      const int sw = (r >> 2) & 1;
      const uint4 lo = *reinterpret_cast<const uint4*>(wrow + 16 * sw);
      const uint4 hi = *reinterpret_cast<const uint4*>(wrow + 16 * (sw ^ 1));
      __syncwarp();
      if (lane == 0) mbar_arrive(empty(s));
      // slot a was last read by the MMAs of k-block kb - kSlots
      if (kb >= C::kSlots) {
        w = mbar_wait_bounded(afree(a), ((kb / C::kSlots) - 1) & 1, p.wait_limit_ns,
                              abort_flag, p.status);
        if (!__all_sync(0xFFFFFFFFu, w)) {
          ok = false;
          break;
        }
      }
      uint32_t u[32];
      unpack_word(lo.x, u + 0);
      unpack_word(lo.y, u + 4);
      unpack_word(lo.z, u + 8);
      unpack_word(lo.w, u + 12);
      unpack_word(hi.x, u + 16);
      unpack_word(hi.y, u + 20);
      unpack_word(hi.z, u + 24);
      unpack_word(hi.w, u + 28);
      tc_st_32x32b_x32(tmem + lane_addr + C::kACol0 + a * 32, u);
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(afull(a));
    }
    if (ok) {
      const bool w = mbar_wait_bounded(accfull, 0, p.wait_limit_ns, abort_flag, p.status);
      ok = __all_sync(0xFFFFFFFFu, w);
    }
    ok = named_bar_and(1, kEpiThreads, ok);
    if (ok && csize > 1) {
      // Split K: dump this CTA's partial sums to shared memory as int32 [token][row]; the
      // cluster adds them after the cluster barrier below.
      tc_fence_after();
      int32_t* part = reinterpret_cast<int32_t*>(s_act);
      for (int c0 = 0; c0 < BN; c0 += C::kChunk) {
        uint32_t acc[32];
        if constexpr (C::kChunk == 32) {
          tc_ld_32x32b_x32(tmem + lane_addr + c0, acc);
        } else {
          tc_ld_32x32b_x16(tmem + lane_addr + c0, acc);
        }
        tc_wait_ld();
#pragma unroll
        for (int jj = 0; jj < C::kChunk; ++jj) part[(c0 + jj) * 128 + r] = static_cast<int32_t>(acc[jj]);
      }
    } else if (ok) {
      tc_fence_after();
      int32_t* stage = reinterpret_cast<int32_t*>(s_act);   // all copies landed, all MMAs done
      const int et = threadIdx.x - 64;                      // 0..127
      for (int c0 = 0; c0 < BN; c0 += C::kChunk) {
        uint32_t acc[32];
        if constexpr (C::kChunk == 32) {
          tc_ld_32x32b_x32(tmem + lane_addr + c0, acc);
        } else {
          tc_ld_32x32b_x16(tmem + lane_addr + c0, acc);
        }
        tc_wait_ld();
#pragma unroll
        for (int jj = 0; jj < C::kChunk; ++jj) stage[jj * 128 + r] = static_cast<int32_t>(acc[jj]);
        named_bar_sync(1, kEpiThreads);
        if (!p.glu) {
          for (int gi = et; gi < C::kChunk * 16; gi += kEpiThreads) {
            const int jj = gi >> 4, c8 = (gi & 15) * 8;
            const int64_t t = t0 + c0 + jj;
            if (t >= p.T) continue;
            const int4 a0 = *reinterpret_cast<const int4*>(stage + jj * 128 + c8);
            const int4 a1 = *reinterpret_cast<const int4*>(stage + jj * 128 + c8 + 4);
            const int av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const int rs = s_rsum[c0 + jj];
            const int64_t off = t * p.ldy + r0 + c8;
            if (p.out_mode == kOutI32) {
              int32_t* y = reinterpret_cast<int32_t*>(p.y) + off;
              *reinterpret_cast<int4*>(y) = make_int4(av[0] - rs, av[1] - rs, av[2] - rs, av[3] - rs);
              *reinterpret_cast<int4*>(y + 4) = make_int4(av[4] - rs, av[5] - rs, av[6] - rs, av[7] - rs);
            } else {
              const float sc = s_scale[c0 + jj];
              float f[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) f[e] = static_cast<float>(av[e] - rs) * sc;
              if (p.out_mode == kOutF16) {
                uint4 o;
                __half2* h = reinterpret_cast<__half2*>(&o);
#pragma unroll
                for (int e = 0; e < 4; ++e) h[e] = __floats2half2_rn(f[2 * e], f[2 * e + 1]);
                *reinterpret_cast<uint4*>(reinterpret_cast<__half*>(p.y) + off) = o;
              } else {
                float* y = reinterpret_cast<float*>(p.y) + off;
                *reinterpret_cast<float4*>(y) = make_float4(f[0], f[1], f[2], f[3]);
                *reinterpret_cast<float4*>(y + 4) = make_float4(f[4], f[5], f[6], f[7]);
              }
            }
          }
        } else {
          for (int gi = et; gi < C::kChunk * 8; gi += kEpiThreads) {
            const int jj = gi >> 3, i8 = (gi & 7) * 8;
            const int64_t t = t0 + c0 + jj;
            if (t >= p.T) continue;
            const int rs = s_rsum[c0 + jj];
            const float sc = s_scale[c0 + jj];
            float hv[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float yg = static_cast<float>(stage[jj * 128 + i8 + e] - rs) * sc;
              const float yu = static_cast<float>(stage[jj * 128 + 64 + i8 + e] - rs) * sc;
              hv[e] = sigmoid_mul(yg, yu);
            }
            const int64_t off = t * p.ldy + static_cast<int64_t>(blockIdx.x) * 64 + i8;
            if (p.out_mode == kOutF16) {
              uint4 o;
              __half2* h = reinterpret_cast<__half2*>(&o);
#pragma unroll
              for (int e = 0; e < 4; ++e) h[e] = __floats2half2_rn(hv[2 * e], hv[2 * e + 1]);
              *reinterpret_cast<uint4*>(reinterpret_cast<__half*>(p.y) + off) = o;
            } else {
              float* y = reinterpret_cast<float*>(p.y) + off;
              *reinterpret_cast<float4*>(y) = make_float4(hv[0], hv[1], hv[2], hv[3]);
              *reinterpret_cast<float4*>(y + 4) = make_float4(hv[4], hv[5], hv[6], hv[7]);
            }
          }
        }
        named_bar_sync(1, kEpiThreads);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (csize > 1) {
    // Every thread of every CTA of the cluster reaches both barriers on every path.
    cluster_sync_all();
    if (warp >= 2) split_k_reduce<BN, TC>(p, csize, t0, r0, s_act, s_scale, s_rsum);
    cluster_sync_all();   // peers' partial sums stay readable until everyone is done
  }
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int BN, int TC = 512>
cudaError_t launch_bn(const GemmCall& c, cudaStream_t s) {
  using Cf = Cfg<BN, TC>;
  static std::once_flag attr_once[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once[dev], [&] {
    attr_err = cudaFuncSetAttribute(ternary_gemm_kernel<BN, TC>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, Cf::kSmem);
  });
  if (attr_err != cudaSuccess) return attr_err;

  CUtensorMap tm_w, tm_a;
  if (!make_tmap_2d_u8(&tm_w, c.Wp, static_cast<uint64_t>(c.K / 4), static_cast<uint64_t>(c.rows),
                       static_cast<uint64_t>(c.K / 4), kWRowBytes, 64,
                       CU_TENSOR_MAP_SWIZZLE_32B))
    return cudaErrorInvalidValue;
  if (!make_tmap_2d_u8(&tm_a, c.A, static_cast<uint64_t>(c.K), static_cast<uint64_t>(c.T),
                       static_cast<uint64_t>(c.K), kKB, BN, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;

  Params p;
  p.T = c.T;
  p.K = c.K;
  p.rows = c.rows;
  p.glu = c.glu;
  p.half = c.glu ? c.rows / 2 : 0;
  p.out_mode = c.out_mode;
  p.ldy = c.glu ? c.rows / 2 : c.rows;
  p.gamma = c.gamma;
  p.rowsum = c.rowsum;
  p.beta = c.beta;
  p.y = c.y;
  p.status = c.status;
  p.wait_limit_ns = c.wait_limit_ns;

  // 128 weight rows per tile: 128 outputs, or 64 gate + 64 multiplier rows for 64 GLU outputs.
  const unsigned ntiles = static_cast<unsigned>(c.rows / 128);
  const unsigned ttiles = static_cast<unsigned>((c.T + BN - 1) / BN);
  // Few tiles (decode): split K over a cluster of up to 8 CTAs so more SMs stream weights.
  const int nkb = c.K / kKB;
  const int64_t tiles = static_cast<int64_t>(ntiles) * ttiles;
  int csize = 1;
  if (tiles < kSplitTargetCtas) {
    const int64_t room = kSplitTargetCtas / tiles;
    while (csize * 2 <= 8 && csize * 2 <= nkb && csize * 2 <= room) csize *= 2;
  }

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ntiles, ttiles, static_cast<unsigned>(csize));
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = Cf::kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attrs[2];
  attrs[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attrs[0].val.programmaticStreamSerializationAllowed = 1;
  attrs[1].id = cudaLaunchAttributeClusterDimension;
  attrs[1].val.clusterDim.x = 1;
  attrs[1].val.clusterDim.y = 1;
  attrs[1].val.clusterDim.z = static_cast<unsigned>(csize);
  cfg.attrs = attrs;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, ternary_gemm_kernel<BN, TC>, tm_w, tm_a, p);
}

}  // namespace

cudaError_t launch_ternary_gemm(const GemmCall& c, cudaStream_t s) {
  // prefill with room for the int8 weight codes: the CTA-pair GEMM
  if (c.w8 != nullptr && prefill_ss_supported(c)) return launch_prefill_ss(c, c.w8, s);
  if (c.T <= 16) return launch_bn<16>(c, s);
  if (c.T <= 32) return launch_bn<32>(c, s);
  if (c.T <= 64) return launch_bn<64>(c, s);
  if (c.T <= 128) return launch_bn<128>(c, s);
  // prefill: 128-token tiles, two CTAs per SM, so that one CTA's epilogue overlaps the
  // other's main loop
  return launch_bn<128, 256>(c, s);
}

namespace {
__global__ void wait_probe_kernel(uint64_t limit_ns, unsigned* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // Nothing ever arrives on this barrier: the wait must give up and report.
    mbar_wait_bounded(smem_u32(&bar), 0, limit_ns, &abort_flag, status);
  }
  __syncthreads();
}
}  // namespace

cudaError_t launch_wait_probe(uint64_t limit_ns, unsigned* status, cudaStream_t s) {
  wait_probe_kernel<<<1, 32, 0, s>>>(limit_ns, status);
  return cudaGetLastError();
}

}  // namespace mmf
