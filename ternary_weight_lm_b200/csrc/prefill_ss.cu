// Prefill contraction (many token tiles) as a CTA-pair int8 GEMM on the 5th-generation tensor
// cores (tcgen05.mma.cta_group::2, kind::i8), both operands brought by TMA.
//
// "MatMul-freie LLMs: Zentrale Konzepte erklärt": section "MatMul durch ternäre Operationen
// ersetzen" (weights in {-1,0,1}: products become adds and subtracts), figure item 4 (scaled
// ternary accumulation) and the GLU paragraph (one branch through SiLU times the other).
//
// It computes what the single-tile contraction computes, with the same exact int32 sums and the
// same epilogue arithmetic:
//   acc[t][n] = sum_k c[n][k] * q[t][k]                (c in {-1,0,1}, q int8: exact in int32)
//   y[t][n]   = acc[t][n] * (gamma_t / 127 * beta)     (or h = silu(y gated) * y multiplier)
//
// Why this shape.  At prefill sizes every token tile re-reads the weights, so the weight codes
// live in L2; per k-block a CTA copies an activation tile and a weight tile from L2 into shared
// memory, and those copies take about a microsecond each under this load.  The tensor pipe is
// fed only if enough bytes are in flight per unit of tensor work.  A CTA pair with tiles of 256
// tokens x 256 weight rows does 128 x 256 x 128 multiply-adds per SM and k-block for 32 KB of
// copies, a third fewer bytes per multiply-add than a 128 x 128 single-CTA tile with 2-bit
// weights unpacked on chip, and no thread of one CTA has to signal the other per k-block (the
// odd CTA's copies complete on the even CTA's barrier; the MMA's commits reach both CTAs).  The
// price is a once-per-call pre-pass that expands the packed 2-bit codes into int8 codes c in
// the workspace (N x K bytes, read back from L2 by every token tile).
//
// Work: tile = 256 tokens x 256 weight rows (GLU: 128 gated + 128 multiplier rows, 128
// outputs).  The even CTA holds tokens 0-127 of the tile (A operand, M rows 0-127) and weight
// rows 0-127 (B operand, N columns 0-127); the odd CTA tokens 128-255 and weight rows 128-255.
// One MMA (M = 256, N = 256, K = 32) issued by the even CTA writes each CTA's TMEM: its own 128
// tokens x all 256 weight rows.  Pairs walk the tiles weight tile fastest (the CTAs running at
// once share a few token tiles of activation codes in L2).
// Warps: 0 TMA producer, 1 TMEM allocation and (even CTA) MMA issue, 2-5 epilogue: TMEM ->
// registers -> dequantisation (and GLU) -> a 128-byte-swizzled shared tile -> TMA store.
// TMEM: two accumulators of 256 columns (the epilogue of tile i overlaps the MMAs of tile i+1).
// Every wait is bounded; on a timeout the block records kStatusTimeout, every role stops, the
// copies, MMAs and stores in flight are drained and TMEM is freed.
//
// The same pipeline with fp16 operands (kind::f16, fp32 accumulators) serves the contractions of
// the straight-through backward.  A stage is still 128 rows x 128 bytes per operand (64 fp16
// values of the contraction), so the shared-memory image, the descriptors and the 32-byte k
// steps are those of the int8 form.  There the contraction may be split over several work items
// (the weight gradient contracts over all tokens but has few output tiles): item i takes the
// tile i mod n_tiles and the split i / n_tiles, and writes its fp32 partial tile into its own
// slab of rows, summed afterwards by another kernel.
#include <cuda_fp16.h>

#include <mutex>

#include "backward.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace mmf {
namespace {

constexpr int kKB = 128;                   // K per k-block (bytes of int8 per operand row)
constexpr int kRows = 128;                 // operand rows per CTA (tokens for A, weights for B)
constexpr int kOpStage = kRows * kKB;      // 16 KB
constexpr int kStage = 2 * kOpStage;       // A + B
constexpr int kS = 6;
constexpr int kThreads = 192;
constexpr int kOutBuf = kRows * 128;       // 128 rows x 128 bytes (64 fp16 / 32 fp32 columns)
constexpr int kBarBytes = 256;
constexpr int kSmem = 1024 + kS * kStage + 2 * kOutBuf + kBarBytes;
constexpr uint64_t kDrainNs = 2000000000ull;
static_assert(8 * (2 * kS + 5) <= kBarBytes, "barrier area");
static_assert(kSmem <= 227 * 1024, "shared memory per block");

struct SParams {
  int64_t T;         // rows of A (tokens; for the weight gradient, output rows)
  int nkb;           // k-blocks of 128 bytes in the contraction
  int ksplit;        // work items per output tile (contraction split); 1 for the int8 form
  int64_t slab;      // output rows between two splits' partial tiles (a multiple of 256)
  int ncols;         // output columns (stores at or beyond are skipped)
  int glu;
  int half;          // GLU: I (row offset of the multiplier half)
  int out_mode;
  int n_wt;          // weight tiles of 256 rows
  int n_tiles;
  const float* gamma;
  const float* beta;
  unsigned* status;
  uint64_t wait_limit_ns;
};

// kind::i8 instruction descriptor with both operands signed (int8 codes c and q).
__host__ __device__ constexpr uint32_t idesc_i8_s8s8(int m, int n) {
  return (2u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(n >> 3) << 17) |
         (static_cast<uint32_t>(m >> 4) << 24);
}

// kind::f16 instruction descriptor: fp32 accumulator, both operands fp16, both K-major.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int m, int n) {
  return (1u << 4) | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(m >> 4) << 24);
}

// Tensor-map tile load into this CTA's shared memory that completes its bytes on a barrier of
// either CTA of the pair (`bar` is a shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pairbar(uint32_t dst, const CUtensorMap* m,
                                                   uint32_t bar, int32_t x, int32_t y,
                                                   uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(x), "r"(y), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void tc_mma_i8_ss_pair_warp(uint32_t d_tmem, uint64_t a_desc,
                                                       uint64_t b_desc, uint32_t idesc,
                                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tc_mma_f16_ss_pair_warp(uint32_t d_tmem, uint64_t a_desc,
                                                        uint64_t b_desc, uint32_t idesc,
                                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

template <bool kF16>
__global__ void __launch_bounds__(kThreads, 1)
prefill_ss_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                  const __grid_constant__ CUtensorMap tm_y, const SParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* s_a = smem;                        // kS x 16 KB, activation codes (A)
  uint8_t* s_b = s_a + kS * kOpStage;         // kS x 16 KB, weight codes (B)
  uint8_t* s_out = s_b + kS * kOpStage;       // 2 x 16 KB output tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_out + 2 * kOutBuf);
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  // full(s) (used in the even CTA): both CTAs' copies of stage s landed.  empty(s) (both): the
  // MMAs that read stage s completed.  accfull(b) (both): accumulator b is final.  accempty(b)
  // (even CTA): the epilogue warps of both CTAs read accumulator b.
  auto full = [&](int s) { return smem_u32(bars + s); };
  auto empty = [&](int s) { return smem_u32(bars + kS + s); };
  auto accfull = [&](int b) { return smem_u32(bars + 2 * kS + b); };
  auto accempty = [&](int b) { return smem_u32(bars + 2 * kS + 2 + b); };
  const uint32_t drainbar = smem_u32(bars + 2 * kS + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  if (threadIdx.x == 0) {
    for (int s = 0; s < kS; ++s) {
      mbar_init(full(s), 1);       // the even CTA's producer (expect_tx for both CTAs' bytes)
      mbar_init(empty(s), 1);      // the pair MMA's commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accfull(b), 1);
      mbar_init(accempty(b), 8);   // the four epilogue warps of each CTA
    }
    mbar_init(drainbar, 1);
    s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_a);
    tma_prefetch_desc(&tm_b);
    tma_prefetch_desc(&tm_y);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(&s_tmem), 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // both CTAs' barriers exist before either signals the other's
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  volatile int* abort_flag = &s_abort;
  if (threadIdx.x == 0) pdl_launch_dependents();
  pdl_wait();

  const int nkb = p.nkb;
  const int n_items = p.n_tiles * p.ksplit;
  const int tile0 = static_cast<int>(blockIdx.x >> 1), tstep = static_cast<int>(gridDim.x >> 1);
  // k-block range of a work item
  auto kb_begin = [&](int item) { return (item / p.n_tiles) * nkb / p.ksplit; };
  auto kb_end = [&](int item) { return (item / p.n_tiles + 1) * nkb / p.ksplit; };

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol_a = l2_policy_evict_normal();   // read by the pairs of one token tile
      const uint64_t pol_b = l2_policy_evict_last();     // every token tile re-reads them
      uint32_t c = 0;
      bool ok = true;
      for (int item = tile0; item < n_items && ok; item += tstep) {
        const int tile = item % p.n_tiles;
        const int wt = tile % p.n_wt, tt = tile / p.n_wt;
        const int tok0 = tt * 2 * kRows + static_cast<int>(rank) * kRows;
        const int brow = p.glu ? (rank == 0 ? wt * kRows : p.half + wt * kRows)
                               : wt * 2 * kRows + static_cast<int>(rank) * kRows;
        const int kbe = kb_end(item);
        for (int kb = kb_begin(item); kb < kbe; ++kb, ++c) {
          const int s = static_cast<int>(c % kS);
          if (c >= kS && !mbar_wait_bounded_cluster(empty(s), ((c / kS) - 1) & 1,
                                                    p.wait_limit_ns, abort_flag, p.status)) {
            ok = false;
            break;
          }
          const uint32_t bar0 = map_peer(full(s), 0);
          if (rank == 0) mbar_arrive_expect_tx(full(s), 2 * kStage);
          // k-block kb starts at element kb * 128 (int8) or kb * 64 (fp16): byte kb * 128
          const int kx = kb * (kF16 ? kKB / 2 : kKB);
          tma_load_2d_pairbar(smem_u32(s_a + s * kOpStage), &tm_a, bar0, kx, tok0, pol_a);
          tma_load_2d_pairbar(smem_u32(s_b + s * kOpStage), &tm_b, bar0, kx, brow, pol_b);
        }
      }
      // Every copy this thread started lands before the block exits: the even CTA sees its
      // full barriers; the odd CTA knows its copies landed once the MMAs that read them
      // completed (their commits reach its empty barriers).
      for (uint32_t i = c > kS ? c - kS : 0; i < c; ++i) {
        if (rank == 0)
          mbar_wait_bounded_cluster(full(static_cast<int>(i % kS)), (i / kS) & 1, kDrainNs,
                                    nullptr, p.status);
        else
          mbar_wait_bounded_cluster(empty(static_cast<int>(i % kS)), (i / kS) & 1, kDrainNs,
                                    nullptr, p.status);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (even CTA)
    if (rank == 0) {
      constexpr uint32_t idesc = kF16 ? idesc_f16_f32(2 * kRows, 2 * kRows)
                                      : idesc_i8_s8s8(2 * kRows, 2 * kRows);
      const uint64_t adesc0 = smem_desc_kmajor_sw128(smem_u32(s_a));
      const uint64_t bdesc0 = smem_desc_kmajor_sw128(smem_u32(s_b));
      uint32_t c = 0;
      int n = 0;
      bool ok = true;
      for (int item = tile0; item < n_items && ok; item += tstep, ++n) {
        const int b = n & 1;
        const int kbb = kb_begin(item), kbe = kb_end(item);
        if (n >= 2) {
          const bool w = mbar_wait_bounded_cluster(accempty(b), ((n >> 1) - 1) & 1,
                                                   p.wait_limit_ns, abort_flag, p.status);
          if (!__all_sync(0xFFFFFFFFu, w)) break;
        }
        tc_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(b * 2 * kRows);
        for (int kb = kbb; kb < kbe; ++kb, ++c) {
          const int s = static_cast<int>(c % kS);
          const bool w = mbar_wait_bounded_cluster(full(s), (c / kS) & 1, p.wait_limit_ns,
                                                   abort_flag, p.status);
          if (!__all_sync(0xFFFFFFFFu, w)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // descriptor start addresses in 16-byte units: a stage is 16 KB per operand, a
          // 32-deep k step is 32 bytes inside the 128-byte swizzled rows
          const uint64_t ad = adesc0 + static_cast<uint64_t>((s * kOpStage) >> 4);
          const uint64_t bd = bdesc0 + static_cast<uint64_t>((s * kOpStage) >> 4);
          if constexpr (kF16) {
            tc_mma_f16_ss_pair_warp(d, ad, bd, idesc, kb > kbb ? 1u : 0u);
            tc_mma_f16_ss_pair_warp(d, ad + 2, bd + 2, idesc, 1u);
            tc_mma_f16_ss_pair_warp(d, ad + 4, bd + 4, idesc, 1u);
            tc_mma_f16_ss_pair_warp(d, ad + 6, bd + 6, idesc, 1u);
          } else {
            tc_mma_i8_ss_pair_warp(d, ad, bd, idesc, kb > kbb ? 1u : 0u);
            tc_mma_i8_ss_pair_warp(d, ad + 2, bd + 2, idesc, 1u);
            tc_mma_i8_ss_pair_warp(d, ad + 4, bd + 4, idesc, 1u);
            tc_mma_i8_ss_pair_warp(d, ad + 6, bd + 6, idesc, 1u);
          }
          tc_commit_pair_warp(empty(s));
        }
        if (ok) tc_commit_pair_warp(accfull(b));
      }
      // nothing this warp issued may still run when either CTA frees its TMEM
      tc_commit_pair_warp(drainbar);
      mbar_wait_bounded_cluster(drainbar, 0, kDrainNs, nullptr, p.status);
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------------------ epilogue (both CTAs)
    // Thread = one token (TMEM lane); it holds that token's 256 accumulators of the tile.
    const int q = warp & 3;
    const int r = q * 32 + lane;                       // TMEM lane = row of this CTA's A
    const int et = threadIdx.x - 64;                   // 0..127
    const uint32_t lane_addr = static_cast<uint32_t>(q * 32) << 16;
    const bool to_i32 = p.out_mode == kOutI32;
    const bool to_f16 = p.out_mode == kOutF16;
    const float beta = to_i32 ? 0.0f : (p.beta ? *p.beta : 1.0f);
    const uint32_t accempty0[2] = {map_peer(accempty(0), 0), map_peer(accempty(1), 0)};
    int nbuf = 0;                                      // output tiles used so far (alternating)
    int last_buf = -1;                                 // tile of the newest committed store
    int n = 0;
    for (int item = tile0; item < n_items; item += tstep, ++n) {
      const int tile = item % p.n_tiles;
      const int wt = tile % p.n_wt, tt = tile / p.n_wt;
      const int64_t tok0 = static_cast<int64_t>(tt) * 2 * kRows + rank * kRows;
      const int64_t t = tok0 + r;
      // row of the output tensor this CTA's 128 rows start at (the split's slab)
      const int64_t yrow0 = tok0 + static_cast<int64_t>(item / p.n_tiles) * p.slab;
      float sc;
      if constexpr (kF16)
        sc = beta;
      else
        sc = (!to_i32 && t < p.T) ? __fmul_rn(__fdiv_rn(p.gamma[t], 127.0f), beta) : 0.0f;
      const int b = n & 1;
      const bool w = mbar_wait_bounded_cluster(accfull(b), (n >> 1) & 1, p.wait_limit_ns,
                                               abort_flag, p.status);
      if (!named_bar_and(1, 128, __all_sync(0xFFFFFFFFu, w))) break;
      tc_fence_after();
      const uint32_t dcol = tmem + lane_addr + static_cast<uint32_t>(b * 2 * kRows);
      // output column blocks of one 128-byte shared tile each: 64 fp16 or 32 fp32/int32
      const int cols_per_buf = to_f16 ? 64 : 32;
      const int n_out = p.glu ? kRows : 2 * kRows;     // outputs of this tile per token
      const int ncb = n_out / cols_per_buf;
      const int col_base = p.glu ? wt * kRows : wt * 2 * kRows;
      for (int cb = 0; cb < ncb; ++cb) {
        // this block's values, as 32-bit words in output order
        uint32_t o[32];
        const int c0 = cb * cols_per_buf;
        if (!p.glu) {
          uint32_t v[32];
          if (to_f16) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              tc_ld_32x32b_x32(dcol + static_cast<uint32_t>(c0 + 32 * hh), v);
              tc_wait_ld();
#pragma unroll
              for (int j = 0; j < 16; ++j)
                o[16 * hh + j] = pack_half2(static_cast<float>(static_cast<int32_t>(v[2 * j])) * sc,
                                            static_cast<float>(static_cast<int32_t>(v[2 * j + 1])) * sc);
            }
          } else {
            tc_ld_32x32b_x32(dcol + static_cast<uint32_t>(c0), v);
            tc_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if constexpr (kF16)
                o[j] = __float_as_uint(__uint_as_float(v[j]) * sc);
              else
                o[j] = to_i32 ? v[j]
                              : __float_as_uint(static_cast<float>(static_cast<int32_t>(v[j])) * sc);
            }
          }
        } else {
          // gated columns [c0, c0 + cols) and multiplier columns 128 + [c0, c0 + cols)
          uint32_t g[32], u[32];
          const int halves = to_f16 ? 2 : 1;
          for (int hh = 0; hh < halves; ++hh) {
            tc_ld_32x32b_x32(dcol + static_cast<uint32_t>(c0 + 32 * hh), g);
            tc_ld_32x32b_x32(dcol + static_cast<uint32_t>(kRows + c0 + 32 * hh), u);
            tc_wait_ld();
            float h[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const float zg = static_cast<float>(static_cast<int32_t>(g[j])) * sc;
              const float zu = static_cast<float>(static_cast<int32_t>(u[j])) * sc;
              h[j] = __fdividef(zg, 1.0f + expf(-zg)) * zu;
            }
            if (to_f16) {
#pragma unroll
              for (int j = 0; j < 16; ++j) o[16 * hh + j] = pack_half2(h[2 * j], h[2 * j + 1]);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(h[j]);
            }
          }
        }
        if (cb == ncb - 1) {
          // every TMEM read of this tile is done: the accumulator may be refilled
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if (rank == 0)
              mbar_arrive(accempty(b));
            else   // relaxed: the loads completed (tcgen05.wait::ld) before this arrive
              mbar_arrive_cluster_relaxed(accempty0[b]);
          }
        }
        // shared tile: row r = token, 128 bytes, 16-byte chunk k stored at k ^ (r mod 8)
        uint8_t* buf = s_out + (nbuf & 1) * kOutBuf;
        // the newest store that used this tile has read it: one other store may still be
        // reading the other tile, unless the newest store used this one (stores skipped past
        // the end break the alternation)
        if (et == 0) {
          if (last_buf == (nbuf & 1))
            bulk_wait_group_read<0>();
          else
            bulk_wait_group_read<1>();
        }
        named_bar_sync(1, 128);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          *reinterpret_cast<uint4*>(buf + r * 128 + ((k ^ (r & 7)) << 4)) =
              make_uint4(o[4 * k], o[4 * k + 1], o[4 * k + 2], o[4 * k + 3]);
        fence_proxy_async_smem();
        named_bar_sync(1, 128);
        if (et == 0 && tok0 < p.T && col_base + c0 < p.ncols) {
          tma_store_2d(&tm_y, smem_u32(buf), col_base + c0, static_cast<int32_t>(yrow0));
          bulk_commit_group();
          last_buf = nbuf & 1;
        }
        ++nbuf;
      }
    }
    if (et == 0) bulk_wait_group<0>();
  }

  // Teardown: every MMA completed (the even CTA's MMA warp drained them), every TMEM read of
  // both CTAs is done, and no signal is still on its way to the other CTA.
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// Packed 2-bit codes (e = c + 1, layout L1: code 16G + 4i + j of a row at bits 8j + 2i of its
// 32-bit word G) -> int8 codes c in K order.  One packed word -> 16 output bytes.
__global__ void __launch_bounds__(256) unpack_codes_i8_kernel(const uint32_t* __restrict__ wp,
                                                              int64_t nwords,
                                                              uint4* __restrict__ w8) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < nwords;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint32_t w = __ldg(wp + i);
    uint4 o;
    o.x = __vsub4(w & 0x03030303u, 0x01010101u);
    o.y = __vsub4((w >> 2) & 0x03030303u, 0x01010101u);
    o.z = __vsub4((w >> 4) & 0x03030303u, 0x01010101u);
    o.w = __vsub4((w >> 6) & 0x03030303u, 0x01010101u);
    w8[i] = o;
  }
}

}  // namespace

size_t prefill_w8_bytes(int64_t N, int64_t K) { return static_cast<size_t>(N) * static_cast<size_t>(K); }

bool prefill_ss_supported(const GemmCall& c) { return c.T > 128 && c.rows % 256 == 0; }

namespace {

// CTA pairs of the pair kernel that fit on the device at once (per device and operand kind).
template <bool kF16>
cudaError_t pair_setup(int* pairs_out, int* sms_out) {
  static std::once_flag once[kMaxDevices];
  static int pairs[kMaxDevices], sms[kMaxDevices];
  static cudaError_t err[kMaxDevices];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::call_once(once[dev], [&] {
    cudaError_t ae = cudaFuncSetAttribute(prefill_ss_kernel<kF16>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (ae == cudaSuccess) ae = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
    int nc = 0;
    if (ae == cudaSuccess) {
      cudaLaunchConfig_t q = {};
      q.gridDim = dim3(2 * static_cast<unsigned>(sms[dev] / 2));
      q.blockDim = dim3(kThreads);
      q.dynamicSmemBytes = kSmem;
      cudaLaunchAttribute ca;
      ca.id = cudaLaunchAttributeClusterDimension;
      ca.val.clusterDim.x = 2;
      ca.val.clusterDim.y = 1;
      ca.val.clusterDim.z = 1;
      q.attrs = &ca;
      q.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&nc, prefill_ss_kernel<kF16>, &q) != cudaSuccess) {
        (void)cudaGetLastError();
        nc = 0;
      }
    }
    pairs[dev] = nc;
    err[dev] = ae;
  });
  if (err[dev] != cudaSuccess) return err[dev];
  if (pairs[dev] <= 0) return cudaErrorInvalidConfiguration;
  *pairs_out = pairs[dev];
  if (sms_out) *sms_out = sms[dev];
  return cudaSuccess;
}

template <bool kF16>
cudaError_t launch_pairs(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const CUtensorMap& tm_y,
                         const SParams& p, int pairs, cudaStream_t s) {
  const int64_t items = static_cast<int64_t>(p.n_tiles) * p.ksplit;
  const int64_t np = items < pairs ? items : pairs;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * np));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, prefill_ss_kernel<kF16>, tm_a, tm_b, tm_y, p);
}

// y[m][n] = sum over the splits of part[split][m][n], for m < M (float4 at a time).
__global__ void __launch_bounds__(256) splitk_sum_kernel(const float4* __restrict__ part,
                                                         int ksplit, int64_t slab_vec,
                                                         int64_t n_vec, float4* __restrict__ y) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n_vec;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float4 a = __ldcs(part + i);
    for (int sp = 1; sp < ksplit; ++sp) {
      const float4 b = __ldcs(part + sp * slab_vec + i);
      a.x += b.x;
      a.y += b.y;
      a.z += b.z;
      a.w += b.w;
    }
    y[i] = a;
  }
}

constexpr int kNominalPairs = 74;   // split choice for a 148-SM part, independent of the device

}  // namespace

cudaError_t launch_prefill_ss(const GemmCall& c, int8_t* w8, cudaStream_t s) {
  int pairs = 0, sms = 0;
  cudaError_t e = pair_setup<false>(&pairs, &sms);
  if (e != cudaSuccess) return e;

  // 1. expand the packed codes into int8 codes (N x K bytes)
  const int64_t nwords = static_cast<int64_t>(c.rows) * (c.K / 16);
  const int64_t want = (nwords + 255) / 256;
  const unsigned ublocks = static_cast<unsigned>(want < 8 * sms ? want : 8 * sms);
  unpack_codes_i8_kernel<<<ublocks, 256, 0, s>>>(reinterpret_cast<const uint32_t*>(c.Wp), nwords,
                                                 reinterpret_cast<uint4*>(w8));
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  // 2. the pair GEMM
  CUtensorMap tm_a, tm_b, tm_y;
  if (!make_tmap_2d_u8(&tm_a, c.A, static_cast<uint64_t>(c.K), static_cast<uint64_t>(c.T),
                       static_cast<uint64_t>(c.K), kKB, kRows, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (!make_tmap_2d_u8(&tm_b, w8, static_cast<uint64_t>(c.K), static_cast<uint64_t>(c.rows),
                       static_cast<uint64_t>(c.K), kKB, kRows, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const int ldy = c.glu ? c.rows / 2 : c.rows;
  const bool f16 = c.out_mode == kOutF16;
  const CUtensorMapDataType ydt = f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                  : c.out_mode == kOutF32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                                          : CU_TENSOR_MAP_DATA_TYPE_INT32;
  if (!make_tmap_2d(&tm_y, ydt, c.y, static_cast<uint64_t>(ldy), static_cast<uint64_t>(c.T),
                    static_cast<uint64_t>(ldy) * (f16 ? 2 : 4), f16 ? 64 : 32, kRows,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;

  SParams p;
  p.T = c.T;
  p.nkb = c.K / kKB;
  p.ksplit = 1;
  p.slab = 0;
  p.ncols = ldy;
  p.glu = c.glu;
  p.half = c.glu ? c.rows / 2 : 0;
  p.out_mode = c.out_mode;
  p.n_wt = c.rows / 256;
  const int64_t n_tt = (c.T + 2 * kRows - 1) / (2 * kRows);
  const int64_t n_tiles = n_tt * p.n_wt;
  if (n_tiles > 0x7fffffff) return cudaErrorInvalidValue;
  p.n_tiles = static_cast<int>(n_tiles);
  p.gamma = c.gamma;
  p.beta = c.beta;
  p.status = c.status;
  p.wait_limit_ns = c.wait_limit_ns;
  return launch_pairs<false>(tm_a, tm_b, tm_y, p, pairs, s);
}

int f16_gemm_split(int64_t M, int rows, int64_t Kc) {
  const int64_t tiles = ((M + 255) / 256) * ((rows + 255) / 256);
  const int64_t nkb = (Kc + 63) / 64;
  const double slab = static_cast<double>((M + 255) / 256 * 256);
  int best = 1;
  double best_us = 0.0;
  for (int sp = 1; sp <= 8; ++sp) {
    if (sp > 1 && nkb / sp < 4) break;
    const int64_t items = tiles * sp;
    const int64_t rounds = (items + kNominalPairs - 1) / kNominalPairs;
    // ~0.41 us per k-block of a 256 x 256 pair tile at the fp16 rate; partial sums written
    // and read once at ~6 TB/s (6e6 bytes per us)
    double us = static_cast<double>(rounds) * static_cast<double>((nkb + sp - 1) / sp) * 0.41;
    if (sp > 1) us += 2.0 * sp * slab * rows * 4.0 / 6.0e6;
    if (sp == 1 || us < best_us) {
      best = sp;
      best_us = us;
    }
  }
  return best;
}

size_t f16_gemm_part_bytes(int64_t M, int rows, int ksplit) {
  if (ksplit <= 1) return 0;
  return static_cast<size_t>(ksplit) * static_cast<size_t>((M + 255) / 256 * 256) *
         static_cast<size_t>(rows) * 4;
}

cudaError_t launch_f16_gemm(const F16GemmCall& c, cudaStream_t s) {
  int pairs = 0, sms = 0;
  cudaError_t e = pair_setup<true>(&pairs, &sms);
  if (e != cudaSuccess) return e;
  const int ks = c.ksplit < 1 ? 1 : c.ksplit;
  const int64_t slab = (c.M + 255) / 256 * 256;
  CUtensorMap tm_a, tm_b, tm_y;
  // operands: 64 fp16 (128 bytes) of the contraction x 128 rows per box; columns past Kc and
  // rows past M or rows read as zeros
  if (!make_tmap_2d(&tm_a, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, c.A, static_cast<uint64_t>(c.Kc),
                    static_cast<uint64_t>(c.M), static_cast<uint64_t>(c.lda) * 2, 64, kRows,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (!make_tmap_2d(&tm_b, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, c.B, static_cast<uint64_t>(c.Kc),
                    static_cast<uint64_t>(c.rows), static_cast<uint64_t>(c.ldb) * 2, 64, kRows,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  float* out = ks > 1 ? c.part : c.y;
  const uint64_t out_rows = ks > 1 ? static_cast<uint64_t>(ks) * static_cast<uint64_t>(slab)
                                   : static_cast<uint64_t>(c.M);
  if (!make_tmap_2d(&tm_y, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, out, static_cast<uint64_t>(c.rows),
                    out_rows, static_cast<uint64_t>(c.rows) * 4, 32, kRows,
                    CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;

  SParams p;
  p.T = c.M;
  p.nkb = static_cast<int>((c.Kc + 63) / 64);
  p.ksplit = ks;
  p.slab = slab;
  p.ncols = c.rows;
  p.glu = 0;
  p.half = 0;
  p.out_mode = kOutF32;
  p.n_wt = (c.rows + 255) / 256;
  const int64_t n_tiles = (slab / 256) * p.n_wt;
  if (n_tiles * ks > 0x7fffffff) return cudaErrorInvalidValue;
  p.n_tiles = static_cast<int>(n_tiles);
  p.gamma = nullptr;
  p.beta = c.scale;
  p.status = c.status;
  p.wait_limit_ns = c.wait_limit_ns;
  e = launch_pairs<true>(tm_a, tm_b, tm_y, p, pairs, s);
  if (e != cudaSuccess || ks == 1) return e;
  const int64_t n_vec = c.M * c.rows / 4;
  const int64_t want = (n_vec + 255) / 256;
  const unsigned blocks = static_cast<unsigned>(want < 8 * sms ? want : 8 * sms);
  splitk_sum_kernel<<<blocks, 256, 0, s>>>(reinterpret_cast<const float4*>(c.part), ks,
                                           slab * c.rows / 4, n_vec, reinterpret_cast<float4*>(c.y));
  return cudaGetLastError();
}

}  // namespace mmf
