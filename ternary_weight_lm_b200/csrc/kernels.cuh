// Host-side launchers of the library's kernels.  Internal to libmmf.so.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

namespace mmf {

enum InDType { kInF32 = 0, kInF16 = 1 };
enum OutMode { kOutF32 = 0, kOutF16 = 1, kOutI32 = 2 };

// Per-device host tables (status word address, one-time kernel attributes) have this many
// slots; a call made with a current device of this index or above fails with a CUDA error
// instead of sharing another device's slot.
constexpr int kMaxDevices = 64;

// Default limit for any one device-side wait before a kernel gives up (nanoseconds).
constexpr uint64_t kWaitLimitNs = 2000000000ull;

// RMSNorm + per-token absmax int8 quantisation (+ row sums of the codes).
cudaError_t launch_act_quant(const void* x, int xdt, int64_t T, int K, const float* g, float eps,
                             int8_t* A, float* gamma, int32_t* rowsum, cudaStream_t s);

// Row sums of given int8 codes A [T x K].
cudaError_t launch_rowsum(const int8_t* A, int64_t T, int K, int32_t* rowsum, cudaStream_t s);

// Weight quantisation: exact |W| sum (bins), beta finalisation, encode + pack.
constexpr size_t kQuantWsBytes = 4096;   // 256 u64 bins + flags
cudaError_t launch_absmean(const void* W, int wdt, int64_t n, void* ws, float* beta,
                           cudaStream_t s);
cudaError_t launch_ternary_pack(const void* W, int wdt, int64_t n, const float* beta,
                                uint8_t* Wp, cudaStream_t s);

// Tensor-core ternary contraction + dequantisation epilogue.
struct GemmCall {
  const int8_t* A;        // [T x K] int8 activation codes
  const uint8_t* Wp;      // [rows x K/4] packed weight codes
  int64_t T;
  int K;
  int rows;               // weight rows (N, or 2I for GLU)
  int glu;                // 1: SiLU-GLU epilogue, output T x rows/2
  const float* gamma;     // [T]
  const int32_t* rowsum;  // [T]
  const float* beta;      // device scalar
  void* y;
  int out_mode;           // OutMode
  unsigned* status;
  uint64_t wait_limit_ns;
  int8_t* w8 = nullptr;   // scratch of prefill_w8_bytes(rows, K) for the int8 weight codes, or
                          // nullptr (then no kernel needs it)
};
cudaError_t launch_ternary_gemm(const GemmCall& c, cudaStream_t s);

// The prefill contraction as a CTA-pair int8 GEMM: needs T > 128, rows % 256 == 0 and w8.
size_t prefill_w8_bytes(int64_t N, int64_t K);
bool prefill_ss_supported(const GemmCall& c);
cudaError_t launch_prefill_ss(const GemmCall& c, int8_t* w8, cudaStream_t s);

// MLGRU recurrence + swish gate norm over T tokens (chunked scan, three launches; one when
// T <= 32).  amap/bmap/carry: workspace arrays of [H x chunks] floats (mlgru_ws_bytes).  With A
// set, o_proj's codes/gamma/rowsum are written instead of o.
struct MlgruCall {
  const void* I;
  const void* F;
  const void* G;
  int xdt;
  int64_t T;
  int H;
  const float* h0;
  const float* norm_w;
  float eps;
  void* o;
  int odt;
  const float* q_norm_w;
  float q_eps;
  int8_t* A;
  float* gamma;
  int32_t* rowsum;
  float* hT;
  float* amap;
  float* bmap;
  float* carry;
};
size_t mlgru_ws_bytes(int64_t T, int64_t H);
cudaError_t launch_mlgru(const MlgruCall& c, cudaStream_t s);

// Device address of the library's status word on the current device (nullptr on failure).
unsigned* device_status_word();

// One block, one wait that nothing satisfies: must give up after limit_ns.
cudaError_t launch_wait_probe(uint64_t limit_ns, unsigned* status, cudaStream_t s);

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).  Sizes
// and box extents in elements of `dt`, the row stride in bytes.
bool make_tmap_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner,
                  uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                  CUtensorMapSwizzle swz);
bool make_tmap_2d_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                     uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                     CUtensorMapSwizzle swz);

}  // namespace mmf
