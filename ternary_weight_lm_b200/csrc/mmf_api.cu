// The C ABI of libmmf.so (declared in include/mmf.h): host-side argument checks, workspace
// layout, tensor-map encoding and kernel launches.  Every check runs before any CUDA call, so
// a rejected call never touches the device.
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/mmf.h"
#include "backward.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

#define MMF_EXPORT extern "C" __attribute__((visibility("default")))

namespace mmf {

// Device status word: kernels OR kStatusTimeout into it when a wait gives up.
__device__ unsigned g_device_status;

namespace {

constexpr int64_t kMaxT = 16777216;
constexpr int64_t kMaxK = 8192;
constexpr int64_t kMaxN = 1 << 20;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

size_t up256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

mmf_status check_dtype(int d) { return (d == MMF_F32 || d == MMF_F16) ? MMF_OK : MMF_ERR_INVALID_ARG; }

mmf_status check_k(int64_t K) {
  if (K < 128 || K > kMaxK || K % 128 != 0) return MMF_ERR_UNSUPPORTED_SHAPE;
  return MMF_OK;
}

mmf_status check_n(int64_t N) {
  if (N < 128 || N > kMaxN || N % 128 != 0) return MMF_ERR_UNSUPPORTED_SHAPE;
  return MMF_OK;
}

mmf_status check_t(int64_t T) {
  if (T < 1 || T > kMaxT) return MMF_ERR_UNSUPPORTED_SHAPE;
  return MMF_OK;
}

struct FwdWs {
  int8_t* A;
  float* gamma;
  int32_t* rowsum;
  int8_t* w8;      // int8 weight codes for the prefill contraction (nullptr when not needed)
};

// int8 weight codes: needed by the prefill contraction (more than 128 tokens)
size_t w8_ws_bytes(int64_t T, int64_t K, int64_t N) {
  return T > 128 ? up256(prefill_w8_bytes(N, K)) : 0;
}

size_t fwd_ws_bytes(int64_t T, int64_t K, int64_t N) {
  return up256(static_cast<size_t>(T) * static_cast<size_t>(K)) +
         2 * up256(static_cast<size_t>(T) * 4) + w8_ws_bytes(T, K, N);
}

FwdWs fwd_ws(void* ws, int64_t T, int64_t K, int64_t N) {
  uint8_t* b = reinterpret_cast<uint8_t*>(ws);
  FwdWs w;
  w.A = reinterpret_cast<int8_t*>(b);
  b += up256(static_cast<size_t>(T) * static_cast<size_t>(K));
  w.gamma = reinterpret_cast<float*>(b);
  b += up256(static_cast<size_t>(T) * 4);
  w.rowsum = reinterpret_cast<int32_t*>(b);
  b += up256(static_cast<size_t>(T) * 4);
  w.w8 = w8_ws_bytes(T, K, N) ? reinterpret_cast<int8_t*>(b) : nullptr;
  return w;
}

unsigned* status_ptr() {
  static unsigned* ptrs[kMaxDevices] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (ptrs[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
    ptrs[dev] = reinterpret_cast<unsigned*>(p);
  }
  return ptrs[dev];
}

mmf_status from_cuda(cudaError_t e) { return e == cudaSuccess ? MMF_OK : MMF_ERR_CUDA; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

mmf_status fwd_common(const void* x, int xdt, int64_t T, int64_t K, const float* norm_w,
                      float eps, const uint8_t* Wp, const float* beta, int64_t rows, void* y,
                      int ydt, void* ws, size_t ws_bytes, bool glu, void* stream) {
  if (!x || !Wp || !beta || !y) return MMF_ERR_INVALID_ARG;
  if (check_dtype(xdt) != MMF_OK || check_dtype(ydt) != MMF_OK) return MMF_ERR_INVALID_ARG;
  if (!(eps > 0.0f) || eps != eps || eps > 1.0f) return MMF_ERR_INVALID_ARG;
  mmf_status st;
  if ((st = check_t(T)) != MMF_OK || (st = check_k(K)) != MMF_OK || (st = check_n(rows)) != MMF_OK)
    return st;
  if (!aligned(x, 16) || !aligned(Wp, 16) || !aligned(y, 16) || !aligned(beta, 4) ||
      (norm_w && !aligned(norm_w, 16)))
    return MMF_ERR_ALIGNMENT;
  if (!ws || ws_bytes < fwd_ws_bytes(T, K, rows)) return MMF_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return MMF_ERR_ALIGNMENT;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned* status = status_ptr();
  if (!status) return MMF_ERR_CUDA;
  FwdWs w = fwd_ws(ws, T, K, rows);
  cudaError_t e = launch_act_quant(x, xdt == MMF_F16 ? kInF16 : kInF32, T, static_cast<int>(K),
                                   norm_w, eps, w.A, w.gamma, w.rowsum, s);
  if (e != cudaSuccess) return MMF_ERR_CUDA;
  GemmCall c;
  c.A = w.A;
  c.Wp = Wp;
  c.T = T;
  c.K = static_cast<int>(K);
  c.rows = static_cast<int>(rows);
  c.glu = glu ? 1 : 0;
  c.gamma = w.gamma;
  c.rowsum = w.rowsum;
  c.beta = beta;
  c.y = y;
  c.out_mode = ydt == MMF_F16 ? kOutF16 : kOutF32;
  c.status = status;
  c.wait_limit_ns = kWaitLimitNs;
  c.w8 = w.w8;
  return from_cuda(launch_ternary_gemm(c, s));
}

}  // namespace

unsigned* device_status_word() { return status_ptr(); }

bool make_tmap_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner,
                  uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                  CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_2d_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                     uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                     CUtensorMapSwizzle swz) {
  return make_tmap_2d(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, inner, outer, row_bytes, box_inner,
                      box_outer, swz);
}

}  // namespace mmf

using namespace mmf;

MMF_EXPORT size_t mmf_quantize_weights_workspace_bytes(int64_t N, int64_t K) {
  (void)N;
  (void)K;
  return kQuantWsBytes;
}

MMF_EXPORT mmf_status mmf_quantize_weights(const void* W, mmf_dtype wdt, int64_t N, int64_t K,
                                           uint8_t* Wp, float* beta, void* ws, size_t ws_bytes,
                                           void* stream) {
  if (!W || !Wp || !beta) return MMF_ERR_INVALID_ARG;
  if (check_dtype(wdt) != MMF_OK) return MMF_ERR_INVALID_ARG;
  mmf_status st;
  if ((st = check_k(K)) != MMF_OK || (st = check_n(N)) != MMF_OK) return st;
  if (!aligned(W, 16) || !aligned(Wp, 16) || !aligned(beta, 4)) return MMF_ERR_ALIGNMENT;
  if (!ws || ws_bytes < kQuantWsBytes) return MMF_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return MMF_ERR_ALIGNMENT;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int dt = wdt == MMF_F16 ? kInF16 : kInF32;
  cudaError_t e = launch_absmean(W, dt, N * K, ws, beta, s);
  if (e != cudaSuccess) return MMF_ERR_CUDA;
  return from_cuda(launch_ternary_pack(W, dt, N * K, beta, Wp, s));
}

MMF_EXPORT mmf_status mmf_ternary_encode(const void* W, mmf_dtype wdt, int64_t N, int64_t K,
                                         const float* beta, uint8_t* Wp, void* stream) {
  if (!W || !Wp || !beta) return MMF_ERR_INVALID_ARG;
  if (check_dtype(wdt) != MMF_OK) return MMF_ERR_INVALID_ARG;
  mmf_status st;
  if ((st = check_k(K)) != MMF_OK || (st = check_n(N)) != MMF_OK) return st;
  if (!aligned(W, 16) || !aligned(Wp, 16) || !aligned(beta, 4)) return MMF_ERR_ALIGNMENT;
  return from_cuda(launch_ternary_pack(W, wdt == MMF_F16 ? kInF16 : kInF32, N * K, beta, Wp,
                                       reinterpret_cast<cudaStream_t>(stream)));
}

MMF_EXPORT size_t mmf_forward_workspace_bytes(int64_t T, int64_t K, int64_t N) {
  if (T < 1 || K < 1 || N < 1) return 0;
  return fwd_ws_bytes(T, K, N);
}

MMF_EXPORT size_t mmf_quantized_workspace_bytes(int64_t T, int64_t K, int64_t N) {
  if (T < 1 || K < 1 || N < 1) return 0;
  return w8_ws_bytes(T, K, N);
}

MMF_EXPORT mmf_status mmf_bitlinear_forward(const void* x, mmf_dtype xdt, int64_t T, int64_t K,
                                            const float* norm_w, float eps, const uint8_t* Wp,
                                            const float* beta, int64_t N, void* y, mmf_dtype ydt,
                                            void* ws, size_t ws_bytes, void* stream) {
  return fwd_common(x, xdt, T, K, norm_w, eps, Wp, beta, N, y, ydt, ws, ws_bytes, false, stream);
}

MMF_EXPORT mmf_status mmf_bitlinear_glu_forward(const void* x, mmf_dtype xdt, int64_t T,
                                                int64_t K, const float* norm_w, float eps,
                                                const uint8_t* Wp, const float* beta, int64_t N2,
                                                void* h, mmf_dtype hdt, void* ws, size_t ws_bytes,
                                                void* stream) {
  return fwd_common(x, xdt, T, K, norm_w, eps, Wp, beta, N2, h, hdt, ws, ws_bytes, true, stream);
}

MMF_EXPORT mmf_status mmf_quantize_activations(const void* x, mmf_dtype xdt, int64_t T, int64_t K,
                                               const float* norm_w, float eps, int8_t* A,
                                               float* gamma, int32_t* rowsum, void* stream) {
  if (!x || !A || !gamma) return MMF_ERR_INVALID_ARG;
  if (check_dtype(xdt) != MMF_OK) return MMF_ERR_INVALID_ARG;
  if (!(eps > 0.0f) || eps != eps || eps > 1.0f) return MMF_ERR_INVALID_ARG;
  mmf_status st;
  if ((st = check_t(T)) != MMF_OK || (st = check_k(K)) != MMF_OK) return st;
  if (!aligned(x, 16) || !aligned(A, 16) || !aligned(gamma, 4) || (rowsum && !aligned(rowsum, 4)) ||
      (norm_w && !aligned(norm_w, 16)))
    return MMF_ERR_ALIGNMENT;
  return from_cuda(launch_act_quant(x, xdt == MMF_F16 ? kInF16 : kInF32, T, static_cast<int>(K),
                                    norm_w, eps, A, gamma, rowsum,
                                    reinterpret_cast<cudaStream_t>(stream)));
}

MMF_EXPORT size_t mmf_mlgru_workspace_bytes(int64_t T, int64_t H) {
  if (T < 1 || T > kMaxT || H < 256 || H > 4096 || H % 256 != 0) return 0;
  return mlgru_ws_bytes(T, H);
}

namespace {

mmf_status mlgru_common(const void* I, const void* F, const void* G, int xdt, int64_t T,
                        int64_t H, const float* h0, const float* norm_w, float eps, float* hT,
                        void* ws, size_t ws_bytes, MlgruCall& c) {
  if (!I || !F || !G) return MMF_ERR_INVALID_ARG;
  if (check_dtype(xdt) != MMF_OK) return MMF_ERR_INVALID_ARG;
  if (!(eps > 0.0f) || eps != eps || eps > 1.0f) return MMF_ERR_INVALID_ARG;
  mmf_status st;
  if ((st = check_t(T)) != MMF_OK) return st;
  if (H < 256 || H > 4096 || H % 256 != 0) return MMF_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(I, 16) || !aligned(F, 16) || !aligned(G, 16) || (h0 && !aligned(h0, 16)) ||
      (norm_w && !aligned(norm_w, 16)) || (hT && !aligned(hT, 16)))
    return MMF_ERR_ALIGNMENT;
  const size_t need = mlgru_ws_bytes(T, H);
  if (need > 0 && (ws == nullptr || ws_bytes < need)) return MMF_ERR_WORKSPACE;
  if (ws == nullptr && ws_bytes != 0) return MMF_ERR_WORKSPACE;
  if (ws != nullptr && !aligned(ws, 256)) return MMF_ERR_ALIGNMENT;
  c = MlgruCall{};
  c.I = I;
  c.F = F;
  c.G = G;
  c.xdt = xdt == MMF_F16 ? kInF16 : kInF32;
  c.T = T;
  c.H = static_cast<int>(H);
  c.h0 = h0;
  c.norm_w = norm_w;
  c.eps = eps;
  c.hT = hT;
  if (need > 0) {
    const size_t one = need / 3;
    uint8_t* b = static_cast<uint8_t*>(ws);
    c.amap = reinterpret_cast<float*>(b);
    c.bmap = reinterpret_cast<float*>(b + one);
    c.carry = reinterpret_cast<float*>(b + 2 * one);
  }
  return MMF_OK;
}

}  // namespace

MMF_EXPORT mmf_status mmf_mlgru_forward(const void* I, const void* F, const void* G,
                                        mmf_dtype xdt, int64_t T, int64_t H, const float* h0,
                                        const float* norm_w, float eps, void* o, mmf_dtype odt,
                                        float* hT, void* ws, size_t ws_bytes, void* stream) {
  if (!o || check_dtype(odt) != MMF_OK) return MMF_ERR_INVALID_ARG;
  MlgruCall c;
  mmf_status st = mlgru_common(I, F, G, xdt, T, H, h0, norm_w, eps, hT, ws, ws_bytes, c);
  if (st != MMF_OK) return st;
  if (!aligned(o, 16)) return MMF_ERR_ALIGNMENT;
  c.o = o;
  c.odt = odt == MMF_F16 ? kInF16 : kInF32;
  return from_cuda(launch_mlgru(c, reinterpret_cast<cudaStream_t>(stream)));
}

MMF_EXPORT mmf_status mmf_mlgru_forward_quantized(const void* I, const void* F, const void* G,
                                                  mmf_dtype xdt, int64_t T, int64_t H,
                                                  const float* h0, const float* norm_w,
                                                  float eps, const float* oproj_norm_w,
                                                  float oproj_eps, int8_t* A, float* gamma,
                                                  int32_t* rowsum, float* hT, void* ws,
                                                  size_t ws_bytes, void* stream) {
  if (!A || !gamma) return MMF_ERR_INVALID_ARG;
  if (!(oproj_eps > 0.0f) || oproj_eps != oproj_eps || oproj_eps > 1.0f) return MMF_ERR_INVALID_ARG;
  MlgruCall c;
  mmf_status st = mlgru_common(I, F, G, xdt, T, H, h0, norm_w, eps, hT, ws, ws_bytes, c);
  if (st != MMF_OK) return st;
  if (!aligned(A, 16) || !aligned(gamma, 4) || (rowsum && !aligned(rowsum, 4)) ||
      (oproj_norm_w && !aligned(oproj_norm_w, 16)))
    return MMF_ERR_ALIGNMENT;
  c.q_norm_w = oproj_norm_w;
  c.q_eps = oproj_eps;
  c.A = A;
  c.gamma = gamma;
  c.rowsum = rowsum;
  return from_cuda(launch_mlgru(c, reinterpret_cast<cudaStream_t>(stream)));
}

MMF_EXPORT mmf_status mmf_bitlinear_forward_quantized(const int8_t* A, const float* gamma,
                                                      const int32_t* rowsum, int64_t T, int64_t K,
                                                      const uint8_t* Wp, const float* beta,
                                                      int64_t N, int glu, void* y, mmf_dtype ydt,
                                                      void* ws, size_t ws_bytes, void* stream) {
  if (!A || !gamma || !rowsum || !Wp || !beta || !y) return MMF_ERR_INVALID_ARG;
  if (check_dtype(ydt) != MMF_OK || (glu != 0 && glu != 1)) return MMF_ERR_INVALID_ARG;
  mmf_status st;
  if ((st = check_t(T)) != MMF_OK || (st = check_k(K)) != MMF_OK || (st = check_n(N)) != MMF_OK)
    return st;
  if (!aligned(A, 16) || !aligned(Wp, 16) || !aligned(y, 16) || !aligned(gamma, 4) ||
      !aligned(rowsum, 4) || !aligned(beta, 4))
    return MMF_ERR_ALIGNMENT;
  // no workspace: the contraction that needs none; otherwise at least the queried size
  if (ws != nullptr && ws_bytes < w8_ws_bytes(T, K, N)) return MMF_ERR_WORKSPACE;
  if (ws == nullptr && ws_bytes != 0) return MMF_ERR_WORKSPACE;
  if (ws != nullptr && !aligned(ws, 256)) return MMF_ERR_ALIGNMENT;
  unsigned* status = status_ptr();
  if (!status) return MMF_ERR_CUDA;
  GemmCall c;
  c.A = A;
  c.Wp = Wp;
  c.T = T;
  c.K = static_cast<int>(K);
  c.rows = static_cast<int>(N);
  c.glu = glu;
  c.gamma = gamma;
  c.rowsum = rowsum;
  c.beta = beta;
  c.y = y;
  c.out_mode = ydt == MMF_F16 ? kOutF16 : kOutF32;
  c.status = status;
  c.wait_limit_ns = kWaitLimitNs;
  c.w8 = (ws != nullptr && w8_ws_bytes(T, K, N) > 0) ? reinterpret_cast<int8_t*>(ws) : nullptr;
  return from_cuda(launch_ternary_gemm(c, reinterpret_cast<cudaStream_t>(stream)));
}

MMF_EXPORT size_t mmf_backward_workspace_bytes(int64_t T, int64_t K, int64_t N) {
  if (check_t(T) != MMF_OK || check_k(K) != MMF_OK || check_n(N) != MMF_OK) return 0;
  return bwd_ws_bytes(T, K, N);
}

MMF_EXPORT mmf_status mmf_bitlinear_backward(const void* x, mmf_dtype xdt, int64_t T, int64_t K,
                                             const float* norm_w, float eps, const int8_t* A,
                                             const float* gamma, const uint8_t* Wp,
                                             const float* beta, int64_t N, const void* dy,
                                             void* dx, mmf_dtype dxdt, float* dW,
                                             float* dnorm_w, void* ws, size_t ws_bytes,
                                             void* stream) {
  if (!x || !Wp || !beta || !dy) return MMF_ERR_INVALID_ARG;
  if (!dx && !dW && !dnorm_w) return MMF_ERR_INVALID_ARG;
  if ((A == nullptr) != (gamma == nullptr)) return MMF_ERR_INVALID_ARG;
  if (check_dtype(xdt) != MMF_OK || check_dtype(dxdt) != MMF_OK) return MMF_ERR_INVALID_ARG;
  if (!(eps > 0.0f) || eps != eps || eps > 1.0f) return MMF_ERR_INVALID_ARG;
  mmf_status st;
  if ((st = check_t(T)) != MMF_OK || (st = check_k(K)) != MMF_OK || (st = check_n(N)) != MMF_OK)
    return st;
  if (!aligned(x, 16) || !aligned(Wp, 16) || !aligned(dy, 16) || !aligned(beta, 4) ||
      (dx && !aligned(dx, 16)) || (dW && !aligned(dW, 16)) || (dnorm_w && !aligned(dnorm_w, 16)) ||
      (A && !aligned(A, 16)) || (gamma && !aligned(gamma, 4)) || (norm_w && !aligned(norm_w, 16)))
    return MMF_ERR_ALIGNMENT;
  if (!ws || ws_bytes < bwd_ws_bytes(T, K, N)) return MMF_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return MMF_ERR_ALIGNMENT;
  unsigned* status = status_ptr();
  if (!status) return MMF_ERR_CUDA;
  BwdCall c;
  c.x = x;
  c.xdt = xdt == MMF_F16 ? kInF16 : kInF32;
  c.T = T;
  c.K = static_cast<int>(K);
  c.norm_w = norm_w;
  c.eps = eps;
  c.A = A;
  c.gamma = gamma;
  c.Wp = Wp;
  c.beta = beta;
  c.N = static_cast<int>(N);
  c.dy = dy;
  c.dx = dx;
  c.dxdt = dxdt == MMF_F16 ? kInF16 : kInF32;
  c.dW = dW;
  c.dnorm_w = dnorm_w;
  c.status = status;
  c.wait_limit_ns = kWaitLimitNs;
  return from_cuda(launch_bitlinear_backward(c, bwd_ws(ws, T, K, N),
                                             reinterpret_cast<cudaStream_t>(stream)));
}

MMF_EXPORT mmf_status mmf_ternary_accumulate_i32(const int8_t* A, int64_t T, int64_t K,
                                                 const uint8_t* Wp, int64_t N, int32_t* acc,
                                                 void* ws, size_t ws_bytes, void* stream) {
  if (!A || !Wp || !acc) return MMF_ERR_INVALID_ARG;
  mmf_status st;
  if ((st = check_t(T)) != MMF_OK || (st = check_k(K)) != MMF_OK || (st = check_n(N)) != MMF_OK)
    return st;
  if (!aligned(A, 16) || !aligned(Wp, 16) || !aligned(acc, 16)) return MMF_ERR_ALIGNMENT;
  if (!ws || ws_bytes < fwd_ws_bytes(T, K, N)) return MMF_ERR_WORKSPACE;
  if (!aligned(ws, 256)) return MMF_ERR_ALIGNMENT;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned* status = status_ptr();
  if (!status) return MMF_ERR_CUDA;
  FwdWs w = fwd_ws(ws, T, K, N);
  cudaError_t e = launch_rowsum(A, T, static_cast<int>(K), w.rowsum, s);
  if (e != cudaSuccess) return MMF_ERR_CUDA;
  GemmCall c;
  c.A = A;
  c.Wp = Wp;
  c.T = T;
  c.K = static_cast<int>(K);
  c.rows = static_cast<int>(N);
  c.glu = 0;
  c.gamma = nullptr;
  c.rowsum = w.rowsum;
  c.beta = nullptr;
  c.y = acc;
  c.out_mode = kOutI32;
  c.status = status;
  c.wait_limit_ns = kWaitLimitNs;
  c.w8 = w.w8;
  return from_cuda(launch_ternary_gemm(c, s));
}

MMF_EXPORT mmf_status mmf_get_device_status(void) {
  unsigned v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(v)) != cudaSuccess) return MMF_ERR_CUDA;
  const unsigned zero = 0;
  if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(zero)) != cudaSuccess) return MMF_ERR_CUDA;
  if (v & kStatusTimeout) return MMF_ERR_TIMEOUT;
  if (v & kStatusBadPlan) return MMF_ERR_PLAN;
  return MMF_OK;
}

MMF_EXPORT mmf_status mmf_debug_wait_timeout_probe(uint64_t limit_ns, void* stream) {
  if (limit_ns < 1000ull || limit_ns > 1000000000ull) return MMF_ERR_INVALID_ARG;
  unsigned* status = status_ptr();
  if (!status) return MMF_ERR_CUDA;
  return from_cuda(launch_wait_probe(limit_ns, status, reinterpret_cast<cudaStream_t>(stream)));
}

MMF_EXPORT const char* mmf_status_string(mmf_status s) {
  switch (s) {
    case MMF_OK: return "MMF_OK";
    case MMF_ERR_INVALID_ARG: return "MMF_ERR_INVALID_ARG";
    case MMF_ERR_UNSUPPORTED_SHAPE: return "MMF_ERR_UNSUPPORTED_SHAPE";
    case MMF_ERR_ALIGNMENT: return "MMF_ERR_ALIGNMENT";
    case MMF_ERR_CUDA: return "MMF_ERR_CUDA";
    case MMF_ERR_TIMEOUT: return "MMF_ERR_TIMEOUT";
    case MMF_ERR_WORKSPACE: return "MMF_ERR_WORKSPACE";
    case MMF_ERR_RESOURCES: return "MMF_ERR_RESOURCES";
    case MMF_ERR_PLAN: return "MMF_ERR_PLAN";
  }
  return "MMF_ERR_UNKNOWN";
}

MMF_EXPORT int mmf_version(void) { return 100; }
