// mmf_bitlinear_forward_noalloc: the forward for callers that cannot allocate device memory.
//
// Some callers have no way to call cudaMalloc: a plugin running inside a host application
// that owns every allocation, a real-time decode loop that must never allocate (allocation
// can synchronise the device or fail under memory pressure), or plain C code with no device
// allocator at hand.  This entry point takes only inputs and outputs; its scratch (the int8
// activation codes, gamma and the code sums) lives in a fixed array that every GPU loading
// the library holds until the process exits.
//
// The array's name in host code is a host-side stand-in, not a device address, so its device
// address is looked up with cudaGetSymbolAddress once per device (with that device current),
// on the first call made on that device.  Make that first call before any stream capture.
//
// The calls share one array and it keeps the last call's contents.  Nothing in it has to
// start at zero: the quantisation kernel writes every byte the contraction reads.  Calls
// whose work overlaps on the GPU (different streams, or threads without ordering between
// them) race on the array; order them on one stream or with events.
#include <mutex>

#include "../../include/mmf.h"
#include "kernels.cuh"

#define MMF_EXPORT extern "C" __attribute__((visibility("default")))

namespace mmf {

// 4 MiB: enough for decode-sized calls (for example 64 tokens x 8192 inputs).
constexpr size_t kNoAllocScratchBytes = 4u << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {

size_t round256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

// Device address of the scratch array for the current device, looked up once per device.
unsigned char* noalloc_scratch_ptr() {
  static unsigned char* ptrs[kMaxDevices] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (ptrs[dev] == nullptr) {
    unsigned char* p = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&p), g_noalloc_scratch) != cudaSuccess)
      return nullptr;
    ptrs[dev] = p;
  }
  return ptrs[dev];
}

bool is_aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

}  // namespace
}  // namespace mmf

using namespace mmf;

MMF_EXPORT mmf_status mmf_bitlinear_forward_noalloc(const void* x, mmf_dtype xdt, int64_t T,
                                                    int64_t K, const float* norm_w, float eps,
                                                    const uint8_t* Wp, const float* beta,
                                                    int64_t N, void* y, mmf_dtype ydt,
                                                    void* stream) {
  if (!x || !Wp || !beta || !y) return MMF_ERR_INVALID_ARG;
  if ((xdt != MMF_F32 && xdt != MMF_F16) || (ydt != MMF_F32 && ydt != MMF_F16))
    return MMF_ERR_INVALID_ARG;
  if (!(eps > 0.0f) || eps != eps || eps > 1.0f) return MMF_ERR_INVALID_ARG;
  if (T < 1 || T > 16777216 || K < 128 || K > 8192 || K % 128 != 0 || N < 128 ||
      N > (1 << 20) || N % 128 != 0)
    return MMF_ERR_UNSUPPORTED_SHAPE;
  if (!is_aligned(x, 16) || !is_aligned(Wp, 16) || !is_aligned(y, 16) || !is_aligned(beta, 4) ||
      (norm_w && !is_aligned(norm_w, 16)))
    return MMF_ERR_ALIGNMENT;
  // Scratch layout: codes [T x K], gamma [T], code sums [T], each rounded up to 256 bytes.
  const size_t a_bytes = round256(static_cast<size_t>(T) * static_cast<size_t>(K));
  const size_t v_bytes = round256(static_cast<size_t>(T) * 4);
  if (a_bytes + 2 * v_bytes > kNoAllocScratchBytes) return MMF_ERR_WORKSPACE;

  unsigned char* scratch = noalloc_scratch_ptr();
  unsigned* status = device_status_word();
  if (!scratch || !status) return MMF_ERR_CUDA;
  int8_t* A = reinterpret_cast<int8_t*>(scratch);
  float* gamma = reinterpret_cast<float*>(scratch + a_bytes);
  int32_t* rowsum = reinterpret_cast<int32_t*>(scratch + a_bytes + v_bytes);

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (launch_act_quant(x, xdt == MMF_F16 ? kInF16 : kInF32, T, static_cast<int>(K), norm_w, eps,
                       A, gamma, rowsum, s) != cudaSuccess)
    return MMF_ERR_CUDA;
  GemmCall c;
  c.A = A;
  c.Wp = Wp;
  c.T = T;
  c.K = static_cast<int>(K);
  c.rows = static_cast<int>(N);
  c.glu = 0;
  c.gamma = gamma;
  c.rowsum = rowsum;
  c.beta = beta;
  c.y = y;
  c.out_mode = ydt == MMF_F16 ? kOutF16 : kOutF32;
  c.status = status;
  c.wait_limit_ns = kWaitLimitNs;
  return launch_ternary_gemm(c, s) == cudaSuccess ? MMF_OK : MMF_ERR_CUDA;
}
