// mhc_prologue_noalloc: the mHC read site with its scratch in a fixed device
// array instead of a caller buffer, for callers that cannot allocate device
// memory: for example code running under a framework or serving runtime whose
// memory pool owns every device allocation and forbids any other, or a
// latency-critical path where the implicit synchronisation of cudaMalloc and
// cudaFree is not acceptable.  This function allocates nothing.
//
// The scratch is the file-scope array below.  Every GPU on which this library
// is loaded holds it (4.7 MB) until the process exits, whether or not it is
// used.  All calls on a device share it and it keeps whatever the last call
// wrote; calls that overlap on the GPU (on two streams, say) race on it and
// must not be issued.  Nothing in it has to start at zero: the first kernel
// writes every value the second one reads.

#include <mutex>
#include <string>

#include "model.h"

namespace loopk {
namespace {

constexpr int64_t kNoAllocMaxTokens = 65536;
constexpr int64_t kScratchFloatsPerToken = 18;  // two halves x (8 projections + 1 sum of squares)

static __device__ __align__(256) float g_noalloc_scratch[kNoAllocMaxTokens * kScratchFloatsPerToken];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float* g_ptr[kMaxDevices] = {};

// The device address of the array on the current device, looked up once per
// device and kept for the life of the process.  In host code
// `g_noalloc_scratch` only names a host-side stand-in, so the address must come
// from cudaGetSymbolAddress.  A cudaDeviceReset on that device invalidates
// the kept address: callers must not use this entry point after resetting a
// device it has run on.
cudaError_t scratch_on_current_device(float** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_ptr[dev]) {
    float* p = nullptr;
    e = cudaGetSymbolAddress((void**)&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_ptr[dev] = p;
  }
  *out = g_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace loopk

using namespace loopk;

extern "C" int32_t mhc_prologue_noalloc(const float* d_streams, int64_t T, int32_t H, const float* d_gamma,
                                        const float* d_phi, const float* d_gain, int32_t iters, float eps,
                                        float* d_coef, void* d_xhat, int32_t xhat_dtype, void* stream) {
  if (!d_streams || !d_gamma || !d_phi || !d_gain || !d_coef || !d_xhat) {
    set_last_error("mhc_prologue_noalloc: NULL argument");
    return LOOP_EINVAL;
  }
  if (T < 0 || H <= 0 || H % 4 != 0 || H > 6144 || iters < 0 || !(eps >= 0.f)) {
    set_last_error("mhc_prologue_noalloc: T >= 0, H a multiple of 4 and <= 6144, iters >= 0, eps >= 0");
    return LOOP_EINVAL;
  }
  if (T > kNoAllocMaxTokens) {
    set_last_error("mhc_prologue_noalloc: T = " + std::to_string(T) + " exceeds the fixed scratch limit of " +
                   std::to_string(kNoAllocMaxTokens) + " tokens; use mhc_prologue with a caller buffer");
    return LOOP_ERANGE;
  }
  if (xhat_dtype != LOOP_F32 && xhat_dtype != LOOP_BF16) {
    set_last_error("mhc_prologue_noalloc: bad xhat_dtype");
    return LOOP_EINVAL;
  }
  float* scratch = nullptr;
  cudaError_t e = scratch_on_current_device(&scratch);
  if (e == cudaSuccess)
    e = launch_mhc_prologue(d_streams, T, H, d_gamma, d_phi, d_gain, iters, eps, d_coef, d_xhat,
                            xhat_dtype == LOOP_BF16, scratch, (cudaStream_t)stream);
  if (e != cudaSuccess) {
    set_last_error(std::string("mhc_prologue_noalloc: ") + cudaGetErrorString(e));
    return LOOP_ECUDA;
  }
  return LOOP_OK;
}
