// LayerNorm backward that allocates nothing: the per-block dgamma/dbeta partial sums live in a
// fixed array in the library's own device memory instead of a caller-provided workspace.
//
// Who needs this: code that cannot call cudaMalloc at the point where it runs the backward --
// frameworks that own every byte of device memory through their own pool allocator (a second
// allocator would break their accounting and fragment the pool), and hot loops where an
// allocation would synchronise the device. Such a caller passes only inputs and outputs.
//
// The array is a file-scope __device__ symbol, so every GPU that loads the library holds it
// until the process exits. Host code must not pass the symbol itself to a kernel (on the host
// it names a host-side shadow, not device memory); the device address is looked up once per
// device with cudaGetSymbolAddress and cached for the life of the process, so a device reset
// (cudaDeviceReset) after the first call on that device is not supported.
//
// This entry point has no status word to report a device-side wait that runs out, so it only
// uses the LayerNorm backward kernels that wait on nothing (never the bulk-copy ring).
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/mgt_layer.h"
#include "mgt_internal.h"

namespace {

constexpr long long kScratchFloats = 1LL << 20;  // 4 MiB of fp32 partial sums
constexpr int kMaxDevices = 64;
constexpr int kMaxBlocks = 296;

static __device__ __align__(256) float g_ln_partial[kScratchFloats];

std::mutex g_mu;
float* g_ptr[kMaxDevices] = {};

// Device address of g_ln_partial on the current device (looked up on the first call there).
mgt_status scratch_for_current_device(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MGT_ECUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_ln_partial) != cudaSuccess || !p) return MGT_ECUDA;
    g_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_ptr[dev];
  return MGT_OK;
}

}  // namespace

extern "C" mgt_status mgt_layernorm_bwd_noalloc(int32_t dtype, int64_t rows, int32_t h,
                                                const void* dy, const void* dres, const void* x,
                                                const float* gamma, const float* mean,
                                                const float* rstd, void* dx, float* dgamma,
                                                float* dbeta, void* stream) {
  if (rows <= 0 || h <= 0 || !dy || !x || !gamma || !mean || !rstd || !dx || !dgamma || !dbeta)
    return MGT_EINVAL;
  if (dtype != MGT_BF16 && dtype != MGT_F32) return MGT_EUNSUPPORTED;
  const int vec = dtype == MGT_BF16 ? 8 : 4;
  const int hmax = dtype == MGT_BF16 ? 16384 : 8192;
  if (h % vec || h > hmax) return MGT_EUNSUPPORTED;
  // The kernels move rows and gamma in 16-byte vectors and the statistics and parameter
  // gradients as floats; reject misaligned views here, before anything reaches the GPU.
  auto aligned = [](const void* p, uintptr_t a) {
    return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
  };
  if (!aligned(dy, 16) || !aligned(x, 16) || !aligned(dx, 16) || !aligned(gamma, 16) ||
      (dres && !aligned(dres, 16)) || !aligned(mean, 4) || !aligned(rstd, 4) ||
      !aligned(dgamma, 4) || !aligned(dbeta, 4))
    return MGT_EUNSUPPORTED;
  // One partial row pair (dgamma, dbeta) per block; as many blocks as the array holds.
  long long nblk = kScratchFloats / (2LL * h);
  if (nblk > kMaxBlocks) nblk = kMaxBlocks;
  if (nblk > rows) nblk = rows;
  float* scratch = nullptr;
  mgt_status st = scratch_for_current_device(&scratch);
  if (st != MGT_OK) return st;
  // Every partial row is written before it is read, so the array needs no clearing. With no
  // status word (err = nullptr) the dispatch picks kernels without device-side waits.
  cudaError_t e = mgt::launch_ln_bwd(dtype == MGT_BF16 ? 1 : 0, rows, h, dy, dres, x, gamma,
                                     mean, rstd, dx, scratch, (int)nblk, dgamma, dbeta,
                                     nullptr, nullptr, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MGT_OK : MGT_ECUDA;
}
