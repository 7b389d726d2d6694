// fa_noalloc.cu -- fa_attn_decode_noalloc: the split-KV decode with its
// scratch in a static device array instead of a caller-provided workspace.
//
// Why: some callers cannot allocate device memory at the point where they
// run decode -- for example a plugin behind a fixed operator interface that
// has no workspace argument, an engine whose memory is all reserved up front
// by its own pool, or a real-time loop where a cudaMalloc (which can
// synchronise the device and fail under memory pressure) is not allowed.
// They still own and pass the inputs and outputs; only the scratch moves
// here.
//
// The scratch is one file-scope __device__ array of kNoAllocScratchBytes
// (8 MiB).  Every GPU that loads this library holds it until the process
// exits.  Host code cannot use the array's name as a device address, so the
// first call on each device (with that device current) looks the address up
// with cudaGetSymbolAddress and caches it; make that first call before any
// stream capture.  The decode kernels write every split's partial result
// before the combine kernel reads it, so nothing in the scratch has to start
// at zero; whatever a previous call left there is overwritten.  All calls
// share the one array: calls whose kernels overlap on the GPU (other streams,
// or other host threads) race on it and must be serialised by the caller.
#include "fa_common.cuh"
#include "fa_internal.h"

#include <mutex>

namespace fa {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mu;
void *g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of g_decode_scratch on the current device (looked up once
// per device).  Returns nullptr on failure.
void *scratch_on_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr) {
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = ptr;
  }
  return g_scratch_ptr[dev];
}

}  // namespace
}  // namespace fa

using namespace fa;

extern "C" {

FA_API size_t fa_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

FA_API int fa_attn_decode_noalloc(const void *q, const void *kcache, const void *vcache,
                                  const int32_t *seqlens, int B, int Lmax, int Hq, int Hkv, int D,
                                  float scale, int mode, const int32_t *mode_dev,
                                  fa_sparse_cfg cfg, void *o, float *lse, int32_t *dev_status,
                                  void *stream) {
  const size_t need = fa_decode_workspace_size(B, Hq, Hkv, Lmax, D);
  if (need == 0) return FA_ERR_INVALID_ARG;            // bad shape (same checks as decode)
  if (need > kNoAllocScratchBytes) return FA_ERR_UNSUPPORTED;  // beyond the static scratch
  void *scratch = scratch_on_current_device();
  if (!scratch) return FA_ERR_CUDA;
  return fa_attn_decode(q, kcache, vcache, seqlens, B, Lmax, Hq, Hkv, D, scale, mode, mode_dev,
                        cfg, o, lse, scratch, kNoAllocScratchBytes, dev_status, stream);
}

}  // extern "C"
