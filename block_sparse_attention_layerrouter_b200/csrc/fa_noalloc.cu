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
// with cudaGetSymbolAddress and caches it together with the id of the CUDA
// context it belongs to; a later call in another context of that device
// (after cudaDeviceReset, say) looks it up again.  Make the first call on a
// device before any stream capture.
//
// Contents: every split of the decode writes its partial result (reference
// max, sum, output) before the combine kernel reads it; a split whose bounded
// wait ran out writes a NaN marker instead, and the combine then writes NaN
// for those heads.  So nothing in the scratch has to start at zero, and no
// output is ever built from what an earlier call left there.  All calls share
// the one array: calls whose kernels overlap on the GPU (other streams, or
// other host threads) race on it and must be serialised by the caller.
#include "fa_common.cuh"
#include "fa_internal.h"

#include <nvtx3/nvToolsExt.h>

#include <mutex>

namespace fa {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

struct DriverFns {
  CtxGetCurrentFn get_current = nullptr;
  CtxGetIdFn get_id = nullptr;
};

const DriverFns &driver_fns() {
  static DriverFns fns;
  static std::once_flag once;
  std::call_once(once, [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fns.get_current = reinterpret_cast<CtxGetCurrentFn>(ptr);
    ptr = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fns.get_id = reinterpret_cast<CtxGetIdFn>(ptr);
  });
  return fns;
}

// Id of the current CUDA context, or 0 if there is none yet (or the driver
// cannot say).
unsigned long long current_context_id() {
  const DriverFns &f = driver_fns();
  if (!f.get_current || !f.get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (f.get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (f.get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

std::mutex g_scratch_mu;
void *g_scratch_ptr[kMaxDevices] = {nullptr};
unsigned long long g_scratch_ctx[kMaxDevices] = {0};

// Device address of g_decode_scratch on the current device, looked up once
// per device and context.  Returns nullptr on failure.
void *scratch_on_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_ptr[dev] == nullptr || ctx == 0 || ctx != g_scratch_ctx[dev]) {
    void *ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess || ptr == nullptr)
      return nullptr;
    g_scratch_ptr[dev] = ptr;
    g_scratch_ctx[dev] = current_context_id();   // the lookup made the context current
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
  nvtxRangePushA("fa_attn_decode_noalloc");
  int rc = check_decode_args(q, kcache, vcache, seqlens, B, Lmax, Hq, Hkv, D, scale, mode, cfg,
                             o);
  if (rc == FA_OK && decode_workspace_bytes(B, Hq, Hkv, Lmax) > kNoAllocScratchBytes)
    rc = FA_ERR_UNSUPPORTED;                          // beyond the static scratch
  if (rc == FA_OK) {
    void *scratch = scratch_on_current_device();
    rc = scratch ? fa_attn_decode(q, kcache, vcache, seqlens, B, Lmax, Hq, Hkv, D, scale, mode,
                                  mode_dev, cfg, o, lse, scratch, kNoAllocScratchBytes,
                                  dev_status, stream)
                 : FA_ERR_CUDA;
  }
  nvtxRangePop();
  return rc;
}

}  // extern "C"
