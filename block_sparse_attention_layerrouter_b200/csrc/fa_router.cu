// fa_router.cu -- the layer router ("Flux Attention", router paragraphs):
// mean-pool the first n_head and last n_tail query tokens per (head, dim),
// flatten head-major, context encoder h = ReLU(W1 x + b1), router head
// [pi_FA, pi_SA] = W2 h + b2, hard routing by argmax (a tie routes to FULL).
//
// Three small launches, all memory/latency bound:
//   pool_kernel   grid (Hq, B): 16 token groups x 16 chunks of 8 dims, fp32
//                 sums reduced in shared memory -> x [B, Hq*D]
//   hidden_kernel grid (ceil(H1/8), B): one warp per hidden unit, coalesced
//                 float4 reads of the W1 row -> h [B, H1]
//   head_kernel   grid (B): one warp per logit, then the argmax -> mode [B]
#include "fa_common.cuh"
#include "fa_internal.h"

namespace fa {
namespace router {

constexpr int HD = 128;

__global__ void __launch_bounds__(256) pool_kernel(const __nv_bfloat16 *q, float *x, int S, int Hq,
                                                   int n_head, int n_tail) {
  __shared__ float red[16][HD];
  const int h = blockIdx.x, b = blockIdx.y;
  const int chunk = threadIdx.x & 15, grp = threadIdx.x >> 4;
  const int n_sel = n_head + n_tail;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int i = grp; i < n_sel; i += 16) {
    const int t = i < n_head ? i : S - n_tail + (i - n_head);
    const uint4 v = *reinterpret_cast<const uint4 *>(
        q + ((static_cast<size_t>(b) * S + t) * Hq + h) * HD + chunk * 8);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      acc[2 * k] += __uint_as_float(w[k] << 16);
      acc[2 * k + 1] += __uint_as_float(w[k] & 0xffff0000u);
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[grp][chunk * 8 + e] = acc[e];
  __syncthreads();
  if (threadIdx.x < HD) {
    float s = 0.f;
#pragma unroll
    for (int g = 0; g < 16; ++g) s += red[g][threadIdx.x];
    x[static_cast<size_t>(b) * Hq * HD + h * HD + threadIdx.x] = s / static_cast<float>(n_sel);
  }
}

__global__ void __launch_bounds__(256) hidden_kernel(const float *x, const float *w1,
                                                     const float *b1, float *hid, int in_f,
                                                     int hidden) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u = blockIdx.x * 8 + warp, b = blockIdx.y;
  if (u >= hidden) return;
  const float *wr = w1 + static_cast<size_t>(u) * in_f;
  const float *xr = x + static_cast<size_t>(b) * in_f;
  float s = 0.f;
  if ((in_f & 3) == 0) {
    for (int i = lane * 4; i < in_f; i += 128) {
      const float4 wv = *reinterpret_cast<const float4 *>(wr + i);
      const float4 xv = *reinterpret_cast<const float4 *>(xr + i);
      s = fmaf(wv.x, xv.x, s);
      s = fmaf(wv.y, xv.y, s);
      s = fmaf(wv.z, xv.z, s);
      s = fmaf(wv.w, xv.w, s);
    }
  } else {
    for (int i = lane; i < in_f; i += 32) s = fmaf(wr[i], xr[i], s);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) {
    const float v = s + (b1 ? b1[u] : 0.f);
    hid[static_cast<size_t>(b) * hidden + u] = v > 0.f ? v : 0.f;
  }
}

__global__ void __launch_bounds__(64) head_kernel(const float *hid, const float *w2,
                                                  const float *b2, float *logits, int32_t *mode,
                                                  int hidden) {
  __shared__ float lg[2];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, b = blockIdx.x;
  const float *wr = w2 + static_cast<size_t>(warp) * hidden;
  const float *hr = hid + static_cast<size_t>(b) * hidden;
  float s = 0.f;
  for (int i = lane; i < hidden; i += 32) s = fmaf(wr[i], hr[i], s);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) {
    const float v = s + (b2 ? b2[warp] : 0.f);
    lg[warp] = v;
    if (logits) logits[2 * b + warp] = v;
  }
  __syncthreads();
  if (threadIdx.x == 0 && mode) mode[b] = (lg[1] > lg[0]) ? FA_MODE_SPARSE : FA_MODE_FULL;
}

}  // namespace router

size_t router_workspace_bytes(int B, int Hq, int D, int hidden) {
  const size_t x = static_cast<size_t>(B) * Hq * D * sizeof(float);
  const size_t h = static_cast<size_t>(B) * hidden * sizeof(float);
  return ((x + 255) & ~static_cast<size_t>(255)) + ((h + 255) & ~static_cast<size_t>(255));
}

int launch_router(const RouterLaunch &a, cudaStream_t stream) {
  using namespace router;
  const size_t xbytes = static_cast<size_t>(a.B) * a.Hq * HD * sizeof(float);
  float *x = reinterpret_cast<float *>(a.workspace);
  float *hid = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(a.workspace) +
                                         ((xbytes + 255) & ~static_cast<size_t>(255)));
  pool_kernel<<<dim3(a.Hq, a.B), 256, 0, stream>>>(reinterpret_cast<const __nv_bfloat16 *>(a.q),
                                                   x, a.S, a.Hq, a.n_head, a.n_tail);
  if (cudaPeekAtLastError() != cudaSuccess) return FA_ERR_CUDA;
  hidden_kernel<<<dim3((a.hidden + 7) / 8, a.B), 256, 0, stream>>>(x, a.w1, a.b1, hid,
                                                                   a.Hq * HD, a.hidden);
  if (cudaPeekAtLastError() != cudaSuccess) return FA_ERR_CUDA;
  head_kernel<<<a.B, 64, 0, stream>>>(hid, a.w2, a.b2, a.logits, a.mode, a.hidden);
  return cudaPeekAtLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace fa
