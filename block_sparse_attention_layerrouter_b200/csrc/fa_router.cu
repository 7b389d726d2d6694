// fa_router.cu -- the layer router ("Flux Attention", router paragraphs):
// mean-pool the first n_head and last n_tail query tokens per (head, dim),
// flatten head-major, context encoder h = ReLU(W1 x + b1), router head
// [pi_FA, pi_SA] = W2 h + b2, hard routing by argmax (a tie routes to FULL).
//
// Three small launches, all memory/latency bound:
//   pool_kernel   grid (Hq, B, 5 token slices): fp32 partial sums per slice
//   hidden_kernel grid (H1, B): sums the slices into x (shared memory), then
//                 one W1 row per CTA with coalesced float4 reads -> h [B, H1]
//   head_kernel   grid (B): one warp per logit, then the argmax -> mode [B]
#include "fa_common.cuh"
#include "fa_internal.h"

namespace fa {
namespace router {

constexpr int HD = 128;
constexpr int kPoolSlices = 5;     // token slices per (head, batch)

// Partial sums of the selected tokens: slice z of (head h, batch b) adds
// up its share of the n_head + n_tail selected tokens for all 128 dims.
__global__ void __launch_bounds__(256) pool_kernel(const __nv_bfloat16 *q, float *part, int S,
                                                   int Hq, int n_head, int n_tail,
                                                   const int32_t *cu) {
  __shared__ float red[16][HD];
  const int h = blockIdx.x, b = blockIdx.y, z = blockIdx.z, B = gridDim.y;
  const int chunk = threadIdx.x & 15, grp = threadIdx.x >> 4;
  const int n_sel = n_head + n_tail;
  const int per = (n_sel + kPoolSlices - 1) / kPoolSlices;
  const int i0 = z * per, i1 = min(n_sel, i0 + per);
  // Sequence b: rows row0 .. row0 + len - 1 (packed batch: from cu_seqlens).
  const size_t row0 = cu ? static_cast<size_t>(cu[b]) : static_cast<size_t>(b) * S;
  const int len = cu ? cu[b + 1] - cu[b] : S;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
  for (int i = i0 + grp; i < i1; i += 16) {
    const int t = i < n_head ? i : len - n_tail + (i - n_head);
    if (t < 0 || t >= len) continue;       // a sequence shorter than n_head + n_tail
    const uint4 v = *reinterpret_cast<const uint4 *>(
        q + ((row0 + t) * Hq + h) * HD + chunk * 8);
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
    part[(static_cast<size_t>(z) * B + b) * Hq * HD + h * HD + threadIdx.x] = s;
  }
}

// One CTA per (hidden unit, batch): x = (sum of the slices) / n_sel into
// shared memory (head-major x[h*D + d]), then ReLU(W1[u] . x + b1[u]).
__global__ void __launch_bounds__(256) hidden_kernel(const float *part, const float *w1,
                                                     const float *b1, float *hid, int in_f,
                                                     int hidden, float inv_n) {
  extern __shared__ float xs[];
  __shared__ float red[8];
  const int u = blockIdx.x, b = blockIdx.y, B = gridDim.y, tid = threadIdx.x;
  for (int i = tid; i < in_f; i += 256) {
    float v = 0.f;
#pragma unroll
    for (int z = 0; z < kPoolSlices; ++z) v += part[(static_cast<size_t>(z) * B + b) * in_f + i];
    xs[i] = v * inv_n;
  }
  __syncthreads();
  const float *wr = w1 + static_cast<size_t>(u) * in_f;
  float s = 0.f;
  if ((in_f & 3) == 0) {
#pragma unroll 4
    for (int i = tid * 4; i < in_f; i += 1024) {
      const float4 wv = *reinterpret_cast<const float4 *>(wr + i);
      s = fmaf(wv.x, xs[i], s);
      s = fmaf(wv.y, xs[i + 1], s);
      s = fmaf(wv.z, xs[i + 2], s);
      s = fmaf(wv.w, xs[i + 3], s);
    }
  } else {
    for (int i = tid; i < in_f; i += 256) s = fmaf(wr[i], xs[i], s);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if ((tid & 31) == 0) red[tid >> 5] = s;
  __syncthreads();
  if (tid == 0) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) t += red[w];
    const float v = t + (b1 ? b1[u] : 0.f);
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

// Soft routing (training-time relaxation): r = exp((pi_FA + g_FA)/tau) /
// sum_i exp((pi_i + g_i)/tau) = 1 / (1 + exp(((pi_SA + g_SA) - (pi_FA + g_FA))/tau)).
__global__ void soft_kernel(const float *logits, const float *gumbel, float inv_tau, float *r,
                            int B) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= B) return;
  float zf = logits[2 * b], zs = logits[2 * b + 1];
  if (gumbel) {
    zf += gumbel[2 * b];
    zs += gumbel[2 * b + 1];
  }
  r[b] = 1.0f / (1.0f + expf((zs - zf) * inv_tau));
}

// ---------------------------------------------------------------- backward
// Chain rule through the soft-routed layer, for an upstream dr = dL/dr per
// sequence (r the weight of the FULL output):
//   dz_FA = dr r (1 - r) / tau = -dz_SA          (r = sigmoid((z_FA - z_SA)/tau))
//   dW2 = dz^T h, db2 = sum_b dz, da = (dz W2) * [h > 0], db1 = sum_b da,
//   dW1 = da^T x, dx = da W1
// (h = ReLU(a) > 0 exactly where a > 0; ReLU'(0) = 0).

// x[b, i] = (sum of the pooling slices) / n_sel, materialised for dW1.
__global__ void __launch_bounds__(256) pooled_kernel(const float *part, float *x, int B, int in_f,
                                                     float inv_n) {
  const long long n = static_cast<long long>(B) * in_f;
  for (long long i = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * 256) {
    float v = 0.f;
#pragma unroll
    for (int z = 0; z < kPoolSlices; ++z) v += part[z * n + i];
    x[i] = v * inv_n;
  }
}

// One CTA per hidden unit u: dz per sequence (recomputed from logits, noise
// and dr), dW2[:, u], da[:, u], db1[u]; unit 0 also writes db2 and dz.
__global__ void __launch_bounds__(128) head_bwd_kernel(const float *logits, const float *gumbel,
                                                       float inv_tau, const float *dr,
                                                       const float *hid, const float *w2, int B,
                                                       int hidden, float *dlogits, float *da,
                                                       float *dw2, float *db1, float *db2) {
  const int u = blockIdx.x;
  float g2a = 0.f, g2b = 0.f, g1 = 0.f;
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    float zf = logits[2 * b], zs = logits[2 * b + 1];
    if (gumbel) {
      zf += gumbel[2 * b];
      zs += gumbel[2 * b + 1];
    }
    const float r = 1.0f / (1.0f + expf((zs - zf) * inv_tau));
    const float dzf = dr[b] * r * (1.0f - r) * inv_tau;
    const float h = hid[static_cast<size_t>(b) * hidden + u];
    g2a += dzf * h;                  // dW2[0, u] (pi_FA row)
    g2b -= dzf * h;                  // dW2[1, u] (pi_SA row): dz_SA = -dz_FA
    const float dh = dzf * (w2[u] - w2[hidden + u]);
    const float a = h > 0.f ? dh : 0.f;
    da[static_cast<size_t>(b) * hidden + u] = a;
    g1 += a;
    if (u == 0) {
      dlogits[2 * b] = dzf;
      dlogits[2 * b + 1] = -dzf;
    }
  }
  __shared__ float red[3][4];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    g2a += __shfl_xor_sync(0xffffffffu, g2a, off);
    g2b += __shfl_xor_sync(0xffffffffu, g2b, off);
    g1 += __shfl_xor_sync(0xffffffffu, g1, off);
  }
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {
    red[0][w] = g2a;
    red[1][w] = g2b;
    red[2][w] = g1;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float s0 = 0.f, s1 = 0.f, s2 = 0.f;
    for (int i = 0; i < 4; ++i) {
      s0 += red[0][i];
      s1 += red[1][i];
      s2 += red[2][i];
    }
    dw2[u] = s0;
    dw2[hidden + u] = s1;
    db1[u] = s2;
  }
  if (u == 0 && threadIdx.x == 0 && db2) {
    float s = 0.f;
    for (int b = 0; b < B; ++b) {
      float zf = logits[2 * b], zs = logits[2 * b + 1];
      if (gumbel) {
        zf += gumbel[2 * b];
        zs += gumbel[2 * b + 1];
      }
      const float r = 1.0f / (1.0f + expf((zs - zf) * inv_tau));
      s += dr[b] * r * (1.0f - r) * inv_tau;
    }
    db2[0] = s;
    db2[1] = -s;
  }
}

// dW1[u, i] = sum_b da[b, u] x[b, i]: one CTA per row u of W1.
__global__ void __launch_bounds__(256) dw1_kernel(const float *da, const float *x, int B, int in_f,
                                                  int hidden, float *dw1) {
  const int u = blockIdx.x;
  for (int i = threadIdx.x; i < in_f; i += 256) {
    float s = 0.f;
    for (int b = 0; b < B; ++b)
      s = fmaf(da[static_cast<size_t>(b) * hidden + u], x[static_cast<size_t>(b) * in_f + i], s);
    dw1[static_cast<size_t>(u) * in_f + i] = s;
  }
}

// dx[b, i] = sum_u da[b, u] W1[u, i]: a CTA covers 32 columns i; its 8 warps
// take every 8th hidden unit (each warp reads 128 contiguous bytes of a W1
// row) and the partial sums meet in shared memory.
__global__ void __launch_bounds__(256) dx_kernel(const float *da, const float *w1, int B, int in_f,
                                                 int hidden, float *dx) {
  __shared__ float part[8][32];
  const int lane = threadIdx.x & 31, ug = threadIdx.x >> 5;
  const int i = blockIdx.x * 32 + lane, b = blockIdx.y;
  const float *dab = da + static_cast<size_t>(b) * hidden;
  float s = 0.f;
  if (i < in_f)
    for (int u = ug; u < hidden; u += 8) s = fmaf(dab[u], w1[static_cast<size_t>(u) * in_f + i], s);
  part[ug][lane] = s;
  __syncthreads();
  if (ug == 0 && i < in_f) {
    float t = 0.f;
#pragma unroll
    for (int g = 0; g < 8; ++g) t += part[g][lane];
    dx[static_cast<size_t>(b) * in_f + i] = t;
  }
}

// y = r O_FA + (1 - r) O_SA per sequence (bf16 rows of 8 elements per thread;
// the products in fp32, rounded once).
__global__ void __launch_bounds__(256) mix_kernel(const __nv_bfloat16 *of, const __nv_bfloat16 *os,
                                                  const float *r, __nv_bfloat16 *y,
                                                  long long per_b, int B) {
  const long long n8 = per_b * B / 8;
  for (long long i = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x; i < n8;
       i += static_cast<long long>(gridDim.x) * 256) {
    const float rb = r[(i * 8) / per_b];
    const uint4 a = reinterpret_cast<const uint4 *>(of)[i];
    const uint4 b = reinterpret_cast<const uint4 *>(os)[i];
    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float lo = rb * __uint_as_float(wa[k] << 16) + (1.0f - rb) * __uint_as_float(wb[k] << 16);
      const float hi = rb * __uint_as_float(wa[k] & 0xffff0000u) +
                       (1.0f - rb) * __uint_as_float(wb[k] & 0xffff0000u);
      w[k] = pack_bf16x2(lo, hi);
    }
    reinterpret_cast<uint4 *>(y)[i] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

}  // namespace router

int launch_soft_mix(const void *o_full, const void *o_sparse, const float *r, void *y, int B,
                    long long per_b, cudaStream_t stream) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return FA_ERR_CUDA;
  const long long n8 = per_b * B / 8;
  const long long blocks = (n8 + 255) / 256;
  router::mix_kernel<<<static_cast<unsigned>(blocks < 4 * sms ? blocks : 4 * sms), 256, 0,
                       stream>>>(reinterpret_cast<const __nv_bfloat16 *>(o_full),
                                 reinterpret_cast<const __nv_bfloat16 *>(o_sparse), r,
                                 reinterpret_cast<__nv_bfloat16 *>(y), per_b, B);
  note_launch();
  return cudaPeekAtLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

void router_ws_parts(void *workspace, int B, int Hq, float **part, float **hid) {
  const size_t pbytes = static_cast<size_t>(router::kPoolSlices) * B * Hq * router::HD * sizeof(float);
  *part = reinterpret_cast<float *>(workspace);
  *hid = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(workspace) +
                                   ((pbytes + 255) & ~static_cast<size_t>(255)));
}

int launch_router_backward(const RouterBwdLaunch &a, cudaStream_t stream) {
  using namespace router;
  const int in_f = a.Hq * HD;
  float *part = nullptr, *hid = nullptr;
  router_ws_parts(a.router_ws, a.B, a.Hq, &part, &hid);
  const long long n = static_cast<long long>(a.B) * in_f;
  pooled_kernel<<<static_cast<unsigned>((n + 255) / 256 < 1184 ? (n + 255) / 256 : 1184), 256, 0,
                  stream>>>(part, a.x, a.B, in_f, 1.0f / static_cast<float>(a.n_sel));
  note_launch();
  if (cudaPeekAtLastError() != cudaSuccess) return FA_ERR_CUDA;
  head_bwd_kernel<<<a.hidden, 128, 0, stream>>>(a.logits, a.gumbel, 1.0f / a.tau, a.dr, hid, a.w2,
                                                a.B, a.hidden, a.dlogits, a.da, a.dw2, a.db1,
                                                a.db2);
  note_launch();
  if (cudaPeekAtLastError() != cudaSuccess) return FA_ERR_CUDA;
  dw1_kernel<<<a.hidden, 256, 0, stream>>>(a.da, a.x, a.B, in_f, a.hidden, a.dw1);
  note_launch();
  if (cudaPeekAtLastError() != cudaSuccess) return FA_ERR_CUDA;
  dx_kernel<<<dim3((in_f + 31) / 32, a.B), 256, 0, stream>>>(a.da, a.w1, a.B, in_f, a.hidden,
                                                              a.dx);
  note_launch();
  return cudaPeekAtLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int launch_router_soft(const float *logits, const float *gumbel, int B, float tau, float *r,
                       cudaStream_t stream) {
  router::soft_kernel<<<(B + 127) / 128, 128, 0, stream>>>(logits, gumbel, 1.0f / tau, r, B);
  note_launch();
  return cudaPeekAtLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

size_t router_workspace_bytes(int B, int Hq, int D, int hidden) {
  const size_t x = static_cast<size_t>(router::kPoolSlices) * B * Hq * D * sizeof(float);
  const size_t h = static_cast<size_t>(B) * hidden * sizeof(float);
  return ((x + 255) & ~static_cast<size_t>(255)) + ((h + 255) & ~static_cast<size_t>(255));
}

int launch_router(const RouterLaunch &a, cudaStream_t stream) {
  using namespace router;
  const int in_f = a.Hq * HD;
  const size_t pbytes = static_cast<size_t>(kPoolSlices) * a.B * in_f * sizeof(float);
  float *part = reinterpret_cast<float *>(a.workspace);
  float *hid = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(a.workspace) +
                                         ((pbytes + 255) & ~static_cast<size_t>(255)));
  const size_t xs_bytes = static_cast<size_t>(in_f) * sizeof(float);
  if (xs_bytes > 48 * 1024 &&
      cudaFuncSetAttribute(hidden_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(xs_bytes)) != cudaSuccess)
    return FA_ERR_CUDA;
  pool_kernel<<<dim3(a.Hq, a.B, kPoolSlices), 256, 0, stream>>>(
      reinterpret_cast<const __nv_bfloat16 *>(a.q), part, a.S, a.Hq, a.n_head, a.n_tail,
      a.cu_seqlens);
  note_launch();
  if (cudaPeekAtLastError() != cudaSuccess) return FA_ERR_CUDA;
  hidden_kernel<<<dim3(a.hidden, a.B), 256, xs_bytes, stream>>>(
      part, a.w1, a.b1, hid, in_f, a.hidden, 1.0f / static_cast<float>(a.n_head + a.n_tail));
  note_launch();
  if (cudaPeekAtLastError() != cudaSuccess) return FA_ERR_CUDA;
  head_kernel<<<a.B, 64, 0, stream>>>(hid, a.w2, a.b2, a.logits, a.mode, a.hidden);
  note_launch();
  return cudaPeekAtLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace fa
