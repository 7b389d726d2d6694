// fa_api.cu -- the extern "C" entry points declared in include/fa_hybrid.h:
// argument checks, TMA descriptor setup and kernel launches.  No allocation,
// no synchronisation, no state beyond one-time driver entry-point lookup.
#include "fa_common.cuh"
#include "fa_internal.h"

#include <nvtx3/nvToolsExt.h>

#include <atomic>
#include <mutex>

namespace fa {

// An NVTX range named after the entry point around each call that enqueues
// work, so a timeline (nsys, ncu's range filter) shows which library call
// launched which kernels.  Without a tool attached it costs a no-op call.
struct NvtxRange {
  explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange &) = delete;
  NvtxRange &operator=(const NvtxRange &) = delete;
};

static std::atomic<unsigned long long> g_kernel_launches{0};
void note_launch() { g_kernel_launches.fetch_add(1, std::memory_order_relaxed); }

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// 4-D TMA map over a bf16 tensor [B, S, H, 128] with boxes of box_cols x 1 x
// box_rows x 1.
int tmap_bhsd(CUtensorMap *map, const void *base, int B, int S, int H, int box_cols, int box_rows,
              CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return -1;
  const cuuint64_t dims[4] = {128, static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(S),
                              static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {128 * 2, static_cast<cuuint64_t>(H) * 256,
                                 static_cast<cuuint64_t>(S) * H * 256};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(box_cols), 1,
                             static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -1;
}

}  // namespace

int make_tmap_bhsd(CUtensorMap *map, const void *base, int B, int S, int H, int box_cols,
                   int box_rows) {
  return tmap_bhsd(map, base, B, S, H, box_cols, box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
}

int make_tmap_bhsd_plain(CUtensorMap *map, const void *base, int B, int S, int H, int box_cols,
                         int box_rows) {
  return tmap_bhsd(map, base, B, S, H, box_cols, box_rows, CU_TENSOR_MAP_SWIZZLE_NONE);
}


int make_tmap_bhsd_u8(CUtensorMap *map, const void *base, int B, int S, int H, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return -1;
  const cuuint64_t dims[4] = {128, static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(S),
                              static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {128, static_cast<cuuint64_t>(H) * 128,
                                 static_cast<cuuint64_t>(S) * H * 128};
  const cuuint32_t box[4] = {128, 1, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void *>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -1;
}

int make_tmap_rows_f32(CUtensorMap *map, void *base, long long rows, int box_cols,
                       int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return -1;
  const cuuint64_t dims[2] = {128, static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {128 * 4};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? 0 : -1;
}

namespace {

constexpr int kHeadDim = 128;

int check_heads(int Hq, int Hkv, int D) {
  if (Hq <= 0 || Hkv <= 0 || D <= 0) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (D != kHeadDim) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

int check_cfg(fa_sparse_cfg c) {
  if (c.block != 64) return c.block <= 0 ? FA_ERR_INVALID_ARG : FA_ERR_UNSUPPORTED;
  if (c.sink < 0 || c.window < c.block) return FA_ERR_INVALID_ARG;
  if (c.sink % c.block || c.window % c.block) return FA_ERR_INVALID_ARG;
  return FA_OK;
}

int check_prefill(const void *q, const void *k, const void *v, void *o, int B, int S, int Hq,
                  int Hkv, int D) {
  if (!q || !k || !v || !o) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return FA_ERR_INVALID_ARG;
  if (B <= 0 || S <= 0) return FA_ERR_INVALID_ARG;
  if (int rc = check_heads(Hq, Hkv, D)) return rc;
  // TMA global dims and the flattened grid must fit.
  if (static_cast<long long>(S) * Hq * kHeadDim * 2 > (1ll << 40)) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

int check_router(const void *q, int B, int S, int Hq, int D, int n_head, int n_tail,
                 const float *w1, int hidden, const float *w2) {
  if (!q || !w1 || !w2) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(w1)) return FA_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || n_head < 0 || n_tail < 0 || n_head + n_tail < 1)
    return FA_ERR_INVALID_ARG;
  if (S < n_head + n_tail) return FA_ERR_UNSUPPORTED;
  if (D != kHeadDim) return FA_ERR_UNSUPPORTED;
  if (hidden < 1 || hidden > 65536) return FA_ERR_INVALID_ARG;
  if (static_cast<long long>(Hq) * kHeadDim * 4 > 200 * 1024) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

}  // namespace

int check_decode_args(const void *q, const void *kcache, const void *vcache,
                      const int32_t *seqlens, int B, int Lmax, int Hq, int Hkv, int D,
                      float scale, int mode, fa_sparse_cfg cfg, const void *o) {
  if (!q || !kcache || !vcache || !seqlens || !o) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(kcache) || !aligned16(vcache) || !aligned16(o))
    return FA_ERR_INVALID_ARG;
  if (B <= 0 || Lmax <= 0) return FA_ERR_INVALID_ARG;
  if (int rc = check_heads(Hq, Hkv, D)) return rc;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return FA_ERR_UNSUPPORTED;
  if (mode != FA_MODE_FULL && mode != FA_MODE_SPARSE) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f)) return FA_ERR_INVALID_ARG;
  return check_cfg(cfg);
}

}  // namespace fa

using namespace fa;

extern "C" {

FA_API const char *fa_status_string(int status) {
  switch (status) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG: invalid argument";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED: shape or option not supported";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE: workspace missing or too small";
    case FA_ERR_CUDA: return "FA_ERR_CUDA: CUDA launch or driver call failed";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT: wait timed out";
    default: return "unknown fa_status";
  }
}

FA_API int fa_version(void) { return 100; }

FA_API unsigned long long fa_kernel_launches(void) {
  return g_kernel_launches.load(std::memory_order_relaxed);
}

FA_API int fa_debug_set_wait_limit_ns(unsigned long long ns) {
  // 0: testing mode -- no TMA loads are issued and waits give up after 1 ms.
  const int skip = ns == 0 ? 1 : 0;
  const uint64_t bound = ns == 0 ? 1000000ull : ns;
  if (set_wait_limit_prefill(bound, skip) != 0 || set_wait_limit_decode(bound, skip) != 0 ||
      set_wait_limit_backward(bound, skip) != 0)
    return FA_ERR_CUDA;
  return FA_OK;
}

FA_API size_t fa_router_workspace_size(int B, int Hq, int D, int hidden) {
  if (B <= 0 || Hq <= 0 || D <= 0 || hidden <= 0) return 0;
  return router_workspace_bytes(B, Hq, D, hidden);
}

FA_API int fa_router_decide(const void *q, int B, int S, int Hq, int D, int n_head_tok, int n_tail_tok,
                     const float *w1, const float *b1, int hidden, const float *w2,
                     const float *b2, float *logits_out, int32_t *mode_out, void *workspace,
                     size_t ws_bytes, void *stream) {
  NvtxRange range_("fa_router_decide");
  if (int rc = check_router(q, B, S, Hq, D, n_head_tok, n_tail_tok, w1, hidden, w2)) return rc;
  if (!logits_out && !mode_out) return FA_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < router_workspace_bytes(B, Hq, D, hidden)) return FA_ERR_WORKSPACE;
  RouterLaunch a{q, B, S, Hq, n_head_tok, n_tail_tok, w1, b1, w2, b2, hidden, logits_out,
                 mode_out, workspace};
  return launch_router(a, static_cast<cudaStream_t>(stream));
}

FA_API int fa_blocksparse_index_size(int S, fa_sparse_cfg cfg, int *n_rows, int *nnz) {
  if (S <= 0 || !n_rows || !nnz) return FA_ERR_INVALID_ARG;
  if (int rc = check_cfg(cfg)) return rc;
  const int rows = (S + cfg.block - 1) / cfg.block;
  const long long n = index_nnz(rows, cfg.sink / cfg.block, cfg.window / cfg.block);
  if (n > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  *n_rows = rows;
  *nnz = static_cast<int>(n);
  return FA_OK;
}

FA_API int fa_blocksparse_index(int S, fa_sparse_cfg cfg, int32_t *row_ptr, int32_t *col_idx,
                         void *stream) {
  NvtxRange range_("fa_blocksparse_index");
  int rows = 0, nnz = 0;
  if (int rc = fa_blocksparse_index_size(S, cfg, &rows, &nnz)) return rc;
  if (!row_ptr || !col_idx) return FA_ERR_INVALID_ARG;
  return launch_index(rows, cfg.sink / cfg.block, cfg.window / cfg.block, row_ptr, col_idx,
                      static_cast<cudaStream_t>(stream));
}

FA_API int fa_attn_prefill_full(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                         int S, int Hq, int Hkv, int D, float scale, int32_t *dev_status,
                         void *stream) {
  NvtxRange range_("fa_attn_prefill_full");
  if (int rc = check_prefill(q, k, v, o, B, S, Hq, Hkv, D)) return rc;
  if (!(scale > 0.f)) return FA_ERR_INVALID_ARG;
  PrefillLaunch a{q, k, v, o, lse, B, S, Hq, Hkv, scale, nullptr, nullptr, nullptr,
                  FA_MODE_FULL, dev_status};
  return launch_prefill(a, static_cast<cudaStream_t>(stream));
}

FA_API int fa_attn_prefill_blocksparse(const void *q, const void *k, const void *v, void *o, float *lse,
                                int B, int S, int Hq, int Hkv, int D, float scale,
                                const int32_t *row_ptr, const int32_t *col_idx, int block,
                                int32_t *dev_status, void *stream) {
  NvtxRange range_("fa_attn_prefill_blocksparse");
  if (int rc = check_prefill(q, k, v, o, B, S, Hq, Hkv, D)) return rc;
  if (!(scale > 0.f)) return FA_ERR_INVALID_ARG;
  if (!row_ptr || !col_idx) return FA_ERR_INVALID_ARG;
  if (block != 64) return block <= 0 ? FA_ERR_INVALID_ARG : FA_ERR_UNSUPPORTED;
  PrefillLaunch a{q, k, v, o, lse, B, S, Hq, Hkv, scale, row_ptr, col_idx, nullptr,
                  FA_MODE_SPARSE, dev_status};
  return launch_prefill(a, static_cast<cudaStream_t>(stream));
}

FA_API size_t fa_decode_workspace_size(int B, int Hq, int Hkv, int Lmax, int D) {
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Lmax <= 0 || D != kHeadDim || Hq % Hkv) return 0;
  return decode_workspace_bytes(B, Hq, Hkv, Lmax);
}

FA_API int fa_attn_decode(const void *q, const void *kcache, const void *vcache, const int32_t *seqlens,
                   int B, int Lmax, int Hq, int Hkv, int D, float scale, int mode,
                   const int32_t *mode_dev, fa_sparse_cfg cfg, void *o, float *lse,
                   void *workspace, size_t ws_bytes, int32_t *dev_status, void *stream) {
  NvtxRange range_("fa_attn_decode");
  if (int rc = check_decode_args(q, kcache, vcache, seqlens, B, Lmax, Hq, Hkv, D, scale, mode,
                                 cfg, o))
    return rc;
  if (!workspace || !aligned16(workspace) || ws_bytes < decode_workspace_bytes(B, Hq, Hkv, Lmax))
    return FA_ERR_WORKSPACE;
  DecodeLaunch a{q, kcache, vcache, seqlens, B, Lmax, Hq, Hkv, scale, mode, mode_dev,
                 cfg.sink, cfg.window, o, lse, workspace, dev_status};
  return launch_decode(a, static_cast<cudaStream_t>(stream));
}

FA_API int fa_kv_append_paged(const void *k_new, const void *v_new, void *k_pages,
                              void *v_pages, int kv_dtype, const float *k_scale,
                              const float *v_scale, const int32_t *block_table, int max_pages,
                              int num_pages, int32_t *seqlens, int B, int Hkv, int D,
                              int32_t *dev_status, void *stream) {
  NvtxRange range_("fa_kv_append_paged");
  if (!k_new || !v_new || !k_pages || !v_pages || !block_table || !seqlens)
    return FA_ERR_INVALID_ARG;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_pages) || !aligned16(v_pages))
    return FA_ERR_INVALID_ARG;
  if (B <= 0 || Hkv <= 0 || max_pages <= 0 || num_pages <= 0) return FA_ERR_INVALID_ARG;
  if (D != kHeadDim) return FA_ERR_UNSUPPORTED;
  if (kv_dtype != FA_KV_BF16 && kv_dtype != FA_KV_FP8_E4M3) return FA_ERR_INVALID_ARG;
  if (kv_dtype == FA_KV_FP8_E4M3 && (!k_scale || !v_scale)) return FA_ERR_INVALID_ARG;
  KvAppendLaunch a{k_new, v_new, k_pages, v_pages, kv_dtype == FA_KV_FP8_E4M3 ? 1 : 0,
                   k_scale, v_scale, block_table, max_pages, num_pages, seqlens, B, Hkv,
                   dev_status};
  return launch_kv_append(a, static_cast<cudaStream_t>(stream));
}

FA_API size_t fa_decode_paged_workspace_size(int B, int Hq, int Hkv, int max_pages, int D) {
  if (max_pages <= 0 || max_pages > (1 << 24)) return 0;
  return fa_decode_workspace_size(B, Hq, Hkv, 64 * max_pages, D);
}

FA_API int fa_attn_decode_paged(const void *q, const void *k_pages, const void *v_pages,
                                int kv_dtype, const float *k_scale, const float *v_scale,
                                const int32_t *block_table, int max_pages, int num_pages,
                                const int32_t *seqlens, int B, int Hq, int Hkv, int D,
                                float scale, int mode, const int32_t *mode_dev,
                                fa_sparse_cfg cfg, void *o, float *lse, void *workspace,
                                size_t ws_bytes, int32_t *dev_status, void *stream) {
  NvtxRange range_("fa_attn_decode_paged");
  if (!q || !k_pages || !v_pages || !block_table || !seqlens || !o) return FA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_pages) || !aligned16(v_pages) || !aligned16(o))
    return FA_ERR_INVALID_ARG;
  if (B <= 0 || max_pages <= 0 || num_pages <= 0 || max_pages > (1 << 24))
    return FA_ERR_INVALID_ARG;
  if (int rc = check_heads(Hq, Hkv, D)) return rc;
  const int G = Hq / Hkv;
  if (G != 1 && G != 2 && G != 4 && G != 8) return FA_ERR_UNSUPPORTED;
  if (mode != FA_MODE_FULL && mode != FA_MODE_SPARSE) return FA_ERR_INVALID_ARG;
  if (kv_dtype != FA_KV_BF16 && kv_dtype != FA_KV_FP8_E4M3) return FA_ERR_INVALID_ARG;
  if (kv_dtype == FA_KV_FP8_E4M3 && (!k_scale || !v_scale)) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f)) return FA_ERR_INVALID_ARG;
  if (int rc = check_cfg(cfg)) return rc;
  const int Lmax = 64 * max_pages;
  if (!workspace || !aligned16(workspace) || ws_bytes < decode_workspace_bytes(B, Hq, Hkv, Lmax))
    return FA_ERR_WORKSPACE;
  DecodeLaunch a{q, k_pages, v_pages, seqlens, B, Lmax, Hq, Hkv, scale, mode, mode_dev,
                 cfg.sink, cfg.window, o, lse, workspace, dev_status};
  a.block_table = block_table;
  a.max_pages = max_pages;
  a.num_pages = num_pages;
  a.fp8 = kv_dtype == FA_KV_FP8_E4M3 ? 1 : 0;
  a.k_scale = k_scale;
  a.v_scale = v_scale;
  return launch_decode(a, static_cast<cudaStream_t>(stream));
}

FA_API size_t fa_hybrid_workspace_size(int B, int Hq, int D, int hidden) {
  return fa_router_workspace_size(B, Hq, D, hidden);
}

FA_API int fa_hybrid_layer(const void *q, const void *k, const void *v, void *o, float *lse, int B,
                    int S, int Hq, int Hkv, int D, float scale, const float *w1, const float *b1,
                    int hidden, const float *w2, const float *b2, fa_sparse_cfg cfg,
                    const int32_t *row_ptr, const int32_t *col_idx, float *logits_out,
                    int32_t *mode_out, void *workspace, size_t ws_bytes, int32_t *dev_status,
                    void *stream) {
  NvtxRange range_("fa_hybrid_layer");
  if (int rc = check_prefill(q, k, v, o, B, S, Hq, Hkv, D)) return rc;
  if (int rc = check_router(q, B, S, Hq, D, 100, 100, w1, hidden, w2)) return rc;
  if (int rc = check_cfg(cfg)) return rc;
  if (!(scale > 0.f)) return FA_ERR_INVALID_ARG;
  if (!row_ptr || !col_idx || !mode_out) return FA_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < router_workspace_bytes(B, Hq, D, hidden)) return FA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  RouterLaunch r{q, B, S, Hq, 100, 100, w1, b1, w2, b2, hidden, logits_out, mode_out, workspace};
  if (int rc = launch_router(r, st)) return rc;
  PrefillLaunch a{q, k, v, o, lse, B, S, Hq, Hkv, scale, row_ptr, col_idx, mode_out,
                  FA_MODE_FULL, dev_status};
  a.expect_nnz = index_nnz((S + cfg.block - 1) / cfg.block, cfg.sink / cfg.block,
                           cfg.window / cfg.block);
  return launch_prefill(a, st);
}

FA_API int fa_router_soft(const float *logits, const float *gumbel, int B, float tau,
                          float *r_out, void *stream) {
  NvtxRange range_("fa_router_soft");
  if (!logits || !r_out || B <= 0) return FA_ERR_INVALID_ARG;
  if (!(tau > 0.f)) return FA_ERR_INVALID_ARG;
  return launch_router_soft(logits, gumbel, B, tau, r_out, static_cast<cudaStream_t>(stream));
}

FA_API int fa_soft_routed_layer(const void *q, const void *k, const void *v, void *o, int B, int S,
                                int Hq, int Hkv, int D, float scale, const float *w1,
                                const float *b1, int hidden, const float *w2, const float *b2,
                                const float *gumbel, float tau, fa_sparse_cfg cfg,
                                const int32_t *row_ptr, const int32_t *col_idx, float *logits_out,
                                float *r_out, void *workspace, size_t ws_bytes,
                                int32_t *dev_status, void *stream) {
  NvtxRange range_("fa_soft_routed_layer");
  if (int rc = check_prefill(q, k, v, o, B, S, Hq, Hkv, D)) return rc;
  if (int rc = check_router(q, B, S, Hq, D, 100, 100, w1, hidden, w2)) return rc;
  if (int rc = check_cfg(cfg)) return rc;
  if (!(scale > 0.f) || !(tau > 0.f)) return FA_ERR_INVALID_ARG;
  if (!row_ptr || !col_idx || !logits_out || !r_out) return FA_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < router_workspace_bytes(B, Hq, D, hidden)) return FA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  RouterLaunch r{q, B, S, Hq, 100, 100, w1, b1, w2, b2, hidden, logits_out, nullptr, workspace};
  if (int rc = launch_router(r, st)) return rc;
  if (int rc = launch_router_soft(logits_out, gumbel, B, tau, r_out, st)) return rc;
  PrefillLaunch full{q, k, v, o, nullptr, B, S, Hq, Hkv, scale, nullptr, nullptr, nullptr,
                     FA_MODE_FULL, dev_status};
  if (int rc = launch_prefill(full, st)) return rc;
  PrefillLaunch sparse{q, k, v, o, nullptr, B, S, Hq, Hkv, scale, row_ptr, col_idx, nullptr,
                       FA_MODE_SPARSE, dev_status};
  sparse.mix_r = r_out;
  sparse.expect_nnz = index_nnz((S + cfg.block - 1) / cfg.block, cfg.sink / cfg.block,
                                cfg.window / cfg.block);
  return launch_prefill(sparse, st);
}

FA_API int fa_soft_mix(const void *o_full, const void *o_sparse, const float *r, void *y, int B,
                       int S, int Hq, int D, void *stream) {
  NvtxRange range_("fa_soft_mix");
  if (!o_full || !o_sparse || !r || !y || B <= 0 || S <= 0 || Hq <= 0) return FA_ERR_INVALID_ARG;
  if (!aligned16(o_full) || !aligned16(o_sparse) || !aligned16(y)) return FA_ERR_INVALID_ARG;
  if (D != kHeadDim) return FA_ERR_UNSUPPORTED;
  return launch_soft_mix(o_full, o_sparse, r, y, B, static_cast<long long>(S) * Hq * D,
                         static_cast<cudaStream_t>(stream));
}

FA_API size_t fa_attn_backward_workspace_size(int B, int S, int Hq, int Hkv, int D) {
  if (B <= 0 || S <= 0 || check_heads(Hq, Hkv, D) != FA_OK) return 0;
  return backward_workspace_bytes(B, S, Hq, Hkv);
}

FA_API int fa_attn_prefill_backward(const void *q, const void *k, const void *v, const void *o,
                                    const float *lse, const void *dout, void *dq, void *dk,
                                    void *dv, int B, int S, int Hq, int Hkv, int D, float scale,
                                    const int32_t *row_ptr, const int32_t *col_idx,
                                    const int32_t *mode_dev, int mode, void *workspace,
                                    size_t ws_bytes, int32_t *dev_status, void *stream) {
  NvtxRange range_("fa_attn_prefill_backward");
  if (int rc = check_prefill(q, k, v, const_cast<void *>(o), B, S, Hq, Hkv, D)) return rc;
  if (!lse || !dout || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  if (!aligned16(dout) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv))
    return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f)) return FA_ERR_INVALID_ARG;
  if (mode != FA_MODE_FULL && mode != FA_MODE_SPARSE) return FA_ERR_INVALID_ARG;
  if (mode == FA_MODE_SPARSE && (!row_ptr || !col_idx)) return FA_ERR_INVALID_ARG;
  if ((row_ptr == nullptr) != (col_idx == nullptr)) return FA_ERR_INVALID_ARG;
  if (!workspace || !aligned16(workspace) || ws_bytes < backward_workspace_bytes(B, S, Hq, Hkv))
    return FA_ERR_WORKSPACE;
  BackwardLaunch a{q, k, v, o, dout, lse, dq, dk, dv, B, S, Hq, Hkv, scale, row_ptr, col_idx,
                   mode_dev, mode, dev_status, workspace};
  return launch_backward(a, static_cast<cudaStream_t>(stream));
}

FA_API size_t fa_soft_routed_backward_workspace_size(int B, int S, int Hq, int Hkv, int D,
                                                     int hidden) {
  if (B <= 0 || S <= 0 || hidden <= 0 || check_heads(Hq, Hkv, D) != FA_OK) return 0;
  return soft_backward_workspace_bytes(B, S, Hq, Hkv, hidden);
}

FA_API int fa_soft_routed_layer_backward(
    const void *q, const void *k, const void *v, const void *o_full, const float *lse_full,
    const void *o_sparse, const float *lse_sparse, const void *dy, int B, int S, int Hq, int Hkv,
    int D, float scale, const float *w1, const float *b1, int hidden, const float *w2,
    const float *b2, const float *gumbel, float tau, const int32_t *row_ptr,
    const int32_t *col_idx, void *dq, void *dk, void *dv, float *dw1, float *db1, float *dw2,
    float *db2, float *r_out, void *workspace, size_t ws_bytes, int32_t *dev_status,
    void *stream) {
  NvtxRange range_("fa_soft_routed_layer_backward");
  if (int rc = check_prefill(q, k, v, const_cast<void *>(o_full), B, S, Hq, Hkv, D)) return rc;
  if (int rc = check_router(q, B, S, Hq, D, 100, 100, w1, hidden, w2)) return rc;
  if (!o_sparse || !lse_full || !lse_sparse || !dy || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  if (!aligned16(o_sparse) || !aligned16(dy) || !aligned16(dq) || !aligned16(dk) ||
      !aligned16(dv))
    return FA_ERR_INVALID_ARG;
  if (!dw1 || !db1 || !dw2 || !db2 || !row_ptr || !col_idx) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !(tau > 0.f)) return FA_ERR_INVALID_ARG;
  if (!workspace || !aligned16(workspace) ||
      ws_bytes < soft_backward_workspace_bytes(B, S, Hq, Hkv, hidden))
    return FA_ERR_WORKSPACE;
  SoftBackwardLaunch a{q, k, v, o_full, o_sparse, dy, lse_full, lse_sparse, B, S, Hq, Hkv, scale,
                       w1, b1, w2, b2, hidden, gumbel, tau, row_ptr, col_idx, dq, dk, dv, dw1,
                       db1, dw2, db2, r_out, workspace, dev_status};
  return launch_soft_backward(a, static_cast<cudaStream_t>(stream));
}

FA_API size_t fa_varlen_workspace_size(int B, int total_tokens) {
  if (B <= 0 || total_tokens <= 0) return 0;
  return varlen_workspace_bytes(B, total_tokens);
}

namespace {
int check_varlen(const void *q, const void *k, const void *v, void *o, const int32_t *cu,
                 int B, int total, int max_seqlen, int Hq, int Hkv, int D) {
  if (!cu) return FA_ERR_INVALID_ARG;
  if (int rc = check_prefill(q, k, v, o, 1, total, Hq, Hkv, D)) return rc;
  if (B <= 0 || B > 4096 || max_seqlen <= 0 || max_seqlen > total) return FA_ERR_INVALID_ARG;
  if ((Hq / Hkv) % 2 != 0) return FA_ERR_UNSUPPORTED;   // the two-tile kernel only
  return FA_OK;
}
}  // namespace

FA_API int fa_attn_prefill_varlen(const void *q, const void *k, const void *v, void *o, float *lse,
                                  const int32_t *cu_seqlens, int B, int total_tokens,
                                  int max_seqlen, int Hq, int Hkv, int D, float scale,
                                  const int32_t *row_ptr, const int32_t *col_idx,
                                  const int32_t *mode_dev, int mode, void *workspace,
                                  size_t ws_bytes, int32_t *dev_status, void *stream) {
  NvtxRange range_("fa_attn_prefill_varlen");
  if (int rc = check_varlen(q, k, v, o, cu_seqlens, B, total_tokens, max_seqlen, Hq, Hkv, D))
    return rc;
  if (!(scale > 0.f)) return FA_ERR_INVALID_ARG;
  if (mode != FA_MODE_FULL && mode != FA_MODE_SPARSE) return FA_ERR_INVALID_ARG;
  const bool any_sparse = mode_dev != nullptr || mode == FA_MODE_SPARSE;
  if (any_sparse && (!row_ptr || !col_idx)) return FA_ERR_INVALID_ARG;
  if (!workspace || ws_bytes < varlen_workspace_bytes(B, total_tokens)) return FA_ERR_WORKSPACE;
  PrefillLaunch a{q, k, v, o, lse, B, max_seqlen, Hq, Hkv, scale, any_sparse ? row_ptr : nullptr,
                  any_sparse ? col_idx : nullptr, mode_dev, mode, dev_status};
  a.cu_seqlens = cu_seqlens;
  a.total_tokens = total_tokens;
  a.varlen_ws = workspace;
  return launch_prefill(a, static_cast<cudaStream_t>(stream));
}

FA_API size_t fa_hybrid_varlen_workspace_size(int B, int total_tokens, int Hq, int D,
                                              int hidden) {
  const size_t r = fa_router_workspace_size(B, Hq, D, hidden);
  const size_t v = fa_varlen_workspace_size(B, total_tokens);
  if (!r || !v) return 0;
  return ((r + 255) & ~static_cast<size_t>(255)) + v;
}

FA_API int fa_hybrid_layer_varlen(const void *q, const void *k, const void *v, void *o,
                                  float *lse, const int32_t *cu_seqlens, int B, int total_tokens,
                                  int max_seqlen, int Hq, int Hkv, int D, float scale,
                                  const float *w1, const float *b1, int hidden, const float *w2,
                                  const float *b2, fa_sparse_cfg cfg, const int32_t *row_ptr,
                                  const int32_t *col_idx, float *logits_out, int32_t *mode_out,
                                  void *workspace, size_t ws_bytes, int32_t *dev_status,
                                  void *stream) {
  NvtxRange range_("fa_hybrid_layer_varlen");
  if (int rc = check_varlen(q, k, v, o, cu_seqlens, B, total_tokens, max_seqlen, Hq, Hkv, D))
    return rc;
  if (int rc = check_router(q, B, max_seqlen, Hq, D, 100, 100, w1, hidden, w2)) return rc;
  if (int rc = check_cfg(cfg)) return rc;
  if (!(scale > 0.f)) return FA_ERR_INVALID_ARG;
  if (!row_ptr || !col_idx || !mode_out) return FA_ERR_INVALID_ARG;
  const size_t rws = router_workspace_bytes(B, Hq, D, hidden);
  const size_t need = ((rws + 255) & ~static_cast<size_t>(255)) + varlen_workspace_bytes(B, total_tokens);
  if (!workspace || ws_bytes < need) return FA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  RouterLaunch r{q, B, max_seqlen, Hq, 100, 100, w1, b1, w2, b2, hidden, logits_out, mode_out,
                 workspace};
  r.cu_seqlens = cu_seqlens;
  if (int rc = launch_router(r, st)) return rc;
  PrefillLaunch a{q, k, v, o, lse, B, max_seqlen, Hq, Hkv, scale, row_ptr, col_idx, mode_out,
                  FA_MODE_FULL, dev_status};
  a.cu_seqlens = cu_seqlens;
  a.total_tokens = total_tokens;
  a.varlen_ws = static_cast<uint8_t *>(workspace) + ((rws + 255) & ~static_cast<size_t>(255));
  a.expect_nnz = index_nnz((max_seqlen + cfg.block - 1) / cfg.block, cfg.sink / cfg.block,
                           cfg.window / cfg.block);
  return launch_prefill(a, st);
}

}  // extern "C"
