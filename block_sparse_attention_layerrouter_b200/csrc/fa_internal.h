// fa_internal.h -- launch descriptors shared by the C-ABI layer and the
// kernel files.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/fa_hybrid.h"

namespace fa {

// 4-D TMA map over a bf16 tensor [B, S, H, 128] (row-major), boxes of
// box_cols x 1 x box_rows x 1 with the 128-byte swizzle.  Returns 0 on success.
int make_tmap_bhsd(CUtensorMap *map, const void *base, int B, int S, int H, int box_cols,
                   int box_rows);
// The same without swizzle (a box is stored row-major in shared memory).
int make_tmap_bhsd_plain(CUtensorMap *map, const void *base, int B, int S, int H, int box_cols,
                         int box_rows);

// 2-D TMA map over an fp32 tensor [rows, 128] (row-major), boxes of
// box_cols x box_rows, no swizzle.  Returns 0 on success.
int make_tmap_rows_f32(CUtensorMap *map, void *base, long long rows, int box_cols, int box_rows);

struct PrefillLaunch {
  const void *q, *k, *v;
  void *o;
  float *lse;
  int B, S, Hq, Hkv;
  float scale;
  const int32_t *row_ptr, *col_idx;  // nullptr: FULL only
  const int32_t *mode_dev;           // nullptr: use mode_default
  int mode_default;
  int32_t *status;
  const float *mix_r = nullptr;      // soft-routing mix weight per batch, or nullptr
  // Packed variable-length batch: S is then the longest sequence, q/k/v/o
  // are [total_tokens, H, D], and `varlen_ws` holds the work-item list.
  const int32_t *cu_seqlens = nullptr;
  int total_tokens = 0;
  void *varlen_ws = nullptr;
  // Entry count the CSR must have (the block rule's count for S and the
  // sparse config), checked on the device; -1: not checked.
  long long expect_nnz = -1;
};
size_t varlen_workspace_bytes(int B, int total_tokens);
int launch_prefill(const PrefillLaunch &a, cudaStream_t stream);

struct DecodeLaunch {
  const void *q, *kcache, *vcache;
  const int32_t *seqlens;
  int B, Lmax, Hq, Hkv;
  float scale;
  int mode;
  const int32_t *mode_dev;
  int sink, window;  // tokens, multiples of 64
  void *o;
  float *lse;
  void *workspace;
  int32_t *status;
  // Paged cache: pool [num_pages, 64, Hkv, D]; Lmax = 64 * max_pages.
  const int32_t *block_table = nullptr;
  int max_pages = 0, num_pages = 0;
  // FP8 (E4M3) cache with per-KV-head dequantisation scales.
  int fp8 = 0;
  const float *k_scale = nullptr, *v_scale = nullptr;
};
struct KvAppendLaunch {
  const void *k_new, *v_new;        // bf16 [B, Hkv, D]
  void *k_pages, *v_pages;
  int fp8;
  const float *k_scale, *v_scale;
  const int32_t *block_table;
  int max_pages, num_pages;
  int32_t *seqlens;                 // in: positions to write; out: + 1
  int B, Hkv;
  int32_t *status;
};
int launch_kv_append(const KvAppendLaunch &a, cudaStream_t stream);
// 4-D TMA map over a byte tensor [B, S, H, 128] (an FP8 cache), boxes of
// 128 x 1 x box_rows x 1 with the 128-byte swizzle.
int make_tmap_bhsd_u8(CUtensorMap *map, const void *base, int B, int S, int H, int box_rows);
// Host-side argument checks of fa_attn_decode (everything but the
// workspace); FA_OK or an fa_status.
int check_decode_args(const void *q, const void *kcache, const void *vcache,
                      const int32_t *seqlens, int B, int Lmax, int Hq, int Hkv, int D,
                      float scale, int mode, fa_sparse_cfg cfg, const void *o);
int decode_num_splits(int B, int Hkv, int Lmax);
int decode_splits_for_tiles(int B, int Hkv, int tiles);
size_t decode_workspace_bytes(int B, int Hq, int Hkv, int Lmax);
int launch_decode(const DecodeLaunch &a, cudaStream_t stream);

struct RouterLaunch {
  const void *q;
  int B, S, Hq, n_head, n_tail;
  const float *w1, *b1, *w2, *b2;
  int hidden;
  float *logits;
  int32_t *mode;
  void *workspace;
  const int32_t *cu_seqlens = nullptr;  // packed sequences (S unused), or nullptr
};
size_t router_workspace_bytes(int B, int Hq, int D, int hidden);
int launch_router_soft(const float *logits, const float *gumbel, int B, float tau, float *r,
                       cudaStream_t stream);
int launch_router(const RouterLaunch &a, cudaStream_t stream);

struct BackwardLaunch {
  const void *q, *k, *v, *o, *dout;
  const float *lse;                  // [B, Hq, S] natural-log LSE of the forward
  void *dq, *dk, *dv;
  int B, S, Hq, Hkv;
  float scale;
  const int32_t *row_ptr, *col_idx;  // nullptr: FULL only
  const int32_t *mode_dev;           // per batch, or nullptr (mode_default)
  int mode_default;
  int32_t *status;
  void *workspace;
  // Soft routing: outputs scaled per batch by gscale[b] (or 1 - gscale[b]);
  // dK/dV added into the existing outputs; dQ accumulated across calls.
  const float *gscale = nullptr;
  int gscale_complement = 0;
  int accumulate_kv = 0;
  int zero_dq_acc = 1;
  int convert_dq = 1;
  const float *pool_dx = nullptr;    // [B, Hq*D] router pooling gradient, or nullptr
  int n_head = 0, n_tail = 0;
};
size_t backward_workspace_bytes(int B, int S, int Hq, int Hkv);
int launch_backward(const BackwardLaunch &a, cudaStream_t stream);

// Router backward (soft routing): gradients of W1, b1, W2, b2 and of the
// pooled input x, from dr = dL/dr per sequence.  `router_ws` holds a router
// forward of the same inputs (pooling slices and ReLU outputs).
struct RouterBwdLaunch {
  const float *logits, *gumbel;
  float tau;
  const float *dr;
  void *router_ws;
  const float *w1, *w2;
  int B, Hq, hidden, n_sel;
  float *x, *dlogits, *da, *dx;        // workspace: [B, Hq*D], [B, 2], [B, hidden], [B, Hq*D]
  float *dw1, *db1, *dw2, *db2;        // outputs
};
void router_ws_parts(void *workspace, int B, int Hq, float **part, float **hid);
int launch_soft_mix(const void *o_full, const void *o_sparse, const float *r, void *y, int B,
                    long long per_b, cudaStream_t stream);
int launch_router_backward(const RouterBwdLaunch &a, cudaStream_t stream);

// Soft-routed layer backward: both attention paths (upstream r dy and
// (1 - r) dy), the router, and the pooling term of dQ.
struct SoftBackwardLaunch {
  const void *q, *k, *v, *o_full, *o_sparse, *dy;
  const float *lse_full, *lse_sparse;
  int B, S, Hq, Hkv;
  float scale;
  const float *w1, *b1, *w2, *b2;
  int hidden;
  const float *gumbel;
  float tau;
  const int32_t *row_ptr, *col_idx;
  void *dq, *dk, *dv;
  float *dw1, *db1, *dw2, *db2;
  float *r_out;                        // nullable
  void *workspace;
  int32_t *status;
};
size_t soft_backward_workspace_bytes(int B, int S, int Hq, int Hkv, int hidden);
int launch_soft_backward(const SoftBackwardLaunch &a, cudaStream_t stream);

// Counts one kernel launch (the total is fa_kernel_launches()).
void note_launch();

// Bound of the kernels' waits (ns) and the testing flag that makes the
// load-issuing roles issue nothing, in each kernel file's constant memory, on
// the current device; 0 on success.
int set_wait_limit_prefill(uint64_t ns, int skip_loads);
int set_wait_limit_decode(uint64_t ns, int skip_loads);
int set_wait_limit_backward(uint64_t ns, int skip_loads);

long long index_nnz(int nrows, int sb, int wb);
int launch_index(int nrows, int sb, int wb, int32_t *row_ptr, int32_t *col_idx,
                 cudaStream_t stream);

}  // namespace fa
