/*
 * fa_hybrid.h -- C ABI of the layer-routed hybrid attention library
 * (libfa_hybrid.so, hand-written CUDA kernels for B200 / sm_100a).
 *
 * The method ("Flux Attention: 효율적인 LLM 추론을 위한 문맥 인식형 하이브리드
 * 어텐션", router and implementation paragraphs): a layer router mean-pools the
 * first and last 100 query tokens of a layer, an MLP context encoder and a
 * router head give two logits pi_FA and pi_SA, the argmax picks the layer's
 * mode, and the layer then runs either exact causal attention or block-sparse
 * attention over 64-token blocks (sink blocks plus a local window).  A sparse
 * layer never loads the KV blocks outside its pattern.
 *
 * Conventions shared by every entry point:
 *  - Tensor pointers are DEVICE memory owned by the caller.  The library
 *    allocates nothing, keeps no state between calls and never synchronises.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream).  Every call only enqueues work on it.
 *  - The return value reports host-side argument checks and launch errors
 *    (fa_status).  On any non-zero return nothing was launched, except
 *    FA_ERR_CUDA, which reports a failed launch.
 *  - Device-side failures (a bounded wait that ran out, an index outside the
 *    query's causal range) are OR-ed into the caller's int32 `dev_status`
 *    (nullable) as FA_DEV_* bits; the caller zeroes it, synchronises, reads it.
 *  - bf16 tensors are row-major with these layouts:
 *      prefill Q, O [B, S, Hq, D];  K, V [B, S, Hkv, D];  LSE fp32 [B, Hq, S]
 *      decode  q, o [B, Hq, D];     K/V caches [B, Lmax, Hkv, D]
 *    Every pointer must be 16-byte aligned.  D must be 128.  Hq % Hkv == 0
 *    and the query head h reads KV head h / (Hq / Hkv).
 *  - Scores are scale * (q . k); the usual scale is 1/sqrt(D) ("Self-Attention
 *    이후", section "셀프 어텐션이 비싼 이유": Q K^T divided by sqrt(d_k)).
 */
#ifndef FA_HYBRID_H
#define FA_HYBRID_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FA_API __attribute__((visibility("default")))
#else
#define FA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = -1,   /* null pointer, bad size, misaligned pointer */
    FA_ERR_UNSUPPORTED = -2,   /* valid but not built: D != 128, G > 8, ... */
    FA_ERR_WORKSPACE = -3,     /* workspace missing or smaller than required */
    FA_ERR_CUDA = -4,          /* a CUDA launch or driver call failed */
    FA_ERR_TIMEOUT = -5        /* reserved for host-side waits (none today) */
} fa_status;

/* Bits OR-ed into *dev_status by the kernels. */
#define FA_DEV_TIMEOUT   1     /* a bounded wait ran out; outputs invalid */
#define FA_DEV_BAD_INDEX 2     /* a block index outside [0, query block] or
                                  out of order was skipped */
#define FA_DEV_DEBUG_BOUNDS 4  /* debug builds only (libfa_hybrid_debug.so):
                                  a store's index fell outside its tensor
                                  and the store was skipped */

typedef enum { FA_MODE_FULL = 0, FA_MODE_SPARSE = 1 } fa_mode;

/* KV cache element type of the paged decode path. */
typedef enum { FA_KV_BF16 = 0, FA_KV_FP8_E4M3 = 1 } fa_kv_dtype;

/* Sparse pattern, in tokens: block = 64 ("Flux Attention", implementation
 * paragraph: 64-token blocks), sink = 128 sink tokens, window = local window
 * counted in whole blocks and including the query's own block.  sink and
 * window must be multiples of block; window >= block. */
typedef struct {
    int32_t block;
    int32_t sink;
    int32_t window;
} fa_sparse_cfg;

/* Human-readable name of a fa_status value; never NULL. */
FA_API const char *fa_status_string(int status);

/* Library ABI version (major * 100 + minor). */
FA_API int fa_version(void);

/* Testing aid: sets the bound of every wait inside this library's kernels
 * (default 2e9 ns) on the current device.  Each wait in a kernel is bounded;
 * a wait that runs out makes the kernel give up (FA_DEV_TIMEOUT in
 * dev_status, the outputs of that call invalid; a decode head whose split
 * gave up reads NaN), let its copies and MMAs in flight finish and return,
 * leaving the device usable.  ns = 0 is the testing mode that makes this
 * happen on purpose: the kernels issue no TMA loads, so every wait on a load
 * runs out, after a bound of 1 ms.  Put the default back afterwards.
 * Synchronous (a copy to device constant memory): not during stream capture
 * or while this library's kernels run.  Returns FA_OK or FA_ERR_CUDA. */
FA_API int fa_debug_set_wait_limit_ns(unsigned long long ns);

/* Number of kernels this library has enqueued in this process so far, on
 * any stream and device (a host-side count taken at each launch; calls
 * rejected by their host-side checks launch nothing and add nothing).  For
 * callers that report how many kernels a step ran: read it before and after.
 * Thread-safe; never touches the GPU. */
FA_API unsigned long long fa_kernel_launches(void);

/* ------------------------------------------------------------ router ---
 * "Flux Attention", router paragraphs: pool tokens [0, n_head) and
 * [S - n_tail, S) of Q (mean, fp32), flatten head-major to x[h*D + d],
 * hidden = ReLU(W1 x + b1), [pi_FA, pi_SA] = W2 hidden + b2, and
 * mode = FA_MODE_SPARSE iff pi_SA > pi_FA (a tie routes to FULL).
 *   q        bf16 [B, S, Hq, D], device
 *   w1       fp32 [hidden, Hq*D], b1 fp32 [hidden], w2 fp32 [2, hidden],
 *            b2 fp32 [2]; device; b1/b2 may be NULL (zero bias)
 *   logits_out fp32 [B, 2] (pi_FA, pi_SA); mode_out int32 [B]; device
 *   workspace  >= fa_router_workspace_size(B, Hq, D, hidden) bytes, device
 * Requires S >= n_head + n_tail, n_head + n_tail >= 1, 1 <= hidden <= 65536. */
FA_API size_t fa_router_workspace_size(int B, int Hq, int D, int hidden);
FA_API int fa_router_decide(const void *q, int B, int S, int Hq, int D,
                     int n_head_tok, int n_tail_tok,
                     const float *w1, const float *b1, int hidden,
                     const float *w2, const float *b2,
                     float *logits_out, int32_t *mode_out,
                     void *workspace, size_t ws_bytes, void *stream);

/* ------------------------------------------------------------- index ---
 * CSR of the key blocks each query block keeps ("Flux Attention",
 * implementation paragraph): row i (query block i, nqb = ceil(S/block) rows)
 * lists, ascending, the sink blocks j < sink/block (j <= i) and the window
 * blocks i - window/block + 1 .. i, each once.
 * fa_blocksparse_index_size is host arithmetic only (no device access). */
FA_API int fa_blocksparse_index_size(int S, fa_sparse_cfg cfg, int *n_rows, int *nnz);
/*   row_ptr int32 [n_rows + 1], col_idx int32 [nnz]; device. */
FA_API int fa_blocksparse_index(int S, fa_sparse_cfg cfg, int32_t *row_ptr,
                         int32_t *col_idx, void *stream);

/* ----------------------------------------------------------- prefill ---
 * Exact causal attention, FlashAttention-style: tiles of QK^T on the tensor
 * cores, online softmax with a running max and sum rescaled by
 * exp(m_old - m_new) (newsletter on Softmax/FlashAttention, section on
 * Online Softmax), then PV; the S x S matrix never reaches memory.
 *   o   bf16 [B, S, Hq, D]; lse fp32 [B, Hq, S] or NULL (natural log of the
 *       softmax denominator of scale*q.k, -inf for a row with no key).
 *   Any S >= 1.  dev_status: see conventions. */
FA_API int fa_attn_prefill_full(const void *q, const void *k, const void *v, void *o,
                         float *lse, int B, int S, int Hq, int Hkv, int D,
                         float scale, int32_t *dev_status, void *stream);

/* Block-sparse attention: query block i attends only the key blocks of CSR
 * row i (row_ptr int32 [ceil(S/block) + 1], col_idx ascending per row, every
 * entry in [0, i]); causal masking inside the diagonal block.  KV blocks
 * outside the list are never loaded.  block must be 64.  An all-ones lower
 * triangle reproduces fa_attn_prefill_full. */
FA_API int fa_attn_prefill_blocksparse(const void *q, const void *k, const void *v,
                                void *o, float *lse, int B, int S, int Hq,
                                int Hkv, int D, float scale,
                                const int32_t *row_ptr, const int32_t *col_idx,
                                int block, int32_t *dev_status, void *stream);

/* ------------------------------------------------------------ decode ---
 * One query token per sequence at position L-1, L = seqlens[b] (device int32
 * [B], 1 <= L <= Lmax; the cache holds L tokens including the current one).
 * FULL attends keys 0..L-1; SPARSE attends the keys the prefill block rule
 * keeps for row L-1 and loads no other KV block ("Flux Attention": a sparse
 * layer bypasses the KV cache outside its pattern).
 *   mode_dev: NULL to use `mode` for every sequence, else device int32 [B]
 *   (e.g. the router's mode_out) read on the device.
 *   o bf16 [B, Hq, D]; lse fp32 [B, Hq] or NULL.
 *   workspace >= fa_decode_workspace_size(B, Hq, Hkv, Lmax, D) bytes, device.
 * Split-KV: each split keeps (reference max, sum, output) with sums relative
 * to its reference; the splits are merged by log-sum-exp, which is exact for
 * any reference at or below the split's true max. */
FA_API size_t fa_decode_workspace_size(int B, int Hq, int Hkv, int Lmax, int D);
FA_API int fa_attn_decode(const void *q, const void *kcache, const void *vcache,
                   const int32_t *seqlens, int B, int Lmax, int Hq, int Hkv,
                   int D, float scale, int mode, const int32_t *mode_dev,
                   fa_sparse_cfg cfg, void *o, float *lse, void *workspace,
                   size_t ws_bytes, int32_t *dev_status, void *stream);

/* ------------------------------------------------------------ backward ---
 * Gradients of the causal attention of fa_attn_prefill_full / _blocksparse
 * for an upstream gradient dO of the output: what training the router through
 * the soft-routing relaxation ("Flux Attention", router paragraphs) needs
 * from each attention path.  With P the masked softmax of scale * Q K^T:
 *   dV = P^T dO,  dS = P * (dO V^T - D),  D_t = dO_t . O_t,
 *   dQ = scale * dS K,  dK = scale * dS^T Q
 * (a KV head's dK/dV sum over the G query heads that read it).
 *   q, o, dout bf16 [B, S, Hq, D]; k, v bf16 [B, S, Hkv, D]; lse fp32
 *   [B, Hq, S] = the forward's LSE (natural log), all device, caller-owned.
 *   dq bf16 [B, S, Hq, D]; dk, dv bf16 [B, S, Hkv, D]: overwritten.
 *   mode: FA_MODE_FULL or FA_MODE_SPARSE for every batch element, or
 *   mode_dev (device int32 [B], e.g. the router's mode_out) when non-NULL;
 *   row_ptr/col_idx: the CSR of fa_blocksparse_index for S (required when
 *   any element may be SPARSE; rows ascending and causal, else the
 *   offending rows are reported as FA_DEV_BAD_INDEX).
 *   workspace >= fa_attn_backward_workspace_size(B, S, Hq, Hkv, D) bytes,
 *   16-byte aligned device memory: an fp32 dQ accumulator [B, S, Hq, D], the
 *   row terms D and the LSE in base 2, the transposed block pattern, fp32
 *   dK/dV partial sums of tiles cut into chunks, and the work-item counter
 *   (reset on the stream by each call, so calls that share one workspace
 *   must be ordered on one stream).
 * D must be 128.  Returns FA_OK or an fa_status; enqueues only. */
FA_API size_t fa_attn_backward_workspace_size(int B, int S, int Hq, int Hkv, int D);
FA_API int fa_attn_prefill_backward(const void *q, const void *k, const void *v,
                                    const void *o, const float *lse, const void *dout,
                                    void *dq, void *dk, void *dv, int B, int S, int Hq,
                                    int Hkv, int D, float scale, const int32_t *row_ptr,
                                    const int32_t *col_idx, const int32_t *mode_dev,
                                    int mode, void *workspace, size_t ws_bytes,
                                    int32_t *dev_status, void *stream);

/* Backward of the soft-routed layer y = r O_FA + (1 - r) O_SA (see
 * fa_soft_routed_layer), for an upstream dy bf16 [B, S, Hq, D]: the router's
 * weight gradients and the attention inputs' gradients through both paths,
 * the pooling included.  By the chain rule:
 *   dr_b = sum dy . (O_FA - O_SA),  dz_FA = -dz_SA = dr r (1 - r) / tau,
 *   dW2 = dz^T h, db2 = sum_b dz, da = (dz W2) * [h > 0] (h = ReLU(W1 x + b1)),
 *   dW1 = da^T x, db1 = sum_b da, dx = da W1,
 *   dQ = r dQ_FA(dy) + (1 - r) dQ_SA(dy) + dx / 200 on the first and last
 *   100 tokens (x is their mean), dK and dV = r d*_FA + (1 - r) d*_SA.
 *   o_full / lse_full, o_sparse / lse_sparse: the outputs and LSE of
 *   fa_attn_prefill_full and fa_attn_prefill_blocksparse on q, k, v.
 *   dq, dk, dv bf16 like q, k, v; dw1 [hidden, Hq*D], db1 [hidden], dw2 [2,
 *   hidden], db2 [2]: fp32, overwritten.  r_out fp32 [B] or NULL.
 *   row_ptr / col_idx: the CSR of the sparse path.  gumbel, tau as in
 *   fa_router_soft.  workspace >= fa_soft_routed_backward_workspace_size(...).
 * ReLU'(0) is taken as 0. */
FA_API size_t fa_soft_routed_backward_workspace_size(int B, int S, int Hq, int Hkv,
                                                     int D, int hidden);
FA_API int fa_soft_routed_layer_backward(
    const void *q, const void *k, const void *v, const void *o_full,
    const float *lse_full, const void *o_sparse, const float *lse_sparse,
    const void *dy, int B, int S, int Hq, int Hkv, int D, float scale,
    const float *w1, const float *b1, int hidden, const float *w2, const float *b2,
    const float *gumbel, float tau, const int32_t *row_ptr, const int32_t *col_idx,
    void *dq, void *dk, void *dv, float *dw1, float *db1, float *dw2, float *db2,
    float *r_out, void *workspace, size_t ws_bytes, int32_t *dev_status, void *stream);

/* ----------------------------------------------- paged / FP8 KV cache ---
 * Decode over a paged KV cache, and the append of the current token.  A page
 * holds 64 consecutive tokens of one sequence (one block of the sparse rule,
 * so a SPARSE layer reads only the pages of its sink and window blocks and
 * never loads any other page: "Flux Attention", KV-cache bypass paragraph).
 *   k_pages, v_pages: device pools [num_pages, 64, Hkv, D] of bf16
 *   (FA_KV_BF16) or E4M3 bytes (FA_KV_FP8_E4M3); token t of sequence b is
 *   slot t % 64 of page block_table[b * max_pages + t / 64].
 *   block_table: device int32 [B, max_pages]; page ids must lie in
 *   [0, num_pages) (an id outside is reported as FA_DEV_BAD_INDEX and its
 *   tokens read as zeros).  A contiguous cache [B, Lmax, Hkv, D] is the
 *   pool with num_pages = B * Lmax / 64 and block_table[b][i] = b * Lmax/64 + i.
 *   k_scale, v_scale: device fp32 [Hkv], FP8 only: stored code c of value x is
 *   RN_e4m3(fp32(x / scale)) (saturating at +-448); x is read back as
 *   e4m3(c) * scale.  Ignored (may be NULL) for bf16.
 * fa_kv_append_paged: writes k_new, v_new (bf16 [B, Hkv, D], device) at
 *   position seqlens[b] of every sequence, quantising for FP8, then sets
 *   seqlens[b] += 1 on the device (seqlens: device int32 [B], in/out).  A
 *   position past max_pages * 64 is reported (FA_DEV_BAD_INDEX) and skipped.
 * fa_attn_decode_paged: as fa_attn_decode (query at position L-1, L =
 *   seqlens[b] <= 64 * max_pages), reading the cache through the block table.
 *   workspace >= fa_decode_paged_workspace_size(B, Hq, Hkv, max_pages, D). */
FA_API int fa_kv_append_paged(const void *k_new, const void *v_new, void *k_pages,
                              void *v_pages, int kv_dtype, const float *k_scale,
                              const float *v_scale, const int32_t *block_table,
                              int max_pages, int num_pages, int32_t *seqlens, int B,
                              int Hkv, int D, int32_t *dev_status, void *stream);
FA_API size_t fa_decode_paged_workspace_size(int B, int Hq, int Hkv, int max_pages, int D);
FA_API int fa_attn_decode_paged(const void *q, const void *k_pages, const void *v_pages,
                                int kv_dtype, const float *k_scale, const float *v_scale,
                                const int32_t *block_table, int max_pages, int num_pages,
                                const int32_t *seqlens, int B, int Hq, int Hkv, int D,
                                float scale, int mode, const int32_t *mode_dev,
                                fa_sparse_cfg cfg, void *o, float *lse, void *workspace,
                                size_t ws_bytes, int32_t *dev_status, void *stream);

/* ------------------------------------------- variable-length batches ---
 * Serving form of the routed layer ("Flux Attention": the router decides per
 * request, before each layer's attention): B sequences of different lengths
 * packed along the token axis, sequence b = tokens [cu_seqlens[b],
 * cu_seqlens[b+1]).  One persistent launch covers every query tile of every
 * sequence, longest causal rows first, each sequence in its own mode.
 *   q, o bf16 [total_tokens, Hq, D]; k, v bf16 [total_tokens, Hkv, D];
 *   lse fp32 [Hq, total_tokens] or NULL; cu_seqlens int32 [B + 1], device,
 *   non-decreasing, cu_seqlens[0] = 0, cu_seqlens[B] = total_tokens;
 *   max_seqlen = the longest sequence (host).  Hq / Hkv must be even.
 *   Sparse sequences use one CSR built for max_seqlen (row i of the block
 *   rule does not depend on the length).
 * fa_attn_prefill_varlen: mode_dev (device int32 [B]) or, if NULL, `mode`
 *   for all; row_ptr/col_idx required unless every sequence is FULL.
 *   workspace >= fa_varlen_workspace_size(B, total_tokens) bytes.
 * fa_hybrid_layer_varlen: the router per sequence (its first and last 100
 *   tokens; every sequence needs >= 200 tokens), then the attention reading
 *   mode_out on the device.  workspace >=
 *   fa_hybrid_varlen_workspace_size(B, total_tokens, Hq, D, hidden). */
FA_API size_t fa_varlen_workspace_size(int B, int total_tokens);
FA_API int fa_attn_prefill_varlen(const void *q, const void *k, const void *v,
                                  void *o, float *lse,
                                  const int32_t *cu_seqlens, int B,
                                  int total_tokens, int max_seqlen, int Hq,
                                  int Hkv, int D, float scale,
                                  const int32_t *row_ptr,
                                  const int32_t *col_idx,
                                  const int32_t *mode_dev, int mode,
                                  void *workspace, size_t ws_bytes,
                                  int32_t *dev_status, void *stream);
FA_API size_t fa_hybrid_varlen_workspace_size(int B, int total_tokens, int Hq,
                                              int D, int hidden);
FA_API int fa_hybrid_layer_varlen(const void *q, const void *k, const void *v,
                                  void *o, float *lse,
                                  const int32_t *cu_seqlens, int B,
                                  int total_tokens, int max_seqlen, int Hq,
                                  int Hkv, int D, float scale, const float *w1,
                                  const float *b1, int hidden, const float *w2,
                                  const float *b2, fa_sparse_cfg cfg,
                                  const int32_t *row_ptr,
                                  const int32_t *col_idx, float *logits_out,
                                  int32_t *mode_out, void *workspace,
                                  size_t ws_bytes, int32_t *dev_status,
                                  void *stream);

/* ------------------------------------------------------ soft routing ---
 * "Flux Attention", router paragraph on training: the Gumbel-softmax
 * relaxation r = exp((pi_FA + g_FA)/tau) / sum_i exp((pi_i + g_i)/tau) and
 * the mixed output y = r * O_FA + (1 - r) * O_SA.  The Gumbel samples g are
 * an input (fp32 [B, 2], nullable = no noise); tau > 0.
 * fa_router_soft: logits fp32 [B, 2] (pi_FA, pi_SA) -> r_out fp32 [B].
 * fa_soft_routed_layer: router logits, r, one FULL launch writing O_FA into
 * o, then one SPARSE launch whose epilogue writes r*O_FA + (1-r)*O_SA over
 * it (O_FA is rounded to bf16 in between).  Forward only; no LSE.
 *   logits_out fp32 [B, 2], r_out fp32 [B]: device, required.
 *   workspace >= fa_router_workspace_size(B, Hq, D, hidden). */
/* fa_soft_mix: y = r * O_FA + (1 - r) * O_SA per sequence, for a training
 * forward that keeps both outputs (and their LSE) for the backward.
 * o_full, o_sparse, y: bf16 [B, S, Hq, D] (y may alias neither input); r fp32
 * [B]; all device.  Rounded to bf16 once. */
FA_API int fa_soft_mix(const void *o_full, const void *o_sparse, const float *r, void *y,
                       int B, int S, int Hq, int D, void *stream);
FA_API int fa_router_soft(const float *logits, const float *gumbel, int B,
                          float tau, float *r_out, void *stream);
FA_API int fa_soft_routed_layer(const void *q, const void *k, const void *v,
                                void *o, int B, int S, int Hq, int Hkv, int D,
                                float scale, const float *w1, const float *b1,
                                int hidden, const float *w2, const float *b2,
                                const float *gumbel, float tau,
                                fa_sparse_cfg cfg, const int32_t *row_ptr,
                                const int32_t *col_idx, float *logits_out,
                                float *r_out, void *workspace, size_t ws_bytes,
                                int32_t *dev_status, void *stream);

/* ------------------------------------------- decode without allocation ---
 * The pages have no counterpart to this entry point; it exists for callers
 * that cannot allocate device memory where they run decode (a plugin behind
 * a fixed operator interface with no workspace argument, an engine whose
 * memory is all reserved up front, a real-time loop where cudaMalloc is not
 * allowed).  Same arguments, checks and results as fa_attn_decode without
 * the workspace: the split-KV scratch lives in one static device array of
 * fa_noalloc_scratch_bytes() (8 MiB) that every GPU loading this library
 * holds until exit.  The call allocates nothing.
 *  - Arguments are checked as by fa_attn_decode first (same status codes);
 *    then FA_ERR_UNSUPPORTED when the shape needs more scratch than the array
 *    holds (fa_decode_workspace_size(B, Hq, Hkv, Lmax, D) > 8 MiB).
 *  - The first call on a device (with that device current) looks up the
 *    array's device address; it is cached with the CUDA context's id and
 *    looked up again in a new context (after a device reset).  Make the first
 *    call on a device before any stream capture.
 *  - All calls share the array.  Nothing in it needs to start at zero: every
 *    split overwrites its slot before the merge reads it (a split that gave
 *    up marks its slot, and those heads read NaN).  Calls whose kernels
 *    overlap on the GPU race on the array and must be serialised. */
FA_API size_t fa_noalloc_scratch_bytes(void);
FA_API int fa_attn_decode_noalloc(const void *q, const void *kcache,
                                  const void *vcache, const int32_t *seqlens,
                                  int B, int Lmax, int Hq, int Hkv, int D,
                                  float scale, int mode,
                                  const int32_t *mode_dev, fa_sparse_cfg cfg,
                                  void *o, float *lse, int32_t *dev_status,
                                  void *stream);

/* ------------------------------------------------------------ hybrid ---
 * One routed layer: fa_router_decide on this layer's Q, then one attention
 * launch that reads the mode from device memory per sequence (no host sync)
 * and runs exact causal attention (FULL) or block-sparse attention over the
 * caller's CSR (SPARSE; build it once with fa_blocksparse_index for this S and
 * cfg).  Arguments as for the calls above; n_head/n_tail are 100/100.
 * The CSR is read on the device only, so the host cannot compare it with
 * cfg: the kernel checks that row_ptr[0] = 0 and that row_ptr[last] is the
 * entry count of the block rule for (S, cfg), and reports a mismatch as
 * FA_DEV_BAD_INDEX (then attends the CSR as given; every entry is still
 * checked against the causal range).  A CSR with the right count but other
 * entries is attended as given.  The same holds for the varlen and
 * soft-routed layers (count for max_seqlen, resp. S).
 *   workspace >= fa_hybrid_workspace_size(B, Hq, D, hidden) bytes. */
FA_API size_t fa_hybrid_workspace_size(int B, int Hq, int D, int hidden);
FA_API int fa_hybrid_layer(const void *q, const void *k, const void *v, void *o,
                    float *lse, int B, int S, int Hq, int Hkv, int D,
                    float scale, const float *w1, const float *b1, int hidden,
                    const float *w2, const float *b2, fa_sparse_cfg cfg,
                    const int32_t *row_ptr, const int32_t *col_idx,
                    float *logits_out, int32_t *mode_out, void *workspace,
                    size_t ws_bytes, int32_t *dev_status, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* FA_HYBRID_H */
