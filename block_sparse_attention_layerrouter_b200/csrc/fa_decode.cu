// fa_decode.cu -- single-token decode attention over a bf16 or FP8 KV cache,
// sm_100a.
//
// o = softmax(scale * q K^T) V for the query at position L-1 of each sequence.
// FULL attends keys 0..L-1; SPARSE attends the sink blocks and the local
// window of the prefill block rule for row L-1 and never loads any other KV
// block ("Flux Attention": a sparse layer bypasses the KV cache outside its
// pattern).  Memory-bound: every byte of K and V it needs is read once.
//
// Grid (split, kv head, batch).  A CTA owns one KV head (all G query heads
// of its group share each K/V tile) and a contiguous share of the sequence's
// 64-key blocks.  Thread 0 streams them with 4-D TMA loads (128-byte swizzle;
// bf16: 2 boxes of 64 keys x 64 dims per K or V tile, one block per stage;
// FP8: 1 box of 64 keys x 128 dims, two blocks per stage) into a 3-stage
// ring; one block barrier per stage releases it.  The dot products run on the
// tensor cores (warp-level mma.sync: the query group is a handful of rows,
// far below the 64-row minimum of a tcgen05 product; the kernel stays bound
// by HBM and the MMAs only replace CUDA-core FMAs and conversions).  Each of
// the 8 warps takes its own keys of every stage:
//   S    = Q K^T     m16n8k16: A = the G query heads (rows G..15 zero), held
//                    in registers for the whole split; B = K rows by
//                    ldmatrix (FP8: codes widened to f16, one cvt per pair).
//   O^T += V^T P^T   bf16: m16n8k8, A = V by ldmatrix.trans; FP8: m16n8k16,
//                    A = byte-paired words of two keys, one cvt per pair.
//                    B = P, straight from the S accumulators (their lane
//                    layout is the B fragment's).
// Each warp keeps per head a reference max (log2 units) that moves only for
// a score more than kRefSlack above it (then it rescales its accumulators),
// the row sum of its rounded P and its O^T (128 dims x the heads); after the
// last tile the warps merge by log-sum-exp in shared memory and the CTA
// writes its partial (reference, sum, unnormalised output) per head; the
// combine kernel merges the splits.
//
// Paged cache: with a block table, tile n of sequence b is page
// block_table[b][n] of a pool [num_pages, 64, Hkv, 128] (one page = one
// 64-token block, so the sparse mode skips whole pages).  FP8 cache: E4M3
// codes with one dequantisation scale per KV head for K and for V; the
// products are in f16 (E4M3 codes are exact in f16; the query is scaled by a
// power of two per head so that its largest element lies in [2^14, 2^15)),
// the K scale and that power are folded into the score scale, the V scale
// into the partial outputs.
#include "fa_common.cuh"
#include "fa_internal.h"

#include <cuda_fp8.h>
#include <climits>
#include <math.h>

namespace fa {
namespace decode {

constexpr int KT = 64;                         // keys per tile = one block = one page
constexpr int HD = 128;
constexpr int BOX_BYTES = KT * 64 * 2;         // 64 keys x 64 dims bf16
constexpr int NT = 256;
constexpr int RING_BYTES = 3 * 4 * BOX_BYTES;  // 96 KB of K/V in flight per CTA
constexpr int MAX_STAGES = 6;
constexpr int PAGE_CACHE = 256;                // page ids of a CTA's tiles kept in smem

// Per KV type: blocks (pages) per iteration, bytes of one block of K or V,
// ring stages.  FP8 takes two blocks (128 keys) per iteration: half the
// bytes per key, so the per-iteration work (barriers, the softmax step) is
// spread over twice the keys.
template <bool FP8>
struct KvT {
  static constexpr int NB = FP8 ? 2 : 1;
  static constexpr int TK = NB * KT;                  // keys per iteration
  static constexpr int BLK = FP8 ? KT * HD : KT * HD * 2;
  static constexpr int KBYTES = NB * BLK;             // K (or V) of one iteration
  static constexpr int STAGE = 2 * KBYTES;
  static constexpr int NST = RING_BYTES / STAGE;
};

struct Params {
  const __nv_bfloat16 *q;
  float *o_part;    // [B, Hq, nsplit, HD]
  float *ml_part;   // [B, Hq, nsplit, 2] (reference max, sum relative to it), log2 units
  const int32_t *seqlens;
  const int32_t *mode;
  int32_t *status;
  int B, Lmax, Hq, Hkv, nsplit;
  int mode_default, sink_blocks, win_blocks;
  float scale_log2;
  const int32_t *block_table;   // [B, max_pages] or nullptr (contiguous cache)
  int max_pages, num_pages;
  const float *k_scale, *v_scale;   // [Hkv] (FP8 cache) or nullptr
};

// Tiles (64-key blocks) a sequence of length L attends, as a virtual list:
// positions [0, a) are blocks [0, a); positions [a, count) are blocks
// lo .. last.  FULL: a = last + 1, count = a.
struct TileList {
  int a, lo, count, L;
  FA_DEV void init(int L_, bool sparse, int sink_blocks, int win_blocks) {
    L = L_;
    const int last = (L - 1) / KT;
    if (!sparse) {
      a = last + 1;
      lo = a;
      count = a;
    } else {
      a = min(sink_blocks, last + 1);
      lo = max(a, last - win_blocks + 1);
      count = a + (last - lo + 1);
    }
  }
  FA_DEV int block(int pos) const { return pos < a ? pos : lo + (pos - a); }
};

// Byte offset of the 16-byte chunk holding dims [8*chunk16, 8*chunk16+8) of
// `key` inside one K or V tile written by TMA with the 128-byte swizzle.
FA_DEV uint32_t tile_offset(int key, int chunk16) {
  const int box = chunk16 >> 3;
  const int phys = (chunk16 & 7) ^ (key & 7);
  return static_cast<uint32_t>(box * BOX_BYTES + key * 128 + phys * 16);
}

// Byte offset of byte `byte` (0..127) of `key`'s row inside one FP8 block
// (one 128-byte row per key, 16-byte units swizzled like the bf16 boxes).
FA_DEV uint32_t fp8_offset(int key, int byte) {
  return static_cast<uint32_t>(key * 128 + (((byte >> 4) ^ (key & 7)) << 4) + (byte & 15));
}

// Page id of block `blk` of sequence b; an id outside the pool is reported
// and replaced by num_pages (a TMA load there reads zeros).
__device__ __noinline__ int page_of(const int32_t *block_table, int max_pages, int num_pages,
                                    int32_t *status, int b, int blk) {
  int pg = block_table[static_cast<size_t>(b) * max_pages + blk];
  if (pg < 0 || pg >= num_pages) {
    report(status, FA_DEV_BAD_INDEX);
    pg = num_pages;
  }
  return pg;
}

// A warp's reference moves only for a score more than this above it (log2
// units): p <= 2^8 stays inside the f16 range of the FP8 path's P.
constexpr float kRefSlack = 8.0f;

FA_DEV void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
FA_DEV void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
FA_DEV uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
// d += A B, m16n8k16, fp32 accumulators; A rows 8..15 (a1, a3) are zero.
template <bool F16>
FA_DEV void mma_k16_top(float (&d)[4], uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
  if constexpr (F16)
    asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
  else
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}
FA_DEV void mma_k16_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                        uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
FA_DEV void mma_k8_bf16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm("mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5}, {%6}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(b0));
}
// Four E4M3 codes (bytes 0..3 of x) -> two f16x2: lo = (byte 0, byte 1),
// hi = (byte 2, byte 3), the lower byte in the lower half.  Exact.
FA_DEV void e4m3x4_to_f16x2(uint32_t x, uint32_t &lo, uint32_t &hi) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, l;\n\tcvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(x));
}
FA_DEV uint32_t pack_f16x2(float lo, float hi) {
  const __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&v);
}

// Shared memory of one decode CTA (offsets from a 1024-byte aligned base):
// K/V ring (after the last tile: the warps' partials) | stage barriers |
// abort flag | page ids.
struct Lay {
  static constexpr int FULL = RING_BYTES;
  static constexpr int FLAGS = FULL + 8 * MAX_STAGES;
  static constexpr int PAGES = FLAGS + 16;
  static constexpr int BYTES = 1024 + PAGES + PAGE_CACHE * 4;
};

template <int G, bool FP8, bool PAGED>
__global__ void __launch_bounds__(NT, 2)
    decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const Params p) {
  static_assert(G >= 1 && G <= 8, "query heads per KV head");
  using T = KvT<FP8>;
  using Y = Lay;
  constexpr int NSTAGE = T::NST, STAGE_BYTES = T::STAGE, NB = T::NB;
  constexpr int NW = NT / 32;
  constexpr int KW = T::TK / NW;       // keys per warp per iteration: 8 (bf16), 16 (FP8)
  constexpr int NT8 = KW / 8;          // n8 score tiles per warp
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint8_t *stages = base;
  uint64_t *full = reinterpret_cast<uint64_t *>(base + Y::FULL);
  volatile int *abort = reinterpret_cast<volatile int *>(base + Y::FLAGS);
  int *page_sm = reinterpret_cast<int *>(base + Y::PAGES);

  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;   // mma fragment row / column pair
  const int L_raw = p.seqlens[b];
  const int L = max(1, min(L_raw, p.Lmax));   // out-of-range lengths are clamped
  if (L != L_raw && threadIdx.x == 0 && blockIdx.x == 0 && blockIdx.y == 0) report(p.status, FA_DEV_BAD_INDEX);
  const int mode = p.mode ? p.mode[b] : p.mode_default;
  TileList tl;
  tl.init(L, mode == FA_MODE_SPARSE, p.sink_blocks, p.win_blocks);
  const int per = ((tl.count + p.nsplit - 1) / p.nsplit + NB - 1) / NB * NB;
  const int pos0 = min(tl.count, split * per);
  const int pos1 = min(tl.count, pos0 + per);
  const int nblocks = pos1 - pos0;
  const int ntiles = (nblocks + NB - 1) / NB;      // iterations

  if (tid == 0) {
    for (int i = 0; i < NSTAGE; ++i) mbar_init(&full[i], 1);
    *abort = 0;
    fence_mbar_init();
  }
  if constexpr (PAGED) {
    for (int i = tid; i < nblocks && i < PAGE_CACHE; i += NT)
      page_sm[i] = page_of(p.block_table, p.max_pages, p.num_pages, p.status, b,
                           tl.block(pos0 + i));
  }
  __syncthreads();

  int issued = 0;
  auto issue = [&](int i) {
    const int st = i % NSTAGE;
    uint8_t *dst = stages + st * STAGE_BYTES;
    mbar_arrive_expect_tx(&full[st], STAGE_BYTES);
    if constexpr (FP8) {
#pragma unroll
      for (int h = 0; h < NB; ++h) {
        const int j = NB * i + h;
        int pg = p.num_pages;
        if (j < nblocks)
          pg = j < PAGE_CACHE ? page_sm[j]
                              : page_of(p.block_table, p.max_pages, p.num_pages, p.status, b,
                                        tl.block(pos0 + j));
        tma_load_4d(dst + h * T::BLK, &tmK, &full[st], 0, kvh, 0, pg);
        tma_load_4d(dst + T::KBYTES + h * T::BLK, &tmV, &full[st], 0, kvh, 0, pg);
      }
    } else {
      int tok = tl.block(pos0 + i) * KT, bidx = b;
      if constexpr (PAGED) {
        bidx = i < PAGE_CACHE ? page_sm[i]
                              : page_of(p.block_table, p.max_pages, p.num_pages, p.status, b,
                                        tl.block(pos0 + i));
        tok = 0;
      }
      tma_load_4d(dst, &tmK, &full[st], 0, kvh, tok, bidx);
      tma_load_4d(dst + BOX_BYTES, &tmK, &full[st], 64, kvh, tok, bidx);
      tma_load_4d(dst + 2 * BOX_BYTES, &tmV, &full[st], 0, kvh, tok, bidx);
      tma_load_4d(dst + 3 * BOX_BYTES, &tmV, &full[st], 64, kvh, tok, bidx);
    }
    issued = i + 1;
  };
  const bool skip_loads = c_skip_loads != 0;
  if (tid == 0 && !skip_loads) {
    for (int i = 0; i < NSTAGE && i < ntiles; ++i) issue(i);
  }

  // ---- query fragments (row g = head g of the group; rows >= G are zero)
  // k-step s: qa[s][0] = dims (2t, 2t+1), qa[s][1] = dims (2t+8, 2t+9) of
  // dims 16s.. (bf16); FP8: dims (4t, 4t+1) and (4t+2, 4t+3) of 16s.., the
  // order in which ldmatrix hands out a 16-byte row of codes.
  const bool hv = g < G;
  const __nv_bfloat16 *qrow = p.q + (static_cast<size_t>(b) * p.Hq + kvh * G + (hv ? g : 0)) * HD;
  uint32_t qa[8][2];
  float sc = p.scale_log2;
  if constexpr (!FP8) {
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      qa[s][0] = hv ? *reinterpret_cast<const uint32_t *>(qrow + 16 * s + 2 * t) : 0u;
      qa[s][1] = hv ? *reinterpret_cast<const uint32_t *>(qrow + 16 * s + 8 + 2 * t) : 0u;
    }
  } else {
    float qf[8][4];
    float mx = 0.f;
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const uint2 w = hv ? *reinterpret_cast<const uint2 *>(qrow + 16 * s + 4 * t) : make_uint2(0, 0);
      qf[s][0] = __uint_as_float(w.x << 16);
      qf[s][1] = __uint_as_float(w.x & 0xffff0000u);
      qf[s][2] = __uint_as_float(w.y << 16);
      qf[s][3] = __uint_as_float(w.y & 0xffff0000u);
#pragma unroll
      for (int e = 0; e < 4; ++e) mx = fmaxf(mx, fabsf(qf[s][e]));
    }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    int ex = 0;
    if (mx > 0.f) frexpf(mx, &ex);            // mx < 2^ex
    // max |q| * 2^sh in [2^14, 2^15), with 2^sh at most 2^64 so that it stays
    // finite in fp32: the cap only acts on heads whose largest |q| is below
    // 2^-49, whose scores are below 2^-40 in magnitude either way.
    const int sh = mx > 0.f ? min(15 - ex, 64) : 0;
    const float pw = ldexpf(1.0f, sh);
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      qa[s][0] = pack_f16x2(qf[s][0] * pw, qf[s][1] * pw);
      qa[s][1] = pack_f16x2(qf[s][2] * pw, qf[s][3] * pw);
    }
    sc = p.scale_log2 * p.k_scale[kvh] * ldexpf(1.0f, -sh);
  }

  float o[8][4];               // O^T: m-tile M (16 dims) x heads (2t, 2t+1)
#pragma unroll
  for (int M = 0; M < 8; ++M)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[M][e] = 0.f;
  float m_ref = -INFINITY;     // reference max of head g in this warp (log2 units)
  float l_sum = 0.f;           // this lane's share of head g's row sum

  // This warp's keys inside an iteration: block wb, keys kb .. kb+KW-1.
  const int wb = FP8 ? (warp >> 2) : 0;
  const int kb = FP8 ? 16 * (warp & 3) : 8 * warp;

  for (int i = 0; i < ntiles; ++i) {
    const int st = i % NSTAGE;
    const bool ok = mbar_wait(&full[st], static_cast<uint32_t>(i / NSTAGE) & 1u, abort, p.status);
    const uint32_t sK = smem_u32(stages + st * STAGE_BYTES) + wb * T::BLK;
    const uint32_t sV = sK + T::KBYTES;
    const int blk_i = NB * i + wb;
    const int key0 = (blk_i < nblocks) ? tl.block(pos0 + blk_i) * KT + kb : INT_MAX / 2;

    // ---- S = Q K^T for this warp's keys
    float s[NT8][4];
#pragma unroll
    for (int j = 0; j < NT8; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[j][e] = 0.f;
#pragma unroll
    for (int j = 0; j < NT8; ++j) {
      const int key = kb + 8 * j + (lane & 7);
      if constexpr (!FP8) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t r[4];
          ldsm_x4(sK + tile_offset(key, 4 * c + (lane >> 3)), r);
          mma_k16_top<false>(s[j], qa[2 * c][0], qa[2 * c][1], r[0], r[1]);
          mma_k16_top<false>(s[j], qa[2 * c + 1][0], qa[2 * c + 1][1], r[2], r[3]);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t r[4];
          const int chunk = 4 * c + (lane >> 3);
          ldsm_x4(sK + fp8_offset(key, 16 * chunk), r);
#pragma unroll
          for (int x = 0; x < 4; ++x) {
            uint32_t b0, b1;
            e4m3x4_to_f16x2(r[x], b0, b1);
            mma_k16_top<true>(s[j], qa[4 * c + x][0], qa[4 * c + x][1], b0, b1);
          }
        }
      }
    }

    // ---- scores (log2 units), reference, probabilities
    float sv[NT8][2];
    float tmax = -INFINITY;
#pragma unroll
    for (int j = 0; j < NT8; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const bool valid = key0 + 8 * j + 2 * t + e < L;
        sv[j][e] = valid ? s[j][e] * sc : -INFINITY;
        tmax = fmaxf(tmax, sv[j][e]);
      }
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 1));
    tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 2));
    const bool up = tmax > m_ref + kRefSlack;
    if (__any_sync(0xffffffffu, up)) {   // rare: move this warp's references
      const float alpha = up ? ((m_ref == -INFINITY) ? 0.f : ex2(m_ref - tmax)) : 1.f;
      if (up) m_ref = tmax;
      l_sum *= alpha;
      // This lane's O^T columns are heads 2t and 2t+1, whose factors sit in
      // lanes 8t and 8t+4.
      const float a0 = __shfl_sync(0xffffffffu, alpha, 8 * t);
      const float a1 = __shfl_sync(0xffffffffu, alpha, 8 * t + 4);
#pragma unroll
      for (int M = 0; M < 8; ++M) {
        o[M][0] *= a0;
        o[M][1] *= a1;
        o[M][2] *= a0;
        o[M][3] *= a1;
      }
    }
    uint32_t pb[NT8];
#pragma unroll
    for (int j = 0; j < NT8; ++j) {
      const float p0 = (sv[j][0] == -INFINITY) ? 0.f : ex2(sv[j][0] - m_ref);
      const float p1 = (sv[j][1] == -INFINITY) ? 0.f : ex2(sv[j][1] - m_ref);
      if constexpr (FP8) {   // f16 keeps 11 bits: the sum of the unrounded p differs by ~2^-12
        pb[j] = pack_f16x2(p0, p1);
        l_sum += p0 + p1;
      } else {
        pb[j] = pack_bf16x2(p0, p1);
        l_sum += __uint_as_float(pb[j] << 16) + __uint_as_float(pb[j] & 0xffff0000u);
      }
    }

    // ---- O^T += V^T P^T
    if constexpr (!FP8) {
      const int key = kb + (lane & 7);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[4];
        ldsm_x4_t(sV + tile_offset(key, 4 * c + (lane >> 3)), r);
        mma_k8_bf16(o[2 * c], r[0], r[1], pb[0]);       // dims 32c + (0..15)
        mma_k8_bf16(o[2 * c + 1], r[2], r[3], pb[0]);   // dims 32c + (16..31)
      }
    } else {
      // Lane (g, t): keys kb + {2t, 2t+1, 2t+8, 2t+9}, dims 32q + 4g + (0..3).
      // m-tile 2q+m: row g = dim 32q + 4g + 2m, row g+8 = dim 32q + 4g + 2m + 1.
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint32_t w[4];
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const int key = kb + 2 * t + (kk & 1) + 8 * (kk >> 1);
          w[kk] = lds32(sV + fp8_offset(key, 32 * q + 4 * g));
        }
        // (key 2t, key 2t+1) byte pairs of dims +0 / +1 (lo) and +2 / +3 (hi).
        uint32_t a[2][4];
        e4m3x4_to_f16x2(__byte_perm(w[0], w[1], 0x5140), a[0][0], a[0][1]);
        e4m3x4_to_f16x2(__byte_perm(w[2], w[3], 0x5140), a[0][2], a[0][3]);
        e4m3x4_to_f16x2(__byte_perm(w[0], w[1], 0x7362), a[1][0], a[1][1]);
        e4m3x4_to_f16x2(__byte_perm(w[2], w[3], 0x7362), a[1][2], a[1][3]);
        mma_k16_f16(o[2 * q], a[0][0], a[0][1], a[0][2], a[0][3], pb[0], pb[1]);
        mma_k16_f16(o[2 * q + 1], a[1][0], a[1][1], a[1][2], a[1][3], pb[0], pb[1]);
      }
    }
    // Past this barrier every warp is done with this stage: it takes tile
    // i + NSTAGE.
    if (__syncthreads_or(!ok)) break;
    if (tid == 0 && !skip_loads && i + NSTAGE < ntiles) issue(i + NSTAGE);
  }
  __syncthreads();   // every thread is done with the stages (reused below)

  if (*abort) {  // a wait ran out: let the copies still in flight land, then leave
    if (tid == 0) {
      for (int x = (issued > NSTAGE ? issued - NSTAGE : 0); x < issued; ++x)
        mbar_wait_drain(&full[x % NSTAGE], static_cast<uint32_t>(x / NSTAGE) & 1u, 200000000ull);
    }
    if (tid < G) {
      const size_t r0 = (static_cast<size_t>(b) * p.Hq + kvh * G + tid) * p.nsplit + split;
      if (in_bounds(p.status, static_cast<long long>(r0) * 2 + 1,
                    static_cast<long long>(p.B) * p.Hq * p.nsplit * 2)) {
        p.ml_part[r0 * 2] = __int_as_float(0x7fc00000);
        p.ml_part[r0 * 2 + 1] = __int_as_float(0x7fc00000);
      }
    }
    __syncthreads();
    return;
  }

  // ---- merge the warps: per head, M = max of the warps' references
  l_sum += __shfl_xor_sync(0xffffffffu, l_sum, 1);
  l_sum += __shfl_xor_sync(0xffffffffu, l_sum, 2);
  float *red_o = reinterpret_cast<float *>(stages);   // [NW][G][HD]
  float *red_m = red_o + NW * G * HD;                  // [NW][G]
  float *red_l = red_m + NW * G;                       // [NW][G]
  float *red_w = red_l + NW * G;                       // [NW][G] merge weights
  float *red_M = red_w + NW * G;                       // [G]
  if (t == 0 && hv) {
    red_m[warp * G + g] = m_ref;
    red_l[warp * G + g] = l_sum;
  }
#pragma unroll
  for (int M = 0; M < 8; ++M)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int h = 2 * t + (e & 1);
      const int d = FP8 ? 32 * (M >> 1) + 4 * g + 2 * (M & 1) + (e >> 1)
                        : 16 * M + g + 8 * (e >> 1);
      if (h < G) red_o[(warp * G + h) * HD + d] = o[M][e];
    }
  __syncthreads();
  if (tid < G) {
    float mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) mx = fmaxf(mx, red_m[w * G + tid]);
    float l = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const float mw = red_m[w * G + tid];
      const float wt = (mw == -INFINITY) ? 0.f : ex2(mw - mx);
      red_w[w * G + tid] = wt;
      l = fmaf(wt, red_l[w * G + tid], l);
    }
    red_M[tid] = mx;
    const size_t mi = ((static_cast<size_t>(b) * p.Hq + kvh * G + tid) * p.nsplit + split) * 2;
    if (in_bounds(p.status, static_cast<long long>(mi) + 1,
                  static_cast<long long>(p.B) * p.Hq * p.nsplit * 2)) {
      p.ml_part[mi] = mx;
      p.ml_part[mi + 1] = l;
    }
  }
  __syncthreads();
  float vs = 1.0f;
  if constexpr (FP8) vs = p.v_scale[kvh];
  const size_t row0 = (static_cast<size_t>(b) * p.Hq + kvh * G) * p.nsplit + split;
  for (int idx = tid; idx < G * HD; idx += NT) {
    const int h = idx / HD, d = idx % HD;
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) sum = fmaf(red_w[w * G + h], red_o[(w * G + h) * HD + d], sum);
    const size_t oi = (row0 + static_cast<size_t>(h) * p.nsplit) * HD + d;
    if (in_bounds(p.status, static_cast<long long>(oi),
                  static_cast<long long>(p.B) * p.Hq * p.nsplit * HD))
      p.o_part[oi] = sum * vs;
  }
}

// Merge the splits of one (batch, head): M = max m_s, w_s = 2^(m_s - M),
// o = sum w_s o_s / sum w_s l_s.  The weights are computed once into shared
// memory; then thread d walks the splits for output dim d (coalesced rows).
// A split that gave up (a bounded wait ran out) left a NaN reference: the
// head's output and LSE are then NaN.
constexpr int kMaxSplits = 256;
__global__ void __launch_bounds__(128) combine_kernel(const float *o_part, const float *ml_part,
                                                      __nv_bfloat16 *o, float *lse, int Hq,
                                                      int nsplit) {
  __shared__ float w_sm[kMaxSplits];
  __shared__ float red[4];
  __shared__ float M_sm, den_sm;
  const int h = blockIdx.x, b = blockIdx.y, d = threadIdx.x, lane = d & 31, warp = d >> 5;
  const size_t row = (static_cast<size_t>(b) * Hq + h);
  const float *ml = ml_part + row * nsplit * 2;
  float mx = -INFINITY;
  bool missing = false;
  for (int s = d; s < nsplit; s += 128) {
    const float m = ml[2 * s];
    missing |= (m != m);
    mx = fmaxf(mx, m);
  }
  missing = __syncthreads_or(missing) != 0;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  if (lane == 0) red[warp] = mx;
  __syncthreads();
  if (d == 0) M_sm = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  __syncthreads();
  const float M = M_sm;
  float den = 0.f;
  for (int s = d; s < nsplit; s += 128) {
    const float m = ml[2 * s];
    const float w = (m == -INFINITY) ? 0.f : ex2(m - M);
    w_sm[s] = w;
    den = fmaf(w, ml[2 * s + 1], den);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
  __syncthreads();
  if (lane == 0) red[warp] = den;
  __syncthreads();
  if (d == 0) den_sm = (red[0] + red[1]) + (red[2] + red[3]);
  __syncthreads();
  den = den_sm;
  float num = 0.f;
  const float *op = o_part + row * nsplit * HD + d;
  for (int s = 0; s < nsplit; ++s) num = fmaf(w_sm[s], op[static_cast<size_t>(s) * HD], num);
  const bool any = (M != -INFINITY) && den > 0.f;
  const float nan = __int_as_float(0x7fc00000);
  o[row * HD + d] = __float2bfloat16_rn(missing ? nan : (any ? num / den : 0.f));
  if (lse && d == 0)
    lse[row] = missing ? nan : (any ? (M + __log2f(den)) * 0.69314718055994531f : -INFINITY);
}

}  // namespace decode

// Splits per (batch, KV head) for a sequence of `tiles` 64-key tiles.  The
// CTA count B*Hkv*splits is chosen to fill whole waves of 2 CTAs on each of
// 148 SMs (a partial last wave leaves SMs idle), with at least 4 tiles per
// CTA and at most kMaxSplits splits; small problems take the most splits.
int decode_splits_for_tiles(int B, int Hkv, int tiles) {
  constexpr int kSlots = 148 * 2;
  const int base = B * Hkv;
  int ns_max = tiles / 4;
  ns_max = ns_max < 1 ? 1 : (ns_max > decode::kMaxSplits ? decode::kMaxSplits : ns_max);
  if (static_cast<long long>(base) * ns_max <= 2 * kSlots) return ns_max;
  const int ns_min = (2 * kSlots + base - 1) / base;
  int best = ns_max;
  double best_eff = -1.0;
  for (int ns = ns_min; ns <= ns_max; ++ns) {
    const double waves = static_cast<double>(base) * ns / kSlots;
    const double eff = waves / static_cast<double>(static_cast<long long>(waves + 0.999999));
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best = ns;
    }
  }
  return best;
}

int decode_num_splits(int B, int Hkv, int Lmax) {
  return decode_splits_for_tiles(B, Hkv, (Lmax + decode::KT - 1) / decode::KT);
}

int set_wait_limit_decode(uint64_t ns, int skip_loads) { return set_wait_limit_local(ns, skip_loads); }

size_t decode_workspace_bytes(int B, int Hq, int Hkv, int Lmax) {
  const size_t ns = static_cast<size_t>(decode_num_splits(B, Hkv, Lmax));
  return static_cast<size_t>(B) * Hq * ns * (decode::HD + 2) * sizeof(float) + 256;
}

int launch_decode(const DecodeLaunch &a, cudaStream_t stream) {
  using namespace decode;
  CUtensorMap tmK, tmV;
  const bool paged = a.block_table != nullptr;
  // The cache as a 4-D tensor (D, Hkv, tokens, batch); a page pool is
  // (D, Hkv, 64, num_pages).
  const int mB = paged ? a.num_pages : a.B, mS = paged ? KT : a.Lmax;
  if (a.fp8) {
    if (make_tmap_bhsd_u8(&tmK, a.kcache, mB, mS, a.Hkv, KT) != 0) return FA_ERR_CUDA;
    if (make_tmap_bhsd_u8(&tmV, a.vcache, mB, mS, a.Hkv, KT) != 0) return FA_ERR_CUDA;
  } else {
    if (make_tmap_bhsd(&tmK, a.kcache, mB, mS, a.Hkv, 64, KT) != 0) return FA_ERR_CUDA;
    if (make_tmap_bhsd(&tmV, a.vcache, mB, mS, a.Hkv, 64, KT) != 0) return FA_ERR_CUDA;
  }
  const int G = a.Hq / a.Hkv;
  // Splits: sized for FULL unless every sequence is known to be SPARSE.
  int ns = decode_num_splits(a.B, a.Hkv, a.Lmax);
  if (a.mode_dev == nullptr && a.mode == FA_MODE_SPARSE) {
    const int sparse_tiles = a.sink / KT + a.window / KT;
    const int ns_sparse = decode_splits_for_tiles(a.B, a.Hkv, sparse_tiles);
    ns = ns_sparse < ns ? ns_sparse : ns;   // the workspace is sized for the FULL count
  }
  Params p;
  p.q = reinterpret_cast<const __nv_bfloat16 *>(a.q);
  float *ws = reinterpret_cast<float *>(a.workspace);
  p.o_part = ws;
  p.ml_part = ws + static_cast<size_t>(a.B) * a.Hq * ns * HD;
  p.seqlens = a.seqlens;
  p.mode = a.mode_dev;
  p.status = a.status;
  p.B = a.B;
  p.Lmax = a.Lmax;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.nsplit = ns;
  p.mode_default = a.mode;
  p.sink_blocks = a.sink / KT;
  p.win_blocks = a.window / KT;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.block_table = a.block_table;
  p.max_pages = a.max_pages;
  p.num_pages = a.num_pages;
  p.k_scale = a.fp8 ? a.k_scale : nullptr;
  p.v_scale = a.fp8 ? a.v_scale : nullptr;
  const dim3 grid(ns, a.Hkv, a.B);
  void (*kern)(const CUtensorMap, const CUtensorMap, const Params) = nullptr;
  int smem = 0;
  // FP8 caches are always paged (a contiguous cache is the identity table).
  if (a.fp8 && !paged) return FA_ERR_UNSUPPORTED;
  switch (G * 4 + (a.fp8 ? 2 : 0) + (paged ? 1 : 0)) {
    case 4: kern = decode_kernel<1, false, false>, smem = Lay::BYTES; break;
    case 8: kern = decode_kernel<2, false, false>, smem = Lay::BYTES; break;
    case 16: kern = decode_kernel<4, false, false>, smem = Lay::BYTES; break;
    case 32: kern = decode_kernel<8, false, false>, smem = Lay::BYTES; break;
    case 5: kern = decode_kernel<1, false, true>, smem = Lay::BYTES; break;
    case 9: kern = decode_kernel<2, false, true>, smem = Lay::BYTES; break;
    case 17: kern = decode_kernel<4, false, true>, smem = Lay::BYTES; break;
    case 33: kern = decode_kernel<8, false, true>, smem = Lay::BYTES; break;
    case 7: kern = decode_kernel<1, true, true>, smem = Lay::BYTES; break;
    case 11: kern = decode_kernel<2, true, true>, smem = Lay::BYTES; break;
    case 19: kern = decode_kernel<4, true, true>, smem = Lay::BYTES; break;
    case 35: kern = decode_kernel<8, true, true>, smem = Lay::BYTES; break;
    default: return FA_ERR_UNSUPPORTED;
  }
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return FA_ERR_CUDA;
  kern<<<grid, NT, smem, stream>>>(tmK, tmV, p);
  note_launch();
  if (cudaPeekAtLastError() != cudaSuccess) return FA_ERR_CUDA;
  combine_kernel<<<dim3(a.Hq, a.B), 128, 0, stream>>>(
      p.o_part, p.ml_part, reinterpret_cast<__nv_bfloat16 *>(a.o), a.lse, a.Hq, ns);
  note_launch();
  return cudaPeekAtLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// ------------------------------------------------------------ KV append
// Writes token position seqlens[b] of every sequence (K and V of all KV
// heads) into its page, quantising to E4M3 (code = RN(fp32(x / scale)),
// saturating) for an FP8 cache, then advances seqlens[b].  A position past
// the block table or a page id outside the pool is reported and skipped.
// One CTA per sequence.
__global__ void __launch_bounds__(256) kv_append_kernel(const __nv_bfloat16 *k_new,
                                                        const __nv_bfloat16 *v_new,
                                                        uint8_t *k_pages, uint8_t *v_pages, int fp8,
                                                        const float *k_scale, const float *v_scale,
                                                        const int32_t *block_table, int max_pages,
                                                        int num_pages, int32_t *seqlens, int Hkv,
                                                        int32_t *status) {
  const int b = blockIdx.x;
  const int pos = seqlens[b];
  const int pi = pos / decode::KT, slot = pos % decode::KT;
  int page = -1;
  if (pos >= 0 && pi < max_pages) page = block_table[static_cast<size_t>(b) * max_pages + pi];
  const bool ok = page >= 0 && page < num_pages;
  if (!ok) {
    if (threadIdx.x == 0) report(status, FA_DEV_BAD_INDEX);
    return;
  }
  const size_t row = (static_cast<size_t>(page) * decode::KT + slot) * Hkv;   // token row
  const int n = Hkv * decode::HD;
  for (int t = 0; t < 2; ++t) {
    const __nv_bfloat16 *src = (t ? v_new : k_new) + static_cast<size_t>(b) * n;
    uint8_t *dst = (t ? v_pages : k_pages);
    const float *sc = t ? v_scale : k_scale;
    for (int i = threadIdx.x * 2; i < n; i += 2 * blockDim.x) {
      if (fp8) {
        const float s = sc[i / decode::HD];
        const float2 x = make_float2(__fdiv_rn(__bfloat162float(src[i]), s),
                                     __fdiv_rn(__bfloat162float(src[i + 1]), s));
        const __nv_fp8x2_storage_t c = __nv_cvt_float2_to_fp8x2(x, __NV_SATFINITE, __NV_E4M3);
        *reinterpret_cast<__nv_fp8x2_storage_t *>(dst + row * decode::HD + i) = c;
      } else {
        *reinterpret_cast<uint32_t *>(dst + (row * decode::HD + i) * 2) =
            *reinterpret_cast<const uint32_t *>(src + i);
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) seqlens[b] = pos + 1;
}

int launch_kv_append(const KvAppendLaunch &a, cudaStream_t stream) {
  kv_append_kernel<<<a.B, 256, 0, stream>>>(
      reinterpret_cast<const __nv_bfloat16 *>(a.k_new),
      reinterpret_cast<const __nv_bfloat16 *>(a.v_new), reinterpret_cast<uint8_t *>(a.k_pages),
      reinterpret_cast<uint8_t *>(a.v_pages), a.fp8, a.k_scale, a.v_scale, a.block_table,
      a.max_pages, a.num_pages, a.seqlens, a.Hkv, a.status);
  note_launch();
  return cudaPeekAtLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace fa
