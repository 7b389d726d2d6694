// fa_decode.cu -- single-token decode attention over a bf16 KV cache, sm_100a.
//
// o = softmax(scale * q K^T) V for the query at position L-1 of each sequence.
// FULL attends keys 0..L-1; SPARSE attends the sink blocks and the local
// window of the prefill block rule for row L-1 and never loads any other KV
// block ("Flux Attention": a sparse layer bypasses the KV cache outside its
// pattern).  Memory-bound: every byte of K and V it needs is read once.
//
// Grid (split, kv head, batch).  A CTA owns one KV head (all G query heads
// of its group share each K/V tile) and a contiguous share of the sequence's
// 64-key tiles.  Thread 0 streams the tiles with 4-D TMA loads (128-byte
// swizzle; bf16: 2 boxes of 64 keys x 64 dims per K or V tile, 3 stages;
// fp8: 1 box of 64 keys x 128 dims, 6 stages) into a ring; all threads
// compute from shared memory:
//   QK^T   thread = (key, 1/PARTS of the head dim), dot products for the G
//          heads, reduced across the PARTS lanes by a butterfly that leaves
//          each head's score on one lane, which also forms its probability
//          2^(s - m) against a per-head reference max m (log2 units);
//   PV     thread = (8 output dims, one of 16 key streams), G accumulators.
// The reference only moves, for the whole CTA, on a tile holding a score more
// than 16 above it (always the first): then the accumulators and row sums
// are rescaled and the tile's probabilities redone.  One block barrier per
// tile otherwise.  Each CTA writes its partial (reference, sum, unnormalised
// output) per head; the combine kernel merges the splits by log-sum-exp.
//
// Paged cache: with a block table, tile n of sequence b is page
// block_table[b][n] of a pool [num_pages, 64, Hkv, 128] (one page = one
// 64-token block, so the sparse mode skips whole pages).  FP8 cache: E4M3
// codes with one dequantisation scale per KV head for K and for V; the K
// scale is folded into the query, the V scale into the partial outputs.
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

template <int G>
struct Cfg {
  static constexpr int PARTS = (G <= 4) ? 8 : 16;       // threads per key in QK^T
  static constexpr int DPT = HD / PARTS;                 // dims per thread
  static constexpr int KPP = NT / PARTS;                 // keys per pass
  static constexpr int MIN_BLOCKS = (G <= 4) ? 2 : 1;
};

FA_DEV void bf16x8_to_f32(const uint4 &v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// Eight bf16 (one 16-byte chunk) -> four packed fp32 pairs (element 2i in
// the low lane of pair i).
FA_DEV void bf16x8_to_f2(const uint4 &v, uint64_t (&f)[4]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) f[i] = f2_make(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xffff0000u));
}

// Byte offset of the 16-byte chunk holding dims [8*chunk16, 8*chunk16+8) of
// `key` inside one K or V tile written by TMA with the 128-byte swizzle.
FA_DEV uint32_t tile_offset(int key, int chunk16) {
  const int box = chunk16 >> 3;
  const int phys = (chunk16 & 7) ^ (key & 7);
  return static_cast<uint32_t>(box * BOX_BYTES + key * 128 + phys * 16);
}

// The same for an FP8 tile (one 128-byte row per key): byte offset of the
// 8 codes of dims [8*g8, 8*g8+8).
FA_DEV uint32_t tile_offset_fp8(int key, int g8) {
  const int phys = (g8 >> 1) ^ (key & 7);
  return static_cast<uint32_t>(key * 128 + phys * 16 + (g8 & 1) * 8);
}

// Eight E4M3 codes (8 bytes) -> four packed fp32 pairs, exact.
FA_DEV void fp8x8_to_f2(const uint2 &v, uint64_t (&f)[4]) {
  const uint32_t w[2] = {v.x, v.y};
#pragma unroll
  for (int i = 0; i < 2; ++i) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(
          static_cast<__nv_fp8x2_storage_t>((w[i] >> (16 * j)) & 0xffffu), __NV_E4M3);
      const float2 fl = __half22float2(*reinterpret_cast<const __half2 *>(&h));
      f[2 * i + j] = f2_make(fl.x, fl.y);
    }
  }
}

// K or V of eight dims of one key (0 .. TK-1) from a stage's K or V part, as
// four fp32 pairs.
template <bool FP8>
FA_DEV void load8(const uint8_t *tile, int key, int g8, uint64_t (&f)[4]) {
  if constexpr (FP8) {
    const uint8_t *blk = tile + (key >> 6) * KvT<true>::BLK;
    fp8x8_to_f2(*reinterpret_cast<const uint2 *>(blk + tile_offset_fp8(key & 63, g8)), f);
  } else {
    bf16x8_to_f2(*reinterpret_cast<const uint4 *>(tile + tile_offset(key, g8)), f);
  }
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

// Shared memory of one decode CTA (offsets from a 1024-byte aligned base):
// K/V ring | stage barriers | abort and re-reference flags | P pairs
// (double-buffered [2][TK][G], each probability stored twice so a packed
// FMA reads it as one 64-bit operand) | raw scores of a re-referenced tile
// [G][TK] | per-head reference max and rescale factor, per-warp row sums |
// page ids.
template <int G, bool FP8>
struct Lay {
  static constexpr int TK = KvT<FP8>::TK;
  static constexpr int FULL = RING_BYTES;
  static constexpr int FLAGS = FULL + 8 * MAX_STAGES;
  static constexpr int P2 = FLAGS + 16;
  static constexpr int SRAW = P2 + 2 * TK * G * 8;
  static constexpr int REF = SRAW + TK * G * 4;
  static constexpr int PAGES = REF + (8 + 8 + 8 * 8) * 4;
  static constexpr int BYTES = 1024 + PAGES + PAGE_CACHE * 4;
};

// A tile is scored against a fixed per-head reference max; only a score
// more than kRefSlack (log2 units) above it, or the first tile, makes the
// whole CTA move the reference (the rare path).  p <= 2^kRefSlack keeps
// every fp32 sum far from overflow.
constexpr float kRefSlack = 16.0f;

template <int G, bool FP8, bool PAGED>
__global__ void __launch_bounds__(NT, Cfg<G>::MIN_BLOCKS)
    decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const Params p) {
  using C = Cfg<G>;
  using T = KvT<FP8>;
  using Y = Lay<G, FP8>;
  constexpr int NSTAGE = T::NST, STAGE_BYTES = T::STAGE, TK = T::TK, NB = T::NB;
  constexpr int PASSES = TK / C::KPP;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  uint8_t *stages = base;
  uint64_t *full = reinterpret_cast<uint64_t *>(base + Y::FULL);
  volatile int *abort = reinterpret_cast<volatile int *>(base + Y::FLAGS);
  // reref[i & 1]: some score of tile i passed its reference.  One flag per
  // tile parity: a thread may already be scoring tile i+1 (and raising its
  // flag) while another still reads tile i's.
  volatile int *reref = abort + 1;
  uint64_t *p2_sm = reinterpret_cast<uint64_t *>(base + Y::P2);
  float *sraw_sm = reinterpret_cast<float *>(base + Y::SRAW);
  float *mref_sm = reinterpret_cast<float *>(base + Y::REF);   // [8]
  float *alpha_sm = mref_sm + 8;                                // [8]
  float *lsum_sm = alpha_sm + 8;                                // [8 warps][G]
  int *page_sm = reinterpret_cast<int *>(base + Y::PAGES);     // [PAGE_CACHE]

  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
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
    reref[0] = 0;
    reref[1] = 0;
    fence_mbar_init();
  }
  if (tid < 8) mref_sm[tid] = -INFINITY;
  // Page ids of this CTA's tiles (paged cache), read once by all threads.
  if constexpr (PAGED) {
    for (int i = tid; i < nblocks && i < PAGE_CACHE; i += NT)
      page_sm[i] = page_of(p.block_table, p.max_pages, p.num_pages, p.status, b,
                           tl.block(pos0 + i));
  }
  __syncthreads();

  int issued = 0;            // tiles whose copies thread 0 has started
  auto issue = [&](int i) {  // iteration i of this CTA into stage i % NSTAGE
    const int st = i % NSTAGE;
    uint8_t *dst = stages + st * STAGE_BYTES;
    mbar_arrive_expect_tx(&full[st], STAGE_BYTES);
    if constexpr (FP8) {     // paged: NB pages; a missing last one reads zeros
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
  // Testing mode: no loads, every wait runs out.
  const bool skip_loads = c_skip_loads != 0;
  if (tid == 0 && !skip_loads) {
    for (int i = 0; i < NSTAGE && i < ntiles; ++i) issue(i);
  }

  // QK^T: the PARTS threads of a key each hold G partial dot products.  Slot
  // j of this thread accumulates query head j ^ hsel, where bit s of `part`
  // contributes G >> (s+1) to hsel: then a butterfly that at each step keeps
  // the lower half of the slots and sends the upper half sums every head with
  // G - 1 shuffles and no selects, leaving head hsel's total in slot 0.
  const int part = tid % C::PARTS;
  int hsel = 0;
#pragma unroll
  for (int s = 0; (G >> (s + 1)) > 0; ++s)
    if ((part >> s) & 1) hsel |= G >> (s + 1);
  const bool writer = part < G;   // one thread per (key, head) scores it
  // Chunk (8 dims) of the head dim for step c8 of this thread's QK^T.  bf16:
  // chunk c8*PARTS + part, so the 8 lanes of a key that share a shared-memory
  // phase read 8 different swizzled slots of one box (no bank conflicts).
  // FP8: the thread's chunks are adjacent (a conflict-free order measured
  // slower there: it costs registers).
  auto chunk_of = [&](int c8) {
    return FP8 ? part * (C::DPT / 8) + c8 : c8 * C::PARTS + part;
  };
  // Query slice of this thread, pre-scaled by scale*log2(e) (and by the K
  // dequantisation scale of this KV head).
  float qscale = p.scale_log2;
  if constexpr (FP8) qscale *= p.k_scale[kvh];
  uint64_t qr[G][C::DPT / 2];   // packed pairs of dims
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const __nv_bfloat16 *qrow =
        p.q + (static_cast<size_t>(b) * p.Hq + kvh * G + (g ^ hsel)) * HD;
#pragma unroll
    for (int c8 = 0; c8 < C::DPT / 8; ++c8) {
      float f[8];
      bf16x8_to_f32(*reinterpret_cast<const uint4 *>(qrow + chunk_of(c8) * 8), f);
#pragma unroll
      for (int e = 0; e < 4; ++e)
        qr[g][c8 * 4 + e] = f2_make(f[2 * e] * qscale, f[2 * e + 1] * qscale);
    }
  }
  const int dc = tid & 15;     // PV: output dims [8*dc, 8*dc+8)
  const int ks = tid >> 4;     // PV: key stream
  uint64_t acc[G][4];           // packed pairs of output dims
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[g][e] = 0ull;
  float mref = -INFINITY;       // writer: reference max of head hsel (log2 units)
  float l_part = 0.f;           // writer: its share of head hsel's row sum

  for (int i = 0; i < ntiles; ++i) {
    const int st = i % NSTAGE;
    // Every thread runs the scores even if its wait failed (the shuffles need
    // the whole warp; the reads stay inside shared memory); the barrier after
    // them agrees on leaving.
    const bool ok = mbar_wait(&full[st], static_cast<uint32_t>(i / NSTAGE) & 1u, abort, p.status);
    const uint8_t *sK = stages + st * STAGE_BYTES;
    const uint8_t *sV = sK + T::KBYTES;
    uint64_t *p2b = p2_sm + (i & 1) * TK * G;
    // Token position of key 0 of each block of this iteration (a missing
    // block: past every length, so its keys are masked).
    int key_base[NB];
#pragma unroll
    for (int h = 0; h < NB; ++h)
      key_base[h] = (NB * i + h < nblocks) ? tl.block(pos0 + NB * i + h) * KT : INT_MAX / 2;

    // ---- scores and probabilities against the reference
    float s_keep[PASSES];
    float l_tile = 0.f;           // writer: this tile's share, added once the reference holds
    bool over = false;
#pragma unroll
    for (int pass = 0; pass < PASSES; ++pass) {
      const int key = pass * C::KPP + tid / C::PARTS;
      uint64_t d2[G];
#pragma unroll
      for (int g = 0; g < G; ++g) d2[g] = 0ull;
#pragma unroll
      for (int c8 = 0; c8 < C::DPT / 8; ++c8) {
        uint64_t k2[4];
        load8<FP8>(sK, key, chunk_of(c8), k2);
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
          for (int e = 0; e < 4; ++e) d2[g] = f2_fma(qr[g][c8 * 4 + e], k2[e], d2[g]);
      }
      float d[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float lo, hi;
        f2_split(d2[g], lo, hi);
        d[g] = lo + hi;
      }
#pragma unroll
      for (int half = G / 2; half >= 1; half >>= 1)
#pragma unroll
        for (int j = 0; j < half; ++j)
          d[j] += __shfl_xor_sync(0xffffffffu, d[j + half], G / (2 * half));
#pragma unroll
      for (int off = G; off < C::PARTS; off <<= 1)
        d[0] += __shfl_xor_sync(0xffffffffu, d[0], off);
      const bool valid = key_base[key / KT] + (key % KT) < L;
      const float s = valid ? d[0] : -INFINITY;
      s_keep[pass] = s;
      if (writer) {
        const bool up = s > mref + kRefSlack;
        over |= up;
        const float pj = (up || s == -INFINITY) ? 0.f : ex2(s - mref);
        l_tile += pj;
        p2b[key * G + hsel] = f2_make(pj, pj);
      }
    }
    if (over) reref[i & 1] = 1;
    // Past this barrier every thread is done with tile i-1 (its PV came before
    // these scores), so its stage takes tile i-1+NSTAGE.
    if (__syncthreads_or(!ok)) break;
    if (tid == 0 && !skip_loads && i >= 1 && i - 1 + NSTAGE < ntiles) issue(i - 1 + NSTAGE);

    // ---- rare: move the reference to the running max, rescale, redo P
    if (reref[i & 1]) {
      if (writer) {
#pragma unroll
        for (int pass = 0; pass < PASSES; ++pass)
          sraw_sm[hsel * TK + pass * C::KPP + tid / C::PARTS] = s_keep[pass];
      }
      __syncthreads();
      if (tid == 0) reref[i & 1] = 0;   // every thread read it before this barrier; the
                                        // next write to it comes after the next tile's barrier
      if (warp < G) {
        float mt = -INFINITY;
#pragma unroll
        for (int j = lane; j < TK; j += 32) mt = fmaxf(mt, sraw_sm[warp * TK + j]);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, off));
        if (lane == 0) {
          const float mo = mref_sm[warp];
          const float mn = fmaxf(mo, mt);
          alpha_sm[warp] = (mo == -INFINITY) ? 0.f : ex2(mo - mn);
          mref_sm[warp] = mn;
        }
      }
      __syncthreads();
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const uint64_t a2 = f2_make(alpha_sm[g], alpha_sm[g]);
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[g][e] = f2_mul(acc[g][e], a2);
      }
      if (writer) {
        l_part *= alpha_sm[hsel];
        mref = mref_sm[hsel];
#pragma unroll
        for (int pass = 0; pass < PASSES; ++pass) {
          const float s = s_keep[pass];
          const float pj = (s == -INFINITY) ? 0.f : ex2(s - mref);
          l_part += pj;
          p2b[(pass * C::KPP + tid / C::PARTS) * G + hsel] = f2_make(pj, pj);
        }
      }
      __syncthreads();
    } else {
      l_part += l_tile;
    }

    // ---- O += P V (P of the G heads of a key: G packed pairs, 16-byte loads)
#pragma unroll
    for (int kk = 0; kk < TK / 16; ++kk) {
      const int key = ks + 16 * kk;
      uint64_t v2[4];
      load8<FP8>(sV, key, dc, v2);
      if constexpr (G == 1) {
        const uint64_t pg = p2b[key];
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[0][e] = f2_fma(pg, v2[e], acc[0][e]);
      } else {
#pragma unroll
        for (int g2 = 0; g2 < G / 2; ++g2) {
          const uint4 w = *reinterpret_cast<const uint4 *>(p2b + key * G + 2 * g2);
          const uint64_t pa = (static_cast<uint64_t>(w.y) << 32) | w.x;
          const uint64_t pb = (static_cast<uint64_t>(w.w) << 32) | w.z;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            acc[2 * g2][e] = f2_fma(pa, v2[e], acc[2 * g2][e]);
            acc[2 * g2 + 1][e] = f2_fma(pb, v2[e], acc[2 * g2 + 1][e]);
          }
        }
      }
    }
  }
  __syncthreads();   // every thread is done with the stages (reused below)

  if (*abort) {  // a wait ran out: let the copies still in flight land, then leave
    if (tid == 0) {
      for (int x = (issued > NSTAGE ? issued - NSTAGE : 0); x < issued; ++x)
        mbar_wait_drain(&full[x % NSTAGE], static_cast<uint32_t>(x / NSTAGE) & 1u, 200000000ull);
    }
    // Mark this split's partials as missing (NaN reference): the combine then
    // writes NaN for these heads instead of merging whatever the workspace
    // held before.
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

  // ---- row sums: the writers of a head share `part`; one total per warp
#pragma unroll
  for (int off = C::PARTS; off < 32; off <<= 1) l_part += __shfl_xor_sync(0xffffffffu, l_part, off);
  if (lane < G) lsum_sm[warp * G + hsel] = l_part;   // lane < G: part = lane, a writer

  // ---- reduce the 16 key streams through shared memory (stage buffers free)
  float *red = reinterpret_cast<float *>(stages);   // [16][G][HD]
  float vs = 1.0f;
  if constexpr (FP8) vs = p.v_scale[kvh];
#pragma unroll
  for (int g = 0; g < G; ++g)
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float lo, hi;
      f2_split(acc[g][e], lo, hi);
      red[(ks * G + g) * HD + dc * 8 + 2 * e] = lo;
      red[(ks * G + g) * HD + dc * 8 + 2 * e + 1] = hi;
    }
  __syncthreads();
  const size_t row0 = (static_cast<size_t>(b) * p.Hq + kvh * G) * p.nsplit + split;
  for (int idx = tid; idx < G * HD; idx += NT) {
    const int g = idx / HD, dd = idx % HD;
    float sum = 0.f;
#pragma unroll
    for (int s = 0; s < 16; ++s) sum += red[(s * G + g) * HD + dd];
    const size_t oi = (row0 + static_cast<size_t>(g) * p.nsplit) * HD + dd;
    if (in_bounds(p.status, static_cast<long long>(oi),
                  static_cast<long long>(p.B) * p.Hq * p.nsplit * HD))
      p.o_part[oi] = sum * vs;
  }
  if (tid < G) {
    float l = 0.f;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) l += lsum_sm[w * G + tid];
    const size_t mi = (row0 + static_cast<size_t>(tid) * p.nsplit) * 2;
    if (in_bounds(p.status, static_cast<long long>(mi) + 1,
                  static_cast<long long>(p.B) * p.Hq * p.nsplit * 2)) {
      p.ml_part[mi] = mref_sm[tid];
      p.ml_part[mi + 1] = l;
    }
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
    case 4: kern = decode_kernel<1, false, false>, smem = Lay<1, false>::BYTES; break;
    case 8: kern = decode_kernel<2, false, false>, smem = Lay<2, false>::BYTES; break;
    case 16: kern = decode_kernel<4, false, false>, smem = Lay<4, false>::BYTES; break;
    case 32: kern = decode_kernel<8, false, false>, smem = Lay<8, false>::BYTES; break;
    case 5: kern = decode_kernel<1, false, true>, smem = Lay<1, false>::BYTES; break;
    case 9: kern = decode_kernel<2, false, true>, smem = Lay<2, false>::BYTES; break;
    case 17: kern = decode_kernel<4, false, true>, smem = Lay<4, false>::BYTES; break;
    case 33: kern = decode_kernel<8, false, true>, smem = Lay<8, false>::BYTES; break;
    case 7: kern = decode_kernel<1, true, true>, smem = Lay<1, true>::BYTES; break;
    case 11: kern = decode_kernel<2, true, true>, smem = Lay<2, true>::BYTES; break;
    case 19: kern = decode_kernel<4, true, true>, smem = Lay<4, true>::BYTES; break;
    case 35: kern = decode_kernel<8, true, true>, smem = Lay<8, true>::BYTES; break;
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
