// fa_prefill.cu -- causal full and block-sparse attention prefill for sm_100a.
//
// What it computes (see include/fa_hybrid.h): O = softmax(scale * Q K^T
// + mask) V per (batch, query head), with the causal mask, and for the sparse
// mode the 64-token block pattern of a CSR row list ("Flux Attention",
// implementation paragraph: 64-token block sparsity, 128 sink tokens).  The
// softmax is the online form of the FlashAttention newsletter (section
// "어려움을 극복하기 위한 Online Softmax"): a running maximum and sum per row,
// with earlier partial results rescaled by exp(m_old - m_new).
//
// Design (one CTA = one 128-row query tile of one (batch, head)):
//   warp 0      TMA producer: Q once, then K and V tiles of 128 keys into a
//               ring of 32 KB slots, in exactly the order the MMAs use them.
//   warp 1      MMA issuer (one thread) and TMEM owner: S_j = Q K_j^T into one
//               of two TMEM score buffers, O += P_j V_j with P read from TMEM.
//   warps 4-7   softmax warpgroup, one thread per query row: reads S_j from
//               TMEM, masks, forms P_j = 2^(s*c - m) (bf16) against a lazy
//               reference m -- the running max of the earlier tiles, moved
//               (with O rescaled in TMEM) only on a tile whose row sum leaves
//               the safe range, and on the first tile -- writes P_j to TMEM,
//               and finally normalises O and stores it (exact: the final
//               division uses the same reference as the sum).
// (prefill2_kernel below: the persistent two-head version of the same.)
// TMEM columns: S0 [0,128) S1 [128,256) O [256,384) P0 [384,448) P1 [448,512).
// All operands are bf16; accumulation and softmax are fp32.
#include "fa_common.cuh"
#include "fa_internal.h"

#include <math.h>

namespace fa {

// ------------------------------------------------ softmax arithmetic ---
// Shared by both prefill kernels: exponentials in log2 units against a
// reference max, two lanes per instruction.

// 2^x on the FMA pipe: round-to-nearest range reduction with the 1.5*2^23
// shifter (x = n + f, f in [-1/2, 1/2]), a degree-3 polynomial for 2^f
// (coefficients fitted here by minimax linear programming on [-1/2, 1/2];
// max relative error 1.0e-4, below bf16 rounding of P), and n added to the
// exponent field.  Inputs below -127 give 0.
#ifndef FA_POLY_PER_8
#define FA_POLY_PER_8 2
#endif
// Key pairs (k, k+1), k even, with (k mod 8) >= 8 - kPolyPer8 take the
// polynomial (so kPolyPer8 counts in steps of 2); the rest use ex2.approx.
constexpr int kPolyPer8 = FA_POLY_PER_8;
constexpr float kExp2C1 = 0.693282962f;
constexpr float kExp2C2 = 0.242210999f;
constexpr float kExp2C3 = 0.0550087839f;
FA_DEV float ex2_poly(float x) {
  x = fmaxf(x, -127.0f);
  const float t = x + 12582912.0f;          // 1.5 * 2^23: low mantissa bits = round(x)
  const float n = t - 12582912.0f;
  const float f = x - n;
  float p = fmaf(kExp2C3, f, kExp2C2);
  p = fmaf(p, f, kExp2C1);
  p = fmaf(p, f, 1.0f);
  return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}
// The same for two lanes at once with the packed fp32x2 instructions.
FA_DEV void ex2_poly2(uint64_t x2, float &r0, float &r1) {
  float a, b;
  f2_split(x2, a, b);
  const uint64_t x = f2_make(fmaxf(a, -127.0f), fmaxf(b, -127.0f));
  const uint64_t t = f2_add(x, f2_make(12582912.0f, 12582912.0f));
  const uint64_t n = f2_add(t, f2_make(-12582912.0f, -12582912.0f));
  const uint64_t f = f2_fma(n, f2_make(-1.0f, -1.0f), x);
  uint64_t p = f2_fma(f2_make(kExp2C3, kExp2C3), f, f2_make(kExp2C2, kExp2C2));
  p = f2_fma(p, f, f2_make(kExp2C1, kExp2C1));
  p = f2_fma(p, f, f2_make(1.0f, 1.0f));
  float p0, p1, t0, t1;
  f2_split(p, p0, p1);
  f2_split(t, t0, t1);
  r0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
  r1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
}

// Row max of N scores: 3-input max over pairs, 8 independent chains.
template <int N>
FA_DEV float row_max(const float (&s)[N]) {
  float mx8[8];
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) mx8[kk] = fmaxf(s[2 * kk], s[2 * kk + 1]);
#pragma unroll
  for (int i = 16; i < N; i += 16)
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) mx8[kk] = fmax3(mx8[kk], s[i + 2 * kk], s[i + 2 * kk + 1]);
  return fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
               fmaxf(mx8[6], mx8[7]));
}

#ifndef FA_LAZY_MAX
#define FA_LAZY_MAX 1
#endif
constexpr bool kLazyMax = FA_LAZY_MAX != 0;
// Largest row sum of one tile's p = 2^(s*c - m) accepted without taking the
// tile's max: p stays far inside the bf16 / fp32 range (2^127).
constexpr float kLazySumLimit = 4294967296.0f;   // 2^32

// p = 2^(s*c - m) for N scores, packed as bf16 pairs into pk; returns the
// row sum.  Two lanes per instruction (the argument and the sums);
// ex2.approx, or the FMA-pipe polynomial for kPolyPer8 keys of 8.
template <int N>
FA_DEV float row_exp2(const float (&s)[N], float c, float m, uint32_t (&pk)[N / 2]) {
  const float m_use = (m == -INFINITY) ? 0.f : m;
  const uint64_t c2 = f2_make(c, c), negm2 = f2_make(-m_use, -m_use);
  uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
  for (int i = 0; i < N / 2; ++i) {
    const int k0 = 2 * i;
    const uint64_t x = f2_fma(f2_make(s[k0], s[k0 + 1]), c2, negm2);
    float p0, p1;
    if ((k0 & 7) >= 8 - kPolyPer8) {
      ex2_poly2(x, p0, p1);
    } else {
      float x0, x1;
      f2_split(x, x0, x1);
      p0 = ex2(x0);
      p1 = ex2(x1);
    }
    acc[i & 3] = f2_add(acc[i & 3], f2_make(p0, p1));
    pk[i] = pack_bf16x2(p0, p1);
  }
  float a0, a1;
  f2_split(f2_add(f2_add(acc[0], acc[1]), f2_add(acc[2], acc[3])), a0, a1);
  return a0 + a1;
}

namespace prefill {

constexpr int BM = 128;                       // query rows per CTA (MMA M)
constexpr int BN = 128;                       // keys per KV tile
constexpr int HD = 128;                       // head dim
constexpr int NSLOT = 5;                      // K/V ring depth
constexpr int TILE_BYTES = BN * HD * 2;       // one K or V tile, 32 KB
constexpr int HALF_BYTES = TILE_BYTES / 2;    // one 64-column TMA box, 16 KB
constexpr int NUM_THREADS = 256;
constexpr int NUM_BARS = 1 + 2 * NSLOT + 2 + 2 + 2 + 1;
constexpr int SMEM_BYTES = 1024 /*align slack*/ + TILE_BYTES /*Q*/ + NSLOT * TILE_BYTES +
                           NUM_BARS * 8 + 16;
constexpr uint32_t TM_S0 = 0, TM_S1 = 128, TM_O = 256, TM_P0 = 384, TM_P1 = 448;
constexpr uint32_t TMEM_COLS = 512;
// Rescale O only when the running max (log2 units) grew by more than this.
constexpr float kRescaleThreshold = 8.0f;
constexpr uint64_t kDrainNs = 200000000ull;  // 0.2 s bound on the abort path

struct Params {
  __nv_bfloat16 *o;
  float *lse;
  const int32_t *row_ptr;  // sparse CSR (nullptr: full mode only)
  const int32_t *col_idx;
  const int32_t *mode;     // per-batch mode on device, or nullptr
  const float *mix_r;      // nullptr, or per-batch weight r: O = r * O_old + (1 - r) * O_new
  // Packed variable-length batch (nullptr: every sequence has length S):
  // sequence b is tokens [cu_seqlens[b], cu_seqlens[b+1]) of [total_tokens, H, D]
  // tensors; `items` lists its query tiles (qt << 12 | b), longest first,
  // and *n_items their count (both written on the device).
  const int32_t *cu_seqlens;
  const int32_t *items;
  const int32_t *n_items;
  int total_tokens;
  int32_t *status;
  int B, S, Hq, G;
  int n_qtiles, nqb;
  int mode_default;
  float scale_log2;        // scale * log2(e)
  int expect_nnz;          // row_ptr[nqb] the CSR must have, or -1 (unchecked)
  int band_q;              // two-tile kernel: q-tiles per band of the KV-head-major item
                           // order, or 0 for the query-tile-major order
};

// The CSR must start at 0 and hold the entry count of the block rule the
// caller configured; one thread of the grid checks it (a mismatch is
// reported; the CSR is still walked as given, entry checks included).
FA_DEV void check_csr_size(const Params &p) {
  if (blockIdx.x == 0 && threadIdx.x == 0 && p.row_ptr != nullptr && p.expect_nnz >= 0) {
    if (p.row_ptr[0] != 0 || p.row_ptr[p.nqb] != p.expect_nnz) report(p.status, FA_DEV_BAD_INDEX);
  }
}

// Writes 32 output columns of one row: o * inv_l as bf16, or, when mix_r is
// given, r * (the bf16 already there) + (1 - r) * o * inv_l (the soft-routing
// mix of the FULL output written by an earlier launch and this SPARSE one).
FA_DEV void store_row_chunk(uint4 *dst, const uint32_t (&o)[32], float inv_l, const float *mix_r,
                            int b) {
  if (mix_r == nullptr) {
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      uint4 w;
      w.x = pack_bf16x2(__uint_as_float(o[8 * v + 0]) * inv_l, __uint_as_float(o[8 * v + 1]) * inv_l);
      w.y = pack_bf16x2(__uint_as_float(o[8 * v + 2]) * inv_l, __uint_as_float(o[8 * v + 3]) * inv_l);
      w.z = pack_bf16x2(__uint_as_float(o[8 * v + 4]) * inv_l, __uint_as_float(o[8 * v + 5]) * inv_l);
      w.w = pack_bf16x2(__uint_as_float(o[8 * v + 6]) * inv_l, __uint_as_float(o[8 * v + 7]) * inv_l);
      dst[v] = w;
    }
    return;
  }
  const float r = mix_r[b], rn = (1.0f - r) * inv_l;
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    const uint4 old = dst[v];
    const uint32_t ow[4] = {old.x, old.y, old.z, old.w};
    uint32_t nw[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float a0 = __uint_as_float(ow[k] << 16), a1 = __uint_as_float(ow[k] & 0xffff0000u);
      nw[k] = pack_bf16x2(fmaf(r, a0, rn * __uint_as_float(o[8 * v + 2 * k])),
                          fmaf(r, a1, rn * __uint_as_float(o[8 * v + 2 * k + 1])));
    }
    dst[v] = make_uint4(nw[0], nw[1], nw[2], nw[3]);
  }
}

// Walks the 128-key tiles a 128-row query tile (query blocks 2qt, 2qt+1)
// attends, ascending, each with a 4-bit block mask: bit 2*qs + ks is set iff
// query block 2qt+qs may attend key block 2n+ks.  FULL mode: tiles 0..qt with
// every bit set.  SPARSE mode: the union of the two CSR rows; an entry outside
// [0, own block] or not ascending is skipped and reported.
struct TileIter {
  const int32_t *col;
  int32_t *status;
  int p0, e0, p1, e1, last0, last1, qb0;
  int n, n_end;
  bool full;

  FA_DEV void init(const Params &p, int qt, bool sparse, int nqb) {
    status = p.status;
    full = !sparse;
    n = 0;
    n_end = qt + 1;
    qb0 = 2 * qt;
    col = p.col_idx;
    last0 = last1 = -1;
    p0 = e0 = p1 = e1 = 0;
    if (sparse) {
      p0 = p.row_ptr[qb0];
      e0 = p.row_ptr[qb0 + 1];
      if (qb0 + 1 < nqb) {
        p1 = e0;
        e1 = p.row_ptr[qb0 + 2];
      }
    }
  }
  FA_DEV int peek(int &pp, int e, int last, int own) {
    while (pp < e) {
      const int c = __ldg(col + pp);
      if (c >= 0 && c <= own && c > last) return c;
      report(status, FA_DEV_BAD_INDEX);
      ++pp;
    }
    return 0x7fffffff;
  }
  FA_DEV bool next(int &tile, uint32_t &bits) {
    if (full) {
      if (n >= n_end) return false;
      tile = n++;
      bits = 0xFu;
      return true;
    }
    int c0 = peek(p0, e0, last0, qb0);
    int c1 = peek(p1, e1, last1, qb0 + 1);
    const int t = min(c0 >> 1, c1 >> 1);
    if (t >= (0x7fffffff >> 1)) return false;
    bits = 0;
    while (c0 >> 1 == t) {
      bits |= 1u << (c0 & 1);
      last0 = c0;
      ++p0;
      c0 = peek(p0, e0, last0, qb0);
    }
    while (c1 >> 1 == t) {
      bits |= 1u << (2 + (c1 & 1));
      last1 = c1;
      ++p1;
      c1 = peek(p1, e1, last1, qb0 + 1);
    }
    tile = t;
    return true;
  }
};

struct Shared {
  uint8_t *q;
  uint8_t *ring;
  uint64_t *q_full, *full, *empty, *s_full, *p_full, *pv_done, *drain;
  uint32_t *tmem_slot;
  volatile int *abort;
};

FA_DEV Shared carve(uint8_t *raw) {
  Shared s;
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  s.q = base;
  s.ring = base + TILE_BYTES;
  uint64_t *bars = reinterpret_cast<uint64_t *>(base + TILE_BYTES + NSLOT * TILE_BYTES);
  s.q_full = bars;
  s.full = bars + 1;
  s.empty = s.full + NSLOT;
  s.s_full = s.empty + NSLOT;
  s.p_full = s.s_full + 2;
  s.pv_done = s.p_full + 2;
  s.drain = s.pv_done + 2;
  s.tmem_slot = reinterpret_cast<uint32_t *>(s.drain + 1);
  s.abort = reinterpret_cast<volatile int *>(s.tmem_slot + 1);
  return s;
}

// ------------------------------------------------------------- producer ---
// Returns the number of ring loads issued (the abort path drains them and
// the Q load), or -1 if it issued nothing at all.
FA_DEV int run_producer(const Shared &sh, const CUtensorMap *tmQ, const CUtensorMap *tmK,
                        const CUtensorMap *tmV, const Params &p, int qt, int b, int h,
                        int kvh, bool sparse) {
  if (c_skip_loads) return -1;   // testing mode: no loads, every wait runs out
  mbar_arrive_expect_tx(sh.q_full, TILE_BYTES);
  tma_load_4d(sh.q, tmQ, sh.q_full, 0, h, qt * BM, b);
  tma_load_4d(sh.q + HALF_BYTES, tmQ, sh.q_full, 64, h, qt * BM, b);

  TileIter it;
  it.init(p, qt, sparse, p.nqb);
  int li = 0;  // loads issued, in consumption order
  auto load = [&](const CUtensorMap *map, int n) -> bool {
    const int slot = li % NSLOT;
    const uint32_t round = static_cast<uint32_t>(li / NSLOT);
    if (!mbar_wait(&sh.empty[slot], (round & 1u) ^ 1u, sh.abort, p.status)) return false;
    uint8_t *dst = sh.ring + slot * TILE_BYTES;
    mbar_arrive_expect_tx(&sh.full[slot], TILE_BYTES);
    tma_load_4d(dst, map, &sh.full[slot], 0, kvh, n * BN, b);
    tma_load_4d(dst + HALF_BYTES, map, &sh.full[slot], 64, kvh, n * BN, b);
    ++li;
    return true;
  };
  int n_cur = 0;
  uint32_t bits;
  bool has = it.next(n_cur, bits);
  bool ok = !has || load(tmK, n_cur);
  while (ok && has) {
    int n_next = 0;
    const bool has_next = it.next(n_next, bits);
    if (has_next && !load(tmK, n_next)) break;
    if (!load(tmV, n_cur)) break;
    n_cur = n_next;
    has = has_next;
  }
  return li;
}

// ------------------------------------------------------------------ MMA ---
FA_DEV void run_mma(const Shared &sh, uint32_t tmem, const Params &p, int qt, bool sparse) {
  constexpr uint32_t kIdescQK = idesc_bf16_f32(BM, BN, false);  // B = K tile, K-major
  constexpr uint32_t kIdescPV = idesc_bf16_f32(BM, HD, true);   // B = V tile, MN-major
  bool ok = mbar_wait(sh.q_full, 0, sh.abort, p.status);
  tc_fence_after_sync();
  const uint32_t q_addr = smem_u32(sh.q);
  int ci = 0;  // ring slots consumed
  auto qk = [&](int j) -> bool {
    const int slot = ci % NSLOT;
    const uint32_t round = static_cast<uint32_t>(ci / NSLOT);
    ++ci;
    if (!mbar_wait(&sh.full[slot], round & 1u, sh.abort, p.status)) return false;
    tc_fence_after_sync();
    const uint32_t k_addr = smem_u32(sh.ring + slot * TILE_BYTES);
    const uint32_t d = tmem + ((j & 1) ? TM_S1 : TM_S0);
#pragma unroll
    for (int kk = 0; kk < HD / 16; ++kk) {
      // 16 bf16 = 32 bytes per K step inside a 128-byte swizzled row; the
      // second 64 columns live in the second TMA box.
      const uint32_t off = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
      mma_bf16_ss(d, smem_desc_sw128(q_addr + off, 16, 1024),
                  smem_desc_sw128(k_addr + off, 16, 1024), kIdescQK, kk > 0 ? 1u : 0u);
    }
    tc_commit(&sh.empty[slot]);
    tc_commit(&sh.s_full[j & 1]);
    return true;
  };
  auto pv = [&](int j) -> bool {
    if (!mbar_wait(&sh.p_full[j & 1], static_cast<uint32_t>(j >> 1) & 1u, sh.abort, p.status))
      return false;
    const int slot = ci % NSLOT;
    const uint32_t round = static_cast<uint32_t>(ci / NSLOT);
    ++ci;
    if (!mbar_wait(&sh.full[slot], round & 1u, sh.abort, p.status)) return false;
    tc_fence_after_sync();
    const uint32_t v_addr = smem_u32(sh.ring + slot * TILE_BYTES);
    const uint32_t a = tmem + ((j & 1) ? TM_P1 : TM_P0);
#pragma unroll
    for (int kk = 0; kk < BN / 16; ++kk) {
      // V tile [key][dim]: dims are the MN (N) mode, keys the K mode.  One K
      // step = 16 keys = two 8-row atoms (2048 bytes); the two 64-dim halves
      // are one TMA box (16 KB) apart (leading byte offset).
      mma_bf16_ts(tmem + TM_O, a + kk * 8, smem_desc_sw128(v_addr + kk * 2048, HALF_BYTES, 1024),
                  kIdescPV, (j > 0 || kk > 0) ? 1u : 0u);
    }
    tc_commit(&sh.empty[slot]);
    tc_commit(&sh.pv_done[j & 1]);
    return true;
  };

  TileIter it;
  it.init(p, qt, sparse, p.nqb);
  int n_cur = 0;
  uint32_t bits;
  bool has = ok && it.next(n_cur, bits);
  if (has) ok = qk(0);
  for (int j = 0; ok && has; ++j) {
    int n_next = 0;
    const bool has_next = it.next(n_next, bits);
    if (has_next && !(ok = qk(j + 1))) break;
    if (!(ok = pv(j))) break;
    has = has_next;
  }
}

// -------------------------------------------------------------- softmax ---
// A wait whose result is the same for every lane of the warp (the TMEM
// loads and stores it guards are warp-collective).
FA_DEV bool warp_wait(uint64_t *bar, uint32_t parity, const Shared &sh, const Params &p) {
  const bool done = mbar_wait(bar, parity, sh.abort, p.status);
  return __all_sync(0xffffffffu, done);
}

// The 128 scores of this thread's row of an S buffer, masked: the 4-bit
// block mask `bits` (sparse tiles) and causality on the diagonal tile.
FA_DEV void load_tile_scores(uint32_t sa, uint32_t bits, bool diag, int r, float (&s)[BN]) {
#pragma unroll
  for (int q4 = 0; q4 < BN / 32; ++q4) {
    uint32_t raw[32];
    tmem_ld32(sa + q4 * 32, raw);
    tmem_ld_wait(raw);
#pragma unroll
    for (int i = 0; i < 32; ++i) s[q4 * 32 + i] = __uint_as_float(raw[i]);
  }
  if (diag || bits != 0xFu) {
    const uint32_t rb = (bits >> ((r >> 6) * 2)) & 3u;
#pragma unroll
    for (int i = 0; i < BN; ++i) {
      const bool keep = ((rb >> (i >> 6)) & 1u) && (!diag || i <= r);
      s[i] = keep ? s[i] : -INFINITY;
    }
  }
}

FA_DEV void run_softmax(const Shared &sh, uint32_t tmem, const Params &p, int qt, int b, int h,
                        bool sparse) {
  const int r = threadIdx.x - 128;                  // row within the tile
  const uint32_t quad = (threadIdx.x >> 5) & 3u;     // TMEM lanes 32*quad..
  const uint32_t lane_base = tmem + ((quad * 32u) << 16);
  const float c = p.scale_log2;
  float m_run = -INFINITY, l_run = 0.f;

  TileIter it;
  it.init(p, qt, sparse, p.nqb);
  int j = 0, n = 0;
  uint32_t bits = 0;
  bool ok = true;
  while (it.next(n, bits)) {
    if (!warp_wait(&sh.s_full[j & 1], static_cast<uint32_t>(j >> 1) & 1u, sh, p)) {
      ok = false;
      break;
    }
    tc_fence_after_sync();
    // Lazy reference max (as in the two-tile kernel): the running max of the
    // earlier tiles, no max over this tile; a row sum past kLazySumLimit (or
    // not finite) means some score rose far above it -- then the warp reads
    // S again, takes the tile's max and redoes the exponentials.  The first
    // tile takes its max first.
    const uint32_t sa = lane_base + ((j & 1) ? TM_S1 : TM_S0);
    const bool diag = (n == qt);
    float m_ref = m_run, m_new = m_run;
    bool need = false;
    uint32_t pk[BN / 2];
    float l_tile;
    {
      float s[BN];
      load_tile_scores(sa, bits, diag, r, s);
      const bool lazy = kLazyMax && !__any_sync(0xffffffffu, m_run == -INFINITY);
      if (!lazy) {
        m_new = fmaxf(m_run, row_max(s) * c);
        need = m_new > m_run + kRescaleThreshold;
        m_ref = need ? m_new : m_run;
      }
      l_tile = row_exp2(s, c, m_ref, pk);
    }
    if (kLazyMax && __any_sync(0xffffffffu, !(l_tile <= kLazySumLimit))) {
      float s[BN];
      load_tile_scores(sa, bits, diag, r, s);
      m_new = fmaxf(m_run, row_max(s) * c);
      need = m_new > m_run;
      m_ref = need ? m_new : m_run;
      l_tile = row_exp2(s, c, m_ref, pk);
    }
    if (j > 0 && __any_sync(0xffffffffu, need)) {
      // O holds sum_{k<j} exp2(s*c - m_run) V; bring it to the new reference.
      // The previous PV must have landed first.
      if (!warp_wait(&sh.pv_done[(j - 1) & 1], static_cast<uint32_t>((j - 1) >> 1) & 1u, sh, p)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      const float alpha = need ? ex2(m_run - m_new) : 1.0f;
#pragma unroll
      for (int q4 = 0; q4 < HD / 32; ++q4) {
        uint32_t o[32];
        tmem_ld32(lane_base + TM_O + q4 * 32, o);
        tmem_ld_wait(o);
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
        tmem_st32(lane_base + TM_O + q4 * 32, o);
      }
      tmem_st_wait();
    }
    if (need) l_run = (m_run == -INFINITY) ? 0.f : l_run * ex2(m_run - m_new);
    m_run = m_ref;
    l_run += l_tile;
    // P buffer j&1 was last read by PV(j-2).
    if (j >= 2 && !warp_wait(&sh.pv_done[j & 1], static_cast<uint32_t>((j - 2) >> 1) & 1u, sh, p)) {
      ok = false;
      break;
    }
    tc_fence_after_sync();
    {
      const uint32_t pa = lane_base + ((j & 1) ? TM_P1 : TM_P0);
      uint32_t lo[32], hi[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        lo[i] = pk[i];
        hi[i] = pk[32 + i];
      }
      tmem_st32(pa, lo);
      tmem_st32(pa + 32, hi);
      tmem_st_wait();
    }
    tc_fence_before_sync();
    mbar_arrive(&sh.p_full[j & 1]);
    ++j;
  }

  // Epilogue: O / l -> bf16, one row per thread.
  const bool have_o =
      ok && j > 0 &&
      warp_wait(&sh.pv_done[(j - 1) & 1], static_cast<uint32_t>((j - 1) >> 1) & 1u, sh, p);
  tc_fence_after_sync();
  const int t = qt * BM + r;
  const bool store = (t < p.S) && !*sh.abort;
  const float inv_l = (l_run > 0.f) ? 1.0f / l_run : 0.f;
  __nv_bfloat16 *orow = p.o + ((static_cast<size_t>(b) * p.S + t) * p.Hq + h) * HD;
#pragma unroll
  for (int q4 = 0; q4 < HD / 32; ++q4) {
    uint32_t o[32];
    if (have_o) {
      tmem_ld32(lane_base + TM_O + q4 * 32, o);
      tmem_ld_wait(o);
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) o[i] = 0u;
    }
    if (store && in_bounds(p.status, ((static_cast<long long>(b) * p.S + t) * p.Hq + h) * HD + q4 * 32,
                           static_cast<long long>(p.B) * p.S * p.Hq * HD)) {
      uint4 *dst = reinterpret_cast<uint4 *>(orow + q4 * 32);
      store_row_chunk(dst, o, inv_l, p.mix_r, b);
    }
  }
  if (store && p.lse &&
      in_bounds(p.status, (static_cast<long long>(b) * p.Hq + h) * p.S + t,
                static_cast<long long>(p.B) * p.Hq * p.S)) {
    const float lse = (l_run > 0.f) ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
    p.lse[(static_cast<size_t>(b) * p.Hq + h) * p.S + t] = lse;
  }
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  const Shared sh = carve(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // CTA -> (query tile, batch, head): longest causal rows first; the query
  // heads of one KV group run side by side so K/V tiles are shared in L2.
  const int bh = p.B * p.Hq;
  const int qt = p.n_qtiles - 1 - static_cast<int>(blockIdx.x) / bh;
  const int rem = static_cast<int>(blockIdx.x) % bh;
  const int b = rem / p.Hq, h = rem % p.Hq, kvh = h / p.G;
  const int mode = p.mode ? p.mode[b] : p.mode_default;
  const bool sparse = (mode == FA_MODE_SPARSE) && p.row_ptr != nullptr;

  if (threadIdx.x == 0) {
    mbar_init(sh.q_full, 1);
    for (int i = 0; i < NSLOT; ++i) {
      mbar_init(&sh.full[i], 1);
      mbar_init(&sh.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sh.s_full[i], 1);
      mbar_init(&sh.p_full[i], 128);
      mbar_init(&sh.pv_done[i], 1);
    }
    mbar_init(sh.drain, 1);
    *sh.abort = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  check_csr_size(p);
  if (warp == 1) {
    tmem_alloc(sh.tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *sh.tmem_slot;

  int loads = 0;
  if (warp == 0) {
    if (lane == 0) loads = run_producer(sh, &tmQ, &tmK, &tmV, p, qt, b, h, kvh, sparse);
  } else if (warp == 1) {
    if (lane == 0) run_mma(sh, tmem, p, qt, sparse);
    __syncwarp();
  } else if (warp >= 4) {
    run_softmax(sh, tmem, p, qt, b, h, sparse);
  }
  tc_fence_before_sync();
  __syncthreads();
  // Every wait of every role is over, so the abort flag is final here.  After
  // an abort, copies and MMAs issued before it may still be in flight: the
  // producer waits (bounded) for its last loads to land and the MMA thread
  // for its MMAs to finish before TMEM is freed and the CTA exits.
  const bool aborted = *sh.abort != 0;
  if (aborted && warp == 0 && lane == 0 && loads >= 0) {
    mbar_wait_drain(sh.q_full, 0, kDrainNs);
    for (int x = (loads > NSLOT ? loads - NSLOT : 0); x < loads; ++x)
      mbar_wait_drain(&sh.full[x % NSLOT], static_cast<uint32_t>(x / NSLOT) & 1u, kDrainNs);
  }
  if (warp == 1) {
    if (aborted && lane == 0) {
      tc_commit(sh.drain);
      mbar_wait_drain(sh.drain, 0, kDrainNs);
    }
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace prefill

// =====================================================================
// Two query tiles per work item: the same 128-row tile of two query heads of
// one GQA group (G even).  The kernel is persistent: one CTA per SM walks its
// share of the items, and the next item's Q/K/V loads and first QK^T overlap
// the current item's epilogue.  Both heads attend the same K/V tiles under the same
// mask, so each K and V tile is loaded once for 256 query rows.
//   warps 0-3   softmax warpgroup of tile 0, warps 4-7 of tile 1
//   warp 8      TMA producer, warp 9 MMA issuer + TMEM owner (10-11 idle)
// TMEM: tile t uses S at columns 256t..256t+127 and O at 256t+128..256t+255;
// P_t (bf16) overwrites the first 64 columns of S_t.  The MMA issue order
//   QK_0(0) QK_1(0) | PV_0(j) QK_0(j+1) PV_1(j) QK_1(j+1) | ...
// makes the tensor core work on one tile while the other tile's softmax
// runs.  MMAs complete in issue order, so "S_t(j) ready" (a commit after
// QK_t(j)) also means PV_t(j-1) has finished: the softmax may rescale O_t
// and overwrite S_t with P_t without any further wait.
// exp2 runs on the special-function unit (ex2.approx) for most keys; a
// polynomial on the FMA pipe takes a share (kPolyPer8 of every 8, in pairs):
// a quarter of the keys by default, which shortens the softmax of a tile
// (the special-function unit alone needs 8 cycles per warp instruction, 1024
// per 128-key row); half the keys there is slower again (the polynomial's
// own instructions then fill the issue slots).
// =====================================================================
namespace prefill2 {

using prefill::Params;
using prefill::TileIter;
constexpr int BM = 128, BN = 128, HD = 128, NQ = 2;
// Epilogue: each softmax warp writes its 32 rows x 32 columns of O (bf16)
// into a staging box in shared memory and one lane stores it with a TMA bulk
// tensor store, instead of 16-byte stores of single rows (each warp-wide
// store instruction of the latter touches 32 rows 8 KB apart).  The staging
// (2 boxes per warp) takes the shared memory of one K/V ring slot.
#ifndef FA_TMA_EPILOGUE
#define FA_TMA_EPILOGUE 1
#endif
constexpr bool kTmaEpilogue = FA_TMA_EPILOGUE != 0;
constexpr int NSLOT = kTmaEpilogue ? 4 : 5;
constexpr int STG_BOX = 32 * 32 * 2;              // 32 rows x 32 bf16 columns
constexpr int STG_BYTES = kTmaEpilogue ? 8 * 2 * STG_BOX : 0;
constexpr int TILE_BYTES = BN * HD * 2;
constexpr int HALF_BYTES = TILE_BYTES / 2;
constexpr int NUM_THREADS = 384;                 // 3 warpgroups
constexpr int WARP_PRODUCER = 8, WARP_MMA = 9;   // warps 10-11 idle
// Register split (setmaxnreg): the two softmax warpgroups grow to
// kSoftmaxRegs, the producer/MMA warpgroup shrinks to kOtherRegs.  The sum
// must not exceed what the block was launched with (384 x the compiled
// count); the launcher checks it before every launch.
constexpr int kSoftmaxRegs = 184, kOtherRegs = 136;
constexpr int NUM_BARS = 2 + 2 * NSLOT + 4 * NQ + 1 + 16;
// For a sparse item the producer, which walks the CSR ahead of everyone to
// load the KV tiles, hands each tile to the MMA and softmax warps through an
// 8-entry ring in shared memory, so they do not walk it themselves:
// (tile << 8) | last << 5 | valid << 4 | 4-bit block mask (0: an item without
// tiles).  A full item's tiles 0..qt need no list.
constexpr int NINFO = 8;
constexpr int SMEM_BYTES =
    1024 + NQ * TILE_BYTES + NSLOT * TILE_BYTES + STG_BYTES + NUM_BARS * 8 + 16 + 4 * NINFO;
static_assert(SMEM_BYTES <= 232448, "shared memory per block");
constexpr uint32_t TMEM_COLS = 512;
constexpr float kRescaleThreshold = 8.0f;
constexpr uint64_t kDrainNs = 200000000ull;

// Shared-memory layout, as offsets from one 1024-byte aligned base:
// Q tiles | K/V ring | epilogue staging | mbarriers | TMEM address | abort word.
struct Smem {
  uint32_t base;
  static constexpr uint32_t kRing = NQ * TILE_BYTES;
  static constexpr uint32_t kStg = kRing + NSLOT * TILE_BYTES;
  static constexpr uint32_t kBars = kStg + STG_BYTES;
  enum : uint32_t {
    Q_FULL = 0, Q_EMPTY = 1, FULL0 = 2, EMPTY0 = FULL0 + NSLOT, S_FULL0 = EMPTY0 + NSLOT,
    P_FULL0 = S_FULL0 + NQ, O_DONE0 = P_FULL0 + NQ, O_FREE0 = O_DONE0 + NQ, DRAIN = O_FREE0 + NQ,
    INFO_FULL0 = DRAIN + 1, INFO_EMPTY0 = INFO_FULL0 + NINFO, NBARS = INFO_EMPTY0 + NINFO
  };
  FA_DEV uint32_t q(int t) const { return base + t * TILE_BYTES; }
  FA_DEV uint32_t ring(int slot) const { return base + kRing + slot * TILE_BYTES; }
  // Staging box `u` (0/1) of softmax warp `w` (0..7).
  FA_DEV uint32_t stg(int w, int u) const { return base + kStg + (2 * w + u) * STG_BOX; }
  FA_DEV uint32_t bar(uint32_t i) const { return base + kBars + 8u * i; }
  FA_DEV uint32_t tmem_slot() const { return base + kBars + 8u * NBARS; }
  FA_DEV uint32_t abort_flag() const { return tmem_slot() + 4u; }
  FA_DEV uint32_t info(int slot) const {
    return base + kBars + 8u * NBARS + 16u + 4u * static_cast<uint32_t>(slot);
  }
};

FA_DEV Smem carve(uint8_t *raw) {
  Smem s;
  s.base = (smem_u32(raw) + 1023u) & ~1023u;
  return s;
}

// Work item -> (query tile, batch, first head of the pair).  Items are
// numbered longest causal rows first.  Two orders:
//  * query-tile-major (band_q = 0): all head pairs of one query tile, then
//    the next tile down; the head pairs of one KV group are adjacent.  The
//    CTAs running together cover every KV head.
//  * KV-head-major bands (long sequences): a band is band_q query tiles; its
//    items are ordered by KV stream (batch, KV head), then query tile, then
//    head pair, so the CTAs running together all stream the K/V tiles of the
//    same KV head, and so do the rounds after them until the band's items of
//    that head run out: the head's K/V stays in L2 instead of being read
//    from HBM again by CTAs that drifted out of L2 reach.  The launcher
//    makes the whole sequence one band.
struct Item {
  int qt, b, h0, kvh;
  bool sparse;
  int L;          // sequence length
  int row0;       // token row of the sequence's first token in Q/K/V/O
  int tma_tok0;   // TMA token coordinate of token 0, and TMA batch coordinate
  int tma_b;
  long long lse0; // LSE index of (head 0, token 0); head stride lse_hs
  int lse_hs;
};
FA_DEV Item item_of(const Params &p, int w) {
  const int hp_count = p.Hq / NQ;
  Item it;
  if (p.cu_seqlens) {
    const int packed = p.items[w / hp_count];
    it.qt = packed >> 12;
    it.b = packed & 4095;
    it.h0 = (w % hp_count) * NQ;
    const int t0 = p.cu_seqlens[it.b];
    it.L = p.cu_seqlens[it.b + 1] - t0;
    it.row0 = t0;
    it.tma_tok0 = t0;
    it.tma_b = 0;
    it.lse0 = t0;
    it.lse_hs = p.total_tokens;
  } else {
    if (p.band_q > 0) {
      const int ppk = p.G / NQ;                       // head pairs per KV head
      const int nkv = p.Hq / p.G;
      const int streams = p.B * nkv;
      const int full_items = p.band_q * ppk * streams;  // items of a full band
      const int full_bands = p.n_qtiles / p.band_q;
      int band, rows, r;
      if (w < full_bands * full_items) {
        band = w / full_items;
        rows = p.band_q;
        r = w % full_items;
      } else {                                        // the last, partial band
        band = full_bands;
        rows = p.n_qtiles - full_bands * p.band_q;
        r = w - full_bands * full_items;
      }
      const int s = r / (rows * ppk), rr = r % (rows * ppk);
      it.qt = p.n_qtiles - 1 - band * p.band_q - rr / ppk;
      it.b = s / nkv;
      it.h0 = (s % nkv) * p.G + (rr % ppk) * NQ;
    } else {
      const int bh = p.B * hp_count;
      it.qt = p.n_qtiles - 1 - w / bh;
      const int rem = w % bh;
      it.b = rem / hp_count;
      it.h0 = (rem % hp_count) * NQ;
    }
    it.L = p.S;
    it.row0 = it.b * p.S;
    it.tma_tok0 = 0;
    it.tma_b = it.b;
    it.lse0 = static_cast<long long>(it.b) * p.Hq * p.S;
    it.lse_hs = p.S;
  }
  it.kvh = it.h0 / p.G;
  const int mode = p.mode ? p.mode[it.b] : p.mode_default;
  it.sparse = (mode == FA_MODE_SPARSE) && p.row_ptr != nullptr;
  return it;
}
FA_DEV int nqb_of(const Item &im) { return (im.L + 63) / 64; }
// The k-th item of this CTA: rounds of gridDim.x items, walked forwards in
// even rounds and backwards in odd ones, so a CTA that drew one of the
// longest items in a round draws one of the shortest in the next.
FA_DEV int item_index(int k, int total) {
  const int G = static_cast<int>(gridDim.x), c = static_cast<int>(blockIdx.x);
  const int w = k * G + ((k & 1) ? (G - 1 - c) : c);
  return w < total ? w : -1;
}

// A wait whose result is the same for every lane of the warp (warp-collective
// instructions follow every wait).
FA_DEV bool warp_wait(uint32_t bar, uint32_t parity, const Smem &sh, const Params &p) {
  const bool done = mbar_wait_a(bar, parity, sh.abort_flag(), p.status);
  return __all_sync(0xffffffffu, done);
}
// The producer and MMA roles run on all 32 lanes of their warp with
// warp-uniform state; one elected lane issues each TMA copy, MMA and commit.
// li / nq: ring loads and Q loads issued (the abort path drains them).
FA_DEV void run_producer(const Smem &sh, const CUtensorMap *tmQ, const CUtensorMap *tmK,
                         const CUtensorMap *tmV, const Params &p, int total, int &li,
                         int &nq) {
  li = 0;           // ring loads issued (continues across items)
  nq = 0;           // Q loads issued
  if (c_skip_loads) return;      // testing mode: no loads, every wait runs out
  int ig = 0;       // tile entries handed to the MMA and softmax warps
  bool ok = true;
  for (int k = 0; ok; ++k) {
    const int w = item_index(k, total);
    if (w < 0) break;
    const Item im = item_of(p, w);
    if (k > 0 && !warp_wait(sh.bar(Smem::Q_EMPTY), static_cast<uint32_t>(k - 1) & 1u, sh, p))
      break;
    mbar_arrive_expect_tx_w(sh.bar(Smem::Q_FULL), NQ * TILE_BYTES);
#pragma unroll
    for (int t = 0; t < NQ; ++t) {
      tma_load_4d_w(sh.q(t), tmQ, sh.bar(Smem::Q_FULL), 0, im.h0 + t,
                    im.tma_tok0 + im.qt * BM, im.tma_b);
      tma_load_4d_w(sh.q(t) + HALF_BYTES, tmQ, sh.bar(Smem::Q_FULL), 64, im.h0 + t,
                    im.tma_tok0 + im.qt * BM, im.tma_b);
    }
    ++nq;
    TileIter it;
    it.init(p, im.qt, im.sparse, nqb_of(im));
    auto publish = [&](int v) -> bool {
      const int slot = ig & (NINFO - 1);
      if (ig >= NINFO &&
          !warp_wait(sh.bar(Smem::INFO_EMPTY0 + slot), static_cast<uint32_t>(ig / NINFO - 1) & 1u,
                     sh, p))
        return false;
      if ((threadIdx.x & 31) == 0) st_shared_s32(sh.info(slot), v);
      __syncwarp();
      if ((threadIdx.x & 31) == 0) mbar_arrive_a(sh.bar(Smem::INFO_FULL0 + slot));
      ++ig;
      return true;
    };
    auto load = [&](const CUtensorMap *map, int n) -> bool {
      const int slot = li % NSLOT;
      const uint32_t round = static_cast<uint32_t>(li / NSLOT);
      if (!warp_wait(sh.bar(Smem::EMPTY0 + slot), (round & 1u) ^ 1u, sh, p)) return false;
      const uint32_t dst = sh.ring(slot), bar = sh.bar(Smem::FULL0 + slot);
      mbar_arrive_expect_tx_w(bar, TILE_BYTES);
      tma_load_4d_w(dst, map, bar, 0, im.kvh, im.tma_tok0 + n * BN, im.tma_b);
      tma_load_4d_w(dst + HALF_BYTES, map, bar, 64, im.kvh, im.tma_tok0 + n * BN, im.tma_b);
      ++li;
      return true;
    };
    int n = 0, n2 = 0;
    uint32_t bits = 0, bits2 = 0;
    bool has = it.next(n, bits);
    if (!has && im.sparse && !(ok = publish(0))) break;
    while (has) {
      const bool has2 = it.next(n2, bits2);
      if ((im.sparse && !publish((n << 8) | (has2 ? 0 : 0x20) | 0x10 | static_cast<int>(bits))) ||
          !load(tmK, n) || !load(tmV, n)) {
        ok = false;
        break;
      }
      n = n2;
      bits = bits2;
      has = has2;
    }
  }
}

// Each product's eight MMAs are issued back to back by one elected lane
// (one election per product rather than per MMA; the issue rate of this
// warp is on the critical path of every tile).
FA_DEV void run_mma(const Smem &sh, uint32_t tmem, const Params &p, int total) {
  constexpr uint32_t kIdescQK = idesc_bf16_f32(BM, BN, false);
  constexpr uint32_t kIdescPV = idesc_bf16_f32(BM, HD, true);
  // Descriptors of the Q tiles (fixed) and of ring slot 0; slot s adds
  // s * TILE_BYTES / 16 to the start-address field, a K step kk adds the
  // byte offset / 16 of its 16-column slice.
  const uint64_t q_desc0 = smem_desc_sw128(sh.q(0), 16, 1024);
  const uint64_t q_desc1 = smem_desc_sw128(sh.q(1), 16, 1024);
  const uint64_t k_desc_base = smem_desc_sw128(sh.ring(0), 16, 1024);
  const uint64_t v_desc_base = smem_desc_sw128(sh.ring(0), HALF_BYTES, 1024);
  int ci = 0;         // ring slots consumed
  int ig = 0;         // tile entries taken from the producer
  // The next tile entry (0 on an abort, with ok = false).
  auto take_info = [&](bool &okk) -> int {
    const int slot = ig & (NINFO - 1);
    if (!warp_wait(sh.bar(Smem::INFO_FULL0 + slot), static_cast<uint32_t>(ig / NINFO) & 1u, sh, p)) {
      okk = false;
      return 0;
    }
    const int v = ld_shared_s32(sh.info(slot));
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive_a(sh.bar(Smem::INFO_EMPTY0 + slot));
    ++ig;
    return v;
  };
  int jp = 0;         // P tiles consumed (per tile index, both advance together)
  int done_items = 0; // items that produced an output (o_done / o_free phases)
  bool ok = true;
  auto take = [&](int &slot) -> bool {
    slot = ci % NSLOT;
    const uint32_t round = static_cast<uint32_t>(ci / NSLOT);
    ++ci;
    if (!warp_wait(sh.bar(Smem::FULL0 + slot), round & 1u, sh, p)) return false;
    tc_fence_after_sync();
    return true;
  };
  auto qk = [&](int t, int slot) {
    const uint64_t qd = t ? q_desc1 : q_desc0;
    const uint64_t kd = k_desc_base + static_cast<uint64_t>(slot * (TILE_BYTES >> 4));
    if (elect_one()) {
#pragma unroll
      for (int kk = 0; kk < HD / 16; ++kk) {
        const uint64_t off = static_cast<uint64_t>(((kk >> 2) * HALF_BYTES + (kk & 3) * 32) >> 4);
        mma_bf16_ss(tmem + 256u * t, qd + off, kd + off, kIdescQK, kk > 0 ? 1u : 0u);
      }
    }
    __syncwarp();
    tc_commit_w(sh.bar(Smem::S_FULL0 + t));
  };
  auto pv = [&](int t, bool first, int slot) -> bool {
    if (!warp_wait(sh.bar(Smem::P_FULL0 + t), static_cast<uint32_t>(jp) & 1u, sh, p))
      return false;
    if (first && done_items > 0 &&
        !warp_wait(sh.bar(Smem::O_FREE0 + t), static_cast<uint32_t>(done_items - 1) & 1u, sh, p))
      return false;
    tc_fence_after_sync();
    const uint64_t vd = v_desc_base + static_cast<uint64_t>(slot * (TILE_BYTES >> 4));
    if (elect_one()) {
#pragma unroll
      for (int kk = 0; kk < BN / 16; ++kk) {
        mma_bf16_ts(tmem + 256u * t + 128u, tmem + 256u * t + kk * 8,
                    vd + static_cast<uint64_t>((kk * 2048) >> 4), kIdescPV,
                    (!first || kk > 0) ? 1u : 0u);
      }
    }
    __syncwarp();
    return true;
  };

  for (int k = 0; ok; ++k) {
    const int w = item_index(k, total);
    if (w < 0) break;
    const Item im = item_of(p, w);
    if (!(ok = warp_wait(sh.bar(Smem::Q_FULL), static_cast<uint32_t>(k) & 1u, sh, p))) break;
    tc_fence_after_sync();
    bool has_next = im.qt > 0, has_next2 = false;     // full item: tiles 0..qt
    if (im.sparse) {
      const int e0 = take_info(ok);
      if (!ok) break;
      if (!(e0 & 0x10)) {             // no KV tile: Q is free again at once
        tc_commit_w(sh.bar(Smem::Q_EMPTY));
        continue;
      }
      has_next = (e0 & 0x20) == 0;
    }
    int k_slot = 0, v_slot = 0;
    if (!(ok = take(k_slot))) break;
    qk(0, k_slot);
    qk(1, k_slot);
    tc_commit_w(sh.bar(Smem::EMPTY0 + k_slot));
    if (!has_next) tc_commit_w(sh.bar(Smem::Q_EMPTY));     // the last QK of this item is issued
    for (int j = 0;; ++j) {
      // V of tile j and K of tile j+1 (the producer is tiles ahead) are taken
      // before the PV waits for P_0, so PV_0(j) and QK_0(j+1) go out back to back.
      if (!(ok = take(v_slot))) break;
      if (has_next) {
        if (im.sparse) {                      // tile j+1: is it the last?
          const int e = take_info(ok);
          if (!ok) break;
          has_next2 = (e & 0x20) == 0;
        } else {
          has_next2 = j + 1 < im.qt;
        }
        if (!(ok = take(k_slot))) break;
      }
      if (!(ok = pv(0, j == 0, v_slot))) break;
      if (has_next) {
        qk(0, k_slot);
      } else {
        tc_commit_w(sh.bar(Smem::O_DONE0));
      }
      if (!(ok = pv(1, j == 0, v_slot))) break;
      ++jp;
      tc_commit_w(sh.bar(Smem::EMPTY0 + v_slot));
      if (!has_next) {
        tc_commit_w(sh.bar(Smem::O_DONE0 + 1));
        break;
      }
      qk(1, k_slot);
      tc_commit_w(sh.bar(Smem::EMPTY0 + k_slot));
      has_next = has_next2;
      if (!has_next) tc_commit_w(sh.bar(Smem::Q_EMPTY));
    }
    ++done_items;
  }
}


// The 128 scores of this thread's row of S_t, masked: the 4-bit block mask
// `bits` (sparse tiles) and causality on the diagonal tile.
FA_DEV void load_scores(uint32_t s_base, uint32_t bits, bool diag, int r, float (&s)[BN]) {
  {
    uint32_t raw[BN];
    tmem_ld128_wait(s_base, raw);
#pragma unroll
    for (int i = 0; i < BN; ++i) s[i] = __uint_as_float(raw[i]);
  }
  if (diag || bits != 0xFu) {
    const uint32_t rb = (bits >> ((r >> 6) * 2)) & 3u;
#pragma unroll
    for (int i = 0; i < BN; ++i) {
      const bool keep = ((rb >> (i >> 6)) & 1u) && (!diag || i <= r);
      s[i] = keep ? s[i] : -INFINITY;
    }
  }
}

// Softmax of one 128-column S tile of head t for the row r of this thread:
// P = 2^(s*c - m) written as bf16 pairs into the first 64 columns of S_t (the
// A operand of the PV product), O rescaled when the reference max moved
// (`rescale_ok`: a PV product of this item has run), running max and sum.
// The reference m: lazily (the default) the running max of the earlier
// tiles, with no max over this tile; the row sum tells when some score rose
// so far above it that p left the safe range (sum > 2^32, or not finite) --
// then the warp reads S again (P is not stored yet), takes the tile's max
// and redoes the exponentials.  An item's first tile takes its max first.
// Eagerly: the tile's max, moved into m only when it passes m by more than
// kRescaleThreshold.
FA_DEV void softmax_tile(uint32_t s_base, uint32_t o_base, uint32_t bits, bool diag, int r,
                         float c, bool rescale_ok, float &m_run, float &l_run) {
  float m_ref = m_run, m_new = m_run;
  bool need = false;
  uint32_t pk[BN / 2];
  float l_tile;
  {
    float s[BN];
    load_scores(s_base, bits, diag, r, s);
    const bool lazy = kLazyMax && !__any_sync(0xffffffffu, m_run == -INFINITY);
    if (!lazy) {
      m_new = fmaxf(m_run, row_max(s) * c);
      need = m_new > m_run + kRescaleThreshold;
      m_ref = need ? m_new : m_run;
    }
    l_tile = row_exp2(s, c, m_ref, pk);
  }
  if (kLazyMax && __any_sync(0xffffffffu, !(l_tile <= kLazySumLimit))) {
    float s[BN];
    load_scores(s_base, bits, diag, r, s);
    m_new = fmaxf(m_run, row_max(s) * c);
    need = m_new > m_run;
    m_ref = need ? m_new : m_run;
    l_tile = row_exp2(s, c, m_ref, pk);
  }
  {
    uint32_t lo[32], hi[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      lo[i] = pk[i];
      hi[i] = pk[32 + i];
    }
    tmem_st32(s_base, lo);
    tmem_st32(s_base + 32, hi);
  }
  // S_t(j) ready implies PV_t(j-1) is done (MMAs complete in order), so
  // O_t may be rescaled here before P_t(j) is released.
  if (rescale_ok && __any_sync(0xffffffffu, need)) {
    const float alpha = need ? ex2(m_run - m_new) : 1.0f;
#pragma unroll
    for (int q4 = 0; q4 < HD / 32; ++q4) {
      uint32_t o[32];
      tmem_ld32(o_base + q4 * 32, o);
      tmem_ld_wait(o);
#pragma unroll
      for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
      tmem_st32(o_base + q4 * 32, o);
    }
  }
  if (need) l_run = (m_run == -INFINITY) ? 0.f : l_run * ex2(m_run - m_new);
  m_run = m_ref;
  l_run += l_tile;
}

FA_DEV void run_softmax(const Smem &sh, uint32_t tmem, const Params &p, const CUtensorMap *tmO,
                        int total, int t) {
  const int r = threadIdx.x - 128 * t;                 // row within the tile
  const uint32_t quad = (threadIdx.x >> 5) & 3u;
  const uint32_t s_base = tmem + ((quad * 32u) << 16) + 256u * t;
  const uint32_t o_base = s_base + 128u;
  const float c = p.scale_log2;
  int js = 0;           // S tiles consumed (continues across items)
  int ig = 0;           // tile entries taken from the producer
  int done_items = 0;   // items whose O this warpgroup has read
  bool ok = true;
  for (int k = 0; ok; ++k) {
    const int w = item_index(k, total);
    if (w < 0) break;
    const Item im = item_of(p, w);
    const int h = im.h0 + t;
    float m_run = -INFINITY, l_run = 0.f;
    int j = 0, n = 0;
    uint32_t bits = 0;
    bool last = false;
    while (!last) {
      if (!im.sparse) {   // a full item: tiles 0..qt
        n = j;
        bits = 0xFu;
        last = j == im.qt;
      } else {   // the next tile from the producer
        const int slot = ig & (NINFO - 1);
        if (!warp_wait(sh.bar(Smem::INFO_FULL0 + slot), static_cast<uint32_t>(ig / NINFO) & 1u, sh,
                       p)) {
          ok = false;
          break;
        }
        const int v = ld_shared_s32(sh.info(slot));
        __syncwarp();
        if ((threadIdx.x & 31) == 0) mbar_arrive_a(sh.bar(Smem::INFO_EMPTY0 + slot));
        ++ig;
        if (!(v & 0x10)) break;       // an item without tiles
        n = v >> 8;
        bits = static_cast<uint32_t>(v) & 15u;
        last = (v & 0x20) != 0;
      }
      if (!warp_wait(sh.bar(Smem::S_FULL0 + t), static_cast<uint32_t>(js) & 1u, sh, p)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      softmax_tile(s_base, o_base, bits, n == im.qt, r, c, j > 0, m_run, l_run);
      tmem_st_wait();
      tc_fence_before_sync();
      __syncwarp();     // one arrive per warp, after all its lanes' P stores
      if ((threadIdx.x & 31) == 0) mbar_arrive_a(sh.bar(Smem::P_FULL0 + t));
      ++j;
      ++js;
    }
    if (!ok) break;

    // Epilogue: read all of O_t at once and hand its TMEM columns back (the
    // next item's first PV may start while this one stores), then O / l ->
    // bf16, one row per thread.
    const bool have_o =
        j > 0 && warp_wait(sh.bar(Smem::O_DONE0 + t), static_cast<uint32_t>(done_items) & 1u, sh, p);
    if (j > 0 && !have_o) break;
    tc_fence_after_sync();
    uint32_t o[HD];
    if (have_o) {
      tmem_ld128_wait(o_base, o);
      tc_fence_before_sync();
      mbar_arrive_a(sh.bar(Smem::O_FREE0 + t));
      ++done_items;
    } else {
#pragma unroll
      for (int i = 0; i < HD; ++i) o[i] = 0u;
    }
    const int tok = im.qt * BM + r;
    // Token rows of O (and LSE entries per head): the packed tensor's, or B * S.
    const long long rows_total =
        p.cu_seqlens ? static_cast<long long>(p.total_tokens) : static_cast<long long>(p.B) * p.S;
    const bool aborted = ld_shared_s32(sh.abort_flag()) != 0;
    const bool store = (tok < im.L) && !aborted;
    const float inv_l = (l_run > 0.f) ? 1.0f / l_run : 0.f;
    __nv_bfloat16 *orow = p.o + ((static_cast<size_t>(im.row0) + tok) * p.Hq + h) * HD;
    // Bulk tensor stores unless the output is mixed into the existing one or
    // the tile of a packed sequence reaches into the next sequence (TMA only
    // clips at the tensor's own end).  Warp-uniform.
    const bool tma = __all_sync(0xffffffffu, kTmaEpilogue && p.mix_r == nullptr && !aborted &&
                                                 (p.cu_seqlens == nullptr ||
                                                  (im.qt + 1) * BM <= im.L));
    const int wq = (threadIdx.x >> 5) & 3;        // rows 32wq .. 32wq+31 of the tile
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int q4 = 0; q4 < HD / 32; ++q4) {
      if (tma) {
        const uint32_t box = sh.stg(4 * t + wq, q4 & 1);
        if (lane == 0) bulk_wait_read1();    // the store that last used this box has read it
        __syncwarp();
        const uint32_t row = box + 64u * static_cast<uint32_t>(lane);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          const uint32_t *ov = o + 32 * q4 + 8 * v;
          const uint32_t w0 = pack_bf16x2(__uint_as_float(ov[0]) * inv_l,
                                          __uint_as_float(ov[1]) * inv_l);
          const uint32_t w1 = pack_bf16x2(__uint_as_float(ov[2]) * inv_l,
                                          __uint_as_float(ov[3]) * inv_l);
          const uint32_t w2 = pack_bf16x2(__uint_as_float(ov[4]) * inv_l,
                                          __uint_as_float(ov[5]) * inv_l);
          const uint32_t w3 = pack_bf16x2(__uint_as_float(ov[6]) * inv_l,
                                          __uint_as_float(ov[7]) * inv_l);
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(row + 16u * v), "r"(w0),
                       "r"(w1), "r"(w2), "r"(w3)
                       : "memory");
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && im.qt * BM + 32 * wq < im.L)   // rows past the end are clipped
          tma_store_4d_commit(tmO, box, q4 * 32, h, im.tma_tok0 + im.qt * BM + 32 * wq, im.tma_b);
      } else if (store && in_bounds(p.status,
                                    ((static_cast<long long>(im.row0) + tok) * p.Hq + h) * HD + q4 * 32,
                                    rows_total * p.Hq * HD)) {
        uint32_t oc[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) oc[i] = o[32 * q4 + i];
        uint4 *dst = reinterpret_cast<uint4 *>(orow + q4 * 32);
        prefill::store_row_chunk(dst, oc, inv_l, p.mix_r, im.b);
      }
    }
    if (store && p.lse &&
        in_bounds(p.status, im.lse0 + static_cast<long long>(h) * im.lse_hs + tok,
                  rows_total * p.Hq)) {
      const float lse = (l_run > 0.f) ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
      p.lse[im.lse0 + static_cast<long long>(h) * im.lse_hs + tok] = lse;
    }
  }
  // Every bulk store of this warp has completed before the CTA exits.
  if (kTmaEpilogue && (threadIdx.x & 31) == 0) bulk_wait_all0();
  __syncwarp();
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    prefill2_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                    const Params p, int total_items) {
  extern __shared__ uint8_t smem_raw[];
  const Smem sh = carve(smem_raw);
  const int warp = threadIdx.x >> 5;

  if (threadIdx.x == 0) {
    mbar_init_a(sh.bar(Smem::Q_FULL), 1);
    mbar_init_a(sh.bar(Smem::Q_EMPTY), 1);
    for (int i = 0; i < NSLOT; ++i) {
      mbar_init_a(sh.bar(Smem::FULL0 + i), 1);
      mbar_init_a(sh.bar(Smem::EMPTY0 + i), 1);
    }
    for (int t = 0; t < NQ; ++t) {
      mbar_init_a(sh.bar(Smem::S_FULL0 + t), 1);
      mbar_init_a(sh.bar(Smem::P_FULL0 + t), 4);     // one arrive per softmax warp
      mbar_init_a(sh.bar(Smem::O_DONE0 + t), 1);
      mbar_init_a(sh.bar(Smem::O_FREE0 + t), 128);
    }
    mbar_init_a(sh.bar(Smem::DRAIN), 1);
    for (int i = 0; i < NINFO; ++i) {
      mbar_init_a(sh.bar(Smem::INFO_FULL0 + i), 1);
      mbar_init_a(sh.bar(Smem::INFO_EMPTY0 + i), 1 + 8);   // the MMA warp + 8 softmax warps
    }
    st_shared_s32(sh.abort_flag(), 0);
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    if (kTmaEpilogue) tma_prefetch_desc(&tmO);
  }
  prefill::check_csr_size(p);
  if (warp == WARP_MMA) {
    tmem_alloc_a(sh.tmem_slot(), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = static_cast<uint32_t>(ld_shared_s32(sh.tmem_slot()));
  if (p.cu_seqlens) total_items = *p.n_items * (p.Hq / NQ);

  int loads = 0, qloads = 0;
  if (warp >= WARP_PRODUCER) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kOtherRegs));
    if (warp == WARP_PRODUCER) {
      run_producer(sh, &tmQ, &tmK, &tmV, p, total_items, loads, qloads);
    } else if (warp == WARP_MMA) {
      run_mma(sh, tmem, p, total_items);
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kSoftmaxRegs));
    run_softmax(sh, tmem, p, &tmO, total_items, warp >> 2);
  }
  tc_fence_before_sync();
  __syncthreads();
  // Every wait of every role is over, so the abort flag is final here.  After
  // an abort, copies and MMAs issued before it may still be in flight: the
  // producer waits (bounded) for its last loads to land and the MMA warp for
  // its MMAs to finish before TMEM is freed and the CTA exits.
  const bool aborted = ld_shared_s32(sh.abort_flag()) != 0;
  if (aborted && warp == WARP_PRODUCER) {
    if (qloads > 0)
      mbar_wait_drain_a(sh.bar(Smem::Q_FULL), static_cast<uint32_t>(qloads - 1) & 1u, kDrainNs);
    for (int x = (loads > NSLOT ? loads - NSLOT : 0); x < loads; ++x)
      mbar_wait_drain_a(sh.bar(Smem::FULL0 + x % NSLOT), static_cast<uint32_t>(x / NSLOT) & 1u,
                        kDrainNs);
  }
  if (warp == WARP_MMA) {
    if (aborted) {
      tc_commit_w(sh.bar(Smem::DRAIN));
      mbar_wait_drain_a(sh.bar(Smem::DRAIN), 0, kDrainNs);
    }
    tc_fence_after_sync();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// Work items of a packed variable-length batch: the query tiles (qt, b) of
// every sequence, ordered by qt descending (longest causal rows first).  The
// position of (v, b) is the number of tiles with a larger qt plus the number
// of earlier sequences that also have a tile v.  One CTA.
__global__ void __launch_bounds__(1024) varlen_items_kernel(const int32_t *cu, int B, int max_items,
                                                            int32_t *n_items, int32_t *items,
                                                            int32_t *status) {
  __shared__ int nq[4096];
  __shared__ int red_max[32], red_sum[32];
  int my_max = 0, my_sum = 0;
  for (int b = threadIdx.x; b < B; b += 1024) {
    const int L = cu[b + 1] - cu[b];
    const int q = L > 0 ? (L + BM - 1) / BM : 0;
    if (L < 0) report(status, FA_DEV_BAD_INDEX);
    nq[b] = q;
    my_max = max(my_max, q);
    my_sum += q;
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    my_max = max(my_max, __shfl_xor_sync(0xffffffffu, my_max, off));
    my_sum += __shfl_xor_sync(0xffffffffu, my_sum, off);
  }
  if ((threadIdx.x & 31) == 0) {
    red_max[threadIdx.x >> 5] = my_max;
    red_sum[threadIdx.x >> 5] = my_sum;
  }
  __syncthreads();
  int max_nq = 0, total = 0;
  for (int w = 0; w < 32; ++w) {
    max_nq = max(max_nq, red_max[w]);
    total += red_sum[w];
  }
  if (total > max_items) {  // cannot happen with consistent cu_seqlens and total_tokens
    if (threadIdx.x == 0) report(status, FA_DEV_BAD_INDEX);
    total = 0;
  }
  if (threadIdx.x == 0) *n_items = total;
  if (total == 0) return;
  for (int v = threadIdx.x; v < max_nq; v += 1024) {
    int pos = 0;
    for (int b = 0; b < B; ++b) pos += max(0, nq[b] - v - 1);
    for (int b = 0; b < B; ++b)
      if (nq[b] > v && in_bounds(status, pos, max_items)) items[pos++] = (v << 12) | b;
  }
}

}  // namespace prefill2

// ----------------------------------------------------------------- host ---
int set_wait_limit_prefill(uint64_t ns, int skip_loads) { return set_wait_limit_local(ns, skip_loads); }

size_t varlen_workspace_bytes(int B, int total_tokens) {
  const size_t max_items = static_cast<size_t>(total_tokens) / prefill2::BM + B + 1;
  return 256 + 4 * max_items;
}

int launch_prefill(const PrefillLaunch &a, cudaStream_t stream) {
  using namespace prefill;
  const bool varlen = a.cu_seqlens != nullptr;
  CUtensorMap tmQ, tmK, tmV;
  // A packed batch is one sequence of total_tokens rows for the TMA maps.
  const int mB = varlen ? 1 : a.B, mS = varlen ? a.total_tokens : a.S;
  if (make_tmap_bhsd(&tmQ, a.q, mB, mS, a.Hq, 64, BM) != 0) return FA_ERR_CUDA;
  if (make_tmap_bhsd(&tmK, a.k, mB, mS, a.Hkv, 64, BN) != 0) return FA_ERR_CUDA;
  if (make_tmap_bhsd(&tmV, a.v, mB, mS, a.Hkv, 64, BN) != 0) return FA_ERR_CUDA;
  CUtensorMap tmO;   // epilogue stores of the two-tile kernel: 32 columns x 32 rows
  if (make_tmap_bhsd_plain(&tmO, a.o, mB, mS, a.Hq, 32, 32) != 0) return FA_ERR_CUDA;
  const int G = a.Hq / a.Hkv;
  const bool two_tiles = (G % 2) == 0;
  if (two_tiles) {
    // setmaxnreg only redistributes what the block was launched with.
    cudaFuncAttributes fattr;
    if (cudaFuncGetAttributes(&fattr, prefill2::prefill2_kernel) != cudaSuccess)
      return FA_ERR_CUDA;
    if (2 * 128 * prefill2::kSoftmaxRegs + 128 * prefill2::kOtherRegs >
        prefill2::NUM_THREADS * fattr.numRegs)
      return FA_ERR_UNSUPPORTED;
  }
  if (cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           SMEM_BYTES) != cudaSuccess ||
      cudaFuncSetAttribute(prefill2::prefill2_kernel,
                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                           prefill2::SMEM_BYTES) != cudaSuccess)
    return FA_ERR_CUDA;
  Params p;
  p.o = reinterpret_cast<__nv_bfloat16 *>(a.o);
  p.lse = a.lse;
  p.row_ptr = a.row_ptr;
  p.col_idx = a.col_idx;
  p.mode = a.mode_dev;
  p.mix_r = a.mix_r;
  p.status = a.status;
  p.cu_seqlens = a.cu_seqlens;
  p.total_tokens = a.total_tokens;
  p.items = nullptr;
  p.n_items = nullptr;
  p.B = a.B;
  p.S = a.S;
  p.Hq = a.Hq;
  p.G = G;
  p.n_qtiles = (a.S + BM - 1) / BM;
  p.nqb = (a.S + 63) / 64;
  p.mode_default = a.mode_default;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.expect_nnz = (a.expect_nnz >= 0 && a.expect_nnz <= 0x7fffffffLL)
                     ? static_cast<int>(a.expect_nnz) : -1;
  p.band_q = 0;
  long long grid =
      static_cast<long long>(p.n_qtiles) * a.B * (two_tiles ? a.Hq / 2 : a.Hq);
  if (varlen) {
    if (!two_tiles || !a.varlen_ws) return FA_ERR_UNSUPPORTED;
    const long long max_items = static_cast<long long>(a.total_tokens) / BM + a.B + 1;
    if (max_items >= (1ll << 19) || a.B > 4096) return FA_ERR_UNSUPPORTED;
    int32_t *ws = reinterpret_cast<int32_t *>(a.varlen_ws);
    p.n_items = ws;
    p.items = ws + 64;
    prefill2::varlen_items_kernel<<<1, 1024, 0, stream>>>(
        a.cu_seqlens, a.B, static_cast<int>(max_items), ws, ws + 64, a.status);
    note_launch();
    if (cudaPeekAtLastError() != cudaSuccess) return FA_ERR_CUDA;
    grid = max_items * (a.Hq / 2);   // upper bound; the kernel reads the real count
  }
  if (grid <= 0 || grid > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  if (two_tiles) {
    // Persistent: one CTA per SM walks the work items.
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return FA_ERR_CUDA;
#ifndef FA_PREFILL_PERSISTENT
#define FA_PREFILL_PERSISTENT 1
#endif
    const long long cap = FA_PREFILL_PERSISTENT ? sms : grid;
    const int ctas = static_cast<int>(grid < cap ? grid : cap);
    // KV-head-major order when the sequence holds at least four rounds of
    // one CTA per SM per KV head (the K/V of one head then no longer fits the
    // L2 share the query-tile-major order leaves it): one band of the whole
    // sequence, so every round streams one KV head after another.  At 256K
    // this read ~200 GB from HBM per FULL launch, against ~480 GB with bands
    // of one round (74 query tiles) and ~900 GB query-tile-major.
#ifndef FA_BAND_ORDER
#define FA_BAND_ORDER 1
#endif
    const int ppk = G / 2;
    const int band = ctas / ppk;
    p.band_q = (FA_BAND_ORDER && !varlen && band >= 1 && p.n_qtiles >= 4 * band) ? p.n_qtiles : 0;
    prefill2::prefill2_kernel<<<ctas, prefill2::NUM_THREADS, prefill2::SMEM_BYTES, stream>>>(
        tmQ, tmK, tmV, tmO, p, static_cast<int>(grid));
    note_launch();
  } else {
    prefill_kernel<<<static_cast<unsigned>(grid), NUM_THREADS, SMEM_BYTES, stream>>>(tmQ, tmK,
                                                                                    tmV, p);
    note_launch();
  }
  return cudaPeekAtLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace fa
