// fa_backward.cu -- gradients of the causal full and block-sparse attention
// (dQ, dK, dV) for an upstream gradient dO of the output; what training the
// router through the soft-routing relaxation ("Flux Attention", router
// paragraphs) differentiates through both attention paths.
//
// With P = softmax(scale * Q K^T) (masked, causal) and O = P V:
//   dV = P^T dO,   dP = dO V^T,   dS = P * (dP - D),  D_t = dO_t . O_t,
//   dQ = scale * dS K,   dK = scale * dS^T Q
// (D_t equals sum_k P_tk dP_tk because O_t = sum_k P_tk v_k.)
//
// Kernels:
//   prep_kernel    D_t and log2(e) * lse_t per (batch, head, token); zeroes
//                  the fp32 dQ accumulator.                      (HBM-bound)
//   csc_*_kernel   for the sparse path: per 128-key tile, the 64-query
//                  blocks whose CSR rows keep one of its two key blocks.
//   bwd_kernel     persistent, one CTA per SM; a work item is one 128-key
//                  tile of one (batch, KV head) (or a chunk of its query
//                  blocks), claimed from a global counter heaviest first, so
//                  CTAs that drew long items take fewer.  It walks the 64-query
//                  blocks that attend the tile, for all G query heads of the
//                  group, with five tcgen05 MMAs per step:
//                    S^T  = K Q^T      (M=128 keys, N=64 queries, K=D)
//                    dP^T = V dO^T     (same shape)
//                    dV  += P^T dO     (A = P^T from TMEM; N=D, K=queries)
//                    dK  += dS^T Q     (A = dS^T from TMEM)
//                    dQ^T = K^T dS^T   (M=D, N=64; A and B MN-major)
//                  dK and dV accumulate in TMEM over the whole item; each
//                  step's dQ^T goes to an fp32 accumulator in HBM through TMA
//                  reduce-adds issued by a separate warpgroup (each warp
//                  stages its 64 x 32 slice in shared memory).  TMEM (512 columns):
//                  S^T x2 (64 each), dP^T/dQ^T x2 (64 each), dV 128, dK 128.
//   convert_kernel dQ = scale * accumulator (+ the router's pooling term),
//                  rounded to bf16.
#include "fa_common.cuh"
#include "fa_internal.h"

namespace fa {
namespace backward {

constexpr int BK = 128;                      // keys per work item
constexpr int BQ = 64;                       // queries per step
constexpr int HD = 128;
constexpr int NST = 3;                       // Q/dO stages
constexpr int NUM_THREADS = 320;             // EW x4 | dQ x4 | producer | MMA
constexpr int WARP_PRODUCER = 8, WARP_MMA = 9;
constexpr int KV_BYTES = BK * HD * 2;        // one K or V tile: 32 KB
constexpr int KV_HALF = KV_BYTES / 2;        // one 64-column TMA box
constexpr int QT_BYTES = BQ * HD * 2;        // one Q or dO tile: 16 KB
constexpr int QT_HALF = QT_BYTES / 2;
constexpr int STAGE_BYTES = 2 * QT_BYTES;    // Q + dO
constexpr int DS_BYTES = BK * BQ * 2;        // one dS^T tile: 16 KB
constexpr int VEC_BYTES = BQ * 4;            // lse2 or D of one step
constexpr int STG_BYTES = BQ * 32 * 4;       // one dQ warp's staging box: 64 x 32 fp32
constexpr uint32_t TMEM_COLS = 512;
constexpr uint64_t kDrainNs = 200000000ull;
constexpr float kLog2e = 1.4426950408889634f;

// Shared memory, offsets from one 1024-byte aligned base:
// K | V | NST x (Q, dO) | 2 x dS^T | 4 x dQ staging | NST x (lse2, D) | barriers |
// TMEM addr | abort.
struct Smem {
  uint32_t base;
  static constexpr uint32_t kK = 0, kV = KV_BYTES, kStages = 2 * KV_BYTES;
  static constexpr uint32_t kDs = kStages + NST * STAGE_BYTES;
  static constexpr uint32_t kStg = kDs + 2 * DS_BYTES;
  static constexpr uint32_t kVec = kStg + 4 * STG_BYTES;
  static constexpr uint32_t kBars = kVec + NST * 2 * VEC_BYTES;
  enum : uint32_t {
    KV_FULL = 0, KV_EMPTY = 1, ST_FULL0 = 2, ST_EMPTY0 = ST_FULL0 + NST,
    S_FULL0 = ST_EMPTY0 + NST, DP_FULL0 = S_FULL0 + 2, EW_DONE0 = DP_FULL0 + 2,
    DQ_FULL0 = EW_DONE0 + 2, DQ_FREE0 = DQ_FULL0 + 2, ACC_FULL = DQ_FREE0 + 2,
    ACC_FREE = ACC_FULL + 1, DRAIN = ACC_FREE + 1, ITEM_FULL0 = DRAIN + 1,
    ITEM_EMPTY0 = ITEM_FULL0 + 4, NBARS = ITEM_EMPTY0 + 4
  };
  FA_DEV uint32_t k() const { return base + kK; }
  FA_DEV uint32_t v() const { return base + kV; }
  FA_DEV uint32_t q(int s) const { return base + kStages + s * STAGE_BYTES; }
  FA_DEV uint32_t dout(int s) const { return q(s) + QT_BYTES; }
  FA_DEV uint32_t ds(int u) const { return base + kDs + u * DS_BYTES; }
  FA_DEV uint32_t stg(int w) const { return base + kStg + w * STG_BYTES; }
  FA_DEV uint32_t lse2(int s) const { return base + kVec + s * 2 * VEC_BYTES; }
  FA_DEV uint32_t dvec(int s) const { return lse2(s) + VEC_BYTES; }
  FA_DEV uint32_t bar(uint32_t i) const { return base + kBars + 8u * i; }
  FA_DEV uint32_t tmem_slot() const { return base + kBars + 8u * NBARS; }
  FA_DEV uint32_t abort_flag() const { return tmem_slot() + 4u; }
  // Work-item ring (NITEM entries) the producer fills for the other roles.
  FA_DEV uint32_t item(int slot) const {
    return tmem_slot() + 16u + 4u * static_cast<uint32_t>(slot);
  }
};
constexpr int NITEM = 4;
constexpr int SMEM_BYTES = 1024 + Smem::kBars + 8 * Smem::NBARS + 16 + 4 * NITEM;
static_assert(SMEM_BYTES <= 232448, "shared memory per block");

struct Params {
  const float *lse2, *dvec;          // [B, Hq, Sp]: log2(e) * lse and D (workspace);
                                     // Sp = S rounded up to 64, pads +inf and 0
  float *dq_acc;                     // [B, Hq, Sp, D] fp32 (workspace)
  __nv_bfloat16 *dk, *dv;            // [B, S, Hkv, D]
  const int32_t *ct_ptr, *ct_q;      // sparse: per key tile, (qb << 2 | key-block bits)
  const int32_t *mode;               // per batch, or nullptr
  int mode_default;
  const float *gscale;               // per batch output factor, or nullptr (1)
  int gscale_complement;             // factor = 1 - gscale[b]
  int accumulate_kv;                 // dK/dV: add into the existing output
  float *dkv_acc;                    // [2, B, Hkv, nkt*128, D] fp32 for split tiles
  int32_t *status;
  int B, S, Sp, Hq, Hkv, G, nqb, nkt;
  int cq_full, cq_sparse, cmax;      // query blocks per chunk (per mode), chunks per tile
  int *item_counter;                 // next unclaimed work item (zeroed before the launch)
  int order;                         // item numbering: kOrderChunk / kOrderTile / kOrderChunkDesc
  float scale, scale_log2;
};

FA_DEV Smem carve(uint8_t *raw) {
  Smem s;
  s.base = (smem_u32(raw) + 1023u) & ~1023u;
  return s;
}

FA_DEV float4 ld_shared_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
FA_DEV void st_shared_u4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}

// Work item w -> (chunk c, key tile, batch, KV head).  A tile's query blocks
// (a descending list) are cut into chunks of at most cq blocks, so no item is
// much longer than the others (the sink tile of the sparse path attends every
// query block); items are numbered chunk index first, key tile next, so the
// CTAs running together work on the same (top) query rows of their lists.  A
// tile with more than one chunk is "split": its chunks add fp32 partial dK/dV
// into dkv_acc, converted after the kernel.
struct Item {
  int kt, b, kvh, nq, ct0, q0, nq_total;
  bool sparse, split;
};
// Work items are claimed in numbering order from a global counter, so each
// CTA takes the next one when it is done (the heaviest items should come
// first).  Numberings:
//  * kOrderChunk: one chunk index across all tiles, then the next -- the full
//    path: chunk 0 holds the last query blocks, which every tile attends (the
//    heaviest), and the CTAs running together reduce into the same dQ rows.
//  * kOrderTile: all chunks of a tile, then the next tile -- the sparse path
//    when the dQ accumulator is small: the sink tiles' chunks (every query
//    block attends them) come first.
//  * kOrderChunkDesc: chunk-major from the last chunk down -- the sparse path
//    with a large accumulator: the sink tiles' later chunks first, and the
//    CTAs still share query rows.
constexpr int kOrderChunk = 0, kOrderTile = 1, kOrderChunkDesc = 2;
FA_DEV int tile_nq(const Params &p, int kt, bool sparse, int &ct0) {
  if (sparse) {
    ct0 = p.ct_ptr[kt];
    return p.ct_ptr[kt + 1] - ct0;
  }
  ct0 = 0;
  return p.nqb - 2 * kt;            // query blocks 2kt .. nqb-1
}
FA_DEV bool batch_sparse(const Params &p, int b) {
  const int mode = p.mode ? p.mode[b] : p.mode_default;
  return (mode == FA_MODE_SPARSE) && p.ct_ptr != nullptr;
}
FA_DEV Item item_of(const Params &p, int w) {
  Item it;
  const int bh = p.B * p.Hkv, per_c = p.nkt * bh;
  int c, rem;
  if (p.order == kOrderTile) {    // all chunks of a tile, then the next tile
    it.kt = w / (p.cmax * bh);
    rem = w % (p.cmax * bh);
    c = rem / bh;
    rem %= bh;
  } else {                        // one chunk index across all tiles, then the next
    c = w / per_c;
    rem = w % per_c;
    it.kt = rem / bh;
    rem %= bh;
    if (p.order == kOrderChunkDesc) c = p.cmax - 1 - c;
  }
  it.b = rem / p.Hkv;
  it.kvh = rem % p.Hkv;
  it.sparse = batch_sparse(p, it.b);
  it.nq_total = tile_nq(p, it.kt, it.sparse, it.ct0);
  const int cq = it.sparse ? p.cq_sparse : p.cq_full;
  it.q0 = c * cq;
  it.nq = max(0, min(cq, it.nq_total - it.q0));
  it.split = it.nq_total > cq;
  return it;
}
// Query block of the item's qi-th step and which of the tile's two key
// blocks it keeps (bit 0: keys 0-63 of the tile, bit 1: keys 64-127).  Steps
// walk the query blocks from the last one down, so the CTAs running at the
// same time sweep the same query rows together and their dQ reductions and
// Q/dO reads stay in L2.
FA_DEV void q_block(const Params &p, const Item &it, int qi, int &qb, uint32_t &bits) {
  const int pos = it.q0 + qi;       // position in the tile's descending list
  if (it.sparse) {
    const int v = p.ct_q[it.ct0 + it.nq_total - 1 - pos];
    qb = v >> 2;
    bits = static_cast<uint32_t>(v) & 3u;
  } else {
    qb = p.nqb - 1 - pos;
    bits = 3u;
  }
}
FA_DEV float out_factor(const Params &p, int b) {
  if (!p.gscale) return 1.0f;
  return p.gscale_complement ? 1.0f - p.gscale[b] : p.gscale[b];
}

FA_DEV bool warp_wait(uint32_t bar, uint32_t parity, const Smem &sh, const Params &p) {
  const bool done = mbar_wait_a(bar, parity, sh.abort_flag(), p.status);
  return __all_sync(0xffffffffu, done);
}

// The k-th work item of this CTA from the producer's ring (-1: no more), or
// -2 after an abort.  One arrive per warp frees the entry.
FA_DEV int next_item(const Smem &sh, const Params &p, int k) {
  const int slot = k & (NITEM - 1);
  if (!warp_wait(sh.bar(Smem::ITEM_FULL0 + slot), static_cast<uint32_t>(k / NITEM) & 1u, sh, p))
    return -2;
  const int w = ld_shared_s32(sh.item(slot));
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive_a(sh.bar(Smem::ITEM_EMPTY0 + slot));
  return w;
}

// ------------------------------------------------------------- producer
// kv_n / li: K/V loads and stage loads issued (the abort path drains them).
FA_DEV void run_producer(const Smem &sh, const CUtensorMap *tmQ, const CUtensorMap *tmO,
                         const CUtensorMap *tmK, const CUtensorMap *tmV, const Params &p,
                         int total, int &kv_n, int &li) {
  kv_n = 0;       // K/V loads issued
  li = 0;         // stage loads issued (continues across items)
  if (c_skip_loads) return;      // testing mode: no loads, every wait runs out
  bool ok = true;
  for (int k = 0; ok; ++k) {
    // Claim the next item that has work (or zero rows to write) from the
    // global counter and publish it to the other roles through the ring.
    int w = 0;
    if ((threadIdx.x & 31) == 0) {
      while (true) {
        w = atomicAdd(p.item_counter, 1);
        if (w >= total) {
          w = -1;
          break;
        }
        const Item t = item_of(p, w);
        if (t.nq > 0 || (t.nq_total == 0 && t.q0 == 0)) break;   // else an empty chunk
      }
    }
    w = __shfl_sync(0xffffffffu, w, 0);
    {
      const int slot = k & (NITEM - 1);
      if (k >= NITEM && !warp_wait(sh.bar(Smem::ITEM_EMPTY0 + slot),
                                   static_cast<uint32_t>(k / NITEM - 1) & 1u, sh, p))
        break;
      if ((threadIdx.x & 31) == 0) st_shared_s32(sh.item(slot), w);
      __syncwarp();
      if ((threadIdx.x & 31) == 0) mbar_arrive_a(sh.bar(Smem::ITEM_FULL0 + slot));
    }
    if (w < 0) break;
    const Item it = item_of(p, w);
    const int n_it = it.nq * p.G;
    if (n_it <= 0) continue;
    if (kv_n > 0 && !warp_wait(sh.bar(Smem::KV_EMPTY), static_cast<uint32_t>(kv_n - 1) & 1u, sh, p))
      break;
    {
      const uint32_t bar = sh.bar(Smem::KV_FULL);
      mbar_arrive_expect_tx_w(bar, 2 * KV_BYTES);
      tma_load_4d_w(sh.k(), tmK, bar, 0, it.kvh, it.kt * BK, it.b);
      tma_load_4d_w(sh.k() + KV_HALF, tmK, bar, 64, it.kvh, it.kt * BK, it.b);
      tma_load_4d_w(sh.v(), tmV, bar, 0, it.kvh, it.kt * BK, it.b);
      tma_load_4d_w(sh.v() + KV_HALF, tmV, bar, 64, it.kvh, it.kt * BK, it.b);
      ++kv_n;
    }
    for (int i = 0; i < n_it; ++i) {
      int qb;
      uint32_t bits;
      q_block(p, it, i / p.G, qb, bits);
      const int h = it.kvh * p.G + i % p.G;
      const int s = li % NST;
      const uint32_t round = static_cast<uint32_t>(li / NST);
      if (!warp_wait(sh.bar(Smem::ST_EMPTY0 + s), (round & 1u) ^ 1u, sh, p)) {
        ok = false;
        break;
      }
      const uint32_t bar = sh.bar(Smem::ST_FULL0 + s);
      mbar_arrive_expect_tx_w(bar, STAGE_BYTES + 2 * VEC_BYTES);
      tma_load_4d_w(sh.q(s), tmQ, bar, 0, h, qb * BQ, it.b);
      tma_load_4d_w(sh.q(s) + QT_HALF, tmQ, bar, 64, h, qb * BQ, it.b);
      tma_load_4d_w(sh.dout(s), tmO, bar, 0, h, qb * BQ, it.b);
      tma_load_4d_w(sh.dout(s) + QT_HALF, tmO, bar, 64, h, qb * BQ, it.b);
      const size_t vo = (static_cast<size_t>(it.b) * p.Hq + h) * p.Sp + static_cast<size_t>(qb) * BQ;
      bulk_load_w(sh.lse2(s), p.lse2 + vo, VEC_BYTES, bar);
      bulk_load_w(sh.dvec(s), p.dvec + vo, VEC_BYTES, bar);
      ++li;
    }
  }
}

// ------------------------------------------------------------------ MMA
// The warp runs warp-wide; each product's MMAs are issued back to back by
// one elected lane (one election per product, not per MMA).
FA_DEV void run_mma(const Smem &sh, uint32_t tmem, const Params &p, int total) {
  constexpr uint32_t kIdS = idesc_bf16_f32_ab(BK, BQ, false, false);   // S^T, dP^T
  constexpr uint32_t kIdKV = idesc_bf16_f32_ab(BK, HD, false, true);   // dV, dK
  constexpr uint32_t kIdQ = idesc_bf16_f32_ab(HD, BQ, true, true);     // dQ^T
  // K-major operands: 128-byte rows, 8-row atoms 1024 bytes apart; a K step
  // of 16 elements is 32 bytes inside a 64-column box.  MN-major operands:
  // 64-element chunks of the M/N dimension one TMA box apart (LBO), groups of
  // 8 K-rows 1024 bytes apart (SBO); a K step of 16 rows is 2048 bytes.
  const uint64_t k_kmaj = smem_desc_sw128(sh.k(), 16, 1024);
  const uint64_t v_kmaj = smem_desc_sw128(sh.v(), 16, 1024);
  const uint64_t k_mn = smem_desc_sw128(sh.k(), KV_HALF, 1024);
  const uint64_t q_kmaj = smem_desc_sw128(sh.q(0), 16, 1024);
  const uint64_t o_kmaj = smem_desc_sw128(sh.dout(0), 16, 1024);
  const uint64_t q_mn = smem_desc_sw128(sh.q(0), QT_HALF, 1024);
  const uint64_t o_mn = smem_desc_sw128(sh.dout(0), QT_HALF, 1024);
  const uint64_t ds_mn = smem_desc_sw128(sh.ds(0), QT_HALF, 1024);
  const uint32_t t_dv = tmem + 256u, t_dk = tmem + 384u;
  int nf = 0, nb = 0;      // steps whose front (S, dP) / back half was issued
  int kv_n = 0, acc_n = 0;
  bool ok = true;

  auto front = [&]() -> bool {
    const int s = nf % NST, u = nf & 1;
    if (!warp_wait(sh.bar(Smem::ST_FULL0 + s), static_cast<uint32_t>(nf / NST) & 1u, sh, p))
      return false;
    tc_fence_after_sync();
    const uint64_t so = static_cast<uint64_t>((s * STAGE_BYTES) >> 4);
    if (elect_one()) {
#pragma unroll
      for (int kk = 0; kk < HD / 16; ++kk) {
        const uint64_t ok_ = static_cast<uint64_t>(((kk >> 2) * KV_HALF + (kk & 3) * 32) >> 4);
        const uint64_t oq = static_cast<uint64_t>(((kk >> 2) * QT_HALF + (kk & 3) * 32) >> 4);
        mma_bf16_ss(tmem + 64u * u, k_kmaj + ok_, q_kmaj + so + oq, kIdS, kk > 0 ? 1u : 0u);
      }
    }
    __syncwarp();
    tc_commit_w(sh.bar(Smem::S_FULL0 + u));
    // dP^T_u is where dQ^T of step nf-2 lives until its readout is done.
    if (nf >= 2 &&
        !warp_wait(sh.bar(Smem::DQ_FREE0 + u), static_cast<uint32_t>((nf >> 1) - 1) & 1u, sh, p))
      return false;
    tc_fence_after_sync();
    if (elect_one()) {
#pragma unroll
      for (int kk = 0; kk < HD / 16; ++kk) {
        const uint64_t ok_ = static_cast<uint64_t>(((kk >> 2) * KV_HALF + (kk & 3) * 32) >> 4);
        const uint64_t oq = static_cast<uint64_t>(((kk >> 2) * QT_HALF + (kk & 3) * 32) >> 4);
        mma_bf16_ss(tmem + 128u + 64u * u, v_kmaj + ok_, o_kmaj + so + oq, kIdS, kk > 0 ? 1u : 0u);
      }
    }
    __syncwarp();
    tc_commit_w(sh.bar(Smem::DP_FULL0 + u));
    ++nf;
    return true;
  };
  auto back = [&](bool first, bool last) -> bool {
    const int s = nb % NST, u = nb & 1;
    if (!warp_wait(sh.bar(Smem::EW_DONE0 + u), static_cast<uint32_t>(nb >> 1) & 1u, sh, p))
      return false;
    if (first && acc_n > 0 &&
        !warp_wait(sh.bar(Smem::ACC_FREE), static_cast<uint32_t>(acc_n - 1) & 1u, sh, p))
      return false;
    tc_fence_after_sync();
    const uint64_t so = static_cast<uint64_t>((s * STAGE_BYTES) >> 4);
    const uint64_t du = static_cast<uint64_t>((u * DS_BYTES) >> 4);
    if (elect_one()) {
#pragma unroll
      for (int kk = 0; kk < BQ / 16; ++kk) {   // dV += P^T dO
        mma_bf16_ts(t_dv, tmem + 64u * u + kk * 8,
                    o_mn + so + static_cast<uint64_t>((kk * 2048) >> 4), kIdKV,
                    (first && kk == 0) ? 0u : 1u);
      }
#pragma unroll
      for (int kk = 0; kk < BQ / 16; ++kk) {   // dK += dS^T Q (dS^T from TMEM)
        mma_bf16_ts(t_dk, tmem + 128u + 64u * u + kk * 8,
                    q_mn + so + static_cast<uint64_t>((kk * 2048) >> 4), kIdKV,
                    (first && kk == 0) ? 0u : 1u);
      }
    }
    __syncwarp();
    tc_commit_w(sh.bar(Smem::ST_EMPTY0 + s));
    if (elect_one()) {
#pragma unroll
      for (int kk = 0; kk < BK / 16; ++kk) {   // dQ^T = K^T dS^T
        mma_bf16_ss(tmem + 128u + 64u * u, k_mn + static_cast<uint64_t>((kk * 2048) >> 4),
                    ds_mn + du + static_cast<uint64_t>((kk * 2048) >> 4), kIdQ, kk > 0 ? 1u : 0u);
      }
    }
    __syncwarp();
    tc_commit_w(sh.bar(Smem::DQ_FULL0 + u));
    if (last) {
      tc_commit_w(sh.bar(Smem::ACC_FULL));
      tc_commit_w(sh.bar(Smem::KV_EMPTY));
    }
    ++nb;
    return true;
  };

  for (int k = 0; ok; ++k) {
    const int w = next_item(sh, p, k);
    if (w == -2) {
      ok = false;
      break;
    }
    if (w < 0) break;
    const Item it = item_of(p, w);
    const int n_it = it.nq * p.G;
    if (n_it <= 0) continue;
    if (!(ok = warp_wait(sh.bar(Smem::KV_FULL), static_cast<uint32_t>(kv_n) & 1u, sh, p))) break;
    tc_fence_after_sync();
    if (!(ok = front())) break;
    for (int i = 0; i < n_it; ++i) {
      if (i + 1 < n_it && !(ok = front())) break;
      if (!(ok = back(i == 0, i + 1 == n_it))) break;
    }
    if (!ok) break;
    ++kv_n;
    ++acc_n;
  }
}

// Rounds 8 fp32 values to bf16 and writes them as one 16-byte chunk.
FA_DEV uint4 pack8(const float *x) {
  return make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                    pack_bf16x2(x[6], x[7]));
}
FA_DEV void unpack8(uint4 v, float *x) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

// One row of dK or dV (128 values in TMEM registers) -> bf16 in HBM.
FA_DEV void store_grad_row(__nv_bfloat16 *dst, const uint32_t (&r)[128], float f, bool acc) {
  uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
  for (int c = 0; c < HD / 8; ++c) {
    float x[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] = __uint_as_float(r[8 * c + e]) * f;
    if (acc) {
      float old[8];
      unpack8(d4[c], old);
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] += old[e];
    }
    d4[c] = pack8(x);
  }
}

// One row of a split tile's dK or dV: fp32 partial sums added into the
// accumulator with 16-byte vector reductions.
FA_DEV void add_grad_row(float *dst, const uint32_t (&r)[128], float f) {
  float4 *d4 = reinterpret_cast<float4 *>(dst);
#pragma unroll
  for (int c = 0; c < HD / 4; ++c)
    atomicAdd(d4 + c, make_float4(__uint_as_float(r[4 * c]) * f, __uint_as_float(r[4 * c + 1]) * f,
                                  __uint_as_float(r[4 * c + 2]) * f,
                                  __uint_as_float(r[4 * c + 3]) * f));
}

// ---------------------------------------- elementwise (one key row per thread)
FA_DEV void run_ew(const Smem &sh, uint32_t tmem, const Params &p, int total) {
  const int r = threadIdx.x;                         // key row within the tile
  const uint32_t lane = ((static_cast<uint32_t>(r) >> 5) * 32u) << 16;
  const float c = p.scale_log2;
  int n = 0, acc_n = 0;
  bool ok = true;
  for (int k = 0; ok; ++k) {
    const int w = next_item(sh, p, k);
    if (w < 0) break;
    const Item it = item_of(p, w);
    const int n_it = it.nq * p.G;
    const int key = it.kt * BK + r;
    const float f = out_factor(p, it.b);
    __nv_bfloat16 *dk_row = p.dk + ((static_cast<size_t>(it.b) * p.S + key) * p.Hkv + it.kvh) * HD;
    __nv_bfloat16 *dv_row = p.dv + ((static_cast<size_t>(it.b) * p.S + key) * p.Hkv + it.kvh) * HD;
    if (n_it <= 0) {          // no query attends this tile: zero gradients
      if (it.nq_total == 0 && key < p.S && !p.accumulate_kv) {
        uint4 *a = reinterpret_cast<uint4 *>(dk_row), *b = reinterpret_cast<uint4 *>(dv_row);
        for (int i = 0; i < HD / 8; ++i) a[i] = b[i] = make_uint4(0u, 0u, 0u, 0u);
      }
      continue;
    }
    for (int i = 0; i < n_it; ++i, ++n) {
      int qb;
      uint32_t bits;
      q_block(p, it, i / p.G, qb, bits);
      const int u = n & 1, s = n % NST;
      const uint32_t ph = static_cast<uint32_t>(n >> 1) & 1u;
      if (!warp_wait(sh.bar(Smem::S_FULL0 + u), ph, sh, p) ||
          !warp_wait(sh.bar(Smem::ST_FULL0 + s), static_cast<uint32_t>(n / NST) & 1u, sh, p)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      const uint32_t t_s = tmem + lane + 64u * u;
      float pv[BQ];
      {
        uint32_t a[32], b[32];
        tmem_ld32(t_s, a);
        tmem_ld32(t_s + 32u, b);
        tmem_ld_wait(a);
        tmem_ld_wait(b);
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          pv[j] = __uint_as_float(a[j]);
          pv[32 + j] = __uint_as_float(b[j]);
        }
      }
      // P = 2^(s * c - lse2) where key <= query and the key block is kept.
      const bool rowbit = ((bits >> (r >> 6)) & 1u) != 0u;
      const int rel = qb * BQ - key;                 // query - key at j = 0
      const bool any = rowbit && (rel + BQ - 1 >= 0);
      const uint32_t lse_s = sh.lse2(s);
#pragma unroll
      for (int j4 = 0; j4 < BQ / 4; ++j4) {
        const float4 L = ld_shared_f4(lse_s + 16u * j4);
        const float l4[4] = {L.x, L.y, L.z, L.w};
#pragma unroll
        for (int e = 0; e < 4; e += 2) {
          const int j = 4 * j4 + e;
          float x0, x1;     // two keys per packed fp32x2 instruction
          f2_split(f2_fma(f2_make(pv[j], pv[j + 1]), f2_make(c, c), f2_make(-l4[e], -l4[e + 1])),
                   x0, x1);
          pv[j] = (any && (j + rel >= 0)) ? ex2(x0) : 0.0f;
          pv[j + 1] = (any && (j + 1 + rel >= 0)) ? ex2(x1) : 0.0f;
        }
      }
      {
        uint32_t pk[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) pk[j] = pack_bf16x2(pv[2 * j], pv[2 * j + 1]);
        tmem_st32(t_s, pk);
      }
      // dS = P (dP - D), into the dS^T tile once MMAs of step n-2 are done with it.
      if (!warp_wait(sh.bar(Smem::DP_FULL0 + u), ph, sh, p) ||
          (n >= 2 && !warp_wait(sh.bar(Smem::DQ_FULL0 + u), static_cast<uint32_t>((n >> 1) - 1) & 1u,
                                sh, p))) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      const uint32_t d_s = sh.dvec(s);
      const uint32_t ds_row = sh.ds(u) + static_cast<uint32_t>(r) * 128u;
#pragma unroll
      for (int hlf = 0; hlf < 2; ++hlf) {
        uint32_t a[32];
        tmem_ld32(tmem + lane + 128u + 64u * u + 32u * hlf, a);
        tmem_ld_wait(a);
        float ds[32];
#pragma unroll
        for (int j4 = 0; j4 < 8; ++j4) {
          const float4 Dv = ld_shared_f4(d_s + 16u * (8 * hlf + j4));
          const float d4[4] = {Dv.x, Dv.y, Dv.z, Dv.w};
#pragma unroll
          for (int e = 0; e < 4; e += 2) {
            const int j = 4 * j4 + e;
            const uint64_t t2 = f2_add(f2_make(__uint_as_float(a[j]), __uint_as_float(a[j + 1])),
                                       f2_make(-d4[e], -d4[e + 1]));
            f2_split(f2_mul(f2_make(pv[32 * hlf + j], pv[32 * hlf + j + 1]), t2), ds[j], ds[j + 1]);
          }
        }
        uint32_t pk[16];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          const uint32_t chunk = static_cast<uint32_t>(4 * hlf + cc);
          const uint4 v = pack8(ds + 8 * cc);
          st_shared_u4(ds_row + ((chunk ^ (static_cast<uint32_t>(r) & 7u)) << 4), v.x, v.y, v.z,
                       v.w);
          pk[4 * cc] = v.x;
          pk[4 * cc + 1] = v.y;
          pk[4 * cc + 2] = v.z;
          pk[4 * cc + 3] = v.w;
        }
        // dS (bf16 pairs) also into the dP columns just read, as the TMEM A
        // operand of dK += dS^T Q.
        tmem_st16(tmem + lane + 128u + 64u * u + 16u * hlf, pk);
      }
      tmem_st_wait();
      fence_proxy_async_smem();
      tc_fence_before_sync();
      __syncwarp();     // one arrive per warp, after all its lanes' stores
      if ((threadIdx.x & 31) == 0) mbar_arrive_a(sh.bar(Smem::EW_DONE0 + u));
    }
    if (!ok) break;
    // Epilogue: dV and scale * dK of this key row.
    if (!warp_wait(sh.bar(Smem::ACC_FULL), static_cast<uint32_t>(acc_n) & 1u, sh, p)) break;
    tc_fence_after_sync();
    bool store = key < p.S && !ld_shared_s32(sh.abort_flag());
    // Debug builds: the gradient row and, for a split tile, its fp32 partial row.
    if (store)
      store = it.split
                  ? in_bounds(p.status, static_cast<long long>(((static_cast<size_t>(it.b) * p.Hkv +
                                                                 it.kvh) * p.nkt * BK + key) * HD),
                              static_cast<long long>(p.B) * p.Hkv * p.nkt * BK * HD)
                  : in_bounds(p.status,
                              ((static_cast<long long>(it.b) * p.S + key) * p.Hkv + it.kvh) * HD,
                              static_cast<long long>(p.B) * p.S * p.Hkv * HD);
    const size_t acc_row = ((static_cast<size_t>(it.b) * p.Hkv + it.kvh) * p.nkt * BK + key) * HD;
    const size_t acc_half = static_cast<size_t>(p.B) * p.Hkv * p.nkt * BK * HD;
    {
      uint32_t a[128];
      tmem_ld128_wait(tmem + lane + 256u, a);
      if (store) {
        if (it.split) add_grad_row(p.dkv_acc + acc_half + acc_row, a, f);
        else store_grad_row(dv_row, a, f, p.accumulate_kv != 0);
      }
    }
    {
      uint32_t a[128];
      tmem_ld128_wait(tmem + lane + 384u, a);
      if (store) {
        if (it.split) add_grad_row(p.dkv_acc + acc_row, a, f * p.scale);
        else store_grad_row(dk_row, a, f * p.scale, p.accumulate_kv != 0);
      }
    }
    tc_fence_before_sync();
    mbar_arrive_a(sh.bar(Smem::ACC_FREE));
    ++acc_n;
  }
}

// ------------------------------------------- dQ readout (one dim per thread)
// Warp w (of 4) holds dims 32w .. 32w+31 of the step's 64 x 128 dQ tile: it
// writes them into its own 64 x 32 staging box and one lane issues a TMA
// reduce-add into the accumulator [B, Hq, Sp, 128]; before the next step
// overwrites the box, the warp waits until that reduce has read it.
FA_DEV void run_dq(const Smem &sh, uint32_t tmem, const CUtensorMap *tmA, const Params &p,
                   int total) {
  const int wq = (threadIdx.x >> 5) & 3, lane_id = threadIdx.x & 31;
  const uint32_t lane = (static_cast<uint32_t>(wq) * 32u) << 16;
  const uint32_t stg = sh.stg(wq) + 4u * static_cast<uint32_t>(lane_id);
  int n = 0;
  bool ok = true;
  for (int k = 0; ok; ++k) {
    const int w = next_item(sh, p, k);
    if (w < 0) break;
    const Item it = item_of(p, w);
    const int n_it = it.nq * p.G;
    const float f = out_factor(p, it.b);
    for (int i = 0; i < n_it; ++i, ++n) {
      int qb;
      uint32_t bits;
      q_block(p, it, i / p.G, qb, bits);
      const int h = it.kvh * p.G + i % p.G;
      const int u = n & 1;
      if (!warp_wait(sh.bar(Smem::DQ_FULL0 + u), static_cast<uint32_t>(n >> 1) & 1u, sh, p)) {
        ok = false;
        break;
      }
      tc_fence_after_sync();
      uint32_t a[32], b[32];
      tmem_ld32(tmem + lane + 128u + 64u * u, a);
      tmem_ld32(tmem + lane + 160u + 64u * u, b);
      tmem_ld_wait(a);
      tmem_ld_wait(b);
      tc_fence_before_sync();
      __syncwarp();
      if ((threadIdx.x & 31) == 0) mbar_arrive_a(sh.bar(Smem::DQ_FREE0 + u));
      bulk_wait_read0();          // the previous reduce has read the staging box
      __syncwarp();
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        asm volatile("st.shared.f32 [%0], %1;" ::"r"(stg + 128u * j),
                     "f"(__uint_as_float(a[j]) * f)
                     : "memory");
        asm volatile("st.shared.f32 [%0], %1;" ::"r"(stg + 128u * (32 + j)),
                     "f"(__uint_as_float(b[j]) * f)
                     : "memory");
      }
      fence_proxy_async_smem();
      __syncwarp();
      const int row = (it.b * p.Hq + h) * p.Sp + qb * BQ;
      tma_reduce_add_2d_w(tmA, sh.stg(wq), 32 * wq, row);
    }
  }
  bulk_wait_all0();               // every reduce of this warp has completed
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmO,
               const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
               const __grid_constant__ CUtensorMap tmA, const Params p, int total_items) {
  extern __shared__ uint8_t smem_raw[];
  const Smem sh = carve(smem_raw);
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init_a(sh.bar(Smem::KV_FULL), 1);
    mbar_init_a(sh.bar(Smem::KV_EMPTY), 1);
    for (int i = 0; i < NST; ++i) {
      mbar_init_a(sh.bar(Smem::ST_FULL0 + i), 1);
      mbar_init_a(sh.bar(Smem::ST_EMPTY0 + i), 1);
    }
    for (int u = 0; u < 2; ++u) {
      mbar_init_a(sh.bar(Smem::S_FULL0 + u), 1);
      mbar_init_a(sh.bar(Smem::DP_FULL0 + u), 1);
      mbar_init_a(sh.bar(Smem::EW_DONE0 + u), 4);     // one arrive per warp
      mbar_init_a(sh.bar(Smem::DQ_FULL0 + u), 1);
      mbar_init_a(sh.bar(Smem::DQ_FREE0 + u), 4);     // one arrive per warp
    }
    mbar_init_a(sh.bar(Smem::ACC_FULL), 1);
    mbar_init_a(sh.bar(Smem::ACC_FREE), 128);
    mbar_init_a(sh.bar(Smem::DRAIN), 1);
    for (int i = 0; i < NITEM; ++i) {
      mbar_init_a(sh.bar(Smem::ITEM_FULL0 + i), 1);
      mbar_init_a(sh.bar(Smem::ITEM_EMPTY0 + i), 9);   // MMA warp, 4 EW and 4 dQ warps
    }
    st_shared_s32(sh.abort_flag(), 0);
    fence_mbar_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmO);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmA);
  }
  if (warp == WARP_MMA) {
    tmem_alloc_a(sh.tmem_slot(), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = static_cast<uint32_t>(ld_shared_s32(sh.tmem_slot()));
  int kv_loads = 0, loads = 0;
  if (warp < 4) {
    run_ew(sh, tmem, p, total_items);
  } else if (warp < 8) {
    run_dq(sh, tmem, &tmA, p, total_items);
  } else if (warp == WARP_PRODUCER) {
    run_producer(sh, &tmQ, &tmO, &tmK, &tmV, p, total_items, kv_loads, loads);
  } else {
    run_mma(sh, tmem, p, total_items);
  }
  tc_fence_before_sync();
  __syncthreads();
  // Every wait of every role is over, so the abort flag is final here.  After
  // an abort, copies and MMAs issued before it may still be in flight: the
  // producer waits (bounded) for its last loads to land and the MMA warp for
  // its MMAs to finish before TMEM is freed and the CTA exits.  (The dQ
  // warps' reduce-adds completed before they left their loop.)
  const bool aborted = ld_shared_s32(sh.abort_flag()) != 0;
  if (aborted && warp == WARP_PRODUCER) {
    if (kv_loads > 0)
      mbar_wait_drain_a(sh.bar(Smem::KV_FULL), static_cast<uint32_t>(kv_loads - 1) & 1u,
                        kDrainNs);
    for (int x = (loads > NST ? loads - NST : 0); x < loads; ++x)
      mbar_wait_drain_a(sh.bar(Smem::ST_FULL0 + x % NST), static_cast<uint32_t>(x / NST) & 1u,
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

// D_t = dO_t . O_t and lse2_t = log2(e) lse_t for every (batch, token, head),
// one warp per row; optionally zeroes the row of the dQ accumulator.  Rows
// t in [S, Sp) of the padded vectors get lse2 = +inf and D = 0, so padded
// query rows have P = 0.
__global__ void __launch_bounds__(256) prep_kernel(const __nv_bfloat16 *o,
                                                   const __nv_bfloat16 *dout, const float *lse,
                                                   int B, int S, int Sp, int Hq, float *dvec,
                                                   float *lse2, float *dq_acc, int zero_acc) {
  const long long prow = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (prow >= static_cast<long long>(B) * Sp * Hq) return;
  {
    const long long h = prow % Hq, bt = prow / Hq, t = bt % Sp, b = bt / Sp;
    if (t >= S) {
      if (lane == 0) {
        dvec[(b * Hq + h) * Sp + t] = 0.f;
        lse2[(b * Hq + h) * Sp + t] = INFINITY;
      }
      if (zero_acc)
        reinterpret_cast<float4 *>(dq_acc + ((b * Hq + h) * Sp + t) * HD)[lane] =
            make_float4(0.f, 0.f, 0.f, 0.f);
      return;
    }
  }
  const long long h_ = prow % Hq, bt_ = prow / Hq, t_ = bt_ % Sp, b_ = bt_ / Sp;
  const long long row = (b_ * S + t_) * Hq + h_;
  const uint2 a = reinterpret_cast<const uint2 *>(o + row * HD)[lane];
  const uint2 g = reinterpret_cast<const uint2 *>(dout + row * HD)[lane];
  float s = __uint_as_float(a.x << 16) * __uint_as_float(g.x << 16);
  s = fmaf(__uint_as_float(a.x & 0xffff0000u), __uint_as_float(g.x & 0xffff0000u), s);
  s = fmaf(__uint_as_float(a.y << 16), __uint_as_float(g.y << 16), s);
  s = fmaf(__uint_as_float(a.y & 0xffff0000u), __uint_as_float(g.y & 0xffff0000u), s);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (zero_acc)
    reinterpret_cast<float4 *>(dq_acc + ((b_ * Hq + h_) * Sp + t_) * HD)[lane] =
        make_float4(0.f, 0.f, 0.f, 0.f);
  if (lane == 0) {
    dvec[(b_ * Hq + h_) * Sp + t_] = s;
    lse2[(b_ * Hq + h_) * Sp + t_] = lse[(b_ * Hq + h_) * S + t_] * kLog2e;
  }
}

// Per 128-key tile kt: the query blocks qb >= 2kt whose CSR row keeps key
// block 2kt (bit 0) or 2kt+1 (bit 1), ascending, as (qb << 2 | bits).  Three
// passes: count per tile (one warp per tile, 32 rows at a time, each lane a
// binary search of its row), an exclusive scan plus the row checks (rows
// must be ascending and inside [0, qb]; a bad row is reported), and the fill
// (the same search, lanes' hits placed in row order with a ballot).
FA_DEV bool row_has(const int32_t *col, int lo, int hi, int c) {
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    const int v = col[mid];
    if (v == c) return true;
    if (v < c) lo = mid + 1; else hi = mid;
  }
  return false;
}
FA_DEV int csc_bits(const int32_t *row_ptr, const int32_t *col_idx, int nqb, int qb, int kt) {
  const int lo = row_ptr[qb], hi = row_ptr[qb + 1];
  int b = row_has(col_idx, lo, hi, 2 * kt) ? 1 : 0;
  if (2 * kt + 1 < nqb && row_has(col_idx, lo, hi, 2 * kt + 1)) b |= 2;
  return b;
}
__global__ void __launch_bounds__(256) csc_count_kernel(const int32_t *row_ptr,
                                                        const int32_t *col_idx, int nqb, int nkt,
                                                        int32_t *cnt) {
  const int kt = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (kt >= nkt) return;
  int c = 0;
  for (int q0 = 2 * kt; q0 < nqb; q0 += 32) {
    const int qb = q0 + lane;
    const bool hit = qb < nqb && csc_bits(row_ptr, col_idx, nqb, qb, kt) != 0;
    c += __popc(__ballot_sync(0xffffffffu, hit));
  }
  if (lane == 0) cnt[kt] = c;
}
__global__ void __launch_bounds__(1024) csc_scan_kernel(const int32_t *row_ptr,
                                                        const int32_t *col_idx, int nqb, int nkt,
                                                        int32_t *ct_ptr, int32_t *status) {
  for (int qb = threadIdx.x; qb < nqb; qb += blockDim.x) {
    int prev = -1;
    for (int e = row_ptr[qb]; e < row_ptr[qb + 1]; ++e) {
      const int c = col_idx[e];
      if (c <= prev || c > qb) {
        report(status, FA_DEV_BAD_INDEX);
        break;
      }
      prev = c;
    }
  }
  // ct_ptr holds the counts on entry; exclusive scan in place (one thread:
  // nkt is at most a few thousand).
  __syncthreads();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int kt = 0; kt < nkt; ++kt) {
      const int c = ct_ptr[kt];
      ct_ptr[kt] = run;
      run += c;
    }
    ct_ptr[nkt] = run;
  }
}
__global__ void __launch_bounds__(256) csc_fill_kernel(const int32_t *row_ptr,
                                                       const int32_t *col_idx, int nqb, int nkt,
                                                       const int32_t *ct_ptr, int32_t *ct_q) {
  const int kt = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (kt >= nkt) return;
  int pos = ct_ptr[kt];
  for (int q0 = 2 * kt; q0 < nqb; q0 += 32) {
    const int qb = q0 + lane;
    const int b = qb < nqb ? csc_bits(row_ptr, col_idx, nqb, qb, kt) : 0;
    const uint32_t m = __ballot_sync(0xffffffffu, b != 0);
    if (b) ct_q[pos + __popc(m & ((1u << lane) - 1u))] = (qb << 2) | b;
    pos += __popc(m);
  }
}

// dQ = scale * accumulator, plus (optionally) the router's pooling gradient
// dx / (n_head + n_tail) on the first n_head and last n_tail tokens; bf16.
// The accumulator is [B, Hq, Sp, D]; dQ is [B, S, Hq, D].
__global__ void __launch_bounds__(256) convert_kernel(const float *acc, __nv_bfloat16 *dq, int B,
                                                      int S, int Sp, int Hq, float scale,
                                                      const float *pool_dx, int n_head,
                                                      int n_tail) {
  const long long n8 = static_cast<long long>(B) * S * Hq * HD / 8;
  const float inv_n = 1.0f / static_cast<float>(n_head + n_tail > 0 ? n_head + n_tail : 1);
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long e = i * 8;                   // element index in [B, S, Hq, D]
    const long long row = e / HD, dd = e % HD;
    const long long h = row % Hq, bt = row / Hq, t = bt % S, bb = bt / S;
    const float *src = acc + ((bb * Hq + h) * Sp + t) * HD + dd;
    const float4 a = reinterpret_cast<const float4 *>(src)[0];
    const float4 b = reinterpret_cast<const float4 *>(src)[1];
    float x[8] = {a.x * scale, a.y * scale, a.z * scale, a.w * scale,
                  b.x * scale, b.y * scale, b.z * scale, b.w * scale};
    if (pool_dx && (t < n_head || t >= S - n_tail)) {
      const float *px = pool_dx + (bb * Hq + h) * HD + dd;
#pragma unroll
      for (int k = 0; k < 8; ++k) x[k] += px[k] * inv_n;
    }
    reinterpret_cast<uint4 *>(dq)[i] = pack8(x);
  }
}

// dK / dV of split tiles: bf16 of the fp32 accumulator (added to the
// existing output when accumulating).  One warp per (batch, key, KV head).
__global__ void __launch_bounds__(256) dkv_convert_kernel(const Params p) {
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= static_cast<long long>(p.B) * p.S * p.Hkv) return;
  const int kvh = static_cast<int>(row % p.Hkv);
  const long long bt = row / p.Hkv;
  const int key = static_cast<int>(bt % p.S), b = static_cast<int>(bt / p.S);
  int ct0;
  const bool sparse = batch_sparse(p, b);
  if (tile_nq(p, key / BK, sparse, ct0) <= (sparse ? p.cq_sparse : p.cq_full)) return;
  const size_t acc_row = ((static_cast<size_t>(b) * p.Hkv + kvh) * p.nkt * BK + key) * HD;
  const size_t acc_half = static_cast<size_t>(p.B) * p.Hkv * p.nkt * BK * HD;
  __nv_bfloat16 *outs[2] = {p.dk, p.dv};
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const float4 a = reinterpret_cast<const float4 *>(p.dkv_acc + t * acc_half + acc_row)[lane];
    float x[4] = {a.x, a.y, a.z, a.w};
    uint2 *dst = reinterpret_cast<uint2 *>(outs[t] + static_cast<size_t>(row) * HD) + lane;
    if (p.accumulate_kv) {
      const uint2 o = *dst;
      x[0] += __uint_as_float(o.x << 16);
      x[1] += __uint_as_float(o.x & 0xffff0000u);
      x[2] += __uint_as_float(o.y << 16);
      x[3] += __uint_as_float(o.y & 0xffff0000u);
    }
    *dst = make_uint2(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]));
  }
}

__global__ void __launch_bounds__(256) zero4_kernel(float4 *x, long long n4) {
  for (long long i = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x; i < n4;
       i += static_cast<long long>(gridDim.x) * 256)
    x[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// dr[b] += sign * sum over (head, token) of D (the padded entries are 0):
// with D = dy . O per row, the FULL pass adds and the SPARSE pass subtracts,
// leaving dr[b] = sum dy * (O_FA - O_SA).
__global__ void __launch_bounds__(256) dsum_kernel(const float *dvec, long long per_b, float sign,
                                                   float *dr) {
  const int b = blockIdx.y;
  const float *src = dvec + b * per_b;
  float s = 0.f;
  for (long long i = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x; i < per_b;
       i += static_cast<long long>(gridDim.x) * 256)
    s += src[i];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  __shared__ float red[8];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < 8; ++w) t += red[w];
    atomicAdd(dr + b, sign * t);
  }
}

__global__ void zero_kernel(float *x, int n) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) x[i] = 0.f;
}

}  // namespace backward

// ----------------------------------------------------------------- host ---
namespace {

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Workspace carve-up of one backward: dQ accumulator, D and lse2 vectors
// (padded to Sp = 64 * nqb per (batch, head)), transposed block pattern.
struct Plan {
  int nqb, nkt, Sp;
  float *acc, *dvec, *lse2, *dkv_acc;
  int32_t *ct_ptr, *ct_q, *counter;
  size_t bytes;
};
Plan make_plan(int B, int S, int Hq, int Hkv, void *workspace) {
  Plan pl;
  pl.nqb = (S + 63) / 64;
  pl.nkt = (pl.nqb + 1) / 2;
  pl.Sp = pl.nqb * 64;
  uint8_t *ws = reinterpret_cast<uint8_t *>(workspace);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t *p = ws ? ws + off : nullptr;
    off += align256(bytes);
    return p;
  };
  pl.acc = reinterpret_cast<float *>(take(static_cast<size_t>(B) * Hq * pl.Sp * backward::HD * 4));
  pl.dvec = reinterpret_cast<float *>(take(static_cast<size_t>(B) * Hq * pl.Sp * 4));
  pl.lse2 = reinterpret_cast<float *>(take(static_cast<size_t>(B) * Hq * pl.Sp * 4));
  pl.ct_ptr = reinterpret_cast<int32_t *>(take((static_cast<size_t>(pl.nkt) + 1) * 4));
  pl.ct_q = reinterpret_cast<int32_t *>(
      take(static_cast<size_t>(pl.nkt) * static_cast<size_t>(pl.nqb) * 4));
  pl.dkv_acc = reinterpret_cast<float *>(
      take(2 * static_cast<size_t>(B) * Hkv * pl.nkt * backward::BK * backward::HD * 4));
  pl.counter = reinterpret_cast<int32_t *>(take(4));
  pl.bytes = off;
  return pl;
}

int sm_count(int *sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return FA_ERR_CUDA;
  return FA_OK;
}

int run_prep(const BackwardLaunch &a, const Plan &pl, cudaStream_t stream) {
  using namespace backward;
  const long long prows = static_cast<long long>(a.B) * pl.Sp * a.Hq;
  prep_kernel<<<static_cast<unsigned>((prows + 7) / 8), 256, 0, stream>>>(
      reinterpret_cast<const __nv_bfloat16 *>(a.o), reinterpret_cast<const __nv_bfloat16 *>(a.dout),
      a.lse, a.B, a.S, pl.Sp, a.Hq, pl.dvec, pl.lse2, pl.acc, a.zero_dq_acc);
  note_launch();
  return cudaPeekAtLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

bool may_be_sparse(const BackwardLaunch &a) {
  return a.row_ptr != nullptr && (a.mode_dev != nullptr || a.mode_default == FA_MODE_SPARSE);
}

int run_csc(const BackwardLaunch &a, const Plan &pl, cudaStream_t stream) {
  using namespace backward;
  const unsigned blocks = static_cast<unsigned>((pl.nkt + 7) / 8);
  csc_count_kernel<<<blocks, 256, 0, stream>>>(a.row_ptr, a.col_idx, pl.nqb, pl.nkt, pl.ct_ptr);
  note_launch();
  if (cudaPeekAtLastError() != cudaSuccess) return FA_ERR_CUDA;
  csc_scan_kernel<<<1, 1024, 0, stream>>>(a.row_ptr, a.col_idx, pl.nqb, pl.nkt, pl.ct_ptr,
                                          a.status);
  note_launch();
  if (cudaPeekAtLastError() != cudaSuccess) return FA_ERR_CUDA;
  csc_fill_kernel<<<blocks, 256, 0, stream>>>(a.row_ptr, a.col_idx, pl.nqb, pl.nkt, pl.ct_ptr,
                                              pl.ct_q);
  note_launch();
  return cudaPeekAtLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int run_main(const BackwardLaunch &a, const Plan &pl, cudaStream_t stream) {
  using namespace backward;
  CUtensorMap tmQ, tmO, tmK, tmV, tmA;
  if (make_tmap_bhsd(&tmQ, a.q, a.B, a.S, a.Hq, 64, BQ) != 0 ||
      make_tmap_bhsd(&tmO, a.dout, a.B, a.S, a.Hq, 64, BQ) != 0 ||
      make_tmap_bhsd(&tmK, a.k, a.B, a.S, a.Hkv, 64, BK) != 0 ||
      make_tmap_bhsd(&tmV, a.v, a.B, a.S, a.Hkv, 64, BK) != 0 ||
      make_tmap_rows_f32(&tmA, pl.acc, static_cast<long long>(a.B) * a.Hq * pl.Sp, 32, BQ) != 0)
    return FA_ERR_CUDA;
  if (cudaFuncSetAttribute(bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) !=
      cudaSuccess)
    return FA_ERR_CUDA;
  const bool sparse = may_be_sparse(a);
  Params p;
  p.lse2 = pl.lse2;
  p.dvec = pl.dvec;
  p.dq_acc = pl.acc;
  p.dk = reinterpret_cast<__nv_bfloat16 *>(a.dk);
  p.dv = reinterpret_cast<__nv_bfloat16 *>(a.dv);
  p.ct_ptr = sparse ? pl.ct_ptr : nullptr;
  p.ct_q = sparse ? pl.ct_q : nullptr;
  p.mode = a.mode_dev;
  p.mode_default = a.mode_default;
  p.gscale = a.gscale;
  p.gscale_complement = a.gscale_complement;
  p.accumulate_kv = a.accumulate_kv;
  p.status = a.status;
  p.B = a.B;
  p.S = a.S;
  p.Sp = pl.Sp;
  p.Hq = a.Hq;
  p.Hkv = a.Hkv;
  p.G = a.Hq / a.Hkv;
  p.nqb = pl.nqb;
  p.nkt = pl.nkt;
  p.scale = a.scale;
  p.scale_log2 = a.scale * kLog2e;
  int sms = 148;
  if (int rc = sm_count(&sms)) return rc;
  // Chunks of at most 32 query blocks (a sixteenth of the sequence's blocks
  // for long sequences).  The sparse path always cuts (its sink tile attends
  // every query block).  The full path keeps whole tiles when its longest
  // tile (nqb blocks) is within one SM's share of all the tiles' blocks and
  // the dQ accumulator is small; with a large accumulator, chunk-major order
  // keeps the CTAs on the same query rows (L2 hits for the reductions).
  const int cq = pl.nqb / 16 > 32 ? pl.nqb / 16 : 32;
  const long long full_blocks =
      static_cast<long long>(a.B) * a.Hkv * (static_cast<long long>(pl.nkt) * pl.nqb -
                                             static_cast<long long>(pl.nkt) * (pl.nkt - 1));
  const long long acc_bytes = static_cast<long long>(a.B) * a.Hq * pl.Sp * HD * 4;
  const bool balanced = static_cast<long long>(pl.nqb) * sms <= full_blocks;
#ifndef FA_BWD_WHOLE_TILE_ACC_MB
#define FA_BWD_WHOLE_TILE_ACC_MB 256
#endif
  p.cq_full = (balanced && acc_bytes <= (static_cast<long long>(FA_BWD_WHOLE_TILE_ACC_MB) << 20))
                  ? pl.nqb : cq;
  // Sparse: at least 64 query blocks per chunk, so a window tile (which at
  // most W/64 + 2 blocks attend) is seldom cut; only the sink tiles are.
  p.cq_sparse = cq > 64 ? cq : 64;
  const bool any_sparse = sparse && (a.mode_dev != nullptr || a.mode_default == FA_MODE_SPARSE);
  const int cq_min =
      any_sparse ? (p.cq_full < p.cq_sparse ? p.cq_full : p.cq_sparse) : p.cq_full;
  p.cmax = (pl.nqb + cq_min - 1) / cq_min;
  p.dkv_acc = pl.dkv_acc;
  p.item_counter = pl.counter;
  p.order = !any_sparse ? kOrderChunk
                        : (acc_bytes <= (256ll << 20) ? kOrderTile : kOrderChunkDesc);
  if (cudaMemsetAsync(pl.counter, 0, sizeof(int32_t), stream) != cudaSuccess) return FA_ERR_CUDA;
  const long long total = static_cast<long long>(p.cmax) * pl.nkt * a.B * a.Hkv;
  if (total <= 0 || total > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  const long long n4 = 2ll * a.B * a.Hkv * pl.nkt * BK * HD / 4;
  if (p.cmax > 1) {
    zero4_kernel<<<static_cast<unsigned>(4 * sms), 256, 0, stream>>>(
        reinterpret_cast<float4 *>(pl.dkv_acc), n4);
    note_launch();
    if (cudaPeekAtLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  const int ctas = static_cast<int>(total < sms ? total : sms);
  bwd_kernel<<<ctas, NUM_THREADS, SMEM_BYTES, stream>>>(tmQ, tmO, tmK, tmV, tmA, p,
                                                        static_cast<int>(total));
  note_launch();
  if (cudaPeekAtLastError() != cudaSuccess) return FA_ERR_CUDA;
  if (p.cmax > 1) {
    const long long rows = static_cast<long long>(a.B) * a.S * a.Hkv;
    dkv_convert_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(p);
    note_launch();
    if (cudaPeekAtLastError() != cudaSuccess) return FA_ERR_CUDA;
  }
  return FA_OK;
}

int run_convert(const BackwardLaunch &a, const Plan &pl, cudaStream_t stream) {
  using namespace backward;
  int sms = 148;
  if (int rc = sm_count(&sms)) return rc;
  const long long n8 = static_cast<long long>(a.B) * a.S * a.Hq * HD / 8;
  const long long blocks = (n8 + 255) / 256;
  convert_kernel<<<static_cast<unsigned>(blocks < 4 * sms ? blocks : 4 * sms), 256, 0, stream>>>(
      pl.acc, reinterpret_cast<__nv_bfloat16 *>(a.dq), a.B, a.S, pl.Sp, a.Hq, a.scale, a.pool_dx,
      a.n_head, a.n_tail);
  note_launch();
  return cudaPeekAtLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace

size_t backward_workspace_bytes(int B, int S, int Hq, int Hkv) {
  return make_plan(B, S, Hq, Hkv, nullptr).bytes;
}

int set_wait_limit_backward(uint64_t ns, int skip_loads) { return set_wait_limit_local(ns, skip_loads); }

int launch_backward(const BackwardLaunch &a, cudaStream_t stream) {
  const Plan pl = make_plan(a.B, a.S, a.Hq, a.Hkv, a.workspace);
  if (int rc = run_prep(a, pl, stream)) return rc;
  if (may_be_sparse(a))
    if (int rc = run_csc(a, pl, stream)) return rc;
  if (int rc = run_main(a, pl, stream)) return rc;
  if (a.convert_dq)
    if (int rc = run_convert(a, pl, stream)) return rc;
  return FA_OK;
}

// Soft-routed layer: y = r O_FA + (1 - r) O_SA, r from the router.  Workspace:
// one attention-backward plan (reused by both passes), the router's forward
// workspace, then x, logits, r, dr, dlogits, da and dx.
namespace {
struct SoftPlan {
  Plan att;
  void *router_ws;
  float *x, *logits, *r, *dr, *dlogits, *da, *dx;
  size_t bytes;
};
SoftPlan make_soft_plan(int B, int S, int Hq, int Hkv, int hidden, void *workspace) {
  SoftPlan sp;
  sp.att = make_plan(B, S, Hq, Hkv, workspace);
  uint8_t *ws = reinterpret_cast<uint8_t *>(workspace);
  size_t off = sp.att.bytes;
  auto take = [&](size_t bytes) {
    uint8_t *p = ws ? ws + off : nullptr;
    off += align256(bytes);
    return p;
  };
  const size_t in_f = static_cast<size_t>(Hq) * backward::HD;
  sp.router_ws = take(router_workspace_bytes(B, Hq, backward::HD, hidden));
  sp.x = reinterpret_cast<float *>(take(B * in_f * 4));
  sp.logits = reinterpret_cast<float *>(take(static_cast<size_t>(B) * 2 * 4));
  sp.r = reinterpret_cast<float *>(take(static_cast<size_t>(B) * 4));
  sp.dr = reinterpret_cast<float *>(take(static_cast<size_t>(B) * 4));
  sp.dlogits = reinterpret_cast<float *>(take(static_cast<size_t>(B) * 2 * 4));
  sp.da = reinterpret_cast<float *>(take(static_cast<size_t>(B) * hidden * 4));
  sp.dx = reinterpret_cast<float *>(take(B * in_f * 4));
  sp.bytes = off;
  return sp;
}
}  // namespace

size_t soft_backward_workspace_bytes(int B, int S, int Hq, int Hkv, int hidden) {
  return make_soft_plan(B, S, Hq, Hkv, hidden, nullptr).bytes;
}

int launch_soft_backward(const SoftBackwardLaunch &a, cudaStream_t stream) {
  using namespace backward;
  const SoftPlan sp = make_soft_plan(a.B, a.S, a.Hq, a.Hkv, a.hidden, a.workspace);
  constexpr int kHead = 100, kTail = 100;
  // Router forward again: pooling slices, ReLU outputs, logits, r.
  RouterLaunch rl{a.q, a.B, a.S, a.Hq, kHead, kTail, a.w1, a.b1, a.w2, a.b2, a.hidden,
                  sp.logits, nullptr, sp.router_ws};
  if (int rc = launch_router(rl, stream)) return rc;
  float *r = a.r_out ? a.r_out : sp.r;
  if (int rc = launch_router_soft(sp.logits, a.gumbel, a.B, a.tau, r, stream)) return rc;
  zero_kernel<<<(a.B + 255) / 256, 256, 0, stream>>>(sp.dr, a.B);
  note_launch();
  if (cudaPeekAtLastError() != cudaSuccess) return FA_ERR_CUDA;
  const long long per_b = static_cast<long long>(a.Hq) * sp.att.Sp;
  const unsigned dsum_blocks = static_cast<unsigned>(per_b / 4096 + 1 < 64 ? per_b / 4096 + 1 : 64);

  // FULL path, upstream r dy: dK/dV written, dQ accumulated (zeroed first).
  BackwardLaunch fa{a.q, a.k, a.v, a.o_full, a.dy, a.lse_full, a.dq, a.dk, a.dv, a.B, a.S, a.Hq,
                    a.Hkv, a.scale, nullptr, nullptr, nullptr, FA_MODE_FULL, a.status,
                    a.workspace};
  fa.gscale = r;
  fa.zero_dq_acc = 1;
  if (int rc = run_prep(fa, sp.att, stream)) return rc;
  dsum_kernel<<<dim3(dsum_blocks, a.B), 256, 0, stream>>>(sp.att.dvec, per_b, 1.0f, sp.dr);
  note_launch();
  if (cudaPeekAtLastError() != cudaSuccess) return FA_ERR_CUDA;
  if (int rc = run_main(fa, sp.att, stream)) return rc;

  // SPARSE path, upstream (1 - r) dy: dK/dV added, dQ accumulated.
  BackwardLaunch sa{a.q, a.k, a.v, a.o_sparse, a.dy, a.lse_sparse, a.dq, a.dk, a.dv, a.B, a.S,
                    a.Hq, a.Hkv, a.scale, a.row_ptr, a.col_idx, nullptr, FA_MODE_SPARSE,
                    a.status, a.workspace};
  sa.gscale = r;
  sa.gscale_complement = 1;
  sa.accumulate_kv = 1;
  sa.zero_dq_acc = 0;
  if (int rc = run_prep(sa, sp.att, stream)) return rc;
  dsum_kernel<<<dim3(dsum_blocks, a.B), 256, 0, stream>>>(sp.att.dvec, per_b, -1.0f, sp.dr);
  note_launch();
  if (cudaPeekAtLastError() != cudaSuccess) return FA_ERR_CUDA;
  if (int rc = run_csc(sa, sp.att, stream)) return rc;
  if (int rc = run_main(sa, sp.att, stream)) return rc;

  // Router: dr -> dlogits -> dW2, db2, dW1, db1 and the pooled-input gradient.
  RouterBwdLaunch rb{sp.logits, a.gumbel, a.tau, sp.dr, sp.router_ws, a.w1, a.w2, a.B, a.Hq,
                     a.hidden, kHead + kTail, sp.x, sp.dlogits, sp.da, sp.dx, a.dw1, a.db1,
                     a.dw2, a.db2};
  if (int rc = launch_router_backward(rb, stream)) return rc;

  // dQ = scale * (accumulated r dQ_FA + (1 - r) dQ_SA) + pooling term.
  sa.pool_dx = sp.dx;
  sa.n_head = kHead;
  sa.n_tail = kTail;
  return run_convert(sa, sp.att, stream);
}

}  // namespace fa
