// sa_pyr_fwd.cuh — PSA multi-level (pyramid) attention forward for sm_100a.
//
// PSA page ("浙江大学突破视频AI瓶颈:金字塔方法提升视频AI效率10倍"): every
// (q-block, k-block) pair is attended at a level l of the pooled KV pyramid,
// and a pooled key that stands for n tokens gets + ln(n) on its logit so the
// probability distribution matches full attention over those tokens.  Its
// "decoupled block-tile" kernel lets logical blocks of different sizes share
// full hardware tiles; here that is done by packing.
//
// Packing: for each 128-row q-tile (one q-block for block 128, two for block
// 64), the kept (k-block j, level l) pairs become segments of BLK >> l pooled
// keys.  Segments are sorted by level, so their lengths are non-increasing
// powers of two that divide 128: they fill 128-key tiles exactly, and no
// segment crosses a tile edge.  With block 64 the two q-blocks of a tile take
// the union of their (j, l) pairs; a segment carries a row mask (which of
// the two q-blocks uses it) that becomes a masking bias for the other rows.
//
// One CTA = two q-tiles with the same roles and TMEM layout as
// sa_attn_fwd.cuh (warp 0 issues every S into the one S buffer, warps 1 and 2
// issue the PV of q-tile 0 / 1, one softmax thread per row, P handed over in
// two halves through named barriers), but each q-tile has its own packed key
// tiles; the entries of the two are interleaved and each entry feeds one
// q-tile.  Warp 3 is the producer: K segments arrive by TMA from one tensor
// map per pyramid level (level 0 is the original K/V) into a 2-slot ring;
// the PV warps gather the V segments of their own next key tile the same way.
// Columns no segment covers are zero-filled so that masked products stay
// finite.  The bias is not added by the softmax: S gets it from one extra
// K = 16 MMA step whose A operand (QX) selects, per q row, the pair of
// columns of its q-block and whose B operand (KX, written per K slot by the
// producer) holds, per key column, the bias in raw logit units as bf16
// hi + lo: ln(count) / scale, or a large negative value where the column is
// masked for that q-block or empty.  The softmax then works on S alone,
// x = s * scale * log2(e), exactly as in the attention kernel.
#pragma once

#include "sa_attn_fwd.cuh"

namespace sa {

constexpr int kPyrMaxBlocks = 1024;                 // k-blocks per sequence
// 12 warps: S issuer, two PV issuers, producer, two softmax warpgroups
constexpr int kPyrWarps = 12;
constexpr int kPyrThreads = kPyrWarps * 32;
constexpr int kPyrMaxSegs = 2 * kPyrMaxBlocks;      // per q-tile (union of 2 q-blocks)
constexpr int kPyrMaxEntries = kPyrMaxBlocks;       // packed key tiles per q-tile
// Entry word of a packed key tile: index of its first segment (bits 0-10),
// uniform flag (bit 11: every segment has the same level and row mask and
// holds full groups, so the bias is one constant per q-block), level (bits
// 12-13) and row mask (bits 14-15) of its first segment.
constexpr uint32_t kEntStartMask = 0x7FFu;
constexpr uint32_t kEntUniform = 1u << 11;
// Raw-logit bias of a masked or empty column, and the row maximum below which
// a row has no valid column in a tile (real logits are many orders smaller).
constexpr float kMaskedBias = -30000.f;
constexpr float kMaskedCut = -10000.f;

struct PyrParams {
  int B, H, N;
  int nb;                 // blocks per sequence
  const uint8_t* levels;  // code map: 0 drop, 1 + l level l
  long long lsb, lsh, lsi;
  float scale_log2;
  int n_pairs;            // q-tile pairs per head
  int n_full;             // CTAs [0, n_full) take a whole pair; each later pair runs as two CTAs, one per q-tile
  __nv_bfloat16* o;
  float* lse;
};

template <int D>
struct PyrSmem {
  static constexpr int kTileBytes = kTileM * D * 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = 2 * kTileBytes;
  static constexpr int kOffV = kOffK + kStages * kTileBytes;
  static constexpr int kOffSeg = kOffV + kStages * kTileBytes;         // [tile][kPyrMaxSegs] u32
  static constexpr int kOffEnt = kOffSeg + 2 * kPyrMaxSegs * 4;        // [tile][kPyrMaxEntries] u16
  // The logit bias enters S through one extra K = 16 MMA step: QX holds, per
  // q row, selector columns (1, 1 on the pair of its q-block), KX per K slot
  // holds, per key column, the bias in raw logit units split into bf16
  // hi + lo for each q-block.  Both are 128 x 16 bf16 in the K-major
  // no-swizzle layout: element (r, c) at (r/8)*256 + (c/8)*128 + (r%8)*16 + (c%8)*2.
  static constexpr int kOffQX = (kOffEnt + 2 * kPyrMaxEntries * 2 + 1023) / 1024 * 1024;
  static constexpr int kOffKX = kOffQX + 4096;                          // [slot] 4 KB
  // q_full, k_full[2], v_full[2][2], k_empty[2], v_empty[2][2], s_ready[2],
  // pv_done_a[2], pv_done_b[2], o_final[2], mma_done[3]
  // (V slots are filled and released by 64-key half: rows [0,64) feed the
  // first half of PV, rows [64,128) the second)
  static constexpr int kNumBars = 1 + 6 * kStages + 2 * 4 + 3;
  static constexpr int kOffKXPat = kOffKX + kStages * 4096;             // 17 KX row patterns
  static constexpr int kOffBar = kOffKXPat + 17 * 16;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kBytes = kOffMisc + 128;
  static constexpr int kAlloc = kBytes + 1024;
};

struct PyrMaps {
  CUtensorMap k[4];
  CUtensorMap v[4];
};

template <int D, int BLK, bool CAUSAL>
__global__ void __launch_bounds__(kPyrThreads, 1)
    pyr_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ PyrMaps maps,
                   const PyrParams p) {
  using L = PyrSmem<D>;
  constexpr int QH = kTileM / BLK;
  constexpr uint32_t kIdescS = idesc_bf16_f32(kTileM, kTileN, false);
  constexpr uint32_t kIdescPV = idesc_bf16_f32(kTileM, D, true);
  constexpr int kHalfBytes = kTileM * 128;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint32_t* segs = reinterpret_cast<uint32_t*>(smem + L::kOffSeg);
  uint16_t* ents = reinterpret_cast<uint16_t*>(smem + L::kOffEnt);
  uint8_t* qx = smem + L::kOffQX;
  uint8_t* kx = smem + L::kOffKX;
  uint4* kxpat = reinterpret_cast<uint4*>(smem + L::kOffKXPat);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = bars + 1 + kStages;          // [slot * 2 + half]
  uint64_t* k_empty = bars + 1 + 3 * kStages;
  uint64_t* v_empty = bars + 1 + 4 * kStages;     // [slot * 2 + half]
  uint64_t* s_ready = bars + 1 + 6 * kStages;
  uint64_t* pv_done_a = s_ready + 2;
  uint64_t* pv_done_b = pv_done_a + 2;
  uint64_t* o_final = pv_done_b + 2;
  uint64_t* mma_done = o_final + 2;   // one per MMA-issuing warp
  volatile int* misc = reinterpret_cast<volatile int*>(smem + L::kOffMisc);
  // misc[0] TMEM base, [1]/[2] segments of q-tile 0/1, [3]/[4] key tiles of q-tile 0/1, [5] abort,
  // [6]/[7] packed columns of q-tile 0/1, [8 + 2t + x] causal: key tile * 256 + column of the
  // diagonal segment of q-block x of q-tile t (-1: none), [12 + 2t + x] key tiles of q-tile t
  // holding a segment of the last block (-1: none)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Work unit u = bh * n_pairs + pair, in launch order.  Units from n_full on
  // (the last, partial wave of a launch) run as two CTAs each; a CTA then
  // treats the pair's other q-tile as absent: no segments, no writes.
  int unit = blockIdx.x, skip_t = -1;
  if (unit >= p.n_full) {
    const int x = unit - p.n_full;
    unit = p.n_full + (x >> 1);
    skip_t = 1 - (x & 1);
  }
  const int bh = unit / p.n_pairs, pair = unit - bh * p.n_pairs;
  const int b = bh / p.H, h = bh - (bh / p.H) * p.H;
  const int qtile0 = 2 * pair;

  if (warp == 0 || warp == 3) {
    // ---- the segment list of q-tile t (warp 0: t = 0, warp 3: t = 1) ----
    // Segments are sorted by group: by level (lengths non-increasing, so they
    // fill 128-key tiles exactly) and, within a level, by row mask: used by
    // both q-blocks, by the first only, by the second only (block 128: one
    // group per level); ascending j within a group.  A key tile whose
    // segments all share a group and hold full pooled groups needs no
    // per-column bias (uniform).  Two passes over j: count the segments of
    // each group, then place each one at its group's offset plus its rank.
    const int t = warp == 0 ? 0 : 1;
    constexpr int NR = QH == 2 ? 3 : 1;   // row-mask groups per level
    constexpr int NG = 4 * NR;
    // The level codes of the two q-blocks (after the causal adjustment) and
    // the per-group running offsets are staged in the V ring, unused until
    // the main loop.
    uint8_t* cd = smem + L::kOffV + t * 2 * kPyrMaxBlocks;
    int* gpos = reinterpret_cast<int*>(smem + L::kOffV + 4 * kPyrMaxBlocks + t * 128);
    int* gcol = gpos + 16;
    const int qbA = (qtile0 + t) * QH;
    const int qbB = qbA + QH - 1;
    const bool validA = qbA < p.nb && t != skip_t, validB = qbB < p.nb && t != skip_t;
    for (int j = lane; j < p.nb; j += 32) {
      const long long rowoff = b * p.lsb + h * p.lsh + j;
      int cA = validA ? p.levels[rowoff + qbA * p.lsi] : 0;
      int cB = validB ? p.levels[rowoff + qbB * p.lsi] : 0;
      if (CAUSAL) {
        // blocks after the q-block are dropped; its own block, if kept, is
        // attended at level 0 (its pooled keys would mix in later tokens)
        cA = j > qbA ? 0 : (j == qbA && cA ? 1 : cA);
        cB = j > qbB ? 0 : (j == qbB && cB ? 1 : cB);
      }
      cd[j] = static_cast<uint8_t>(cA);
      cd[kPyrMaxBlocks + j] = static_cast<uint8_t>(cB);
    }
    __syncwarp();
    // group of each of a block's (at most two) segments, -1 for none
    auto groups_of = [&](int j, int& gA, int& gB) {
      gA = -1;
      gB = -1;
      if (j >= p.nb) return;
      const int cA = cd[j], cB = cd[kPyrMaxBlocks + j];
      if (QH == 1 || cA == cB) {
        if (cA) gA = (cA - 1) * NR;
      } else {
        if (cA) gA = (cA - 1) * NR + 1;
        if (cB) gB = (cB - 1) * NR + 2;
      }
    };
    // pass 1: segments per group, as 16-bit fields of three 64-bit words
    unsigned long long cw[3] = {0ull, 0ull, 0ull};
    for (int base = 0; base < p.nb; base += 32) {
      int gA, gB;
      groups_of(base + lane, gA, gB);
#pragma unroll
      for (int w = 0; w < 3; ++w) {
        if (gA >= 0 && (gA >> 2) == w) cw[w] += 1ull << (16 * (gA & 3));
        if (gB >= 0 && (gB >> 2) == w) cw[w] += 1ull << (16 * (gB & 3));
      }
    }
#pragma unroll
    for (int w = 0; w < 3; ++w)
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) cw[w] += __shfl_xor_sync(0xffffffffu, cw[w], o);
    int n = 0, cols = 0;
#pragma unroll
    for (int g = 0; g < NG; ++g) {
      const int c = static_cast<int>((cw[g >> 2] >> (16 * (g & 3))) & 0xFFFFull);
      if (lane == g) {
        gpos[g] = n;
        gcol[g] = cols;
      }
      n += c;
      cols += c * (BLK >> (g / NR));
    }
    if (lane == 0) {
      misc[8 + 2 * t] = -1;
      misc[9 + 2 * t] = -1;
      misc[12 + 2 * t] = -1;
      misc[13 + 2 * t] = -1;
    }
    __syncwarp();
    // pass 2: each segment at its group's running offset plus its rank among
    // the chunk's lanes of the same group (lanes hold ascending j)
    for (int base = 0; base < p.nb; base += 32) {
      const int j = base + lane;
      int gA, gB;
      groups_of(j, gA, gB);
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        const int g = x == 0 ? gA : gB;
        const unsigned peers = __match_any_sync(0xffffffffu, g);
        const int rank = __popc(peers & ((1u << lane) - 1u));
        if (g >= 0) {
          const int lvl = g / NR;
          const uint32_t rm = NR == 1 ? 3u : (g % NR == 0 ? 3u : static_cast<uint32_t>(g % NR));
          const int pos = gpos[g] + rank;
          const int cg = gcol[g] + rank * (BLK >> lvl);
          segs[t * kPyrMaxSegs + pos] = static_cast<uint32_t>(j) | (static_cast<uint32_t>(lvl) << 16) | (rm << 18) |
                                        (static_cast<uint32_t>(cg & (kTileN - 1)) << 24);
          if ((cg & (kTileN - 1)) == 0) ents[t * kPyrMaxEntries + cg / kTileN] = static_cast<uint16_t>(pos);
          if (CAUSAL && lvl == 0) {
            const int where = (cg / kTileN) * 256 + (cg & (kTileN - 1));
            if ((rm & 1u) && j == qbA) misc[8 + 2 * t] = where;
            if ((rm & 2u) && j == qbB) misc[9 + 2 * t] = where;
          }
          if (j == p.nb - 1) misc[12 + 2 * t + x] = cg / kTileN;   // a tile holding a segment of the last block
        }
        __syncwarp();
        if (g >= 0 && rank == 0) {
          gpos[g] += __popc(peers);
          gcol[g] += __popc(peers) * (BLK >> (g / NR));
        }
        __syncwarp();
      }
    }
    // key-tile descriptors, packed above the first-segment index (11 bits):
    // bit 11 uniform, bits 12-13 level, bits 14-15 row mask
    const bool last_partial = p.N - (p.nb - 1) * BLK < BLK;
    const int part0 = misc[12 + 2 * t], part1 = misc[13 + 2 * t];
    const int nt = (cols + kTileN - 1) / kTileN;
    for (int k = lane; k < nt; k += 32) {
      // (the start bits are masked: a neighbour lane may already have added
      // the descriptor bits of tile k + 1)
      const int s0 = ents[t * kPyrMaxEntries + k] & kEntStartMask;
      const int s1 = (k + 1 < nt ? (ents[t * kPyrMaxEntries + k + 1] & kEntStartMask) : n) - 1;
      const uint32_t g0 = (segs[t * kPyrMaxSegs + s0] >> 16) & 15u;
      const uint32_t g1 = (segs[t * kPyrMaxSegs + s1] >> 16) & 15u;
      const bool full = (k + 1) * kTileN <= cols;
      const bool uni = g0 == g1 && full && !(last_partial && (k == part0 || k == part1));
      ents[t * kPyrMaxEntries + k] = static_cast<uint16_t>(s0 | (uni ? kEntUniform : 0u) | (g0 << 12));
    }
    if (lane == 0) {
      misc[1 + t] = n;
      misc[3 + t] = nt;
      misc[6 + t] = cols;
    }
    if (warp == 0 && lane == 0) {
      misc[5] = 0;
      for (int i = 0; i < L::kNumBars; ++i)   // k_full: the K loads' arrival and the KX writes' arrival
        mbar_init(&bars[i], (&bars[i] == &k_full[0] || &bars[i] == &k_full[1]) ? 2u : 1u);
      fence_mbar_init();
      tma_prefetch_desc(&tmQ);
    }
  } else if (warp == 1) {
    tmem_alloc(const_cast<uint32_t*>(reinterpret_cast<volatile uint32_t*>(misc)), 512);
    tmem_relinquish();
  } else {
    // QX (warp 2): q rows of the tile's first q-block select columns 0-1, of
    // its second 2-3 (block 128: every row 0-1); the KX columns 8-15 of both
    // slots are 0
    for (int i = lane; i < 128; i += 32) {
      const bool second = QH == 2 && i >= 64;
      uint4 w;
      w.x = second ? 0u : 0x3F803F80u;   // bf16 1.0 in columns 0 and 1
      w.y = second ? 0x3F803F80u : 0u;   // columns 2 and 3
      w.z = 0u;
      w.w = 0u;
      const int off = (i >> 3) * 256 + (i & 7) * 16;
      *reinterpret_cast<uint4*>(qx + off) = w;
      *reinterpret_cast<uint4*>(qx + off + 128) = make_uint4(0, 0, 0, 0);
      for (int sl = 0; sl < kStages; ++sl) *reinterpret_cast<uint4*>(kx + sl * 4096 + off + 128) = make_uint4(0, 0, 0, 0);
    }
    // KX row patterns of full groups: index 4 * level + useA + 2 * useB, and
    // 16 for a column that holds no key
    if (lane < 17) {
      const float inv_sl2 = 1.f / p.scale_log2;
      const int lv = lane >> 2;
      const bool useA = lane < 16 && (lane & 1), useB = lane < 16 && (lane & 2);
      const float b = static_cast<float>(lv) * inv_sl2;
      const float bA = useA ? b : kMaskedBias, bB = useB ? b : kMaskedBias;
      const __nv_bfloat16 hA = __float2bfloat16(bA), hB = __float2bfloat16(bB);
      const __nv_bfloat16 lA = __float2bfloat16(bA - __bfloat162float(hA));
      const __nv_bfloat16 lB = __float2bfloat16(bB - __bfloat162float(hB));
      kxpat[lane] = make_uint4(
          static_cast<uint32_t>(__bfloat16_as_ushort(hA)) | (static_cast<uint32_t>(__bfloat16_as_ushort(lA)) << 16),
          static_cast<uint32_t>(__bfloat16_as_ushort(hB)) | (static_cast<uint32_t>(__bfloat16_as_ushort(lB)) << 16), 0u,
          0u);
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = static_cast<uint32_t>(misc[0]);
  const int ntile0 = misc[3], ntile1 = misc[4];   // packed key tiles of q-tile 0 / 1
  const int n_entries = ntile0 + ntile1;
  // entry e -> (tile, key tile): tiles alternate while both have key tiles left
  auto entry_of = [&](int e, int& t, int& k) {
    const int m = min(ntile0, ntile1);
    if (e < 2 * m) {
      t = e & 1;
      k = e >> 1;
    } else {
      t = ntile0 > ntile1 ? 0 : 1;
      k = m + (e - 2 * m);
    }
  };
  const uint32_t sK = smem_addr(smem + L::kOffK);
  const uint32_t sV = smem_addr(smem + L::kOffV);

  if (warp < kSoftmaxWarp0) {
    setmaxnreg_dec<56>();
    // ------------------------------------------- segment gather helpers ---
    // An entry's segments, one lane per segment (a 128-key tile holds at
    // most 128 / 8 = 16), with the columns the list builder assigned.
    struct Seg {
      uint32_t sg;
      int lvl, len, col, row, fill;
      bool mine;
    };
    auto seg_of = [&](int t, int k) -> Seg {   // segments of key tile k of q-tile t
      const int nt = t == 0 ? ntile0 : ntile1;
      const int start = ents[t * kPyrMaxEntries + k] & kEntStartMask;
      const int end = k + 1 < nt ? (ents[t * kPyrMaxEntries + k + 1] & kEntStartMask) : misc[1 + t];
      Seg g;
      g.fill = k + 1 < nt ? kTileN : misc[6 + t] - kTileN * k;
      g.mine = lane < end - start;
      g.sg = g.mine ? segs[t * kPyrMaxSegs + start + lane] : 0u;
      g.lvl = static_cast<int>((g.sg >> 16) & 3u);
      g.len = g.mine ? (BLK >> g.lvl) : 0;
      g.col = static_cast<int>((g.sg >> 24) & (kTileN - 1));
      g.row = static_cast<int>(g.sg & 0xFFFFu) * g.len;
      return g;
    };
    // wait (lane 0) for a slot's previous phase; false after an error
    auto slot_free = [&](uint64_t* bar, int e) -> bool {
      if (e < kStages) return true;
      const uint32_t par = ((e / kStages) - 1) & 1;
      if (__all_sync(0xffffffffu, mbar_test(bar, par))) return true;   // the common case
      const bool w = lane == 0 ? (misc[5] == 0 && mbar_wait(bar, par)) : true;
      return __shfl_sync(0xffffffffu, w, 0);
    };
    // zero rows [r0, r1) of a K or V slot so masked products stay finite
    auto zero_rows = [&](uint8_t* st, int r0, int r1) {
      if (r0 < r1) {
        const int per_half = (r1 - r0) * 8;   // 16-byte chunks per 64-column half
        for (int idx = lane; idx < per_half * (D / 64); idx += 32) {
          const int hd = idx >= per_half ? 1 : 0;
          const int rem = idx - hd * per_half;
          reinterpret_cast<uint4*>(st + hd * kHalfBytes + (r0 + (rem >> 3)) * 128)[rem & 7] = make_uint4(0, 0, 0, 0);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      }
    };
    // TMA of the segment pieces whose columns lie in [c0, c1); a segment
    // longer than 64 keys (level 0 of block 128) goes in two 64-row pieces
    // (the level maps' boxes are at most 64 rows), so no piece crosses 64
    auto issue = [&](const Seg& g, const CUtensorMap* lvmaps, uint64_t* full, uint8_t* st, int c0, int c1) {
      const int rows = max(0, min(g.fill, c1) - c0);
      if (lane == 0) mbar_arrive_expect_tx(full, static_cast<uint32_t>(rows) * D * 2);
      __syncwarp();
      if (g.mine) {
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int cq = g.col + 64 * q;
          if ((q == 0 || g.len > 64) && cq >= c0 && cq < c1) {
#pragma unroll
            for (int hd = 0; hd < D / 64; ++hd)
              tma_load_3d(&lvmaps[g.lvl], full, st + hd * kHalfBytes + cq * 128, hd * 64, g.row + 64 * q, bh);
          }
        }
      }
    };
    // V half h (keys [64h, 64h+64)) of entry e into its slot
    auto load_v_half = [&](const Seg& g, int e, int h) -> bool {
      const int s = e % kStages;
      if (!slot_free(&v_empty[s * 2 + h], e)) return false;
      uint8_t* vst = smem + L::kOffV + s * L::kTileBytes;
      zero_rows(vst, max(g.fill, 64 * h), 64 * h + 64);
      issue(g, maps.v, &v_full[s * 2 + h], vst, 64 * h, 64 * h + 64);
      return true;
    };
    const float NEG_INF = -__int_as_float(0x7f800000);
    // The bias of each key column, log2(pooled token count) / (scale log2 e) in
    // raw logit units, for the tile's two q-blocks, into the K slot's KX rows
    // (hi and lo bf16 parts, columns 0-1 for q-block A, 2-3 for B; columns
    // 4-15 stay zero).  Lane L writes key columns [4L, 4L+4): the segment that
    // covers them is found from a mask of segment start columns (segments are
    // in column order) and its fields are fetched by shuffle.  The value is the
    // level unless the segment holds the end of the sequence (a short last
    // group, or rows past the level's end); kMaskedBias on masked or empty
    // columns.
    const float inv_sl2 = 1.f / p.scale_log2;
    auto write_kx = [&](const Seg& g, uint8_t* kxs) {
      const uint32_t starts = __reduce_or_sync(0xffffffffu, g.mine ? (1u << (g.col >> 2)) : 0u);
      const int c0 = 4 * lane;
      const int owner = __popc(starts & ((2u << lane) - 1u)) - 1;   // the segment's rank = its lane
      const int src = owner < 0 ? 0 : owner;
      const uint32_t sg_o = __shfl_sync(0xffffffffu, g.sg, src);
      const int col_o = __shfl_sync(0xffffffffu, g.col, src);
      const int row_o = __shfl_sync(0xffffffffu, g.row, src);
      const int lv = static_cast<int>((sg_o >> 16) & 3u);
      const uint32_t rm = (sg_o >> 18) & 3u;
      const int useA = rm & 1u, useB = QH == 1 ? (rm & 1u) : ((rm >> 1) & 1u);
      const int gr0 = row_o + (c0 - col_o);
      if (c0 >= g.fill || ((gr0 + 4) << lv) <= p.N) {
        // empty, or four full groups of one level: a precomputed row pattern
        const uint4 w = kxpat[c0 >= g.fill ? 16 : 4 * lv + useA + 2 * useB];
#pragma unroll
        for (int i = 0; i < 4; ++i) *reinterpret_cast<uint4*>(kxs + ((c0 + i) >> 3) * 256 + ((c0 + i) & 7) * 16) = w;
      } else {
        // the segment that holds the end of the sequence: short last group
        // (fewer than 2^lv tokens) and rows past the level's end
        const int rows_l = (p.N + (1 << lv) - 1) >> lv;
#pragma unroll 1
        for (int i = 0; i < 4; ++i) {
          float braw = kMaskedBias;
          const int gr = gr0 + i;
          if (gr < rows_l) {
            const int count = min(1 << lv, p.N - (gr << lv));
            braw = (count == (1 << lv) ? static_cast<float>(lv) : log2f(static_cast<float>(count))) * inv_sl2;
          }
          const float bA = useA ? braw : kMaskedBias, bB = useB ? braw : kMaskedBias;
          const __nv_bfloat16 hA = __float2bfloat16(bA), hB = __float2bfloat16(bB);
          const __nv_bfloat16 lA = __float2bfloat16(bA - __bfloat162float(hA));
          const __nv_bfloat16 lB = __float2bfloat16(bB - __bfloat162float(hB));
          const int r = c0 + i;   // key column = row of KX
          *reinterpret_cast<uint4*>(kxs + (r >> 3) * 256 + (r & 7) * 16) = make_uint4(
              static_cast<uint32_t>(__bfloat16_as_ushort(hA)) | (static_cast<uint32_t>(__bfloat16_as_ushort(lA)) << 16),
              static_cast<uint32_t>(__bfloat16_as_ushort(hB)) | (static_cast<uint32_t>(__bfloat16_as_ushort(lB)) << 16),
              0u, 0u);
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
    };
    if (warp == 3) {
      // ----------------------------------- producer of Q, K and KX (warp 3) ---
      if (n_entries > 0) {
        if (lane == 0) {
          const uint32_t qbytes = static_cast<uint32_t>((ntile0 > 0) + (ntile1 > 0)) * L::kTileBytes;
          mbar_arrive_expect_tx(q_full, qbytes);
#pragma unroll
          for (int t = 0; t < 2; ++t) {
            if ((t == 0 ? ntile0 : ntile1) == 0) continue;
#pragma unroll
            for (int hd = 0; hd < D / 64; ++hd)
              tma_load_3d(&tmQ, q_full, smem + L::kOffQ + t * L::kTileBytes + hd * kHalfBytes, hd * 64,
                          (qtile0 + t) * kTileM, bh);
          }
        }
        int k_issued = 0;
        bool ok = true;
        for (int e = 0; e < n_entries; ++e) {
          int t, k;
          entry_of(e, t, k);
          const Seg g = seg_of(t, k);
          const int s = e % kStages;
          if (!slot_free(&k_empty[s], e)) {
            ok = false;
            break;
          }
          uint8_t* kst = smem + L::kOffK + s * L::kTileBytes;
          zero_rows(kst, g.fill, kTileN);
          issue(g, maps.k, &k_full[s], kst, 0, kTileN);
          k_issued = e + 1;
          // KX is written while the K segments are in flight (mixed tiles
          // only: a uniform tile's bias is added by the softmax); its arrival
          // is the second of the k_full phase (made visible to the MMA by it)
          if (!(ents[t * kPyrMaxEntries + k] & kEntUniform)) write_kx(g, kx + s * 4096);
          if (lane == 0) mbar_arrive(&k_full[s]);
        }
        if (!ok && lane == 0) misc[5] = 1;
        // Loads still in flight must land before the CTA can exit.
        if (lane == 0) {
          for (int e = (k_issued > kStages ? k_issued - kStages : 0); e < k_issued; ++e)
            mbar_wait(&k_full[e % kStages], (e / kStages) & 1);
          mbar_wait(q_full, 0);
        }
      }
    } else if (warp == 0) {
      // ---------------------------------------------------- S issue (warp 0) ---
      // Entry e's S = Q_t K_e^T goes into the one S buffer once the softmax that
      // consumed entry e-1's S has loaded it; warp-wide, one elected lane issues.
      if (n_entries > 0) {
        bool ok = __all_sync(0xffffffffu, mbar_wait(q_full, 0));
        if (!ok && lane == 0) misc[5] = 1;
        const uint64_t dq0 = smem_desc(smem_addr(smem + L::kOffQ), 16, 1024);
        const uint64_t dk0 = smem_desc(sK, 16, 1024);
        const uint64_t dqx = smem_desc_kmajor_noswizzle(smem_addr(qx), 128, 256);
        const uint64_t dkx0 = smem_desc_kmajor_noswizzle(smem_addr(kx), 128, 256);
        constexpr uint64_t kStageStep = L::kTileBytes >> 4;
        int prev_t = 0;
        for (int e = 0; e < n_entries; ++e) {
          int t, k;
          entry_of(e, t, k);
          const int s = e % kStages;
          if (e > 0) named_bar_sync(kBarSFree + prev_t, kHandoff);
          ok = ok && !__any_sync(0xffffffffu, misc[5] != 0);
          bool seen = false;
          if (ok) {
            seen = __all_sync(0xffffffffu, mbar_wait(&k_full[s], (e / kStages) & 1));
            if (!seen) {
              ok = false;
              if (lane == 0) misc[5] = 1;
            }
          }
          if (ok) {
            tc_fence_after();
            const uint64_t dq = dq0 + t * kStageStep;
            const uint64_t dk = dk0 + s * kStageStep;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t off = static_cast<uint64_t>((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4;
              mma_ss_warp(tmem, dq + off, dk + off, kIdescS, kk > 0 ? 1u : 0u);
            }
            // + the bias of a mixed tile: selector columns of the row's q-block
            // times its hi + lo parts
            if (!(ents[t * kPyrMaxEntries + k] & kEntUniform))
              mma_ss_warp(tmem, dqx, dkx0 + s * (4096 >> 4), kIdescS, 1u);
          }
          // committed also after an error, so that the softmax keeps its place
          mma_commit_warp(&s_ready[t]);
          // the K slot is free once this S completes (only if its load landed)
          if (seen) mma_commit_warp(&k_empty[s]);
          prev_t = t;
        }
        named_bar_sync(kBarSFree + prev_t, kHandoff);   // the last S has been loaded
        mma_commit_warp(&mma_done[0]);
        mbar_wait(&mma_done[0], 0);
      }
    } else {
      // ------------------------- V loads and PV issue for q-tile t (warps 1, 2) ---
      // O_t += P_t V in two halves, each as soon as the softmax warpgroup has
      // written that half of P_t.  This warp also loads V of its own next
      // entry, each 64-key half as soon as the slot's half is free, so that
      // the V of an entry is in flight while the previous entry's softmax runs.
      const int t = warp - 1;
      const int cnt = t == 0 ? ntile0 : ntile1;
      if (n_entries > 0 && cnt > 0) {
        const uint64_t dv0 = smem_desc(sV, kHalfBytes, 1024);
        constexpr uint64_t kStageStep = L::kTileBytes >> 4;
        const uint32_t a_tmem = tmem + 128 + 64 * t;
        const uint32_t o_tmem = tmem + 256 + t * D;
        auto next_own = [&](int e) -> int {   // first entry >= e of this tile, or n_entries
          for (; e < n_entries; ++e) {
            int te, k;
            entry_of(e, te, k);
            if (te == t) break;
          }
          return e;
        };
        auto aborted = [&]() -> bool { return __any_sync(0xffffffffu, misc[5] != 0); };
        // Every V half that was issued is waited for (also after an error), so
        // that no load is in flight when the CTA exits.
        int e = next_own(0);
        int k_own = 0;
        Seg g = seg_of(t, 0);
        bool cur_lo = load_v_half(g, e, 0);
        bool cur_hi = cur_lo && load_v_half(g, e, 1);
        int done = 0;
        while (e < n_entries) {
          const int s = e % kStages;
          const uint64_t dv = dv0 + s * kStageStep;
          const int en = next_own(e + 1);
          Seg gn;
          if (en < n_entries) gn = seg_of(t, k_own + 1);
          named_bar_sync(kBarPA + t, kHandoff);
          bool landed = cur_lo && __all_sync(0xffffffffu, mbar_wait(&v_full[s * 2], (e / kStages) & 1));
          bool ok = landed && !aborted();
          if (ok) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ts_warp(o_tmem, a_tmem + kk * 8, dv + ((kk * 16 * 128) >> 4), kIdescPV,
                          (done == 0 && kk == 0) ? 0u : 1u);
            mma_commit_warp(&v_empty[s * 2]);   // first V half free
          }
          mma_commit_warp(&pv_done_a[t]);   // also after an error, so that no waiter stalls
          named_bar_sync(kBarPB + t, kHandoff);
          landed = cur_hi && __all_sync(0xffffffffu, mbar_wait(&v_full[s * 2 + 1], (e / kStages) & 1));
          ok = ok && landed && !aborted();
          if (ok) {
            tc_fence_after();
#pragma unroll
            for (int kk = 4; kk < 8; ++kk)
              mma_ts_warp(o_tmem, a_tmem + kk * 8, dv + ((kk * 16 * 128) >> 4), kIdescPV, 1u);
            mma_commit_warp(&v_empty[s * 2 + 1]);   // second V half free
          }
          mma_commit_warp(&pv_done_b[t]);
          if (++done == cnt) mma_commit_warp(&o_final[t]);
          if (!ok && lane == 0) misc[5] = 1;
          // V of the next entry, after this entry's hand-offs so that the
          // softmax never waits at PB for these gathers
          const bool nxt_lo = en < n_entries && !aborted() && load_v_half(gn, en, 0);
          const bool nxt_hi = nxt_lo && !aborted() && load_v_half(gn, en, 1);
          if (en < n_entries && !(nxt_lo && nxt_hi) && lane == 0) misc[5] = 1;
          e = en;
          g = gn;
          ++k_own;
          cur_lo = nxt_lo;
          cur_hi = nxt_hi;
        }
        mma_commit_warp(&mma_done[1 + t]);
        mbar_wait(&mma_done[1 + t], 0);
      }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
      tc_fence_after();
      tmem_dealloc(tmem, 512);
    }
    return;
  }

  setmaxnreg_inc<224>();
  {
    // ------------------------------------------------------------- softmax ---
    const int t = (warp - kSoftmaxWarp0) >> 2;
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const int row = (qtile0 + t) * kTileM + r;
    const bool row_valid = row < p.N && t != skip_t;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const uint32_t s_addr = lane_base;
    const uint32_t p_addr = lane_base + 128 + 64 * t;
    const uint32_t o_addr = lane_base + 256 + t * D;
    const int cnt = t == 0 ? ntile0 : ntile1;
    const float sl2 = p.scale_log2;
    const float NEG_INF = -__int_as_float(0x7f800000);
    // causal: where this row's own block sits in the packed key tiles
    const int xq = (BLK == 64) ? (r >> 6) : 0;
    const int diag = CAUSAL ? misc[8 + 2 * t + xq] : -1;
    const int r_in_blk = r & (BLK - 1);

    const float inv_sl2 = 1.f / sl2;
    float m_used = NEG_INF, l_sum = 0.f;
    int et = 0;            // entries of this q-tile processed
    bool ok = true;
    if (cnt > 0) {
      for (int e = 0; e < n_entries; ++e) {
        int te, k;
        entry_of(e, te, k);
        if (te != t) continue;
        // A uniform tile (same level and row mask throughout, full groups):
        // its bias is one constant, ln(2^l) (l * inv_sl2 in raw logit units),
        // added here instead of by the bias MMA, and the rows of a q-block
        // that does not use the tile skip it (their P is zero).
        const uint32_t ed = ents[t * kPyrMaxEntries + k];
        const bool use = !(ed & kEntUniform) || QH == 1 || ((ed >> (14 + xq)) & 1u);
        // the tile's bias in raw logit units (0 for a mixed tile, whose S carries it)
        const float bias = (ed & kEntUniform) ? static_cast<float>((ed >> 12) & 3u) * inv_sl2 : 0.f;
        // The previous PV of this tile reads P_t and accumulates into O_t: each
        // half of P_t is rewritten once that half of the PV has completed, and
        // O_t is rescaled once all of it has.
        auto wait_pv = [&](uint64_t* bar) {
          if (et > 0) {
            if (!mbar_wait(bar, (et - 1) & 1)) {
              misc[5] = 1;
              ok = false;
            }
            tc_fence_after();
          }
        };
        if (!use) {
          // these rows' P is zero (no S load, no exponentials); the hand-offs
          // run as for any entry
          named_bar_sync(kBarSFree + t, kHandoff);
          uint32_t zk[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) zk[i] = 0u;
          wait_pv(&pv_done_a[t]);
          tmem_st32(p_addr, reinterpret_cast<const float*>(zk));
          tmem_st_wait();
          tc_fence_before();
          named_bar_sync(kBarPA + t, kHandoff);
          wait_pv(&pv_done_b[t]);
          tmem_st32(p_addr + 32, reinterpret_cast<const float*>(zk));
          tmem_st_wait();
          tc_fence_before();
          named_bar_sync(kBarPB + t, kHandoff);
          ++et;
          continue;
        }
        // After an error the loop still runs to the end (its hand-offs keep
        // the issuing warps' sequences in step); it only stops trusting TMEM.
        if (!mbar_wait(&s_ready[t], et & 1)) {
          misc[5] = 1;
          ok = false;
        }
        tc_fence_after();
        float s[kTileN];
        tmem_ld128(s_addr, s);
        // the S buffer is free for the next entry's S
        tc_fence_before();
        named_bar_sync(kBarSFree + t, kHandoff);
        if (CAUSAL && diag >= 0 && (diag >> 8) == k) {
          // causal: the diagonal segment's key x (from the block start) is
          // visible to the row only if x <= the row's position in its block
          const int c0 = diag & 255;
#pragma unroll
          for (int c = 0; c < kTileN; ++c)
            if (c >= c0 && c < c0 + BLK && c - c0 > r_in_blk) s[c] = NEG_INF;
        }
        // a mixed tile's s already carries the bias (raw logit units): q.k +
        // log2(count) / (scale log2 e), and about -30000 on masked and empty
        // columns; a uniform tile's bias is `bias` on every column (and its
        // row maximum is a real logit, never below the cut)
        float a[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) a[u] = fmaxf(s[2 * u], s[2 * u + 1]);
#pragma unroll
        for (int c = 16; c < kTileN; c += 16) {
#pragma unroll
          for (int u = 0; u < 8; ++u) a[u] = fmax3(a[u], s[c + 2 * u], s[c + 2 * u + 1]);
        }
        float mx = fmaxf(fmax3(a[0], a[1], a[2]), fmax3(a[3], a[4], fmax3(a[5], a[6], a[7])));
        mx = mx < kMaskedCut ? NEG_INF : mx + bias;   // -inf: no valid column for this row in this tile
        float factor = 1.f;
        if (mx > m_used && (m_used == NEG_INF || (mx - m_used) * sl2 > 8.f)) {
          factor = (m_used == NEG_INF) ? 0.f : fast_exp2((m_used - mx) * sl2);
          m_used = mx;
          l_sum *= factor;
        }
        const bool rescale = et > 0 && __any_sync(0xffffffffu, factor != 1.f);
        if (rescale) {
          wait_pv(&pv_done_b[t]);
#pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            float ov[32];
            tmem_ld32(o_addr + c * 32, ov);
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] *= factor;
            tmem_st32(o_addr + c * 32, ov);
          }
          tmem_st_wait();
        }
        // x = (s + bias - m) sl2
        const float neg_m = (m_used == NEG_INF) ? 0.f : (bias - m_used) * sl2;
        {
          uint32_t pk[32];
          l_sum += exp_pack_64(s, sl2, neg_m, pk);
          if (!rescale) wait_pv(&pv_done_a[t]);
          tmem_st32(p_addr, reinterpret_cast<const float*>(pk));
          tmem_st_wait();
          tc_fence_before();
          named_bar_sync(kBarPA + t, kHandoff);
        }
        {
          uint32_t pk[32];
          l_sum += exp_pack_64(s + 64, sl2, neg_m, pk);
          if (!rescale) wait_pv(&pv_done_b[t]);
          tmem_st32(p_addr + 32, reinterpret_cast<const float*>(pk));
          tmem_st_wait();
          tc_fence_before();
          named_bar_sync(kBarPB + t, kHandoff);
        }
        ++et;
      }
    }

    // ------------------------------------------------------------ epilogue ---
    ok = __all_sync(0xffffffffu, ok && misc[5] == 0);
    if (cnt > 0 && ok) {
      ok = __all_sync(0xffffffffu, mbar_wait(&o_final[t], 0));
      if (!ok) misc[5] = 1;
      tc_fence_after();
    }
    if (m_used == NEG_INF) l_sum = 0.f;
    const float inv_l = l_sum > 0.f ? 1.f / l_sum : 0.f;
    __nv_bfloat16* orow = p.o + (static_cast<size_t>(bh) * p.N + (row_valid ? row : 0)) * D;
#pragma unroll 1
    for (int c = 0; c < D / 32; ++c) {
      float ov[32];
      if (cnt > 0 && ok) {
        tmem_ld32(o_addr + c * 32, ov);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) ov[i] = 0.f;
      }
      if (row_valid) {
        uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint4 w;
          w.x = pack_bf16x2(ov[q4 * 8 + 0] * inv_l, ov[q4 * 8 + 1] * inv_l);
          w.y = pack_bf16x2(ov[q4 * 8 + 2] * inv_l, ov[q4 * 8 + 3] * inv_l);
          w.z = pack_bf16x2(ov[q4 * 8 + 4] * inv_l, ov[q4 * 8 + 5] * inv_l);
          w.w = pack_bf16x2(ov[q4 * 8 + 6] * inv_l, ov[q4 * 8 + 7] * inv_l);
          dst[q4] = w;
        }
      }
    }
    if (p.lse && row_valid)
      p.lse[static_cast<size_t>(bh) * p.N + row] =
          l_sum > 0.f ? (log2f(l_sum) + m_used * sl2) * 0.69314718055994531f : NEG_INF;
  }
  tc_fence_before();
  __syncthreads();
}

}  // namespace sa
