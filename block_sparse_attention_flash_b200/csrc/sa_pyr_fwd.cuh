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
// the two q-blocks uses it) that becomes a -inf bias for the other rows.
//
// One CTA = two q-tiles (ping-pong as in sa_attn_fwd.cuh), 16 softmax warps with
// two threads per row (the halves swap row maxima once per key tile), but each q-tile has
// its own packed key tiles; the entries of the two are interleaved.  K and V
// segments arrive by TMA from one tensor map per pyramid level (level 0 is
// the original K/V), into 2-stage rings released separately.  The producer
// warp also writes, per stage, the per-column bias (log2 of the pooled token
// count, -inf where a column is masked or empty) for both row halves, and
// zero-fills columns no segment covers so that masked products stay finite.
// The softmax works in log2 units: x = s * scale * log2(e) + log2(count).
#pragma once

#include "sa_attn_fwd.cuh"

namespace sa {

constexpr int kPyrMaxBlocks = 1024;                 // k-blocks per sequence
// 20 warps: producer, MMA, 2 idle, then 16 softmax warps (two threads per row)
constexpr int kPyrWarps = 20;
constexpr int kPyrThreads = kPyrWarps * 32;
constexpr int kPyrMaxSegs = 2 * kPyrMaxBlocks;      // per q-tile (union of 2 q-blocks)

struct PyrParams {
  int B, H, N;
  int nb;                 // blocks per sequence
  int pool_rows[4];       // rows of the level-l tensor: ceil(N / 2^l)
  const uint8_t* levels;  // code map: 0 drop, 1 + l level l
  long long lsb, lsh, lsi;
  float scale_log2;
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
  static constexpr int kOffBias = kOffSeg + 2 * kPyrMaxSegs * 4;       // [stage][half A/B][128] f32
  static constexpr int kOffRed = kOffBias + kStages * 2 * kTileN * 4;
  static constexpr int kRedFloats = 2 * 2 * 2 * kTileM;
  static constexpr int kNumBars = 1 + 5 * kStages + 2 + 2 + 2 + 1;
  static constexpr int kOffBar = kOffRed + kRedFloats * 4;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kBytes = kOffMisc + 64;
  static constexpr int kAlloc = kBytes + 1024;
};

struct PyrMaps {
  CUtensorMap k[4];
  CUtensorMap v[4];
};

template <int D, int BLK>
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
  float* bias = reinterpret_cast<float*>(smem + L::kOffBias);
  float* red = reinterpret_cast<float*>(smem + L::kOffRed);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = bars + 1 + kStages;
  uint64_t* k_empty = bars + 1 + 2 * kStages;
  uint64_t* v_empty = bars + 1 + 3 * kStages;
  uint64_t* b_full = bars + 1 + 4 * kStages;
  uint64_t* s_ready = bars + 1 + 5 * kStages;
  uint64_t* p_ready = s_ready + 2;
  uint64_t* o_final = p_ready + 2;
  uint64_t* mma_done = o_final + 2;
  volatile int* misc = reinterpret_cast<volatile int*>(smem + L::kOffMisc);
  // misc[0] TMEM base, [1]/[2] segments of q-tile 0/1, [3]/[4] key tiles of q-tile 0/1, [5] abort

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x, bh = blockIdx.y;
  const int b = bh / p.H, h = bh - (bh / p.H) * p.H;
  const int qtile0 = 2 * pair;

  if (warp == 0) {
    // ---- per q-tile segment lists, sorted by level (pass l collects level l) ----
#pragma unroll 1
    for (int t = 0; t < 2; ++t) {
      int n = 0, cols = 0;
      const int qbA = (qtile0 + t) * QH;
      const int qbB = qbA + QH - 1;
      const bool validA = qbA < p.nb, validB = qbB < p.nb;
#pragma unroll 1
      for (int lvl = 0; lvl < 4; ++lvl) {
        for (int base = 0; base < p.nb; base += 32) {
          const int j = base + lane;
          uint32_t rm = 0;
          if (j < p.nb) {
            const long long rowoff = b * p.lsb + h * p.lsh + j;
            const int cA = validA ? p.levels[rowoff + qbA * p.lsi] : 0;
            const int cB = validB ? p.levels[rowoff + qbB * p.lsi] : 0;
            rm = (cA == lvl + 1 ? 1u : 0u) | (cB == lvl + 1 ? 2u : 0u);
          }
          const unsigned ball = __ballot_sync(0xffffffffu, rm != 0);
          if (rm) segs[t * kPyrMaxSegs + n + __popc(ball & ((1u << lane) - 1u))] =
              static_cast<uint32_t>(j) | (static_cast<uint32_t>(lvl) << 16) | (rm << 18);
          n += __popc(ball);
          cols += __popc(ball) * (BLK >> lvl);
        }
      }
      if (lane == 0) {
        misc[1 + t] = n;
        misc[3 + t] = (cols + kTileN - 1) / kTileN;
      }
    }
    if (lane == 0) {
      misc[5] = 0;
      for (int i = 0; i < L::kNumBars; ++i) {
        const bool softmax_arrivals = (&bars[i] == &p_ready[0]) || (&bars[i] == &p_ready[1]);
        mbar_init(&bars[i], softmax_arrivals ? 256u : 1u);
      }
      fence_mbar_init();
      tma_prefetch_desc(&tmQ);
    }
  } else if (warp == 1) {
    tmem_alloc(const_cast<uint32_t*>(reinterpret_cast<volatile uint32_t*>(misc)), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = static_cast<uint32_t>(misc[0]);
  const int ntile[2] = {misc[3], misc[4]};
  const int n_entries = ntile[0] + ntile[1];
  // entry e -> (tile, key tile): tiles alternate while both have key tiles left
  auto entry_of = [&](int e, int& t, int& k) {
    const int m = min(ntile[0], ntile[1]);
    if (e < 2 * m) {
      t = e & 1;
      k = e >> 1;
    } else {
      t = ntile[0] > ntile[1] ? 0 : 1;
      k = m + (e - 2 * m);
    }
  };
  const uint32_t sQ = smem_addr(smem + L::kOffQ);
  const uint32_t sK = smem_addr(smem + L::kOffK);
  const uint32_t sV = smem_addr(smem + L::kOffV);

  if (warp < kSoftmaxWarp0) {
    setmaxnreg_dec<32>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer ---
    if (n_entries > 0) {
      if (lane == 0) {
        const uint32_t qbytes = static_cast<uint32_t>((ntile[0] > 0) + (ntile[1] > 0)) * L::kTileBytes;
        mbar_arrive_expect_tx(q_full, qbytes);
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (ntile[t] == 0) continue;
#pragma unroll
          for (int hd = 0; hd < D / 64; ++hd)
            tma_load_3d(&tmQ, q_full, smem + L::kOffQ + t * L::kTileBytes + hd * kHalfBytes, hd * 64,
                        (qtile0 + t) * kTileM, bh);
        }
      }
      int cursor[2] = {0, 0};   // next segment of each q-tile
      int issued = 0;
      bool ok = true;
      for (int e = 0; e < n_entries && ok; ++e) {
        int t, k;
        entry_of(e, t, k);
        const int s = e % kStages;
        const uint32_t par = ((e / kStages) - 1) & 1;
        // segments of this key tile: [s0, s1)
        const uint32_t* tseg = segs + t * kPyrMaxSegs;
        const int nseg = misc[1 + t];
        const int s0 = cursor[t];
        int s1 = s0, fill = 0;
        while (s1 < nseg) {
          const int len = BLK >> ((tseg[s1] >> 16) & 3u);
          if (fill + len > kTileN) break;
          fill += len;
          ++s1;
        }
        cursor[t] = s1;
        if (e >= kStages) {
          bool w = lane == 0 ? (misc[5] == 0 && mbar_wait(&k_empty[s], par)) : true;
          if (!__shfl_sync(0xffffffffu, w, 0)) {
            ok = false;
            break;
          }
        }
        // empty columns [fill, 128): zero K rows so masked products stay finite
        uint8_t* kst = smem + L::kOffK + s * L::kTileBytes;
        uint8_t* vst = smem + L::kOffV + s * L::kTileBytes;
        if (fill < kTileN) {
          for (int idx = lane; idx < (kTileN - fill) * 8 * (D / 64); idx += 32) {
            const int hd = idx / ((kTileN - fill) * 8);
            const int rem = idx - hd * (kTileN - fill) * 8;
            reinterpret_cast<uint4*>(kst + hd * kHalfBytes + (fill + rem / 8) * 128)[rem % 8] = make_uint4(0, 0, 0, 0);
          }
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          __syncwarp();
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(&k_full[s], static_cast<uint32_t>(fill) * D * 2);
          int col = 0;
          for (int g = s0; g < s1; ++g) {
            const uint32_t sg = tseg[g];
            const int lvl = (sg >> 16) & 3u;
            const int len = BLK >> lvl;
            const int row = static_cast<int>(sg & 0xFFFFu) * len;
#pragma unroll
            for (int hd = 0; hd < D / 64; ++hd)
              tma_load_3d(&maps.k[lvl], &k_full[s], kst + hd * kHalfBytes + col * 128, hd * 64, row, bh);
            col += len;
          }
        }
        // V slot and the bias table of this stage are free once PV of entry e-2 is done
        if (e >= kStages) {
          bool w = lane == 0 ? mbar_wait(&v_empty[s], par) : true;
          if (!__shfl_sync(0xffffffffu, w, 0)) {
            ok = false;
            if (lane == 0) mbar_wait(&k_full[s], (e / kStages) & 1);
            break;
          }
        }
        if (fill < kTileN) {
          for (int idx = lane; idx < (kTileN - fill) * 8 * (D / 64); idx += 32) {
            const int hd = idx / ((kTileN - fill) * 8);
            const int rem = idx - hd * (kTileN - fill) * 8;
            reinterpret_cast<uint4*>(vst + hd * kHalfBytes + (fill + rem / 8) * 128)[rem % 8] = make_uint4(0, 0, 0, 0);
          }
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
        // per-column log2(count) bias for row halves A and B
        float* bst = bias + s * 2 * kTileN;
        {
          const float NEG_INF = -__int_as_float(0x7f800000);
          int col = 0;
          for (int g = s0; g < s1; ++g) {
            const uint32_t sg = tseg[g];
            const int lvl = (sg >> 16) & 3u;
            const int len = BLK >> lvl;
            const uint32_t rm = (sg >> 18) & 3u;
            const int g0 = static_cast<int>(sg & 0xFFFFu) * len;
            for (int c = lane; c < len; c += 32) {
              const int gr = g0 + c;
              float bv = NEG_INF;
              if (gr < p.pool_rows[lvl]) {
                const int count = min(1 << lvl, p.N - (gr << lvl));
                bv = log2f(static_cast<float>(count));
              }
              bst[col + c] = (rm & 1u) ? bv : NEG_INF;
              bst[kTileN + col + c] = (QH == 1 ? (rm & 1u) : (rm & 2u)) ? bv : NEG_INF;
            }
            col += len;
          }
          for (int c = fill + lane; c < kTileN; c += 32) {
            bst[c] = NEG_INF;
            bst[kTileN + c] = NEG_INF;
          }
        }
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&b_full[s]);
          mbar_arrive_expect_tx(&v_full[s], static_cast<uint32_t>(fill) * D * 2);
          int col = 0;
          for (int g = s0; g < s1; ++g) {
            const uint32_t sg = tseg[g];
            const int lvl = (sg >> 16) & 3u;
            const int len = BLK >> lvl;
            const int row = static_cast<int>(sg & 0xFFFFu) * len;
#pragma unroll
            for (int hd = 0; hd < D / 64; ++hd)
              tma_load_3d(&maps.v[lvl], &v_full[s], vst + hd * kHalfBytes + col * 128, hd * 64, row, bh);
            col += len;
          }
        }
        issued = e + 1;
      }
      if (!ok && lane == 0) misc[5] = 1;
      if (lane == 0) {
        for (int e = (issued > kStages ? issued - kStages : 0); e < issued; ++e) {
          const int s = e % kStages;
          mbar_wait(&k_full[s], (e / kStages) & 1);
          mbar_wait(&v_full[s], (e / kStages) & 1);
        }
        mbar_wait(q_full, 0);
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issue ---
    if (lane == 0 && n_entries > 0) {
      bool ok = mbar_wait(q_full, 0);
      int pend[2] = {-1, -1};
      int done_pv[2] = {0, 0};
      uint32_t pphase[2] = {0u, 0u};
      auto issue_pv = [&](int t) -> bool {
        const int e = pend[t];
        const int s = e % kStages;
        if (!mbar_wait(&p_ready[t], pphase[t])) return false;
        pphase[t] ^= 1u;
        if (!mbar_wait(&v_full[s], (e / kStages) & 1)) return false;
        tc_fence_after();
        const uint32_t d_tmem = tmem + 256 + t * D;
        const uint32_t a_tmem = tmem + t * 128;
        const uint32_t vbase = sV + s * L::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < kTileN / 16; ++kk)
          mma_ts(d_tmem, a_tmem + kk * 8, smem_desc(vbase + kk * 16 * 128, kHalfBytes, 1024), kIdescPV,
                 (done_pv[t] == 0 && kk == 0) ? 0u : 1u);
        mma_commit(&v_empty[s]);
        if (++done_pv[t] == ntile[t]) mma_commit(&o_final[t]);
        pend[t] = -1;
        return true;
      };
      for (int e = 0; ok && e < n_entries; ++e) {
        int t, k;
        entry_of(e, t, k);
        const int s = e % kStages;
        // A PV two or more entries old holds the V slot (and bias table) of
        // the stage the producer refills next: issue it now.  This matters
        // once one q-tile has run out of key tiles and the other continues.
        if (pend[t ^ 1] >= 0 && pend[t ^ 1] <= e - kStages && !issue_pv(t ^ 1)) {
          ok = false;
          break;
        }
        // S_t(e) overwrites the TMEM columns P_t of the previous entry occupies
        if (pend[t] >= 0 && !issue_pv(t)) {
          ok = false;
          break;
        }
        if (!mbar_wait(&k_full[s], (e / kStages) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + t * 128;
        const uint32_t qbase = sQ + t * L::kTileBytes;
        const uint32_t kbase = sK + s * L::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
          mma_ss(d_tmem, smem_desc(qbase + off, 16, 1024), smem_desc(kbase + off, 16, 1024), kIdescS,
                 kk > 0 ? 1u : 0u);
        }
        mma_commit(&s_ready[t]);
        mma_commit(&k_empty[s]);
        pend[t] = e;
        if (misc[5]) ok = false;
      }
      for (int t = 0; ok && t < 2; ++t)
        if (pend[t] >= 0 && !issue_pv(t)) ok = false;
      if (!ok) misc[5] = 1;
      mma_commit(mma_done);
      mbar_wait(mma_done, 0);
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

  setmaxnreg_inc<112>();
  {
    // ------------------------------------------------------------- softmax ---
    const int sw = warp - kSoftmaxWarp0;
    const int t = sw >> 3;
    const int hf = (sw >> 2) & 1;
    const int sub = warp & 3;
    const int r = sub * 32 + lane;
    const int row = (qtile0 + t) * kTileM + r;
    const bool row_valid = row < p.N;
    const int rh = (QH == 2) ? (r >> 6) : 0;   // which q-block of the tile (bias half)
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(sub * 32) << 16);
    const uint32_t s_addr = lane_base + t * 128 + hf * 64;
    const uint32_t p_addr = lane_base + t * 128 + hf * 32;
    constexpr int kOCols = D / 2;
    const uint32_t o_addr = lane_base + 256 + t * D + hf * kOCols;
    const int cnt = ntile[t];
    const float sl2 = p.scale_log2;
    const float NEG_INF = -__int_as_float(0x7f800000);
    const int bar_id = 1 + t;
    float* red_t = red + t * (2 * 2 * kTileM);

    float m_used = NEG_INF, l_part = 0.f;
    uint32_t sphase = 0;
    int et = 0;
    bool ok = true;
    if (cnt > 0) {
      for (int e = 0; e < n_entries; ++e) {
        int te, k;
        entry_of(e, te, k);
        if (te != t) continue;
        const int st = e % kStages;
        bool w_ok = mbar_wait(&s_ready[t], sphase);
        w_ok = w_ok && mbar_wait(&b_full[st], (e / kStages) & 1);
        w_ok = __all_sync(0xffffffffu, w_ok);
        sphase ^= 1u;
        tc_fence_after();
        float s[64];
        if (w_ok) {
          tmem_ld64(s_addr, s);
        } else {
#pragma unroll
          for (int c = 0; c < 64; ++c) s[c] = 0.f;
        }
        // x = s * scale * log2e + log2(count), -inf on masked / empty columns
        const float4* bsrc = reinterpret_cast<const float4*>(bias + st * 2 * kTileN + rh * kTileN + hf * 64);
#pragma unroll
        for (int c4 = 0; c4 < 16; ++c4) {
          const float4 bv = bsrc[c4];
          s[4 * c4 + 0] = fmaf(s[4 * c4 + 0], sl2, bv.x);
          s[4 * c4 + 1] = fmaf(s[4 * c4 + 1], sl2, bv.y);
          s[4 * c4 + 2] = fmaf(s[4 * c4 + 2], sl2, bv.z);
          s[4 * c4 + 3] = fmaf(s[4 * c4 + 3], sl2, bv.w);
        }
        float a0 = fmaxf(s[0], s[1]), a1 = fmaxf(s[2], s[3]);
        float a2 = fmaxf(s[4], s[5]), a3 = fmaxf(s[6], s[7]);
#pragma unroll
        for (int c = 8; c < 64; c += 8) {
          a0 = fmax3(a0, s[c + 0], s[c + 1]);
          a1 = fmax3(a1, s[c + 2], s[c + 3]);
          a2 = fmax3(a2, s[c + 4], s[c + 5]);
          a3 = fmax3(a3, s[c + 6], s[c + 7]);
        }
        const float m_mine = fmax3(a0, a1, fmaxf(a2, a3));
        float* red_p = red_t + (et & 1) * (2 * kTileM);
        red_p[hf * kTileM + r] = m_mine;
        tc_fence_before();
        ok = named_bar_and(bar_id, 256, w_ok && misc[5] == 0);
        tc_fence_after();
        if (!ok) {
          misc[5] = 1;
          break;
        }
        const float mx = fmaxf(m_mine, red_p[(hf ^ 1) * kTileM + r]);
        float factor = 1.f;
        if (mx > m_used && (m_used == NEG_INF || mx - m_used > 8.f)) {
          factor = (m_used == NEG_INF) ? 0.f : fast_exp2(m_used - mx);
          m_used = mx;
          l_part *= factor;
        }
        if (et > 0 && __any_sync(0xffffffffu, factor != 1.f)) {
#pragma unroll 1
          for (int c = 0; c < kOCols / 32; ++c) {
            float ov[32];
            tmem_ld32(o_addr + c * 32, ov);
#pragma unroll
            for (int i = 0; i < 32; ++i) ov[i] *= factor;
            tmem_st32(o_addr + c * 32, ov);
          }
          tmem_st_wait();
        }
        const float neg_m = (m_used == NEG_INF) ? 0.f : -m_used;
        const float2 nmv = make_float2(neg_m, neg_m);
        float2 acc[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) acc[a] = make_float2(0.f, 0.f);
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float2 x = add2(make_float2(s[2 * i], s[2 * i + 1]), nmv);
          float2 pe;
          if ((i & 15) >= kPolyPairFrom) {
            pe = exp2_poly2(x);
          } else {
            pe.x = fast_exp2(x.x);
            pe.y = fast_exp2(x.y);
          }
          acc[i & 3] = add2(acc[i & 3], pe);
          pk[i] = pack_bf16x2(pe.x, pe.y);
        }
        tmem_st32(p_addr, reinterpret_cast<const float*>(pk));
        const float2 at = add2(add2(acc[0], acc[1]), add2(acc[2], acc[3]));
        l_part += at.x + at.y;
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_ready[t]);
        ++et;
      }
    }

    // ------------------------------------------------------------ epilogue ---
    if (cnt > 0 && ok) {
      ok = mbar_wait(&o_final[t], 0);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) misc[5] = 1;
      tc_fence_after();
    }
    float* red_l = red_t;
    named_bar_sync(bar_id, 256);
    red_l[hf * kTileM + r] = l_part;
    named_bar_sync(bar_id, 256);
    const float l_sum = l_part + red_l[(hf ^ 1) * kTileM + r];
    const float inv_l = l_sum > 0.f ? 1.f / l_sum : 0.f;
    __nv_bfloat16* orow = p.o + (static_cast<size_t>(bh) * p.N + (row_valid ? row : 0)) * D + hf * kOCols;
#pragma unroll 1
    for (int c = 0; c < kOCols / 32; ++c) {
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
    if (p.lse && row_valid && hf == 0)
      p.lse[static_cast<size_t>(bh) * p.N + row] =
          l_sum > 0.f ? (log2f(l_sum) + m_used) * 0.69314718055994531f : NEG_INF;
  }

  tc_fence_before();
  __syncthreads();
}

}  // namespace sa
