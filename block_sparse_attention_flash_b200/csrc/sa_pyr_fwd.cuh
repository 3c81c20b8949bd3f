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
// One CTA = two q-tiles with the same roles as sa_attn_fwd.cuh (one MMA issuer
// per q-tile, one softmax thread per row, P handed over in two halves, the two
// softmax warpgroups taking turns), but each q-tile has its own packed key
// tiles; the entries of the two are interleaved.  K and V
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
// 12 warps: producer, two MMA issuers, one idle, two softmax warpgroups
constexpr int kPyrWarps = 12;
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
  // q_full, k_full[2], v_full[2], k_empty[2], v_empty[2], b_full[2],
  // s_ready[2], pa[2], pb[2], o_final[2], mma_done[2], go[2]
  static constexpr int kNumBars = 1 + 5 * kStages + 2 * 6;
  static constexpr int kOffBar = kOffBias + kStages * 2 * kTileN * 4;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kBytes = kOffMisc + 128;
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
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = bars + 1 + kStages;
  uint64_t* k_empty = bars + 1 + 2 * kStages;
  uint64_t* v_empty = bars + 1 + 3 * kStages;
  uint64_t* b_full = bars + 1 + 4 * kStages;
  uint64_t* s_ready = bars + 1 + 5 * kStages;
  uint64_t* pa = s_ready + 2;
  uint64_t* pb = pa + 2;
  uint64_t* o_final = pb + 2;
  uint64_t* mma_done = o_final + 2;
  uint64_t* go = mma_done + 2;
  volatile int* misc = reinterpret_cast<volatile int*>(smem + L::kOffMisc);
  // misc[0] TMEM base, [1]/[2] segments of q-tile 0/1, [3]/[4] key tiles of q-tile 0/1, [5] abort
  volatile int* grp = misc + 8;   // producer scratch: owning lane of each 8-column group

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
        uint32_t count = 1;
        if (&bars[i] == &k_empty[0] || &bars[i] == &k_empty[1] || &bars[i] == &v_empty[0] ||
            &bars[i] == &v_empty[1])
          count = 2;  // one arrival from each q-tile's MMA issuer
        if (&bars[i] == &pa[0] || &bars[i] == &pa[1] || &bars[i] == &pb[0] || &bars[i] == &pb[1] ||
            &bars[i] == &go[0] || &bars[i] == &go[1])
          count = 128;  // every softmax thread of the tile
        mbar_init(&bars[i], count);
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
  const uint32_t sK = smem_addr(smem + L::kOffK);
  const uint32_t sV = smem_addr(smem + L::kOffV);

  if (warp < kSoftmaxWarp0) {
    setmaxnreg_dec<56>();
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
      const float NEG_INF = -__int_as_float(0x7f800000);
      for (int e = 0; e < n_entries && ok; ++e) {
        int t, k;
        entry_of(e, t, k);
        const int s = e % kStages;
        const uint32_t par = ((e / kStages) - 1) & 1;
        // One lane per segment (a 128-key tile holds at most 128 / 8 = 16):
        // a warp scan of the lengths gives each segment's column.
        const uint32_t* tseg = segs + t * kPyrMaxSegs;
        const int nseg = misc[1 + t];
        const int gi = cursor[t] + lane;
        const uint32_t sg = (lane < 16 && gi < nseg) ? tseg[gi] : 0u;
        const int lvl = static_cast<int>((sg >> 16) & 3u);
        const int len = (lane < 16 && gi < nseg) ? (BLK >> lvl) : 0;
        int incl = len;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        const int col = incl - len;
        const bool mine = len > 0 && incl <= kTileN;
        const unsigned ball = __ballot_sync(0xffffffffu, mine);
        const int nmine = __popc(ball);
        const int fill = nmine > 0 ? __shfl_sync(0xffffffffu, incl, nmine - 1) : 0;
        cursor[t] += nmine;
        const int row = static_cast<int>(sg & 0xFFFFu) * len;

        if (e >= kStages) {
          bool w = lane == 0 ? (misc[5] == 0 && mbar_wait(&k_empty[s], par)) : true;
          if (!__shfl_sync(0xffffffffu, w, 0)) {
            ok = false;
            break;
          }
        }
        uint8_t* kst = smem + L::kOffK + s * L::kTileBytes;
        uint8_t* vst = smem + L::kOffV + s * L::kTileBytes;
        // empty columns [fill, 128): zero K rows so masked products stay finite
        if (fill < kTileN) {
          for (int idx = lane; idx < (kTileN - fill) * 8 * (D / 64); idx += 32) {
            const int hd = idx / ((kTileN - fill) * 8);
            const int rem = idx - hd * (kTileN - fill) * 8;
            reinterpret_cast<uint4*>(kst + hd * kHalfBytes + (fill + rem / 8) * 128)[rem % 8] = make_uint4(0, 0, 0, 0);
          }
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
        if (lane == 0) mbar_arrive_expect_tx(&k_full[s], static_cast<uint32_t>(fill) * D * 2);
        __syncwarp();
        if (mine) {
#pragma unroll
          for (int hd = 0; hd < D / 64; ++hd)
            tma_load_3d(&maps.k[lvl], &k_full[s], kst + hd * kHalfBytes + col * 128, hd * 64, row, bh);
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
        // per-column log2(pooled token count) for row halves A and B: every
        // lane takes columns lane, lane+32, ...; the owner of each 8-column
        // group is looked up in grp[] and its fields fetched by shuffle
        float* bst = bias + s * 2 * kTileN;
        if (mine)
          for (int g = col / 8; g < (col + len) / 8; ++g) grp[g] = lane;
        __syncwarp();
#pragma unroll
        for (int cc = 0; cc < kTileN / 32; ++cc) {
          const int c = cc * 32 + lane;
          const int src = c < fill ? grp[c / 8] : 0;
          const uint32_t sg_o = __shfl_sync(0xffffffffu, sg, src);
          const int col_o = __shfl_sync(0xffffffffu, col, src);
          const int row_o = __shfl_sync(0xffffffffu, row, src);
          float bA = NEG_INF, bB = NEG_INF;
          if (c < fill) {
            const int lv = static_cast<int>((sg_o >> 16) & 3u);
            const uint32_t rm = (sg_o >> 18) & 3u;
            const int gr = row_o + (c - col_o);
            float bv = NEG_INF;
            if (gr < p.pool_rows[lv]) {
              const int count = min(1 << lv, p.N - (gr << lv));
              bv = count == (1 << lv) ? static_cast<float>(lv) : log2f(static_cast<float>(count));
            }
            bA = (rm & 1u) ? bv : NEG_INF;
            bB = (QH == 1 ? (rm & 1u) : (rm & 2u)) ? bv : NEG_INF;
          }
          bst[c] = bA;
          bst[kTileN + c] = bB;
        }
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&b_full[s]);
          mbar_arrive_expect_tx(&v_full[s], static_cast<uint32_t>(fill) * D * 2);
        }
        __syncwarp();
        if (mine) {
#pragma unroll
          for (int hd = 0; hd < D / 64; ++hd)
            tma_load_3d(&maps.v[lvl], &v_full[s], vst + hd * kHalfBytes + col * 128, hd * 64, row, bh);
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
  } else if (warp <= 2) {
    // ---------------------------------------------- MMA issue, q-tile t ---
    const int t = warp - 1;
    if (lane == 0 && n_entries > 0) {
      const int cnt = ntile[t];
      bool ok = mbar_wait(q_full, 0);
      const uint64_t dq = smem_desc(smem_addr(smem + L::kOffQ + t * L::kTileBytes), 16, 1024);
      const uint64_t dk0 = smem_desc(sK, 16, 1024);
      const uint64_t dv0 = smem_desc(sV, kHalfBytes, 1024);
      constexpr uint64_t kStageStep = L::kTileBytes >> 4;
      const uint32_t s_tmem = tmem + t * 128;
      const uint32_t o_tmem = tmem + 256 + t * D;
      int pend = -1, done = 0;
      uint32_t pph = 0;
      auto issue_pv = [&]() -> bool {
        const int ps = pend % kStages;
        const uint64_t dv = dv0 + ps * kStageStep;
        if (!mbar_wait(&pa[t], pph) || !mbar_wait(&v_full[ps], (pend / kStages) & 1)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ts(o_tmem, s_tmem + kk * 8, dv + ((kk * 16 * 128) >> 4), kIdescPV, (done == 0 && kk == 0) ? 0u : 1u);
        if (!mbar_wait(&pb[t], pph)) return false;
        tc_fence_after();
#pragma unroll
        for (int kk = 4; kk < 8; ++kk)
          mma_ts(o_tmem, s_tmem + kk * 8, dv + ((kk * 16 * 128) >> 4), kIdescPV, 1u);
        pph ^= 1u;
        mma_commit(&v_empty[ps]);
        if (++done == cnt) mma_commit(&o_final[t]);
        pend = -1;
        return true;
      };
      for (int e = 0; ok && e < n_entries; ++e) {
        int te, k;
        entry_of(e, te, k);
        const int s = e % kStages;
        const uint32_t par = (e / kStages) & 1;
        if (pend >= 0 && !issue_pv()) {
          ok = false;
          break;
        }
        // every entry's K must have landed before this tile reports the slot free
        if (!mbar_wait(&k_full[s], par)) {
          ok = false;
          break;
        }
        if (te == t) {
          tc_fence_after();
          const uint64_t dk = dk0 + s * kStageStep;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t off = static_cast<uint64_t>((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4;
            mma_ss(s_tmem, dq + off, dk + off, kIdescS, kk > 0 ? 1u : 0u);
          }
          mma_commit(&s_ready[t]);
          mma_commit(&k_empty[s]);
          pend = e;
        } else {
          mma_commit(&k_empty[s]);
          if (!mbar_wait(&v_full[s], par)) {
            ok = false;
            break;
          }
          mma_commit(&v_empty[s]);
        }
        if (misc[5]) ok = false;
      }
      if (ok && pend >= 0 && !issue_pv()) ok = false;
      if (!ok) misc[5] = 1;
      mma_commit(&mma_done[t]);
      mbar_wait(&mma_done[t], 0);
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
    const bool row_valid = row < p.N;
    const int rh = (QH == 2) ? (r >> 6) : 0;   // which q-block of the tile (bias half)
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const uint32_t s_addr = lane_base + t * 128;
    const uint32_t o_addr = lane_base + 256 + t * D;
    const int cnt = ntile[t];
    const float sl2 = p.scale_log2;
    const float NEG_INF = -__int_as_float(0x7f800000);

    float m_used = NEG_INF, l_sum = 0.f;
    uint32_t sphase = 0, gphase = 0;
    int et = 0;
    bool ok = true;
    if (cnt > 0) {
      for (int e = 0; e < n_entries; ++e) {
        int te, k;
        entry_of(e, te, k);
        if (te != t) continue;
        const int st = e % kStages;
        bool w_ok = true;
        if (e > 0) {                       // wait for our turn
          w_ok = mbar_wait(&go[t], gphase);
          gphase ^= 1u;
        }
        w_ok = w_ok && mbar_wait(&s_ready[t], sphase) && mbar_wait(&b_full[st], (e / kStages) & 1);
        ok = __all_sync(0xffffffffu, w_ok) && misc[5] == 0;
        if (!ok) {
          misc[5] = 1;
          break;
        }
        sphase ^= 1u;
        tc_fence_after();
        float s[kTileN];
        tmem_ld128(s_addr, s);
        // x = s * scale * log2e + log2(count), -inf on masked / empty columns
        const float4* bsrc = reinterpret_cast<const float4*>(bias + st * 2 * kTileN + rh * kTileN);
#pragma unroll
        for (int c4 = 0; c4 < 32; ++c4) {
          const float4 bv = bsrc[c4];
          s[4 * c4 + 0] = fmaf(s[4 * c4 + 0], sl2, bv.x);
          s[4 * c4 + 1] = fmaf(s[4 * c4 + 1], sl2, bv.y);
          s[4 * c4 + 2] = fmaf(s[4 * c4 + 2], sl2, bv.z);
          s[4 * c4 + 3] = fmaf(s[4 * c4 + 3], sl2, bv.w);
        }
        float a[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) a[u] = fmaxf(s[2 * u], s[2 * u + 1]);
#pragma unroll
        for (int c = 16; c < kTileN; c += 16) {
#pragma unroll
          for (int u = 0; u < 8; ++u) a[u] = fmax3(a[u], s[c + 2 * u], s[c + 2 * u + 1]);
        }
        const float mx = fmaxf(fmax3(a[0], a[1], a[2]), fmax3(a[3], a[4], fmax3(a[5], a[6], a[7])));
        float factor = 1.f;
        if (mx > m_used && (m_used == NEG_INF || mx - m_used > 8.f)) {
          factor = (m_used == NEG_INF) ? 0.f : fast_exp2(m_used - mx);
          m_used = mx;
          l_sum *= factor;
        }
        if (et > 0 && __any_sync(0xffffffffu, factor != 1.f)) {
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
        const float neg_m = (m_used == NEG_INF) ? 0.f : -m_used;
        {
          uint32_t pk[32];
          l_sum += exp_pack_64(s, 1.f, neg_m, pk);
          tmem_st32(s_addr, reinterpret_cast<const float*>(pk));
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(&pa[t]);
        }
        {
          uint32_t pk[32];
          l_sum += exp_pack_64(s + 64, 1.f, neg_m, pk);
          tmem_st32(s_addr + 32, reinterpret_cast<const float*>(pk));
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(&pb[t]);
        }
        if (e + 1 < n_entries) {           // pass the turn to the next entry's tile
          int tn, kn;
          entry_of(e + 1, tn, kn);
          mbar_arrive(&go[tn]);
        }
        ++et;
      }
    }

    // ------------------------------------------------------------ epilogue ---
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
          l_sum > 0.f ? (log2f(l_sum) + m_used) * 0.69314718055994531f : NEG_INF;
  }
  tc_fence_before();
  __syncthreads();
}

}  // namespace sa
