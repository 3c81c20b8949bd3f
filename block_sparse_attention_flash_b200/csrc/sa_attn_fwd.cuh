// sa_attn_fwd.cuh — block-sparse attention forward for sm_100a with the
// LiteAttention skip update fused into the online softmax.
//
// Work unit: one CTA owns two 128-row q-tiles (rows [256*pair, 256*pair+256))
// of one (b, h) and walks the union of their kept 128-column kv tiles in
// ascending order.  Each kv tile is loaded once by TMA and feeds both q-tiles.
//
// Roles (640 threads = 20 warps, one CTA per SM; warps 2-3 only join the
// final barrier, they keep the softmax warps aligned to TMEM lane quarters):
//   warp 0       builds the kv-tile list from the mask / skip bytes, then one
//                lane issues the TMA loads (Q once, K and V through 2-stage
//                rings released separately; skipped tiles are never loaded:
//                LiteAttention write-up, sections 3 and 6);
//   warp 1       owns TMEM (512 columns) and one lane issues every
//                tcgen05.mma: S_t = Q_t K^T (both operands from shared memory)
//                and O_t += P_t V (A operand P_t read from TMEM, where the
//                softmax wrote it over S_t);
//   warps 4-11   online softmax of q-tile 0, warps 12-19 of q-tile 1.  Two
//                threads per row: warps [4,8) take columns 0-63 of rows
//                32*(warp%4) .. +31 (a warp may only touch its own TMEM lane
//                quarter), warps [8,12) columns 64-127; the two halves swap
//                their row maxima through shared memory once per kv tile.
//                They evaluate the skip condition on the maxima they compute
//                anyway (LiteAttention write-up, section 5), record it per
//                warp and reduce across warps only at kernel end (section 6).
//
// TMEM columns: S0 [0,128), S1 [128,256), O0 [256,256+D), O1 [384,384+D).
// Shared memory: Q0, Q1, K[2], V[2] tiles of 128 x D bf16 in the 128-byte
// swizzled layout TMA writes (each 64-column half is a [128 x 128 B] slab),
// the kv list, the per-warp skip votes, the row-max exchange and mbarriers.
//
// Block size 64: a 128-row tile holds q-blocks 2i, 2i+1 and a 128-column kv
// tile holds k-blocks 2j, 2j+1; the list keeps per-quadrant bits and the
// softmax masks the quadrants a q-block does not keep.
#pragma once

#include "sa_common.cuh"

namespace sa {

constexpr int kTileM = 128;
constexpr int kTileN = 128;
constexpr int kStages = 2;
constexpr int kMaxKvTiles = 4096;
constexpr int kAttnWarps = 20;
constexpr int kAttnThreads = kAttnWarps * 32;
constexpr int kSoftmaxWarp0 = 4;
// Within each 16-pair chunk of a row, pairs [kPolyPairFrom, 16) take 2^x from
// the FMA-pipe polynomial instead of the MUFU unit (balances the two pipes).
constexpr int kPolyPairFrom = 12;

struct AttnParams {
  int B, H, N;
  int nb;           // blocks per sequence, ceil(N / block)
  int n_kv_tiles;   // ceil(N / 128)
  const uint8_t* mask;
  long long msb, msh, msi;
  const uint8_t* skip_in;
  uint8_t* skip_out;
  int write_skip;   // skip_out != NULL
  int carry_skip;   // skip_out != NULL && skip_out != skip_in
  float scale_log2; // scale * log2(e)
  float eps_raw;    // eps / scale: the skip threshold in raw q.k units
  __nv_bfloat16* o;
  float* lse;
};

template <int D>
struct AttnSmem {
  static constexpr int kTileBytes = kTileM * D * 2;
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = 2 * kTileBytes;
  static constexpr int kOffV = kOffK + kStages * kTileBytes;
  static constexpr int kOffList = kOffV + kStages * kTileBytes;
  static constexpr int kVoteWords = kMaxKvTiles / 32;      // per softmax warp
  static constexpr int kOffVotes = kOffList + kMaxKvTiles * 4;
  static constexpr int kOffRed = kOffVotes + 16 * kVoteWords * 4;
  static constexpr int kRedFloats = 2 * 2 * 2 * kTileM;    // [tile][parity][half][row]
  static constexpr int kNumBars = 1 + 4 * kStages + 2 + 2 + 2 + 1;
  static constexpr int kOffBar = kOffRed + kRedFloats * 4;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kBytes = kOffMisc + 64;
  static constexpr int kAlloc = kBytes + 1024;
};

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Named barrier over `nthreads` threads that also returns the AND of `v`
// over all of them, so that every participant takes the same branch.
__device__ __forceinline__ bool named_bar_and(int id, int nthreads, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %2, 0;\n\t"
      "bar.red.and.pred po, %1, %3, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"(id), "r"(static_cast<uint32_t>(v)), "r"(nthreads)
      : "memory");
  return r != 0;
}

template <int D, int BLK>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using L = AttnSmem<D>;
  constexpr int QH = kTileM / BLK;  // q-blocks per q-tile
  constexpr int KH = kTileN / BLK;  // k-blocks per kv tile
  constexpr uint32_t kIdescS = idesc_bf16_f32(kTileM, kTileN, false);
  constexpr uint32_t kIdescPV = idesc_bf16_f32(kTileM, D, true);
  constexpr int kHalfBytes = kTileM * 128;  // one 64-column slab of a tile

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint32_t* list = reinterpret_cast<uint32_t*>(smem + L::kOffList);
  uint32_t* votes = reinterpret_cast<uint32_t*>(smem + L::kOffVotes);
  float* red = reinterpret_cast<float*>(smem + L::kOffRed);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = bars + 1 + kStages;
  uint64_t* k_empty = bars + 1 + 2 * kStages;
  uint64_t* v_empty = bars + 1 + 3 * kStages;
  uint64_t* s_ready = bars + 1 + 4 * kStages;
  uint64_t* p_ready = s_ready + 2;
  uint64_t* o_final = p_ready + 2;
  uint64_t* mma_done = o_final + 2;
  volatile int* misc = reinterpret_cast<volatile int*>(smem + L::kOffMisc);
  // misc[0] TMEM base, [1] list length, [2] / [3] kv tiles of q-tile 0 / 1, [4] abort flag

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x, bh = blockIdx.y;
  const int b = bh / p.H, h = bh - (bh / p.H) * p.H;
  const int qtile0 = 2 * pair;

  for (int i = threadIdx.x; i < 16 * L::kVoteWords; i += kAttnThreads) votes[i] = 0;

  if (warp == 0) {
    // ---- kv-tile list: union over the two q-tiles, per-quadrant keep bits ----
    int n = 0, c0 = 0, c1 = 0;
    for (int base = 0; base < p.n_kv_tiles; base += 32) {
      const int jt = base + lane;
      uint32_t bits = 0;
      if (jt < p.n_kv_tiles) {
#pragma unroll
        for (int t = 0; t < 2; ++t) {
#pragma unroll
          for (int qh = 0; qh < QH; ++qh) {
            const int qb = (qtile0 + t) * QH + qh;
            if (qb >= p.nb) continue;
#pragma unroll
            for (int kh = 0; kh < KH; ++kh) {
              const int kb = jt * KH + kh;
              if (kb >= p.nb) continue;
              const uint8_t keep = p.mask ? p.mask[b * p.msb + h * p.msh + qb * p.msi + kb] : uint8_t(1);
              const size_t sidx = (static_cast<size_t>(bh) * p.nb + qb) * p.nb + kb;
              const uint8_t sk = p.skip_in ? p.skip_in[sidx] : uint8_t(0);
              if (keep && !sk) {
                bits |= (BLK == 128 ? 0xFu : (1u << (qh * 2 + kh))) << (16 + 4 * t);
              } else if (p.carry_skip) {
                p.skip_out[sidx] = sk;
              }
            }
          }
        }
      }
      const unsigned ball = __ballot_sync(0xffffffffu, bits != 0);
      if (bits) list[n + __popc(ball & ((1u << lane) - 1u))] = static_cast<uint32_t>(jt) | bits;
      n += __popc(ball);
      c0 += __popc(__ballot_sync(0xffffffffu, (bits >> 16) & 0xFu));
      c1 += __popc(__ballot_sync(0xffffffffu, (bits >> 20) & 0xFu));
    }
    if (lane == 0) {
      misc[1] = n;
      misc[2] = c0;
      misc[3] = c1;
      misc[4] = 0;
      for (int i = 0; i < L::kNumBars; ++i) {
        const bool softmax_arrivals = (&bars[i] == &p_ready[0]) || (&bars[i] == &p_ready[1]);
        mbar_init(&bars[i], softmax_arrivals ? 256u : 1u);
      }
      fence_mbar_init();
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
    }
  } else if (warp == 1) {
    tmem_alloc(const_cast<uint32_t*>(reinterpret_cast<volatile uint32_t*>(misc)), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = static_cast<uint32_t>(misc[0]);
  const int n_list = misc[1];
  const uint32_t sQ = smem_addr(smem + L::kOffQ);
  const uint32_t sK = smem_addr(smem + L::kOffK);
  const uint32_t sV = smem_addr(smem + L::kOffV);

  if (warp < kSoftmaxWarp0) {
    // Register split: this warpgroup gives up registers the softmax rows use.
    // Each role runs to its own final barrier so the two register budgets
    // never meet in shared code.
    setmaxnreg_dec<32>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer ---
    if (lane == 0 && n_list > 0) {
      const int cnt0 = misc[2], cnt1 = misc[3];
      const uint32_t qbytes = static_cast<uint32_t>((cnt0 > 0) + (cnt1 > 0)) * L::kTileBytes;
      mbar_arrive_expect_tx(q_full, qbytes);
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if ((t == 0 ? cnt0 : cnt1) == 0) continue;
#pragma unroll
        for (int hd = 0; hd < D / 64; ++hd)
          tma_load_3d(&tmQ, q_full, smem + L::kOffQ + t * L::kTileBytes + hd * kHalfBytes, hd * 64,
                      (qtile0 + t) * kTileM, bh);
      }
      int issued = 0;
      for (int e = 0; e < n_list; ++e) {
        const int s = e % kStages;
        const uint32_t par = ((e / kStages) - 1) & 1;
        if (e >= kStages && (misc[4] || !mbar_wait(&k_empty[s], par))) {
          misc[4] = 1;
          break;
        }
        const int row = static_cast<int>(list[e] & 0xFFFFu) * kTileN;
        mbar_arrive_expect_tx(&k_full[s], L::kTileBytes);
#pragma unroll
        for (int hd = 0; hd < D / 64; ++hd)
          tma_load_3d(&tmK, &k_full[s], smem + L::kOffK + s * L::kTileBytes + hd * kHalfBytes, hd * 64, row, bh);
        if (e >= kStages && !mbar_wait(&v_empty[s], par)) {
          misc[4] = 1;
          issued = e;
          mbar_wait(&k_full[s], (e / kStages) & 1);
          break;
        }
        mbar_arrive_expect_tx(&v_full[s], L::kTileBytes);
#pragma unroll
        for (int hd = 0; hd < D / 64; ++hd)
          tma_load_3d(&tmV, &v_full[s], smem + L::kOffV + s * L::kTileBytes + hd * kHalfBytes, hd * 64, row, bh);
        issued = e + 1;
      }
      // Loads still in flight must land before the CTA can exit.
      for (int e = (issued > kStages ? issued - kStages : 0); e < issued; ++e) {
        const int s = e % kStages;
        mbar_wait(&k_full[s], (e / kStages) & 1);
        mbar_wait(&v_full[s], (e / kStages) & 1);
      }
      if ((cnt0 | cnt1) != 0) mbar_wait(q_full, 0);
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issue ---
    if (lane == 0 && n_list > 0) {
      const int cnt[2] = {misc[2], misc[3]};
      bool ok = mbar_wait(q_full, 0);
      if (!ok) misc[4] = 1;
      int pend[2] = {-1, -1};
      int done_pv[2] = {0, 0};
      uint32_t pphase[2] = {0u, 0u};
      int users[kStages];
#pragma unroll
      for (int s = 0; s < kStages; ++s) users[s] = 0;

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
        for (int kk = 0; kk < kTileN / 16; ++kk) {
          const uint64_t bdesc = smem_desc(vbase + kk * 16 * 128, kHalfBytes, 1024);
          mma_ts(d_tmem, a_tmem + kk * 8, bdesc, kIdescPV, (done_pv[t] == 0 && kk == 0) ? 0u : 1u);
        }
        if (--users[s] == 0) mma_commit(&v_empty[s]);
        if (++done_pv[t] == cnt[t]) mma_commit(&o_final[t]);
        pend[t] = -1;
        return true;
      };

      for (int e = 0; ok && e < n_list; ++e) {
        const int s = e % kStages;
        const uint32_t bits = list[e];
        const int last_t = ((bits >> 20) & 0xFu) ? 1 : 0;
        bool k_waited = false;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          if (pend[t] >= 0 && !issue_pv(t)) {
            ok = false;
            break;
          }
          if (((bits >> (16 + 4 * t)) & 0xFu) == 0) continue;
          if (!k_waited) {
            if (!mbar_wait(&k_full[s], (e / kStages) & 1)) {
              ok = false;
              break;
            }
            k_waited = true;
            users[s] = 0;
          }
          ++users[s];
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
          if (t == last_t) mma_commit(&k_empty[s]);
          pend[t] = e;
        }
        if (misc[4]) ok = false;
      }
      for (int t = 0; ok && t < 2; ++t)
        if (pend[t] >= 0 && !issue_pv(t)) ok = false;
      if (!ok) misc[4] = 1;
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
    const int sw = warp - kSoftmaxWarp0;       // 0..15
    const int t = sw >> 3;                     // q-tile
    const int hf = (sw >> 2) & 1;              // column half of the S tile
    const int sub = warp & 3;                  // TMEM lane quarter = row group
    const int r = sub * 32 + lane;
    const int row = (qtile0 + t) * kTileM + r;
    const bool row_valid = row < p.N;
    const int qh = (BLK == 64) ? (r >> 6) : 0;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(sub * 32) << 16);
    const uint32_t s_addr = lane_base + t * 128 + hf * 64;     // this thread's 64 S columns
    const uint32_t p_addr = lane_base + t * 128 + hf * 32;     // its 32 packed P columns
    constexpr int kOCols = D / 2;                               // O columns this thread owns
    const uint32_t o_addr = lane_base + 256 + t * D + hf * kOCols;
    const int cnt = misc[2 + t];
    const float sl2 = p.scale_log2;
    const float NEG_INF = -__int_as_float(0x7f800000);
    const int bar_id = 1 + t;
    float* red_t = red + t * (2 * 2 * kTileM);

    float m_used = NEG_INF, m_true = NEG_INF, l_part = 0.f;
    uint32_t sphase = 0;
    int et = 0;
    bool ok = true;
    uint32_t* my_votes = votes + ((t * 4 + sub) * 2 + hf) * L::kVoteWords;

    if (cnt > 0) {
      for (int e = 0; e < n_list; ++e) {
        const uint32_t ent = list[e];
        const uint32_t bits = (ent >> (16 + 4 * t)) & 0xFu;
        if (!bits) continue;
        const int jt = static_cast<int>(ent & 0xFFFFu);
        // A bounded wait that runs out is only acted on at the barrier below,
        // which every thread of the tile reaches, so no thread is left waiting.
        const bool w_ok = __all_sync(0xffffffffu, mbar_wait(&s_ready[t], sphase));
        sphase ^= 1u;
        tc_fence_after();

        float s[64];
        if (w_ok) {
          tmem_ld64(s_addr, s);
        } else {
#pragma unroll
          for (int c = 0; c < 64; ++c) s[c] = NEG_INF;
        }

        // mask columns past N and quadrants this row's q-block does not keep
        const int valid_cols = min(64, p.N - jt * kTileN - hf * 64);
        const bool keep_half = BLK == 128 ? true : ((bits >> (qh * 2 + hf)) & 1u);
        if (valid_cols < 64 || !keep_half) {
#pragma unroll
          for (int c = 0; c < 64; ++c) s[c] = (keep_half && c < valid_cols) ? s[c] : NEG_INF;
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
        // swap half maxima with the partner thread (same row, other half)
        float* red_p = red_t + (et & 1) * (2 * kTileM);
        red_p[hf * kTileM + r] = m_mine;
        tc_fence_before();
        ok = named_bar_and(bar_id, 256, w_ok && misc[4] == 0);
        tc_fence_after();
        if (!ok) {
          misc[4] = 1;
          break;
        }
        const float m_other = red_p[(hf ^ 1) * kTileM + r];
        const float mx0 = hf == 0 ? m_mine : m_other;
        const float mx1 = hf == 0 ? m_other : m_mine;
        const float mx = fmaxf(mx0, mx1);

        if (p.write_skip) {
          if (BLK == 128) {
            if (hf == 0) {
              const bool pred = !row_valid || (mx < m_true - p.eps_raw);
              const bool all = __all_sync(0xffffffffu, pred);
              if (lane == 0 && all) my_votes[e >> 5] |= 1u << (e & 31);
            }
          } else if ((bits >> (qh * 2 + hf)) & 1u) {
            // k-block 2j is visited before 2j+1: half 1 tests against the
            // running max including half 0 (-inf when half 0 is masked)
            const float m_test = hf == 0 ? m_true : fmaxf(m_true, mx0);
            const bool pred = !row_valid || (m_mine < m_test - p.eps_raw);
            const bool all = __all_sync(0xffffffffu, pred);
            if (lane == 0 && all) my_votes[e >> 5] |= 1u << (e & 31);
          }
          m_true = fmaxf(m_true, mx);
        }

        // online softmax with a lazily updated reference maximum
        float factor = 1.f;
        if (mx > m_used && (m_used == NEG_INF || (mx - m_used) * sl2 > 8.f)) {
          factor = (m_used == NEG_INF) ? 0.f : fast_exp2((m_used - mx) * sl2);
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
        // p = 2^(s*scale*log2e - m): pairs through packed fp32 ops; pairs
        // kPolyPairFrom..15 of every 16 use the FMA-pipe polynomial.
        const float neg_m = (m_used == NEG_INF) ? 0.f : -m_used * sl2;
        const float2 sl2v = make_float2(sl2, sl2), nmv = make_float2(neg_m, neg_m);
        float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int c = ch * 32 + 2 * i;
            const float2 x = fma2(make_float2(s[c], s[c + 1]), sl2v, nmv);
            float2 pe;
            if (i >= kPolyPairFrom) {
              pe = exp2_poly2(x);
            } else {
              pe.x = fast_exp2(x.x);
              pe.y = fast_exp2(x.y);
            }
            if (i & 1) acc1 = add2(acc1, pe);
            else acc0 = add2(acc0, pe);
            pk[i] = pack_bf16x2(pe.x, pe.y);
          }
          tmem_st16(p_addr + ch * 16, pk);
        }
        const float2 at = add2(acc0, acc1);
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
      if (!ok) misc[4] = 1;
      tc_fence_after();
    }
    // row sum = both halves' partial sums
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
    if (p.lse && row_valid && hf == 0) {
      const float neg_m = (m_used == NEG_INF) ? 0.f : -m_used * sl2;
      p.lse[static_cast<size_t>(bh) * p.N + row] =
          l_sum > 0.f ? (log2f(l_sum) - neg_m) * 0.69314718055994531f : NEG_INF;
    }

    // ----------------------------------- skip bits: cross-warp AND at the end ---
    if (p.write_skip && cnt > 0 && ok && !misc[4]) {
      const int tid = sw * 32 + lane - t * 256;   // 0..255 within the tile
      // votes of the tile: [sub][half][words]
      const uint32_t* tv = votes + t * 8 * L::kVoteWords;
      for (int e = tid; e < n_list; e += 256) {
        const uint32_t ent = list[e];
        const uint32_t bits = (ent >> (16 + 4 * t)) & 0xFu;
        if (!bits) continue;
        const int jt = static_cast<int>(ent & 0xFFFFu);
        const uint32_t word = e >> 5, bit = e & 31;
#pragma unroll
        for (int qq = 0; qq < QH; ++qq) {
#pragma unroll
          for (int kh = 0; kh < KH; ++kh) {
            if (BLK == 64 && !((bits >> (qq * 2 + kh)) & 1u)) continue;
            const int qb = (qtile0 + t) * QH + qq;
            const int kb = jt * KH + kh;
            uint32_t all = 1u;
            if (BLK == 128) {
#pragma unroll
              for (int sb = 0; sb < 4; ++sb) all &= tv[(sb * 2 + 0) * L::kVoteWords + word] >> bit;
            } else {
#pragma unroll
              for (int sb = 2 * qq; sb < 2 * qq + 2; ++sb) all &= tv[(sb * 2 + kh) * L::kVoteWords + word] >> bit;
            }
            p.skip_out[(static_cast<size_t>(bh) * p.nb + qb) * p.nb + kb] = static_cast<uint8_t>(all & 1u);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
}

}  // namespace sa
