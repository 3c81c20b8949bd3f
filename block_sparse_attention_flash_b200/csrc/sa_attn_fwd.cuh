// sa_attn_fwd.cuh — block-sparse attention forward for sm_100a with the
// LiteAttention skip update fused into the online softmax.
//
// Work unit: one CTA owns two 128-row q-tiles (rows [256*pair, 256*pair+256))
// of one (b, h) and walks the union of their kept 128-column kv tiles in
// ascending (or radial-centric) order.  Each kv tile is loaded once by TMA and
// feeds both q-tiles.
//
// Roles (384 threads = 12 warps, one CTA per SM):
//   warp 0       builds the kv-tile list from the mask / skip bytes, loads Q
//                and K by TMA (2-slot ring) and issues every S = Q_t K^T
//                (tcgen05.mma, both operands in shared memory) into the one S
//                buffer, which the two q-tiles use in turn (skipped tiles are
//                never loaded: LiteAttention write-up, sections 3 and 6);
//   warp 3       loads V by TMA (2-slot ring);
//   warps 1, 2   issue O_t += P_t V for q-tile 0 / 1 (A operand P_t in TMEM,
//                V in shared memory); warp 1 also owns TMEM (512 columns);
//   warps 4-7    online softmax of q-tile 0, warps 8-11 of q-tile 1, one row
//                per thread (a warp may only touch its own TMEM lane quarter).
//                A softmax warpgroup hands the S buffer back as soon as its
//                tcgen05.ld has landed, so the next S (of the other q-tile)
//                is computed while it works; P goes to the tile's own P
//                columns in two 64-column halves, each handed to the PV warp
//                at once, so the first half of PV runs while the second half
//                is computed.  The skip condition is evaluated on the row
//                maxima the softmax computes anyway (LiteAttention write-up,
//                section 5), recorded per warp and reduced across warps at
//                kernel end (section 6).
// Hand-offs between a softmax warpgroup and an issuing warp are named
// barriers (a few tens of cycles), data arrival and MMA completion are
// mbarriers.  All MMA issue is warp-wide with one elected lane, so the
// operands stay in uniform registers.  The producer/MMA warpgroup hands
// registers to the softmax warpgroups (setmaxnreg); each role runs to its own
// final barrier.
//
// TMEM columns: S [0,128), P0 [128,192), P1 [192,256) (bf16 pairs),
// O0 [256,256+D), O1 [256+D,256+2D).
// Shared memory: Q0, Q1, K[2], V[2] tiles of 128 x D bf16 in the 128-byte
// swizzled layout TMA writes (each 64-column half is a [128 x 128 B] slab),
// the kv list, the per-warp skip votes and the mbarriers.
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
constexpr int kAttnWarps = 12;
constexpr int kAttnThreads = kAttnWarps * 32;
constexpr int kSoftmaxWarp0 = 4;

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
  int radial;       // visit kv tiles in radial-centric order (else ascending)
  int causal;       // key c visible to row r only if c <= r (blocks j > i dropped); selects the kernel
  int n_pairs;      // q-tile pairs per head
  int n_full;       // CTAs [0, n_full) take a whole pair; each later pair runs as two CTAs, one per q-tile
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
  static constexpr int kVoteWords = kMaxKvTiles * 2 / 32;  // per softmax warp
  static constexpr int kOffVotes = kOffList + kMaxKvTiles * 4;
  // q_full, k_full[2], v_full[2], v_empty[2], s_ready[2], pv_done_a[2],
  // pv_done_b[2], o_final[2], mma_done[3]
  static constexpr int kNumBars = 1 + 3 * kStages + 2 * 4 + 3;
  static constexpr int kOffBar = kOffVotes + 8 * kVoteWords * 4;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kBytes = kOffMisc + 64;
  static constexpr int kAlloc = kBytes + 1024;
};

// Named barriers (id 0 is __syncthreads): per-warpgroup epilogue syncs, and
// the hand-offs between softmax warpgroup t (128 threads) and an MMA-issuing
// warp (32 threads).  Each id joins the same two parties every time, both
// sides use bar.sync, and every party runs its full, list-determined
// sequence of syncs (also after an error, skipping only its MMAs and loads),
// so the syncs pair up in order and none can wait forever.
constexpr int kBarEpi = 1;      // + t, 128 threads
constexpr int kBarSFree = 3;    // + t: the S buffer loaded by softmax t <-> S issuer
constexpr int kBarPA = 5;       // + t: first half of P_t written <-> PV issuer t
constexpr int kBarPB = 7;       // + t: second half of P_t written <-> PV issuer t
constexpr int kHandoff = 160;

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// p = 2^x for 64 logits s[c] (x = s * sl2 + neg_m), packed to 32 bf16 pairs;
// returns the fp32 sum.  The scale-and-shift and the sums run on packed
// f32x2 FMA / ADD (two lanes per instruction): the softmax loop is partly
// bound by instruction issue, and halving these instructions measured 4.8 %
// faster end to end at 75.6K tokens.  2^x itself comes from the MUFU ex2
// (moving a share of it to an FMA-pipe polynomial measured slower: 12.5 % of
// the pairs -2.4 %, 25 % -5.5 %).
__device__ __forceinline__ float exp_pack_64(const float* s, float sl2, float neg_m, uint32_t* pk) {
  float2 acc[4];
#pragma unroll
  for (int a = 0; a < 4; ++a) acc[a] = make_float2(0.f, 0.f);
  const float2 sl2v = make_float2(sl2, sl2), nmv = make_float2(neg_m, neg_m);
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const float2 x = fma2(make_float2(s[2 * i], s[2 * i + 1]), sl2v, nmv);
    const float p0 = fast_exp2(x.x), p1 = fast_exp2(x.y);
    acc[i & 3] = add2(acc[i & 3], make_float2(p0, p1));
    pk[i] = pack_bf16x2(p0, p1);
  }
  const float2 t = add2(add2(acc[0], acc[1]), add2(acc[2], acc[3]));
  return t.x + t.y;
}

template <int D, int BLK, bool CAUSAL>
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
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = k_full + kStages;
  uint64_t* v_empty = v_full + kStages;
  uint64_t* s_ready = v_empty + kStages;
  uint64_t* pv_done_a = s_ready + 2;
  uint64_t* pv_done_b = pv_done_a + 2;
  uint64_t* o_final = pv_done_b + 2;
  uint64_t* mma_done = o_final + 2;   // one per MMA-issuing warp
  volatile int* misc = reinterpret_cast<volatile int*>(smem + L::kOffMisc);
  // misc[0] TMEM base, [1] list length, [2] / [3] kv tiles of q-tile 0 / 1, [4] abort flag

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Work unit u = bh * n_pairs + pair, in launch order.  Units from n_full on
  // (the last, partial wave of a launch) run as two CTAs each; a CTA then
  // treats the pair's other q-tile as absent: no list bits, no writes.
  int unit = blockIdx.x, skip_t = -1;
  if (unit >= p.n_full) {
    const int x = unit - p.n_full;
    unit = p.n_full + (x >> 1);
    skip_t = 1 - (x & 1);
  }
  const int bh = unit / p.n_pairs, pair = unit - bh * p.n_pairs;
  const int b = bh / p.H, h = bh - (bh / p.H) * p.H;
  const int qtile0 = 2 * pair;

  for (int i = threadIdx.x; i < 8 * L::kVoteWords; i += kAttnThreads) votes[i] = 0;

  if (warp == 0) {
    // ---- kv-tile list: union over the two q-tiles, per-quadrant keep bits ----
    // Ascending: slot s is kv tile s.  Radial-centric: the CTA's 256 query
    // rows have diagonal kv tiles qtile0 and qtile0 + 1 (distance 0); slot
    // 2*dd is tile qtile0 - dd and slot 2*dd + 1 tile qtile0 + 1 + dd, so the
    // slots run by ascending distance, ties by ascending tile, and a slot
    // outside [0, n_kv_tiles) holds nothing.
    const int n_slots = p.radial ? 2 * max(qtile0, p.n_kv_tiles - qtile0 - 1) + 2 : p.n_kv_tiles;
    int n = 0, c0 = 0, c1 = 0;
    for (int base = 0; base < n_slots; base += 32) {
      const int sl = base + lane;
      const int jt = !p.radial ? sl : (sl < 2 ? qtile0 + sl : ((sl & 1) ? qtile0 + 1 + (sl >> 1) : qtile0 - (sl >> 1)));
      uint32_t bits = 0;
      if (sl < n_slots && jt >= 0 && jt < p.n_kv_tiles) {
#pragma unroll
        for (int t = 0; t < 2; ++t) {
#pragma unroll
          for (int qh = 0; qh < QH; ++qh) {
            const int qb = (qtile0 + t) * QH + qh;
            if (qb >= p.nb || t == skip_t) continue;
#pragma unroll
            for (int kh = 0; kh < KH; ++kh) {
              const int kb = jt * KH + kh;
              if (kb >= p.nb) continue;
              const uint8_t keep = p.mask ? p.mask[b * p.msb + h * p.msh + qb * p.msi + kb] : uint8_t(1);
              const size_t sidx = (static_cast<size_t>(bh) * p.nb + qb) * p.nb + kb;
              const uint8_t sk = p.skip_in ? p.skip_in[sidx] : uint8_t(0);
              if (keep && !sk && (!CAUSAL || kb <= qb)) {
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
        // v_empty: one arrival per q-tile per entry (its PV commit; the
        // commit is doubled when the other q-tile skips the entry)
        const uint32_t count = (&bars[i] == &v_empty[0] || &bars[i] == &v_empty[1]) ? 2u : 1u;
        mbar_init(&bars[i], count);
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

  if (warp < kSoftmaxWarp0) {
    setmaxnreg_dec<56>();
    auto active = [&](int e, int t) -> bool { return ((list[e] >> (16 + 4 * t)) & 0xFu) != 0; };
    auto aborted = [&]() -> bool { return __any_sync(0xffffffffu, misc[4] != 0); };
    if (warp == 0) {
      // ------------------------------------------- K loads and S issue (warp 0) ---
      // S number i (the (entry, q-tile) pairs in list order) goes into the one
      // S buffer once the softmax that consumed S number i-1 has loaded it.
      // At that point every earlier S has completed, so the K slot of an entry
      // whose last S was i-1 is free and K of the entry two ahead goes into it.
      if (n_list > 0) {
        const int cnt0 = misc[2], cnt1 = misc[3];
        const int n_s = cnt0 + cnt1;
        if (lane == 0) {
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
        }
        auto load_k = [&](int e) {
          if (lane == 0) {
            const int s = e % kStages;
            mbar_arrive_expect_tx(&k_full[s], L::kTileBytes);
#pragma unroll
            for (int hd = 0; hd < D / 64; ++hd)
              tma_load_3d(&tmK, &k_full[s], smem + L::kOffK + s * L::kTileBytes + hd * kHalfBytes, hd * 64,
                          static_cast<int>(list[e] & 0xFFFFu) * kTileN, bh);
          }
        };
        int k_issued = n_list < kStages ? n_list : kStages;   // K loads issued
        int k_seen = 0;                                        // K loads observed landed
        for (int e = 0; e < k_issued; ++e) load_k(e);
        bool ok = __all_sync(0xffffffffu, mbar_wait(q_full, 0));
        if (!ok && lane == 0) misc[4] = 1;
        const uint64_t dq0 = smem_desc(smem_addr(smem + L::kOffQ), 16, 1024);
        const uint64_t dk0 = smem_desc(smem_addr(smem + L::kOffK), 16, 1024);
        constexpr uint64_t kStageStep = L::kTileBytes >> 4;   // descriptor units
        int se = 0, st = active(0, 0) ? 0 : 1;
        int prev_e = 0, prev_t = 0;
        bool prev_last = false;
        for (int i = 0; i < n_s; ++i) {
          if (i > 0) named_bar_sync(kBarSFree + prev_t, kHandoff);
          ok = ok && !aborted();
          if (ok && se >= k_seen) {
            ok = __all_sync(0xffffffffu, mbar_wait(&k_full[se % kStages], (se / kStages) & 1));
            if (ok) k_seen = se + 1;
            else if (lane == 0) misc[4] = 1;
          }
          if (ok) {
            tc_fence_after();
            const uint64_t dq = dq0 + st * kStageStep;
            const uint64_t dk = dk0 + (se % kStages) * kStageStep;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t off = static_cast<uint64_t>((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4;
              mma_ss_warp(tmem, dq + off, dk + off, kIdescS, kk > 0 ? 1u : 0u);
            }
          }
          // committed also after an error (with nothing issued), so that the
          // softmax keeps its place in the sequence of hand-offs
          mma_commit_warp(&s_ready[st]);
          // The next K load is issued only now: issuing a TMA load can hold
          // the issuing warp for hundreds of cycles, and S(i) is on the path.
          if (i > 0 && prev_last && prev_e + kStages < n_list && !aborted()) {
            load_k(prev_e + kStages);
            k_issued = prev_e + kStages + 1;
          }
          prev_e = se;
          prev_t = st;
          prev_last = st == 1 || !active(se, 1);
          if (prev_last) {
            ++se;
            st = (se < n_list && active(se, 0)) ? 0 : 1;
          } else {
            st = 1;
          }
        }
        named_bar_sync(kBarSFree + prev_t, kHandoff);   // the softmax has loaded the last S
        // K loads never observed (error path) must land before the CTA exits
        for (int e = k_seen; e < k_issued; ++e) mbar_wait(&k_full[e % kStages], (e / kStages) & 1);
        mma_commit_warp(&mma_done[0]);
        mbar_wait(&mma_done[0], 0);
      }
    } else if (warp == 3) {
      // ------------------------------------------------------- V loads (warp 3) ---
      if (lane == 0 && n_list > 0) {
        int issued = 0;
        for (int e = 0; e < n_list; ++e) {
          const int s = e % kStages;
          if (e >= kStages && (misc[4] || !mbar_wait(&v_empty[s], ((e / kStages) - 1) & 1))) {
            misc[4] = 1;
            break;
          }
          mbar_arrive_expect_tx(&v_full[s], L::kTileBytes);
#pragma unroll
          for (int hd = 0; hd < D / 64; ++hd)
            tma_load_3d(&tmV, &v_full[s], smem + L::kOffV + s * L::kTileBytes + hd * kHalfBytes, hd * 64,
                        static_cast<int>(list[e] & 0xFFFFu) * kTileN, bh);
          issued = e + 1;
        }
        // Loads still in flight must land before the CTA can exit.
        for (int e = (issued > kStages ? issued - kStages : 0); e < issued; ++e)
          mbar_wait(&v_full[e % kStages], (e / kStages) & 1);
      }
    } else {
      // ------------------------------------ PV issue for q-tile t (warps 1, 2) ---
      // O_t += P_t V, in two halves, each as soon as the softmax warpgroup has
      // written that half of P_t (A operand from TMEM, V from shared memory).
      const int t = warp - 1;
      const int cnt = misc[2 + t];
      if (n_list > 0 && cnt > 0) {
        const uint64_t dv0 = smem_desc(smem_addr(smem + L::kOffV), kHalfBytes, 1024);
        constexpr uint64_t kStageStep = L::kTileBytes >> 4;
        const uint32_t a_tmem = tmem + 128 + 64 * t;
        const uint32_t o_tmem = tmem + 256 + t * D;
        int k = 0;
        for (int e = 0; e < n_list; ++e) {
          if (!active(e, t)) continue;
          const int s = e % kStages;
          const uint64_t dv = dv0 + s * kStageStep;
          named_bar_sync(kBarPA + t, kHandoff);
          bool ok = !aborted();
          if (ok) {
            ok = __all_sync(0xffffffffu, mbar_wait(&v_full[s], (e / kStages) & 1));
            if (!ok && lane == 0) misc[4] = 1;
          }
          if (ok) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ts_warp(o_tmem, a_tmem + kk * 8, dv + ((kk * 16 * 128) >> 4), kIdescPV,
                          (k == 0 && kk == 0) ? 0u : 1u);
          }
          mma_commit_warp(&pv_done_a[t]);   // also after an error, so that no waiter stalls
          named_bar_sync(kBarPB + t, kHandoff);
          if (ok && !aborted()) {
            tc_fence_after();
#pragma unroll
            for (int kk = 4; kk < 8; ++kk)
              mma_ts_warp(o_tmem, a_tmem + kk * 8, dv + ((kk * 16 * 128) >> 4), kIdescPV, 1u);
          }
          // committed also after an error, so that no waiter stalls
          mma_commit_warp(&pv_done_b[t]);
          mma_commit_warp(&v_empty[s]);
          if (!active(e, 1 - t)) mma_commit_warp(&v_empty[s]);   // the other tile's share
          if (k + 1 == cnt) mma_commit_warp(&o_final[t]);
          ++k;
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
    const int qh = (BLK == 64) ? (r >> 6) : 0;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const uint32_t s_addr = lane_base;
    const uint32_t p_addr = lane_base + 128 + 64 * t;
    const uint32_t o_addr = lane_base + 256 + t * D;
    const int cnt = misc[2 + t];
    const float sl2 = p.scale_log2;
    const float NEG_INF = -__int_as_float(0x7f800000);

    float m_used = NEG_INF, m_true = NEG_INF, l_sum = 0.f;
    int et = 0;   // kv tiles this q-tile has processed
    bool ok = true;
    uint32_t* my_votes = votes + (t * 4 + wq) * L::kVoteWords;

    if (cnt > 0) {
      for (int e = 0; e < n_list; ++e) {
        const uint32_t ent = list[e];
        const uint32_t bits = (ent >> (16 + 4 * t)) & 0xFu;
        if (!bits) continue;
        const int jt = static_cast<int>(ent & 0xFFFFu);
        // After an error the loop still runs to the end (its hand-offs keep
        // the issuing warps' sequences in step); it only stops trusting TMEM.
        if (!mbar_wait(&s_ready[t], et & 1)) {
          misc[4] = 1;
          ok = false;
        }
        tc_fence_after();

        float s[kTileN];
        tmem_ld128(s_addr, s);
        // the S buffer is free for the next S (of either q-tile)
        tc_fence_before();
        named_bar_sync(kBarSFree + t, kHandoff);

        const int valid_cols = min(kTileN, p.N - jt * kTileN);
        if (valid_cols < kTileN || (BLK == 64 && bits != 0xFu)) {
          const bool k0 = BLK == 128 ? true : ((bits >> (qh * 2 + 0)) & 1u);
          const bool k1 = BLK == 128 ? true : ((bits >> (qh * 2 + 1)) & 1u);
#pragma unroll
          for (int c = 0; c < kTileN; ++c) {
            const bool keep = (c < valid_cols) && (c < 64 ? k0 : k1);
            s[c] = keep ? s[c] : NEG_INF;
          }
        }
        // causal: in the diagonal tile (kv tile = q-tile) key c needs c <= r
        // (a separate loop, so that the common path is unchanged)
        if (CAUSAL && jt == qtile0 + t) {
#pragma unroll
          for (int c = 0; c < kTileN; ++c) s[c] = c <= r ? s[c] : NEG_INF;
        }
        // row maxima of the two 64-column halves: four independent chains each
        float mxh[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const float* sh = s + 64 * hh;
          float a0 = fmaxf(sh[0], sh[1]), a1 = fmaxf(sh[2], sh[3]);
          float a2 = fmaxf(sh[4], sh[5]), a3 = fmaxf(sh[6], sh[7]);
#pragma unroll
          for (int c = 8; c < 64; c += 8) {
            a0 = fmax3(a0, sh[c + 0], sh[c + 1]);
            a1 = fmax3(a1, sh[c + 2], sh[c + 3]);
            a2 = fmax3(a2, sh[c + 4], sh[c + 5]);
            a3 = fmax3(a3, sh[c + 6], sh[c + 7]);
          }
          mxh[hh] = fmax3(a0, a1, fmaxf(a2, a3));
        }
        const float mx0 = mxh[0], mx1 = mxh[1];
        const float mx = fmaxf(mx0, mx1);

        if (p.write_skip) {
          if (BLK == 128) {
            const bool pred = !row_valid || (mx < m_true - p.eps_raw);
            const bool all = __all_sync(0xffffffffu, pred);
            if (lane == 0 && all) my_votes[e >> 5] |= 1u << (e & 31);
            m_true = fmaxf(m_true, mx);
          } else {
#pragma unroll
            for (int kh = 0; kh < 2; ++kh) {
              if ((bits >> (qh * 2 + kh)) & 1u) {
                const float mk = kh == 0 ? mx0 : mx1;
                const bool pred = !row_valid || (mk < m_true - p.eps_raw);
                const bool all = __all_sync(0xffffffffu, pred);
                const int bi = e * 2 + kh;
                if (lane == 0 && all) my_votes[bi >> 5] |= 1u << (bi & 31);
                m_true = fmaxf(m_true, mk);
              }
            }
          }
        }

        // online softmax with a lazily updated reference maximum
        float factor = 1.f;
        if (mx > m_used && (m_used == NEG_INF || (mx - m_used) * sl2 > 8.f)) {
          factor = (m_used == NEG_INF) ? 0.f : fast_exp2((m_used - mx) * sl2);
          m_used = mx;
          l_sum *= factor;
        }
        // The previous PV of this tile reads P_t and accumulates into O_t: each
        // half of P_t is rewritten once that half of the PV has completed, and
        // O_t is rescaled once all of it has.
        auto wait_pv = [&](uint64_t* bar) {
          if (et > 0) {
            if (!mbar_wait(bar, (et - 1) & 1)) {
              misc[4] = 1;
              ok = false;
            }
            tc_fence_after();
          }
        };
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
        const float neg_m = (m_used == NEG_INF) ? 0.f : -m_used * sl2;
        // first 64 columns -> P[0, 32): the MMA warp starts PV on them at once
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
    ok = __all_sync(0xffffffffu, ok && misc[4] == 0);
    if (cnt > 0 && ok) {
      ok = __all_sync(0xffffffffu, mbar_wait(&o_final[t], 0));
      if (!ok) misc[4] = 1;
      tc_fence_after();
    }
    // A row that never saw a valid column keeps m_used = -inf: it is empty
    // (O = 0, LSE = -inf) whatever its exponentials left in l_sum.
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
    if (p.lse && row_valid) {
      const float neg_m = (m_used == NEG_INF) ? 0.f : -m_used * sl2;
      p.lse[static_cast<size_t>(bh) * p.N + row] =
          l_sum > 0.f ? (log2f(l_sum) - neg_m) * 0.69314718055994531f : NEG_INF;
    }

    // ----------------------------------- skip bits: cross-warp AND at the end ---
    if (p.write_skip && cnt > 0) {
      named_bar_sync(kBarEpi + t, 128);
      if (ok && !misc[4]) {
        const int tid = wq * 32 + lane;
        uint32_t* tv = votes + t * 4 * L::kVoteWords;
        for (int e = tid; e < n_list; e += 128) {
          const uint32_t ent = list[e];
          const uint32_t bits = (ent >> (16 + 4 * t)) & 0xFu;
          if (!bits) continue;
          const int jt = static_cast<int>(ent & 0xFFFFu);
#pragma unroll
          for (int qq = 0; qq < QH; ++qq) {
#pragma unroll
            for (int kh = 0; kh < KH; ++kh) {
              if (BLK == 64 && !((bits >> (qq * 2 + kh)) & 1u)) continue;
              const int qb = (qtile0 + t) * QH + qq;
              const int kb = jt * KH + kh;
              const int bi = (BLK == 128) ? e : e * 2 + kh;
              uint32_t all = 1u;
              if (BLK == 128) {
#pragma unroll
                for (int w = 0; w < 4; ++w) all &= tv[w * L::kVoteWords + (bi >> 5)] >> (bi & 31);
              } else {
#pragma unroll
                for (int w = 2 * qq; w < 2 * qq + 2; ++w) all &= tv[w * L::kVoteWords + (bi >> 5)] >> (bi & 31);
              }
              p.skip_out[(static_cast<size_t>(bh) * p.nb + qb) * p.nb + kb] = static_cast<uint8_t>(all & 1u);
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
}

}  // namespace sa
