// sa_attn_bwd.cuh — backward pass of block-sparse attention for sm_100a.
//
// Gradients of O = softmax(scale * Q K^T restricted to the kept blocks) V with
// respect to Q, K and V, given dO and the forward's LSE (needed by the LoRA
// length extension of the Radial Attention write-up, "MIT实验室推出Radial
// Attention", training-cost paragraph; the formulas are the derivative of the
// forward definition):
//   P = exp(S - LSE) on kept columns, D_r = dO_r . O_r,
//   dV = P^T dO,  dS = P * (dO V^T - D),  dK = scale dS^T Q,  dQ = scale dS K.
//
// Three launches, no atomics (the result does not depend on scheduling):
//   bwd_delta_kernel   D_r = dO_r . O_r (HBM-bound: reads O and dO once);
//   bwd_dkdv_kernel    one CTA per 128-key kv tile: walks the q-tiles that
//                      keep any of its blocks, S^T = K Q^T and dP^T = V dO^T
//                      into TMEM, P^T and dS^T packed to bf16 in place, then
//                      dV += P^T dO and dK += dS^T Q with the A operand in TMEM;
//   bwd_dq_kernel      one CTA per 128-row q-tile: walks its kept kv tiles,
//                      S = Q K^T and dP = dO V^T, dS packed in place, then
//                      dQ += dS K with the A operand in TMEM.
// The MMAs take one of three forms: both operands K-major in shared memory
// (S^T, dP^T in dK/dV), A from TMEM and B K-major in shared memory (S, dP in
// dQ, with Q and dO copied into TMEM), or A from TMEM and B MN-major in shared
// memory (dV, dK, dQ).  The same 128 x D tile, as TMA writes it, serves as a
// K-major B operand (Q in S^T, K in S) and as an MN-major B operand (Q in dK,
// dO in dV, K in dQ).  Each S is computed in two 64-column halves.
//
// Roles (320 threads = 10 warps, one CTA per SM for the TMEM it holds):
//   warps 0-3   one thread per row of the CTA's tile (key row in dK/dV, query
//               row in dQ): P and dS of the first 64-column half of each S;
//   warps 4-7   the same rows, second half (the two halves run concurrently);
//               both warpgroups share the epilogue;
//   warp 8      builds the tile list from the mask, issues the TMA loads
//               (2-stage ring) and stages the per-query LSE / D vectors;
//   warp 9      allocates TMEM and issues every MMA (warp-wide, one elected lane).
// Hand-offs: tcgen05.commit to mbarriers from the MMA warp; one named barrier
// per half (its warpgroup + warp 9) when that half's P / dS are in TMEM.
// Every party runs the full, list-determined sequence of syncs, also after an
// error (skipping only its loads and MMAs), and every mbarrier wait is bounded.
#pragma once

#include "sa_attn_fwd.cuh"

namespace sa {

constexpr int kBwdWarps = 10;
constexpr int kBwdThreads = kBwdWarps * 32;
constexpr int kBwdLoadWarp = 8;
constexpr int kBwdMmaWarp = 9;
// P / dS of the first / second 64-column half packed in TMEM: warps 0-3 /
// warps 4-7 <-> MMA warp
constexpr int kBarBwdA = 1;
constexpr int kBarBwdB = 2;
constexpr int kBwdHandoff = 160;

struct BwdParams {
  int B, H, N;
  int nb;             // blocks per sequence
  int n_tiles;        // ceil(N / 128)
  const uint8_t* mask;
  long long msb, msh, msi;
  const float* lse;   // [B,H,N] natural-log LSE of the forward
  const float* delta; // [B,H,N] D_r = dO_r . O_r
  float scale;        // logit scale
  float scale_log2;   // scale * log2(e)
  int causal;         // key c visible to row r only if c <= r (blocks j > i dropped)
  __nv_bfloat16* dq;
  __nv_bfloat16* dk;
  __nv_bfloat16* dv;
};

// D_r = sum_a dO[r,a] O[r,a] in fp32; D / 8 threads per row, 16-byte loads.
template <int D>
__global__ void __launch_bounds__(256) bwd_delta_kernel(const __nv_bfloat16* __restrict__ o,
                                                        const __nv_bfloat16* __restrict__ dout,
                                                        float* __restrict__ delta, long long rows) {
  constexpr int kTpr = D / 8;                       // threads per row
  constexpr int kRowsPerBlock = 256 / kTpr;
  const int sub = threadIdx.x % kTpr;
  for (long long r = static_cast<long long>(blockIdx.x) * kRowsPerBlock + threadIdx.x / kTpr; r < rows;
       r += static_cast<long long>(gridDim.x) * kRowsPerBlock) {
    const uint4 a = reinterpret_cast<const uint4*>(o + r * D)[sub];
    const uint4 g = reinterpret_cast<const uint4*>(dout + r * D)[sub];
    const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&g);
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 af = __bfloat1622float2(a2[i]), gf = __bfloat1622float2(g2[i]);
      acc = fmaf(af.x, gf.x, acc);
      acc = fmaf(af.y, gf.y, acc);
    }
#pragma unroll
    for (int off = kTpr / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (sub == 0) delta[r] = acc;
  }
}

template <int D>
struct BwdSmem {
  static constexpr int kTileBytes = kTileM * D * 2;
  // dK/dV kernel: K, V of the CTA's kv tile, then a ring of Q / dO tiles with
  // their [-lse * log2(e) | D] vectors (2 x 128 fp32 per stage).
  // dQ kernel: Q, dO of the CTA's q-tile, then a ring of K / V tiles.
  static constexpr int kOffFix0 = 0;
  static constexpr int kOffFix1 = kTileBytes;
  static constexpr int kOffRing0 = 2 * kTileBytes;                      // [stage]
  static constexpr int kOffRing1 = kOffRing0 + kStages * kTileBytes;    // [stage]
  static constexpr int kOffVec = kOffRing1 + kStages * kTileBytes;      // [stage][2][128] f32
  static constexpr int kOffList = kOffVec + kStages * 2 * 128 * 4;
  // fix_full, ring_full[2], ring_empty[2], ready[2], half_done[2], final_done,
  // fix_tmem (dQ kernel: Q and dO copied into TMEM)
  static constexpr int kNumBars = 1 + 2 * kStages + 6;
  static constexpr int kOffBar = kOffList + kMaxKvTiles * 4;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kBytes = kOffMisc + 64;
  static constexpr int kAlloc = kBytes + 1024;
};

// p = 2^(s * sl2 + nl) on kept columns (0 elsewhere), ds = p * (dp - dl), for
// 32 columns; both packed to bf16 pairs.  nl = -lse * log2(e) and dl = D are
// per column (dK/dV kernel: pointers into shared memory, 16-byte aligned) or
// per row (dQ kernel: nls / dls).  kAll: every column kept (no selects).
template <bool kPerColumn, bool kAll>
__device__ __forceinline__ void grad_chunk(const float* sv, const float* dp, float sl2, const float* nl,
                                           const float* dl, float nls, float dls, uint32_t keep_bits,
                                           uint32_t* pk, uint32_t* dk) {
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    float x[4], g[4], pv[4];
    if (kPerColumn) {
      const float4 l4 = reinterpret_cast<const float4*>(nl)[q];
      const float4 g4 = reinterpret_cast<const float4*>(dl)[q];
      x[0] = fmaf(sv[4 * q + 0], sl2, l4.x);
      x[1] = fmaf(sv[4 * q + 1], sl2, l4.y);
      x[2] = fmaf(sv[4 * q + 2], sl2, l4.z);
      x[3] = fmaf(sv[4 * q + 3], sl2, l4.w);
      g[0] = g4.x;
      g[1] = g4.y;
      g[2] = g4.z;
      g[3] = g4.w;
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        x[j] = fmaf(sv[4 * q + j], sl2, nls);
        g[j] = dls;
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j)
      pv[j] = (kAll || ((keep_bits >> (4 * q + j)) & 1u)) ? fast_exp2(x[j]) : 0.f;
    pk[2 * q] = pack_bf16x2(pv[0], pv[1]);
    pk[2 * q + 1] = pack_bf16x2(pv[2], pv[3]);
    dk[2 * q] = pack_bf16x2(pv[0] * (dp[4 * q] - g[0]), pv[1] * (dp[4 * q + 1] - g[1]));
    dk[2 * q + 1] = pack_bf16x2(pv[2] * (dp[4 * q + 2] - g[2]), pv[3] * (dp[4 * q + 3] - g[3]));
  }
}

template <bool kPerColumn>
__device__ __forceinline__ void grad_chunk_any(const float* sv, const float* dp, float sl2, const float* nl,
                                               const float* dl, float nls, float dls, uint32_t keep_bits,
                                               uint32_t* pk, uint32_t* dk) {
  if (keep_bits == 0xffffffffu)
    grad_chunk<kPerColumn, true>(sv, dp, sl2, nl, dl, nls, dls, keep_bits, pk, dk);
  else
    grad_chunk<kPerColumn, false>(sv, dp, sl2, nl, dl, nls, dls, keep_bits, pk, dk);
}

// Bits i of a 32-column chunk with i >= lo (all for lo <= 0, none for lo >= 32).
__device__ __forceinline__ uint32_t causal_from(int lo) {
  return lo <= 0 ? 0xffffffffu : (lo >= 32 ? 0u : ~((1u << lo) - 1u));
}

// Half hh (columns [64 hh, 64 hh + 64)) of this thread's S and dP rows: P
// packed over the half's first 32 S columns (when kStoreP) and dS over the
// half's first 32 columns at ds_base.  The second chunk's loads are issued
// before the first chunk's stores (disjoint columns); each chunk's stores
// land on columns its own or the previous chunk already read.
template <bool kPerColumn, bool kStoreP>
__device__ __forceinline__ void grad_half(uint32_t ts, uint32_t tdp, uint32_t ds_base, int hh, float sl2,
                                          const float* l2, const float* dl, float l2s, float dls, uint32_t keep0,
                                          uint32_t keep1) {
  float s0[32], d0[32], s1[32], d1[32];
  uint32_t pk[16], dk[16];
  const uint32_t cs = ts + 64 * hh, cd = tdp + 64 * hh, cq = ds_base + 64 * hh;
  tmem_ld32x2_nowait(cs, cd, s0, d0);
  tmem_ld_wait2(s0, d0);
  tmem_ld32x2_nowait(cs + 32, cd + 32, s1, d1);
  grad_chunk_any<kPerColumn>(s0, d0, sl2, kPerColumn ? l2 + 64 * hh : nullptr,
                             kPerColumn ? dl + 64 * hh : nullptr, l2s, dls, keep0, pk, dk);
  if (kStoreP) tmem_st16(cs, pk);
  tmem_st16(cq, dk);
  tmem_ld_wait2(s1, d1);
  grad_chunk_any<kPerColumn>(s1, d1, sl2, kPerColumn ? l2 + 64 * hh + 32 : nullptr,
                             kPerColumn ? dl + 64 * hh + 32 : nullptr, l2s, dls, keep1, pk, dk);
  if (kStoreP) tmem_st16(cs + 16, pk);
  tmem_st16(cq + 16, dk);
}

// One thread's fp32 TMEM row (columns [taddr, taddr + D)) times `mul`, to
// bf16 at dst (16-byte aligned) when `store`, or zeros when `zero`.  Called by
// whole warps with warp-uniform `zero` (the TMEM loads are warp-collective).
template <int D>
__device__ __forceinline__ void store_row(uint32_t taddr, float mul, __nv_bfloat16* dst, bool zero, bool store) {
#pragma unroll
  for (int c = 0; c < D / 32; ++c) {
    float v[32];
    if (zero) {
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = 0.f;
    } else {
      tmem_ld32(taddr + 32 * c, v);
    }
    if (!store) continue;
    uint4* out = reinterpret_cast<uint4*>(dst + 32 * c);
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
      uint4 w;
      w.x = pack_bf16x2(v[q4 * 8 + 0] * mul, v[q4 * 8 + 1] * mul);
      w.y = pack_bf16x2(v[q4 * 8 + 2] * mul, v[q4 * 8 + 3] * mul);
      w.z = pack_bf16x2(v[q4 * 8 + 4] * mul, v[q4 * 8 + 5] * mul);
      w.w = pack_bf16x2(v[q4 * 8 + 6] * mul, v[q4 * 8 + 7] * mul);
      out[q4] = w;
    }
  }
}


// ------------------------------------------------------------ dK / dV ---
// CTA = (kv tile jt, head bh).  TMEM columns: dV [0, D), dK [D, 2D),
// S^T [2D, 2D + 128) and dP^T [2D + 128, 2D + 256), each in two 64-query
// halves; P^T / dS^T of a half are packed to bf16 over the half's first 32
// columns.  Per entry (q-tile) the MMA warp issues, for each half: S^T_h and
// dP^T_h (N = 64), and once its warpgroup has packed the half, dV += P^T_h dO_h
// and dK += dS^T_h Q_h (K = 64).  The next entry's S^T_h goes into a half as
// soon as the gradient MMAs that read it have completed, so one half's MMAs
// run while the warpgroups work on the halves.
template <int D, int BLK>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                    const BwdParams p) {
  using L = BwdSmem<D>;
  constexpr int QH = kTileM / BLK;  // q-blocks per q-tile
  constexpr int KH = kTileN / BLK;  // k-blocks per kv tile
  constexpr uint32_t kIdescH = idesc_bf16_f32(kTileN, 64, false);   // S^T / dP^T half: 128 keys x 64 queries
  constexpr uint32_t kIdescG = idesc_bf16_f32(kTileN, D, true);
  constexpr int kHalfBytes = kTileM * 128;  // one 64-column slab of a tile

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint32_t* list = reinterpret_cast<uint32_t*>(smem + L::kOffList);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* kv_full = bars;
  uint64_t* q_full = bars + 1;
  uint64_t* q_empty = q_full + kStages;
  uint64_t* ready = q_empty + kStages;       // [2]: S^T_h and dP^T_h of the current entry computed
  uint64_t* half_done = ready + 2;           // [2]: the gradient MMAs of half h completed
  uint64_t* final_done = half_done + 2;
  volatile int* misc = reinterpret_cast<volatile int*>(smem + L::kOffMisc);
  // misc[0] TMEM base, [1] list length, [2] abort flag

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int jt = blockIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / p.H, h = bh - (bh / p.H) * p.H;
  auto aborted = [&]() -> bool { return misc[2] != 0; };

  if (warp == kBwdLoadWarp) {
    // ---- q-tile list: the q-tiles keeping any (q-block, k-block) quadrant ----
    int n = 0;
    for (int base = 0; base < p.n_tiles; base += 32) {
      const int it = base + lane;
      uint32_t bits = 0;
      if (it < p.n_tiles) {
#pragma unroll
        for (int qh = 0; qh < QH; ++qh) {
          const int qb = it * QH + qh;
          if (qb >= p.nb) continue;
#pragma unroll
          for (int kh = 0; kh < KH; ++kh) {
            const int kb = jt * KH + kh;
            if (kb >= p.nb) continue;
            const uint8_t keep = p.mask ? p.mask[b * p.msb + h * p.msh + qb * p.msi + kb] : uint8_t(1);
            if (keep && (!p.causal || kb <= qb)) bits |= (BLK == 128 ? 0xFu : (1u << (qh * 2 + kh)));
          }
        }
      }
      const unsigned ball = __ballot_sync(0xffffffffu, bits != 0);
      if (bits) list[n + __popc(ball & ((1u << lane) - 1u))] = static_cast<uint32_t>(it) | (bits << 16);
      n += __popc(ball);
    }
    if (lane == 0) {
      misc[1] = n;
      misc[2] = 0;
      // q_full: the TMA bytes' arrival and the LSE / D writer's arrival
      for (int i = 0; i < L::kNumBars; ++i) mbar_init(&bars[i], (&bars[i] >= q_full && &bars[i] < q_empty) ? 2u : 1u);
      fence_mbar_init();
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
    }
  } else if (warp == kBwdMmaWarp) {
    tmem_alloc(const_cast<uint32_t*>(reinterpret_cast<volatile uint32_t*>(misc)), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = static_cast<uint32_t>(misc[0]);
  const int n_list = misc[1];
  const uint32_t tm_dv = tmem, tm_dk = tmem + D, tm_s = tmem + 2 * D, tm_dp = tmem + 2 * D + 128;

  if (warp == kBwdLoadWarp) {
    // ------------------------------------------------------------- loads ---
    if (n_list > 0) {
      if (lane == 0) {
        mbar_arrive_expect_tx(kv_full, 2 * L::kTileBytes);
#pragma unroll
        for (int hd = 0; hd < D / 64; ++hd) {
          tma_load_3d(&tmK, kv_full, smem + L::kOffFix0 + hd * kHalfBytes, hd * 64, jt * kTileN, bh);
          tma_load_3d(&tmV, kv_full, smem + L::kOffFix1 + hd * kHalfBytes, hd * 64, jt * kTileN, bh);
        }
      }
      for (int e = 0; e < n_list; ++e) {
        const int s = e % kStages;
        const int it = static_cast<int>(list[e] & 0xFFFFu);
        // per-query vectors of the tile, read before the wait for the stage:
        // -lse * log2(e) (-inf past N) and D
        float lv[4], dv4[4];
        const size_t rbase = static_cast<size_t>(bh) * p.N;
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          const int row = it * kTileM + k4 * 32 + lane;
          const bool valid = row < p.N;
          lv[k4] = valid ? p.lse[rbase + row] * -1.4426950408889634f : -__int_as_float(0x7f800000);
          dv4[k4] = valid ? p.delta[rbase + row] : 0.f;
        }
        // the MMAs of entry e - 2 (the last readers of this stage) have completed
        if (e >= kStages && !mbar_wait(&q_empty[s], ((e / kStages) - 1) & 1) && lane == 0) misc[2] = 1;
        if (__any_sync(0xffffffffu, aborted())) continue;
        if (lane == 0) {
          mbar_arrive_expect_tx(&q_full[s], 2 * L::kTileBytes);
#pragma unroll
          for (int hd = 0; hd < D / 64; ++hd) {
            tma_load_3d(&tmQ, &q_full[s], smem + L::kOffRing0 + s * L::kTileBytes + hd * kHalfBytes, hd * 64,
                        it * kTileM, bh);
            tma_load_3d(&tmDO, &q_full[s], smem + L::kOffRing1 + s * L::kTileBytes + hd * kHalfBytes, hd * 64,
                        it * kTileM, bh);
          }
        }
        float* vec = reinterpret_cast<float*>(smem + L::kOffVec) + s * 256;
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          vec[k4 * 32 + lane] = lv[k4];
          vec[128 + k4 * 32 + lane] = dv4[k4];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&q_full[s]);
      }
    }
  } else if (warp == kBwdMmaWarp) {
    // -------------------------------------------------------- MMA issue ---
    if (n_list > 0) {
      bool ok = __all_sync(0xffffffffu, mbar_wait(kv_full, 0));
      if (!ok && lane == 0) misc[2] = 1;
      const uint64_t dk_a = smem_desc(smem_addr(smem + L::kOffFix0), 16, 1024);   // K, A operand
      const uint64_t dv_a = smem_desc(smem_addr(smem + L::kOffFix1), 16, 1024);   // V, A operand
      const uint64_t dq_k = smem_desc(smem_addr(smem + L::kOffRing0), 16, 1024);  // Q, K-major B
      const uint64_t ddo_k = smem_desc(smem_addr(smem + L::kOffRing1), 16, 1024); // dO, K-major B
      const uint64_t dq_mn = smem_desc(smem_addr(smem + L::kOffRing0), kHalfBytes, 1024);   // Q, MN-major B
      const uint64_t ddo_mn = smem_desc(smem_addr(smem + L::kOffRing1), kHalfBytes, 1024);  // dO, MN-major B
      constexpr uint64_t kStageStep = L::kTileBytes >> 4;
      // S^T_hh, dP^T_hh of entry e: queries [64 hh, 64 hh + 64) = rows 64 hh.. of
      // each 64-column slab of the Q / dO tile (8 KB into the slab)
      auto issue_sdp = [&](int e, int hh) {
        const uint64_t base = (e % kStages) * kStageStep + (static_cast<uint64_t>(hh * 64 * 128) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4;
          mma_ss_warp(tm_s + 64 * hh, dk_a + off, dq_k + base + off, kIdescH, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4;
          mma_ss_warp(tm_dp + 64 * hh, dv_a + off, ddo_k + base + off, kIdescH, kk > 0 ? 1u : 0u);
        }
      };
      // dV += P^T_hh dO_hh and dK += dS^T_hh Q_hh: K = the half's 64 queries
      auto issue_grad = [&](int e, int hh) {
        const uint64_t base = (e % kStages) * kStageStep;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t off = static_cast<uint64_t>((hh * 64 + kk * 16) * 128) >> 4;
          const uint32_t acc = (e > 0 || hh > 0 || kk > 0) ? 1u : 0u;
          mma_ts_warp(tm_dv, tm_s + 64 * hh + kk * 8, ddo_mn + base + off, kIdescG, acc);
          mma_ts_warp(tm_dk, tm_dp + 64 * hh + kk * 8, dq_mn + base + off, kIdescG, acc);
        }
      };
      auto wait_q = [&](int e) {
        ok = __all_sync(0xffffffffu, ok && !aborted());
        if (ok) {
          ok = __all_sync(0xffffffffu, mbar_wait(&q_full[e % kStages], (e / kStages) & 1));
          if (!ok && lane == 0) misc[2] = 1;
        }
        if (ok) tc_fence_after();
      };
      auto wait_half = [&](int hh, int e) {
        if (!__all_sync(0xffffffffu, mbar_wait(&half_done[hh], e & 1))) {
          if (lane == 0) misc[2] = 1;
          ok = false;
        }
        ok = __all_sync(0xffffffffu, ok && !aborted());
        if (ok) tc_fence_after();
      };
      wait_q(0);
      if (ok) issue_sdp(0, 0);
      mma_commit_warp(&ready[0]);   // every commit also after an error, so that no waiter stalls
      if (ok) issue_sdp(0, 1);
      mma_commit_warp(&ready[1]);
      // Per half: once its warpgroup has packed it, the gradient MMAs; once
      // those have completed (they read the half's columns), the next
      // entry's S / dP of the half.  The other half's MMAs keep the pipe busy
      // while this warp waits.
      for (int e = 0; e < n_list; ++e) {
        named_bar_sync(kBarBwdA, kBwdHandoff);
        if (__all_sync(0xffffffffu, ok && !aborted())) {
          tc_fence_after();
          issue_grad(e, 0);
        }
        mma_commit_warp(&half_done[0]);
        if (e + 1 < n_list) {
          wait_half(0, e);
          wait_q(e + 1);
          if (ok) issue_sdp(e + 1, 0);
          mma_commit_warp(&ready[0]);
        }
        named_bar_sync(kBarBwdB, kBwdHandoff);
        if (__all_sync(0xffffffffu, ok && !aborted())) {
          tc_fence_after();
          issue_grad(e, 1);
        }
        mma_commit_warp(&half_done[1]);
        mma_commit_warp(&q_empty[e % kStages]);
        if (e + 1 < n_list) {
          wait_half(1, e);
          if (ok) issue_sdp(e + 1, 1);
          mma_commit_warp(&ready[1]);
        }
      }
      mma_commit_warp(final_done);   // every MMA of the CTA has completed
    }
  } else {
    // ------------------------------- P^T, dS^T of one half; the epilogue ---
    const int hh = warp >> 2;                        // half of each S^T this warpgroup packs
    const int r = (warp & 3) * 32 + lane;            // key row of the kv tile
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int key = jt * kTileN + r;
    const bool key_valid = key < p.N;
    const int kh = BLK == 128 ? 0 : (r >> 6);
    const float sl2 = p.scale_log2;
    bool ok = true;
    for (int e = 0; e < n_list; ++e) {
      const uint32_t bits = list[e] >> 16;
      const int it = static_cast<int>(list[e] & 0xFFFFu);
      const int s = e % kStages;
      const float* vec = reinterpret_cast<const float*>(smem + L::kOffVec) + s * 256;
      const int valid_q = min(kTileM, p.N - it * kTileM);
      if (!mbar_wait(&ready[hh], e & 1)) {
        misc[2] = 1;
        ok = false;
      }
      if (ok && !aborted() && !mbar_wait(&q_full[s], (e / kStages) & 1)) {
        misc[2] = 1;
        ok = false;
      }
      tc_fence_after();
      // half hh: query columns [64 hh, 64 hh + 64), q-block half hh for block 64
      const bool quad = BLK == 128 ? true : ((bits >> (hh * 2 + kh)) & 1u);
      const int nv0 = min(32, max(0, valid_q - 64 * hh)), nv1 = min(32, max(0, valid_q - 64 * hh - 32));
      uint32_t keep0 = (key_valid && quad) ? (nv0 == 32 ? 0xffffffffu : ((1u << nv0) - 1u)) : 0u;
      uint32_t keep1 = (key_valid && quad) ? (nv1 == 32 ? 0xffffffffu : ((1u << nv1) - 1u)) : 0u;
      if (p.causal && it == jt) {
        // diagonal tile: query column c sees this key (row r) only if c >= r
        keep0 &= causal_from(r - 64 * hh);
        keep1 &= causal_from(r - 64 * hh - 32);
      }
      grad_half<true, true>(tm_s + lane_off, tm_dp + lane_off, tm_dp + lane_off, hh, sl2, vec, vec + 128, 0.f, 0.f,
                            keep0, keep1);
      tmem_st_wait();
      tc_fence_before();
      named_bar_sync(hh == 0 ? kBarBwdA : kBarBwdB, kBwdHandoff);
    }
    // epilogue: warps 0-3 write dV, warps 4-7 dK, once every MMA has completed
    if (n_list > 0 && !mbar_wait(final_done, 0)) {
      misc[2] = 1;
      ok = false;
    }
    tc_fence_after();
    if (n_list == 0 || __all_sync(0xffffffffu, ok && !aborted())) {
      const size_t off = (static_cast<size_t>(bh) * p.N + (key_valid ? key : 0)) * D;
      if (hh == 0)
        store_row<D>(tm_dv + lane_off, 1.f, p.dv + off, n_list == 0, key_valid);
      else
        store_row<D>(tm_dk + lane_off, p.scale, p.dk + off, n_list == 0, key_valid);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kBwdMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ----------------------------------------------------------------- dQ ---
// CTA = (q-tile it, head bh).  TMEM columns: dQ [0, D), S [128, 256) and
// dP [256, 384), each in two 64-key halves; dS of a half is packed to bf16
// over the half's first 32 S columns; Q and dO as bf16 pairs at [384, 384 +
// D/2) and [384 + D/2, 384 + D), copied there once per CTA from the TMA
// tiles, so that S_h = Q K_h^T and dP_h = dO V_h^T read only K_h / V_h from
// shared memory (an N = 64 MMA with both operands in shared memory is bound
// by the shared-memory bandwidth).  The same two-half pipeline as the
// dK / dV kernel: S_h, dP_h (N = 64 keys), then dQ += dS_h K_h (K = 64).
template <int D, int BLK>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmDO,
                  const BwdParams p) {
  using L = BwdSmem<D>;
  constexpr int QH = kTileM / BLK;
  constexpr int KH = kTileN / BLK;
  constexpr uint32_t kIdescH = idesc_bf16_f32(kTileM, 64, false);   // S / dP half: 128 queries x 64 keys
  constexpr uint32_t kIdescG = idesc_bf16_f32(kTileM, D, true);
  constexpr int kHalfBytes = kTileM * 128;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint32_t* list = reinterpret_cast<uint32_t*>(smem + L::kOffList);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kOffBar);
  uint64_t* qd_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + kStages;
  uint64_t* ready = kv_empty + kStages;
  uint64_t* half_done = ready + 2;
  uint64_t* final_done = half_done + 2;
  uint64_t* qd_tmem = final_done + 1;        // Q and dO rows stored into TMEM (256 arrivals)
  volatile int* misc = reinterpret_cast<volatile int*>(smem + L::kOffMisc);
  // misc[0] TMEM base, [1] list length, [2] abort flag

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int it = blockIdx.x;
  const int bh = blockIdx.y;
  const int b = bh / p.H, h = bh - (bh / p.H) * p.H;
  auto aborted = [&]() -> bool { return misc[2] != 0; };

  if (warp == kBwdLoadWarp) {
    // ---- kv-tile list of this q-tile, per-quadrant keep bits ----
    int n = 0;
    for (int base = 0; base < p.n_tiles; base += 32) {
      const int jt = base + lane;
      uint32_t bits = 0;
      if (jt < p.n_tiles) {
#pragma unroll
        for (int qh = 0; qh < QH; ++qh) {
          const int qb = it * QH + qh;
          if (qb >= p.nb) continue;
#pragma unroll
          for (int kh = 0; kh < KH; ++kh) {
            const int kb = jt * KH + kh;
            if (kb >= p.nb) continue;
            const uint8_t keep = p.mask ? p.mask[b * p.msb + h * p.msh + qb * p.msi + kb] : uint8_t(1);
            if (keep && (!p.causal || kb <= qb)) bits |= (BLK == 128 ? 0xFu : (1u << (qh * 2 + kh)));
          }
        }
      }
      const unsigned ball = __ballot_sync(0xffffffffu, bits != 0);
      if (bits) list[n + __popc(ball & ((1u << lane) - 1u))] = static_cast<uint32_t>(jt) | (bits << 16);
      n += __popc(ball);
    }
    if (lane == 0) {
      misc[1] = n;
      misc[2] = 0;
      for (int i = 0; i < L::kNumBars; ++i) mbar_init(&bars[i], &bars[i] == qd_tmem ? 256u : 1u);
      fence_mbar_init();
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmDO);
    }
  } else if (warp == kBwdMmaWarp) {
    tmem_alloc(const_cast<uint32_t*>(reinterpret_cast<volatile uint32_t*>(misc)), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem = static_cast<uint32_t>(misc[0]);
  const int n_list = misc[1];
  const uint32_t tm_dq = tmem, tm_s = tmem + 128, tm_dp = tmem + 256;
  const uint32_t tm_q = tmem + 384, tm_do = tmem + 384 + D / 2;

  if (warp == kBwdLoadWarp) {
    // ------------------------------------------------------------- loads ---
    if (n_list > 0) {
      if (lane == 0) {
        mbar_arrive_expect_tx(qd_full, 2 * L::kTileBytes);
#pragma unroll
        for (int hd = 0; hd < D / 64; ++hd) {
          tma_load_3d(&tmQ, qd_full, smem + L::kOffFix0 + hd * kHalfBytes, hd * 64, it * kTileM, bh);
          tma_load_3d(&tmDO, qd_full, smem + L::kOffFix1 + hd * kHalfBytes, hd * 64, it * kTileM, bh);
        }
      }
      for (int e = 0; e < n_list; ++e) {
        const int s = e % kStages;
        if (e >= kStages && !mbar_wait(&kv_empty[s], ((e / kStages) - 1) & 1) && lane == 0) misc[2] = 1;
        if (__any_sync(0xffffffffu, aborted())) continue;
        const int jt = static_cast<int>(list[e] & 0xFFFFu);
        if (lane == 0) {
          mbar_arrive_expect_tx(&kv_full[s], 2 * L::kTileBytes);
#pragma unroll
          for (int hd = 0; hd < D / 64; ++hd) {
            tma_load_3d(&tmK, &kv_full[s], smem + L::kOffRing0 + s * L::kTileBytes + hd * kHalfBytes, hd * 64,
                        jt * kTileN, bh);
            tma_load_3d(&tmV, &kv_full[s], smem + L::kOffRing1 + s * L::kTileBytes + hd * kHalfBytes, hd * 64,
                        jt * kTileN, bh);
          }
        }
      }
    }
  } else if (warp == kBwdMmaWarp) {
    // -------------------------------------------------------- MMA issue ---
    if (n_list > 0) {
      bool ok = __all_sync(0xffffffffu, mbar_wait(qd_tmem, 0));   // Q, dO in TMEM
      if (!ok && lane == 0) misc[2] = 1;
      const uint64_t dk_k = smem_desc(smem_addr(smem + L::kOffRing0), 16, 1024);   // K, K-major B
      const uint64_t dv_k = smem_desc(smem_addr(smem + L::kOffRing1), 16, 1024);   // V, K-major B
      const uint64_t dk_mn = smem_desc(smem_addr(smem + L::kOffRing0), kHalfBytes, 1024);  // K, MN-major B
      constexpr uint64_t kStageStep = L::kTileBytes >> 4;
      // S_hh, dP_hh of entry e: keys [64 hh, 64 hh + 64) of its kv tile
      auto issue_sdp = [&](int e, int hh) {
        const uint64_t base = (e % kStages) * kStageStep + (static_cast<uint64_t>(hh * 64 * 128) >> 4);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4;
          mma_ts_warp(tm_s + 64 * hh, tm_q + kk * 8, dk_k + base + off, kIdescH, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = static_cast<uint64_t>((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4;
          mma_ts_warp(tm_dp + 64 * hh, tm_do + kk * 8, dv_k + base + off, kIdescH, kk > 0 ? 1u : 0u);
        }
      };
      // dQ += dS_hh K_hh: K = the half's 64 keys
      auto issue_grad = [&](int e, int hh) {
        const uint64_t base = (e % kStages) * kStageStep;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t off = static_cast<uint64_t>((hh * 64 + kk * 16) * 128) >> 4;
          mma_ts_warp(tm_dq, tm_s + 64 * hh + kk * 8, dk_mn + base + off, kIdescG,
                      (e > 0 || hh > 0 || kk > 0) ? 1u : 0u);
        }
      };
      auto wait_kv = [&](int e) {
        ok = __all_sync(0xffffffffu, ok && !aborted());
        if (ok) {
          ok = __all_sync(0xffffffffu, mbar_wait(&kv_full[e % kStages], (e / kStages) & 1));
          if (!ok && lane == 0) misc[2] = 1;
        }
        if (ok) tc_fence_after();
      };
      auto wait_half = [&](int hh, int e) {
        if (!__all_sync(0xffffffffu, mbar_wait(&half_done[hh], e & 1))) {
          if (lane == 0) misc[2] = 1;
          ok = false;
        }
        ok = __all_sync(0xffffffffu, ok && !aborted());
        if (ok) tc_fence_after();
      };
      wait_kv(0);
      if (ok) issue_sdp(0, 0);
      mma_commit_warp(&ready[0]);   // every commit also after an error, so that no waiter stalls
      if (ok) issue_sdp(0, 1);
      mma_commit_warp(&ready[1]);
      // Per half: once its warpgroup has packed it, the gradient MMAs; once
      // those have completed (they read the half's columns), the next
      // entry's S / dP of the half.  The other half's MMAs keep the pipe busy
      // while this warp waits.
      for (int e = 0; e < n_list; ++e) {
        named_bar_sync(kBarBwdA, kBwdHandoff);
        if (__all_sync(0xffffffffu, ok && !aborted())) {
          tc_fence_after();
          issue_grad(e, 0);
        }
        mma_commit_warp(&half_done[0]);
        if (e + 1 < n_list) {
          wait_half(0, e);
          wait_kv(e + 1);
          if (ok) issue_sdp(e + 1, 0);
          mma_commit_warp(&ready[0]);
        }
        named_bar_sync(kBarBwdB, kBwdHandoff);
        if (__all_sync(0xffffffffu, ok && !aborted())) {
          tc_fence_after();
          issue_grad(e, 1);
        }
        mma_commit_warp(&half_done[1]);
        mma_commit_warp(&kv_empty[e % kStages]);
        if (e + 1 < n_list) {
          wait_half(1, e);
          if (ok) issue_sdp(e + 1, 1);
          mma_commit_warp(&ready[1]);
        }
      }
      mma_commit_warp(final_done);   // every MMA of the CTA has completed
    }
  } else {
    // ---------------------------------------- dS of one half; the epilogue ---
    const int hh = warp >> 2;                        // half of each S this warpgroup packs
    const int r = (warp & 3) * 32 + lane;            // query row of the q-tile
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const int row = it * kTileM + r;
    const bool row_valid = row < p.N;
    const int qh = BLK == 128 ? 0 : (r >> 6);
    const float sl2 = p.scale_log2;
    const size_t rix = static_cast<size_t>(bh) * p.N + (row_valid ? row : 0);
    const float l2 = row_valid ? p.lse[rix] * -1.4426950408889634f : 0.f;   // -lse * log2(e)
    const float dl = row_valid ? p.delta[rix] : 0.f;
    bool ok = true;
    if (n_list > 0) {
      // row r of Q (warps 0-3) or dO (warps 4-7) from the 128-byte swizzled TMA
      // tile (16-byte chunk j of a row at chunk j ^ (r % 8)) into TMEM as bf16
      // pairs: the A operand layout of the MMAs above
      if (!mbar_wait(qd_full, 0)) {
        misc[2] = 1;
        ok = false;
      }
      const uint8_t* tile = smem + (hh == 0 ? L::kOffFix0 : L::kOffFix1);
#pragma unroll
      for (int hd = 0; hd < D / 64; ++hd) {
        uint32_t w[32];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint4 c = *reinterpret_cast<const uint4*>(tile + hd * kHalfBytes + r * 128 + ((j ^ (r & 7)) << 4));
          w[4 * j] = c.x;
          w[4 * j + 1] = c.y;
          w[4 * j + 2] = c.z;
          w[4 * j + 3] = c.w;
        }
        tmem_st32((hh == 0 ? tm_q : tm_do) + lane_off + 32 * hd, reinterpret_cast<const float*>(w));
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(qd_tmem);
    }
    for (int e = 0; e < n_list; ++e) {
      const uint32_t bits = list[e] >> 16;
      const int jt = static_cast<int>(list[e] & 0xFFFFu);
      const int valid_k = min(kTileN, p.N - jt * kTileN);
      if (!mbar_wait(&ready[hh], e & 1)) {
        misc[2] = 1;
        ok = false;
      }
      tc_fence_after();
      // half hh: key columns [64 hh, 64 hh + 64), k-block half hh for block 64
      const bool quad = BLK == 128 ? true : ((bits >> (qh * 2 + hh)) & 1u);
      const int nv0 = min(32, max(0, valid_k - 64 * hh)), nv1 = min(32, max(0, valid_k - 64 * hh - 32));
      uint32_t keep0 = (row_valid && quad) ? (nv0 == 32 ? 0xffffffffu : ((1u << nv0) - 1u)) : 0u;
      uint32_t keep1 = (row_valid && quad) ? (nv1 == 32 ? 0xffffffffu : ((1u << nv1) - 1u)) : 0u;
      if (p.causal && jt == it) {
        // diagonal tile: key column c is visible to row r only if c <= r
        keep0 &= ~causal_from(r - 64 * hh + 1);
        keep1 &= ~causal_from(r - 64 * hh - 32 + 1);
      }
      grad_half<false, false>(tm_s + lane_off, tm_dp + lane_off, tm_s + lane_off, hh, sl2, nullptr, nullptr, l2, dl,
                              keep0, keep1);
      tmem_st_wait();
      tc_fence_before();
      named_bar_sync(hh == 0 ? kBarBwdA : kBarBwdB, kBwdHandoff);
    }
    // epilogue: warps 0-3 write dQ columns [0, D/2), warps 4-7 [D/2, D)
    if (n_list > 0 && !mbar_wait(final_done, 0)) {
      misc[2] = 1;
      ok = false;
    }
    tc_fence_after();
    if (n_list == 0 || __all_sync(0xffffffffu, ok && !aborted())) {
      store_row<D / 2>(tm_dq + lane_off + hh * (D / 2), p.scale, p.dq + rix * D + hh * (D / 2), n_list == 0,
                       row_valid);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kBwdMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace sa
