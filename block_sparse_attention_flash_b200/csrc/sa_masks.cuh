// sa_masks.cuh — block-mask construction and pyramid pooling kernels.
//
//   radial_mask_kernel     static radial mask (Radial Attention page, static
//                          exponential-decay mask paragraphs)
//   block_means_kernel     mean of each token block of Q and K (VMoBA write-up,
//                          block scoring with pooled queries/keys)
//   block_scores_tc_kernel S_ij = scale * qbar_i . kbar_j (one small GEMM per
//                          head, fp32 accuracy from three tf32 tensor-core passes)
//   tau_select_warp_kernel per q-block row, one warp: tau-mass selection
//                          (VMoBA write-up, threshold dynamic selection)
//   level_select_warp_kernel  per q-block row, one warp: PSA level quotas (PSA
//                          page, multi-level mask generator)
//   block_select_kernel    either, one CTA per row, for rows above 1024 blocks
//   pyramid_pool_kernel    mean of 2, 4, 8 consecutive tokens (PSA page,
//                          pyramid KV by progressive average pooling)
//
// The readers are HBM-bound; loads are 16-byte vectors, consecutive threads
// read consecutive 16-byte chunks of a row, and each thread keeps several rows
// in flight before it reduces.
#pragma once

#include "sa_common.cuh"

namespace sa {

// ------------------------------------------------------------ radial mask ---
__global__ void radial_mask_kernel(int nb, int F, int block, int S, uint8_t* __restrict__ out) {
  const int i = blockIdx.x;
  const long long fi_tok = static_cast<long long>(i) * block;
  const int fi = static_cast<int>(fi_tok / F);
  const int pi = static_cast<int>((fi_tok % F) / block);
  for (int j = threadIdx.x; j < nb; j += blockDim.x) {
    const long long fj_tok = static_cast<long long>(j) * block;
    const int fj = static_cast<int>(fj_tok / F);
    const int pj = static_cast<int>((fj_tok % F) / block);
    const int dt = abs(fi - fj);
    uint8_t keep;
    if (dt <= 1) {
      keep = 1;
    } else {
      const int k = 31 - __clz(dt);  // floor(log2 dt)
      keep = (static_cast<long long>(abs(pi - pj)) << k) < static_cast<long long>(S) ? 1 : 0;
    }
    out[static_cast<size_t>(i) * nb + j] = keep;
  }
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float* f) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 v = __bfloat1622float2(h[i]);
    f[2 * i] = v.x;
    f[2 * i + 1] = v.y;
  }
}

// ------------------------------------------------------------ block means ---
// grid (nb, B*H, 2): z = 0 averages Q, z = 1 averages K.  128 threads: thread
// (rg, ch) sums 16-byte chunk ch of rows rg, rg + RG, ...; smem reduces over rg.
// Each fp32 mean x is written as two tf32 parts for the scores GEMM: hi = x
// with its 13 low mantissa bits cleared (exact in tf32) and lo = x - hi
// (exact in fp32); hi + lo = x.
__device__ __forceinline__ float tf32_hi(float v) { return __uint_as_float(__float_as_uint(v) & 0xFFFFE000u); }

template <int D>
__global__ void __launch_bounds__(128) block_means_kernel(const __nv_bfloat16* __restrict__ q,
                                                          const __nv_bfloat16* __restrict__ k, int N, int block,
                                                          int nb, float* __restrict__ qhi, float* __restrict__ qlo,
                                                          float* __restrict__ khi, float* __restrict__ klo) {
  constexpr int CH = D / 8;      // 16-byte chunks per row
  constexpr int RG = 128 / CH;   // row groups
  __shared__ float red[RG][D];
  // the scores kernel after this one may be scheduled once every CTA here
  // has started; it waits for this grid's completion before reading
  asm volatile("griddepcontrol.launch_dependents;");
  const int i = blockIdx.x, bh = blockIdx.y, z = blockIdx.z;
  const __nv_bfloat16* x = (z == 0 ? q : k) + (static_cast<size_t>(bh) * N + static_cast<size_t>(i) * block) * D;
  const int rows = min(block, N - i * block);
  const int ch = threadIdx.x % CH, rg = threadIdx.x / CH;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  int r = rg;
  for (; r + 3 * RG < rows; r += 4 * RG) {
    uint4 u[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) u[j] = __ldg(reinterpret_cast<const uint4*>(x + static_cast<size_t>(r + j * RG) * D) + ch);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float f[8];
      bf16x8_to_f32(u[j], f);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += f[e];
    }
  }
  for (; r < rows; r += RG) {
    float f[8];
    bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(x + static_cast<size_t>(r) * D) + ch), f);
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += f[e];
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[rg][ch * 8 + e] = acc[e];
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += 128) {
    float s = 0.f;
#pragma unroll
    for (int g = 0; g < RG; ++g) s += red[g][c];
    const size_t o = (static_cast<size_t>(bh) * nb + i) * D + c;
    const float m = s / static_cast<float>(rows);
    const float hi = tf32_hi(m);
    (z == 0 ? qhi : khi)[o] = hi;
    (z == 0 ? qlo : klo)[o] = m - hi;
  }
}

// ------------------------------------------- block scores on tensor cores ---
// grid (ceil(nb/256), ceil(nb/128), B*H), 128 threads, one 128 x 256 tile of
// S = scale * Qbar Kbar^T per CTA, fp32 out.  The means arrive as tf32 parts
// (x = hi + lo, block_means_kernel), and
//   S ~= hi_q hi_k^T + hi_q lo_k^T + lo_q hi_k^T
// runs as three tcgen05 kind::tf32 MMA passes accumulating in fp32 in TMEM
// (the dropped lo_q lo_k^T term and the tf32 rounding of lo are below 2^-20
// of each product, close to fp32's own rounding).  The d dimension goes in
// chunks of 32 (one 128-byte row of a 128-byte-swizzled K-major operand)
// through a 2-stage ring that TMA fills (Q hi / lo: 128 rows, K hi / lo: 256
// rows; rows past a head's last block read as zero); per chunk one elected
// lane issues 12 MMAs (3 passes x 4 steps of K = 8) and releases the stage.
// Epilogue: one thread per row loads its 256 fp32 accumulators from TMEM,
// scales and stores the columns below nb.
constexpr int kScoresStage = 2 * 16384 + 2 * 32768;   // A hi, A lo (128 rows), B hi, B lo (256 rows) x 128 B
constexpr int kScoresTcSmem = 2 * kScoresStage;

struct ScoresMaps {
  CUtensorMap qhi, qlo, khi, klo;   // fp32 [B*H][nb][D], box 32 columns x 128 (Q) or 256 (K) rows
};

template <int D>
__global__ void __launch_bounds__(128, 1) block_scores_tc_kernel(const __grid_constant__ ScoresMaps maps, int nb,
                                                                 float scale, float* __restrict__ scores) {
  constexpr int kChunks = D / 32;
  // kind::tf32: D f32 (bits 4-5 = 1), A and B tf32 (bits 7-9, 10-12 = 2), both
  // K-major, N = 256 (bits 17-22 = N >> 3), M = 128 (bits 24-28 = M >> 4)
  constexpr uint32_t kIdesc = (1u << 4) | (2u << 7) | (2u << 10) | ((256u >> 3) << 17) | ((128u >> 4) << 24);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t full_bar[2], empty_bar[2], done_bar;
  __shared__ uint32_t tmem_base;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.z, i0 = blockIdx.y * 128, j0 = blockIdx.x * 256;
  if (warp == 2) {
    tmem_alloc(&tmem_base, 256);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
    }
    mbar_init(&done_bar, 1);
    fence_mbar_init();
    tma_prefetch_desc(&maps.qhi);
    tma_prefetch_desc(&maps.qlo);
    tma_prefetch_desc(&maps.khi);
    tma_prefetch_desc(&maps.klo);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // launched with programmatic stream serialization: the set-up above may run
  // beside the block means; wait until they are complete and visible, then
  // let the selection after this kernel be scheduled
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;");
  const uint32_t tmem = tmem_base;
  if (warp == 0) {
    // ------------------------------------------------------ TMA producer ---
    if (lane == 0) {
      for (int c = 0; c < kChunks; ++c) {
        const int st = c & 1;
        if (c >= 2 && !mbar_wait(&empty_bar[st], ((c >> 1) - 1) & 1)) break;
        uint8_t* base = smem + st * kScoresStage;
        mbar_arrive_expect_tx(&full_bar[st], static_cast<uint32_t>(kScoresStage));
        tma_load_3d(&maps.qhi, &full_bar[st], base, c * 32, i0, bh);
        tma_load_3d(&maps.qlo, &full_bar[st], base + 16384, c * 32, i0, bh);
        tma_load_3d(&maps.khi, &full_bar[st], base + 32768, c * 32, j0, bh);
        tma_load_3d(&maps.klo, &full_bar[st], base + 65536, c * 32, j0, bh);
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------- MMA issue ---
    bool ok = true;
    for (int c = 0; c < kChunks; ++c) {
      const int st = c & 1;
      ok = ok && __all_sync(0xffffffffu, mbar_wait(&full_bar[st], (c >> 1) & 1));
      if (ok) {
        tc_fence_after();
        const uint32_t sbase = smem_addr(smem + st * kScoresStage);
        const uint64_t d_ahi = smem_desc(sbase, 16, 1024), d_alo = smem_desc(sbase + 16384, 16, 1024);
        const uint64_t d_bhi = smem_desc(sbase + 32768, 16, 1024), d_blo = smem_desc(sbase + 65536, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t off = static_cast<uint64_t>(kk * 32) >> 4;
          mma_tf32_warp(tmem, d_ahi + off, d_bhi + off, kIdesc, (c > 0 || kk > 0) ? 1u : 0u);
          mma_tf32_warp(tmem, d_ahi + off, d_blo + off, kIdesc, 1u);
          mma_tf32_warp(tmem, d_alo + off, d_bhi + off, kIdesc, 1u);
        }
      }
      mma_commit_warp(&empty_bar[st]);   // also after an error, so that the producer never stalls
    }
    mma_commit_warp(&done_bar);
  }
  // epilogue: thread = row i0 + 32 warp + lane, columns j0 .. j0 + 255
  const bool ok = mbar_wait(&done_bar, 0);
  tc_fence_after();
  const int i = i0 + warp * 32 + lane;
  float* srow = scores + (static_cast<size_t>(bh) * nb + (i < nb ? i : 0)) * nb;
#pragma unroll 1
  for (int cc = 0; cc < 8; ++cc) {
    float v[32];
    tmem_ld32(tmem + (static_cast<uint32_t>(warp * 32) << 16) + cc * 32, v);
    const int jb = j0 + cc * 32;
    if (i < nb && ok && jb < nb) {
      if (jb + 32 <= nb && (nb & 3) == 0) {
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4)
          *reinterpret_cast<float4*>(srow + jb + q4 * 4) =
              make_float4(v[q4 * 4] * scale, v[q4 * 4 + 1] * scale, v[q4 * 4 + 2] * scale, v[q4 * 4 + 3] * scale);
      } else {
#pragma unroll
        for (int t = 0; t < 32; ++t)
          if (jb + t < nb) srow[jb + t] = v[t] * scale;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ---------------------------------------------------------- block select ---
constexpr int kSelectThreads = 256;
constexpr int kMaxSelect = 4096;

// Order-preserving map of a float to an unsigned key (larger float -> larger key).
__device__ __forceinline__ uint32_t float_order_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float block_reduce_max(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  v = (l < kSelectThreads / 32) ? red[l] : -__int_as_float(0x7f800000);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float block_reduce_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  v = (l < kSelectThreads / 32) ? red[l] : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__host__ __device__ inline int select_pow2(int nb) {
  int P = 32;
  while (P < nb) P <<= 1;
  return P;
}
__host__ __device__ inline size_t select_smem_bytes(int nb) {
  return static_cast<size_t>(select_pow2(nb)) * 13;
}

// One CTA per (b, h, i).  Keys (descending score, then ascending j) are
// bitonic-sorted in shared memory; TAU mode takes an exclusive prefix sum of
// the probabilities in that order, LEVELS mode uses the rank directly.
__global__ void __launch_bounds__(kSelectThreads) block_select_kernel(const float* __restrict__ scores, int nb,
                                                                      int mode, float tau, int c0, int c1, int c2,
                                                                      uint8_t* __restrict__ mask_out) {
  // dynamic shared memory: keys[P] (8 B), prob[P] (4 B), out_row[P] (1 B)
  extern __shared__ unsigned long long select_smem[];
  __shared__ float red[32];
  __shared__ float part[kSelectThreads];
  int P = 32;
  while (P < nb) P <<= 1;
  unsigned long long* keys = select_smem;
  float* prob = reinterpret_cast<float*>(keys + P);
  uint8_t* out_row = reinterpret_cast<uint8_t*>(prob + P);
  const size_t row = blockIdx.x;
  const float* srow = scores + row * nb;

  float mx = -__int_as_float(0x7f800000);
  for (int j = threadIdx.x; j < P; j += kSelectThreads) {
    if (j < nb) {
      const float sc = srow[j];
      prob[j] = sc;
      mx = fmaxf(mx, sc);
      keys[j] = (static_cast<unsigned long long>(~float_order_key(sc)) << 32) | static_cast<unsigned>(j);
    } else {
      keys[j] = ~0ull;
    }
  }
  if (mode == SA_MASK_TAU) {
    mx = block_reduce_max(mx, red);
    float sum = 0.f;
    for (int j = threadIdx.x; j < nb; j += kSelectThreads) {
      const float e = expf(prob[j] - mx);
      prob[j] = e;
      sum += e;
    }
    sum = block_reduce_sum(sum, red);
    const float inv = 1.f / sum;
    for (int j = threadIdx.x; j < nb; j += kSelectThreads) prob[j] *= inv;
  }
  __syncthreads();

  // bitonic sort, ascending keys
  for (int k = 2; k <= P; k <<= 1) {
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      for (int i = threadIdx.x; i < P; i += kSelectThreads) {
        const int ixj = i ^ jj;
        if (ixj > i) {
          const unsigned long long a = keys[i], b = keys[ixj];
          const bool up = (i & k) == 0;
          if ((a > b) == up) {
            keys[i] = b;
            keys[ixj] = a;
          }
        }
      }
      __syncthreads();
    }
  }

  if (mode == SA_MASK_TAU) {
    // exclusive scan of prob in sorted order: each thread a contiguous run
    const int per = (nb + kSelectThreads - 1) / kSelectThreads;
    const int r0 = threadIdx.x * per, r1 = min(nb, r0 + per);
    float s = 0.f;
    for (int r = r0; r < r1; ++r) s += prob[static_cast<unsigned>(keys[r])];
    part[threadIdx.x] = s;
    __syncthreads();
    if (threadIdx.x < 32) {
      // scan of the 256 partial sums by one warp (8 per lane)
      float v[8];
      float tot = 0.f;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        v[u] = part[threadIdx.x * 8 + u];
        tot += v[u];
      }
      float inc = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, inc, o);
        if (threadIdx.x >= o) inc += y;
      }
      float run = inc - tot;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float x = v[u];
        part[threadIdx.x * 8 + u] = run;
        run += x;
      }
    }
    __syncthreads();
    float before = part[threadIdx.x];
    for (int r = r0; r < r1; ++r) {
      const unsigned j = static_cast<unsigned>(keys[r]);
      out_row[j] = before < tau ? 1 : 0;
      before += prob[j];
    }
  } else {
    for (int r = threadIdx.x; r < nb; r += kSelectThreads) {
      const unsigned j = static_cast<unsigned>(keys[r]);
      out_row[j] = r < c0 ? 1 : (r < c1 ? 2 : (r < c2 ? 3 : 4));
    }
  }
  __syncthreads();
  uint8_t* mrow = mask_out + row * nb;
  for (int j = threadIdx.x; j < nb; j += kSelectThreads) mrow[j] = out_row[j];
}

// LEVELS rows without a sort (rows of at most 32*E blocks, one warp per row).
// A block's level follows its rank r in (descending score, ascending j)
// order: code 1 for r < c0, 2 for r < c1, 3 for r < c2, else 4.  For each
// cut c the 32-bit score key K_c of the block of rank c - 1 is found bit by
// bit from the most significant end: the smallest K with count(key <= K) >=
// c (32 rounds of a warp count, the three cuts side by side).  A block is
// below cut c if its key is below K_c, or if its key equals K_c (equal
// scores) and fewer than c blocks precede it: those with a smaller key, then
// the tied ones in ascending j.  Lane l holds blocks j = 32 k + l (k < E), so
// the row is read and the codes written with coalesced accesses.
template <int E>
__device__ __forceinline__ void level_select_row(const float* __restrict__ srow, int nb, int c0, int c1, int c2,
                                                 uint8_t* __restrict__ mrow, int lane) {
  uint32_t key[E];
#pragma unroll
  for (int k = 0; k < E; ++k) {
    const int i = 32 * k + lane;
    key[k] = i < nb ? ~float_order_key(srow[i]) : 0xFFFFFFFFu;   // ascending key = descending score
  }
  const uint32_t cut[3] = {static_cast<uint32_t>(max(c0, 0)), static_cast<uint32_t>(max(c1, 0)),
                           static_cast<uint32_t>(max(c2, 0))};
  uint32_t kst[3] = {0u, 0u, 0u};
#pragma unroll 1
  for (int b = 31; b >= 0; --b) {
    const uint32_t low = (1u << b) - 1u;
#pragma unroll
    for (int c = 0; c < 3; ++c) {
      const uint32_t cand = kst[c] | low;
      uint32_t n = 0;
#pragma unroll
      for (int k = 0; k < E; ++k) n += (32 * k + lane < nb && key[k] <= cand) ? 1u : 0u;
      n = __reduce_add_sync(0xffffffffu, n);
      if (n < cut[c]) kst[c] |= 1u << b;
    }
  }
  uint32_t less[3];
#pragma unroll
  for (int c = 0; c < 3; ++c) {
    uint32_t n = 0;
#pragma unroll
    for (int k = 0; k < E; ++k) n += (32 * k + lane < nb && key[k] < kst[c]) ? 1u : 0u;
    less[c] = __reduce_add_sync(0xffffffffu, n);
  }
  uint32_t tie_before[3] = {0u, 0u, 0u};
  const unsigned lower = (1u << lane) - 1u;
#pragma unroll
  for (int k = 0; k < E; ++k) {
    const int i = 32 * k + lane;
    uint8_t code = 1;
#pragma unroll
    for (int c = 0; c < 3; ++c) {
      const bool tied = i < nb && key[k] == kst[c];
      const unsigned ball = __ballot_sync(0xffffffffu, tied);
      const bool below =
          key[k] < kst[c] || (tied && less[c] + tie_before[c] + static_cast<uint32_t>(__popc(ball & lower)) < cut[c]);
      code += below ? 0 : 1;
      tie_before[c] += static_cast<uint32_t>(__popc(ball));
    }
    if (i < nb) mrow[i] = code;
  }
}

// At E = 16 (rows of up to 512 blocks) the registers are capped so that 11
// CTAs share an SM: the 1,536 CTAs of 12 heads of 512 rows then run as one
// wave (50.1 against 55.5 us at 480p).  The same cap costs the tau kernel
// spills and time, so it keeps its 64 registers.
template <int E>
__global__ void __launch_bounds__(128, E == 16 ? 11 : 1) level_select_warp_kernel(const float* __restrict__ scores, int nb,
                                                                long long nrows, int c0, int c1, int c2,
                                                                uint8_t* __restrict__ mask_out) {
  // launched with programmatic stream serialization after the scores kernel
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * 4 + warp;
  if (row >= nrows) return;
  level_select_row<E>(scores + row * nb, nb, c0, c1, c2, mask_out + row * nb, lane);
}

// TAU rows without a sort (rows of at most 32*E blocks, one warp per row):
// the kept set is the shortest prefix, in (descending score, ascending j)
// order, whose probability mass reaches tau.  Its last key K* is the smallest
// 32-bit score key whose cumulative mass reaches tau; it is found bit by bit
// from the most significant end (32 rounds of a masked warp sum).  Blocks
// with a key below K* are kept; blocks whose key equals K* (equal scores) are
// kept in ascending j while the mass before them is < tau.  Lane l holds
// blocks j = 32 k + l (k < E), so the row is read with coalesced loads.
template <int E>
__device__ __forceinline__ void tau_select_row(const float* __restrict__ srow, int nb, float tau,
                                               uint8_t* __restrict__ mrow, int lane) {
  float sc[E], pr[E];
  uint32_t key[E];
  float mx = -__int_as_float(0x7f800000);
#pragma unroll
  for (int k = 0; k < E; ++k) {
    const int i = 32 * k + lane;
    sc[k] = i < nb ? srow[i] : -__int_as_float(0x7f800000);
    mx = fmaxf(mx, sc[k]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float sum = 0.f;
#pragma unroll
  for (int k = 0; k < E; ++k) {
    const int i = 32 * k + lane;
    pr[k] = i < nb ? expf(sc[k] - mx) : 0.f;
    sum += pr[k];
    key[k] = i < nb ? ~float_order_key(sc[k]) : 0xFFFFFFFFu;   // ascending key = descending score
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float inv = 1.f / sum;
#pragma unroll
  for (int k = 0; k < E; ++k) pr[k] *= inv;
  // smallest K with mass(key <= K) >= tau (all ones when the total stays below tau)
  uint32_t kstar = 0u;
#pragma unroll 1
  for (int b = 31; b >= 0; --b) {
    const uint32_t cand = kstar | ((1u << b) - 1u);
    float m = 0.f;
#pragma unroll
    for (int k = 0; k < E; ++k) m += key[k] <= cand ? pr[k] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m += __shfl_xor_sync(0xffffffffu, m, o);
    if (!(m >= tau)) kstar |= 1u << b;
  }
  // mass strictly before K*
  float below = 0.f;
#pragma unroll
  for (int k = 0; k < E; ++k) below += key[k] < kstar ? pr[k] : 0.f;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) below += __shfl_xor_sync(0xffffffffu, below, o);
  // blocks tied at K*, in ascending j: chunk by chunk, lanes in order
  int tie_before = 0;
  const unsigned lower = (1u << lane) - 1u;
#pragma unroll
  for (int k = 0; k < E; ++k) {
    const int i = 32 * k + lane;
    const bool tied = key[k] == kstar && i < nb;
    const unsigned ball = __ballot_sync(0xffffffffu, tied);
    if (i < nb) {
      uint8_t keep = key[k] < kstar ? 1 : 0;
      if (tied) keep = below + static_cast<float>(tie_before + __popc(ball & lower)) * pr[k] < tau ? 1 : 0;
      mrow[i] = keep;
    }
    tie_before += __popc(ball);
  }
}

template <int E>
__global__ void __launch_bounds__(128) tau_select_warp_kernel(const float* __restrict__ scores, int nb,
                                                              long long nrows, float tau,
                                                              uint8_t* __restrict__ mask_out) {
  // launched with programmatic stream serialization after the scores kernel
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = static_cast<long long>(blockIdx.x) * 4 + warp;
  if (row >= nrows) return;
  tau_select_row<E>(scores + row * nb, nb, tau, mask_out + row * nb, lane);
}

// ----------------------------------------------------------- pyramid pool ---
// grid (ceil(N / (8 * GPB)), B*H, 2); z = 0 pools K, z = 1 pools V.  Thread
// (g, ch) owns the 8-token group g of the CTA and 16-byte chunk ch: it loads
// the 8 rows once and writes the c = 2, 4 and 8 means of that chunk.
template <int D>
__global__ void __launch_bounds__(128) pyramid_pool_kernel(const __nv_bfloat16* __restrict__ k,
                                                           const __nv_bfloat16* __restrict__ v, int N,
                                                           __nv_bfloat16* __restrict__ k2,
                                                           __nv_bfloat16* __restrict__ k4,
                                                           __nv_bfloat16* __restrict__ k8,
                                                           __nv_bfloat16* __restrict__ v2,
                                                           __nv_bfloat16* __restrict__ v4,
                                                           __nv_bfloat16* __restrict__ v8) {
  constexpr int CH = D / 8;
  constexpr int GPB = 128 / CH;  // 8-token groups per CTA
  const int bh = blockIdx.y, z = blockIdx.z;
  const int g = blockIdx.x * GPB + threadIdx.x / CH;
  const int ch = threadIdx.x % CH;
  const int r0 = g * 8;
  if (r0 >= N) return;
  const int rows = min(8, N - r0);
  const __nv_bfloat16* x = (z == 0 ? k : v) + (static_cast<size_t>(bh) * N + r0) * D;
  float f[8][8];
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    if (r < rows) {
      bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(x + static_cast<size_t>(r) * D) + ch), f[r]);
    } else {
#pragma unroll
      for (int e = 0; e < 8; ++e) f[r][e] = 0.f;
    }
  }
  __nv_bfloat16* o2 = z == 0 ? k2 : v2;
  __nv_bfloat16* o4 = z == 0 ? k4 : v4;
  __nv_bfloat16* o8 = z == 0 ? k8 : v8;
  const size_t n2 = (N + 1) / 2, n4 = (N + 3) / 4, n8 = (N + 7) / 8;
  auto store = [&](__nv_bfloat16* base, size_t nrows, size_t prow, const float* s, float inv) {
    if (prow >= nrows) return;
    uint4 w;
    w.x = pack_bf16x2(s[0] * inv, s[1] * inv);
    w.y = pack_bf16x2(s[2] * inv, s[3] * inv);
    w.z = pack_bf16x2(s[4] * inv, s[5] * inv);
    w.w = pack_bf16x2(s[6] * inv, s[7] * inv);
    reinterpret_cast<uint4*>(base + (static_cast<size_t>(bh) * nrows + prow) * D)[ch] = w;
  };
  float s2[4][8], s4[2][8], s8[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
#pragma unroll
    for (int u = 0; u < 4; ++u) s2[u][e] = f[2 * u][e] + f[2 * u + 1][e];
    s4[0][e] = s2[0][e] + s2[1][e];
    s4[1][e] = s2[2][e] + s2[3][e];
    s8[e] = s4[0][e] + s4[1][e];
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int cnt = min(2, max(0, rows - 2 * u));
    if (cnt > 0) store(o2, n2, static_cast<size_t>(r0 / 2 + u), s2[u], 1.f / cnt);
  }
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int cnt = min(4, max(0, rows - 4 * u));
    if (cnt > 0) store(o4, n4, static_cast<size_t>(r0 / 4 + u), s4[u], 1.f / cnt);
  }
  store(o8, n8, static_cast<size_t>(r0 / 8), s8, 1.f / rows);
}

// ------------------------------------------------ global block selection ---
// VMoBA write-up, "global block selection" and "threshold dynamic selection"
// paragraphs: the (q-block, k-block) pairs of a head compete with each other
// rather than within a row, and the head's own concentration decides how many
// survive.  Reading: P_ij = softmax_j(S_ij) per row; all pairs of the head are
// visited by descending P (ties: lower i * Nb + j first) and a pair is kept
// iff the mass visited before it is < tau * Nb (the head's total mass is Nb).
//
// Row statistics (max, 1 / sum of exp) first, one warp per row.
__global__ void __launch_bounds__(128) global_row_stats_kernel(const float* __restrict__ scores, int nb, long long nrows,
                                                               float2* __restrict__ stats) {
  const long long row = static_cast<long long>(blockIdx.x) * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= nrows) return;
  const float* srow = scores + row * nb;
  float mx = -__int_as_float(0x7f800000);
  for (int j = lane; j < nb; j += 32) mx = fmaxf(mx, srow[j]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  float sum = 0.f;
  for (int j = lane; j < nb; j += 32) sum += expf(srow[j] - mx);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  if (lane == 0) stats[row] = make_float2(mx, 1.f / sum);
}

// Then one CTA per head finds the last kept pair by a most-significant-first
// radix search over the 64-bit key (fp32 bits of P, then the complement of the
// pair index): pass k histograms, by the key's next 8 bits, the mass of the
// pairs that match the bits fixed so far; the bin where the mass counted from
// the top first reaches tau * Nb holds the last kept pair.  After 8 passes the
// key is known and a pair is kept iff its key is >= it.  P is recomputed from
// the scores in every pass with the same instructions, so it is the same value
// each time.
constexpr int kGlobalThreads = 1024;
constexpr int kGlobalWarps = kGlobalThreads / 32;

__device__ __forceinline__ unsigned long long global_key(const float* srow_scores, const float2 st, int j, int lin) {
  const float p = expf(srow_scores[j] - st.x) * st.y;
  return (static_cast<unsigned long long>(__float_as_uint(p)) << 32) | (0xFFFFFFFFu - static_cast<uint32_t>(lin));
}

__global__ void __launch_bounds__(kGlobalThreads) global_select_kernel(const float* __restrict__ scores,
                                                                       const float2* __restrict__ stats, int nb,
                                                                       float tau, uint8_t* __restrict__ mask) {
  __shared__ float hist[kGlobalWarps][256];
  __shared__ float bin_mass[256];
  __shared__ unsigned long long s_prefix;
  __shared__ double s_above;
  __shared__ int s_keep_all;
  const int bh = blockIdx.x;
  const int warp = threadIdx.x >> 5;
  const float* sc = scores + static_cast<size_t>(bh) * nb * nb;
  const float2* st = stats + static_cast<size_t>(bh) * nb;
  const int total = nb * nb;
  const double target = static_cast<double>(tau) * nb;
  if (threadIdx.x == 0) {
    s_prefix = 0ull;
    s_above = 0.0;
    s_keep_all = 0;
  }
  for (int pass = 0; pass < 8; ++pass) {
    const int shift = 56 - 8 * pass;
    for (int i = threadIdx.x; i < kGlobalWarps * 256; i += kGlobalThreads) (&hist[0][0])[i] = 0.f;
    __syncthreads();
    const unsigned long long prefix = s_prefix;
    const unsigned long long hi_mask = pass == 0 ? 0ull : (~0ull << (shift + 8));
    for (int e = threadIdx.x; e < total; e += kGlobalThreads) {
      const int i = e / nb, j = e - (e / nb) * nb;
      const unsigned long long key = global_key(sc + static_cast<size_t>(i) * nb, st[i], j, e);
      if ((key & hi_mask) == prefix) {
        const float p = __uint_as_float(static_cast<uint32_t>(key >> 32));
        atomicAdd(&hist[warp][(key >> shift) & 255u], p);
      }
    }
    __syncthreads();
    if (threadIdx.x < 256) {
      float m = 0.f;
      for (int w = 0; w < kGlobalWarps; ++w) m += hist[w][threadIdx.x];
      bin_mass[threadIdx.x] = m;
    }
    __syncthreads();
    if (threadIdx.x == 0 && !s_keep_all) {
      // bins from the top: the first whose inclusive cumulative mass reaches the target
      double cum = s_above;
      int bin = -1;
      for (int b = 255; b >= 0; --b) {
        if (cum + bin_mass[b] >= target) {
          bin = b;
          break;
        }
        cum += bin_mass[b];
      }
      if (bin < 0) {
        s_keep_all = 1;   // the head's mass never reaches the target: keep every pair
      } else {
        s_prefix = prefix | (static_cast<unsigned long long>(bin) << shift);
        s_above = cum;
      }
    }
    __syncthreads();
    if (s_keep_all) break;
  }
  const unsigned long long cut = s_prefix;
  const bool all = s_keep_all != 0;
  uint8_t* mk = mask + static_cast<size_t>(bh) * total;
  for (int e = threadIdx.x; e < total; e += kGlobalThreads) {
    const int i = e / nb, j = e - (e / nb) * nb;
    mk[e] = (all || global_key(sc + static_cast<size_t>(i) * nb, st[i], j, e) >= cut) ? uint8_t(1) : uint8_t(0);
  }
}

// Many-CTA form of the same search for large heads (Nb > 64): G CTAs per
// head each histogram a slice of the head's pairs into the head's global bins
// (one launch per pass), and one CTA per head then picks the bin.  State per
// head: [0] key prefix, [1] mass above the prefix (double bits), [2] keep-all.
constexpr int kGlobalSliceThreads = 512;

__global__ void global_init_kernel(float* __restrict__ hist, unsigned long long* __restrict__ state) {
  const int bh = blockIdx.x;
  for (int b = threadIdx.x; b < 256; b += blockDim.x) hist[bh * 256 + b] = 0.f;
  if (threadIdx.x < 4) state[bh * 4 + threadIdx.x] = 0ull;
}

__global__ void __launch_bounds__(kGlobalSliceThreads) global_hist_kernel(
    const float* __restrict__ scores, const float2* __restrict__ stats, int nb, int pass,
    const unsigned long long* __restrict__ state, float* __restrict__ hist) {
  __shared__ float wh[kGlobalSliceThreads / 32][256];
  const int bh = blockIdx.y;
  if (state[bh * 4 + 2]) return;
  const int warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < (kGlobalSliceThreads / 32) * 256; i += kGlobalSliceThreads) (&wh[0][0])[i] = 0.f;
  __syncthreads();
  const int shift = 56 - 8 * pass;
  const unsigned long long prefix = state[bh * 4];
  const unsigned long long hi_mask = pass == 0 ? 0ull : (~0ull << (shift + 8));
  const float* sc = scores + static_cast<size_t>(bh) * nb * nb;
  const float2* st = stats + static_cast<size_t>(bh) * nb;
  const int total = nb * nb;
  const int per = (total + gridDim.x - 1) / gridDim.x;
  const int e0 = blockIdx.x * per, e1 = min(total, e0 + per);
  for (int e = e0 + threadIdx.x; e < e1; e += kGlobalSliceThreads) {
    const int i = e / nb, j = e - (e / nb) * nb;
    const unsigned long long key = global_key(sc + static_cast<size_t>(i) * nb, st[i], j, e);
    if ((key & hi_mask) == prefix) atomicAdd(&wh[warp][(key >> shift) & 255u], __uint_as_float(static_cast<uint32_t>(key >> 32)));
  }
  __syncthreads();
  if (threadIdx.x < 256) {
    float m = 0.f;
    for (int w = 0; w < kGlobalSliceThreads / 32; ++w) m += wh[w][threadIdx.x];
    if (m != 0.f) atomicAdd(&hist[bh * 256 + threadIdx.x], m);
  }
}

__global__ void global_decide_kernel(float* __restrict__ hist, unsigned long long* __restrict__ state, int nb,
                                     float tau, int pass) {
  const int bh = blockIdx.x;
  if (threadIdx.x == 0 && !state[bh * 4 + 2]) {
    const int shift = 56 - 8 * pass;
    const double target = static_cast<double>(tau) * nb;
    double cum = __longlong_as_double(static_cast<long long>(state[bh * 4 + 1]));
    int bin = -1;
    for (int b = 255; b >= 0; --b) {
      const double m = hist[bh * 256 + b];
      if (cum + m >= target) {
        bin = b;
        break;
      }
      cum += m;
    }
    if (bin < 0) {
      state[bh * 4 + 2] = 1ull;
    } else {
      state[bh * 4] |= static_cast<unsigned long long>(bin) << shift;
      state[bh * 4 + 1] = static_cast<unsigned long long>(__double_as_longlong(cum));
    }
  }
  __syncthreads();
  for (int b = threadIdx.x; b < 256; b += blockDim.x) hist[bh * 256 + b] = 0.f;
}

__global__ void __launch_bounds__(kGlobalSliceThreads) global_mark_kernel(
    const float* __restrict__ scores, const float2* __restrict__ stats, int nb,
    const unsigned long long* __restrict__ state, uint8_t* __restrict__ mask) {
  const int bh = blockIdx.y;
  const unsigned long long cut = state[bh * 4];
  const bool all = state[bh * 4 + 2] != 0ull;
  const float* sc = scores + static_cast<size_t>(bh) * nb * nb;
  const float2* st = stats + static_cast<size_t>(bh) * nb;
  const int total = nb * nb;
  const int per = (total + gridDim.x - 1) / gridDim.x;
  const int e0 = blockIdx.x * per, e1 = min(total, e0 + per);
  uint8_t* mk = mask + static_cast<size_t>(bh) * total;
  for (int e = e0 + threadIdx.x; e < e1; e += kGlobalSliceThreads) {
    const int i = e / nb, j = e - (e / nb) * nb;
    mk[e] = (all || global_key(sc + static_cast<size_t>(i) * nb, st[i], j, e) >= cut) ? uint8_t(1) : uint8_t(0);
  }
}

}  // namespace sa

