// sa_permute.cuh — token permutations of the (t, h, w) grid for sm_100a.
//
// PAROAttention write-up ("模式感知重排序", the pattern-aware reordering
// paragraphs): a video's tokens can be flattened in any of the 6 orders of
// the three axes, chosen per attention head, so that the tokens a head
// attends to together become contiguous and its attention map turns into
// blocks.  VMoBA write-up ("层级循环分块策略", layer-wise recurrent block
// partition): tokens are grouped into temporal (1D), spatial (2D) or
// spatio-temporal (3D) cells.  Both are one operation: order the tokens by
// (cell coordinates, coordinates inside the cell), each tuple taken in the
// head's axis order (slowest axis first).  Cells of 1 x 1 x 1 give PARO's
// pure axis orders; axis order t, h, w with cells of ct frames x Hh x Ww
// (1D), T x ch x cw (2D) or ct x ch x cw (3D) give VMoBA's partitions.  The
// attention kernels run unchanged on the permuted sequence; the inverse
// permutation brings O back to raster order.
//
// The kernel is a row gather (HBM-bound: every row read once, written once).
// The source row of an output row is computed from the grid and cell sizes
// with integer arithmetic (no index table), once per row.
#pragma once

#include "sa_common.cuh"

namespace sa {

constexpr int kPermMaxTensors = 4;

// axis order codes, slowest axis first (0 = t, 1 = h, 2 = w)
__host__ __device__ constexpr uint32_t perm_axes(int code) {
  // packed as a0 | a1 << 2 | a2 << 4
  return code == 0 ? (0u | 1u << 2 | 2u << 4)    // t h w (raster)
       : code == 1 ? (0u | 2u << 2 | 1u << 4)    // t w h
       : code == 2 ? (1u | 0u << 2 | 2u << 4)    // h t w
       : code == 3 ? (1u | 2u << 2 | 0u << 4)    // h w t
       : code == 4 ? (2u | 0u << 2 | 1u << 4)    // w t h
                   : (2u | 1u << 2 | 0u << 4);   // w h t
}

struct PermParams {
  const __nv_bfloat16* src[kPermMaxTensors];
  __nv_bfloat16* dst[kPermMaxTensors];
  int n_tensors;
  int H;
  int N;                  // T * Hh * Ww
  int g[3];               // grid extents (T, Hh, Ww)
  int c[3];               // cell extents (ct, ch, cw), dividing g
  int order;              // axis order code for every head, when head_order is NULL
  const uint8_t* head_order;
  int inverse;            // 0: dst[n'] = src[raster of n'], 1: dst[raster] = src[n']
};

__device__ __forceinline__ int sel3(int a, int v0, int v1, int v2) { return a == 0 ? v0 : (a == 1 ? v1 : v2); }

// Permuted position n' of the token at raster coordinates (xt, xh, xw) under
// axis order `ax`: (cell rank) * cell volume + rank inside the cell.
__device__ __forceinline__ int perm_rank(const PermParams& p, uint32_t ax, int xt, int xh, int xw) {
  int cell = 0, in = 0;
#pragma unroll
  for (int i = 0; i < 3; ++i) {
    const int a = (ax >> (2 * i)) & 3;
    const int x = sel3(a, xt, xh, xw), g = sel3(a, p.g[0], p.g[1], p.g[2]), c = sel3(a, p.c[0], p.c[1], p.c[2]);
    cell = cell * (g / c) + x / c;
    in = in * c + x % c;
  }
  return cell * (p.c[0] * p.c[1] * p.c[2]) + in;
}

// Raster coordinates of the token at permuted position np (inverse of perm_rank).
__device__ __forceinline__ void perm_coords(const PermParams& p, uint32_t ax, int np, int& xt, int& xh, int& xw) {
  const int vol = p.c[0] * p.c[1] * p.c[2];
  int cell = np / vol, in = np - (np / vol) * vol;
#pragma unroll
  for (int i = 2; i >= 0; --i) {
    const int a = (ax >> (2 * i)) & 3;
    const int g = sel3(a, p.g[0], p.g[1], p.g[2]), c = sel3(a, p.c[0], p.c[1], p.c[2]);
    const int m = g / c;
    const int x = (cell % m) * c + in % c;
    cell /= m;
    in /= c;
    if (a == 0) xt = x;
    else if (a == 1) xh = x;
    else xw = x;
  }
}

// Grid: x = chunks of 256 output rows, y = b * H + h, z = tensor.  Each warp
// owns 32 consecutive output rows: lane L works out the source row of row L
// (the index arithmetic runs once per row), then the warp moves the 32 rows,
// 32 / (D / 8) rows per instruction, all loads issued before the stores.
template <int D>
__global__ void __launch_bounds__(256) token_permute_kernel(const __grid_constant__ PermParams p) {
  constexpr int kTpr = D / 8;                  // lanes per row (16-byte chunks)
  constexpr int kRowsPerInst = 32 / kTpr;      // rows moved per warp instruction
  constexpr int kInsts = 32 / kRowsPerInst;    // instructions for the warp's 32 rows
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int bh = blockIdx.y, t = blockIdx.z;
  const int row0 = (blockIdx.x * 8 + warp) * 32;
  if (row0 >= p.N) return;
  const uint32_t ax = perm_axes(p.head_order ? p.head_order[bh % p.H] : p.order);
  int src_n = 0;
  const int n = row0 + lane;
  if (n < p.N) {
    int xt = 0, xh = 0, xw = 0;
    if (!p.inverse) {
      perm_coords(p, ax, n, xt, xh, xw);        // output position n is n'
      src_n = (xt * p.g[1] + xh) * p.g[2] + xw;
    } else {
      xt = n / (p.g[1] * p.g[2]);               // output position n is raster
      xh = (n / p.g[2]) % p.g[1];
      xw = n % p.g[2];
      src_n = perm_rank(p, ax, xt, xh, xw);
    }
  }
  const __nv_bfloat16* src = p.src[t] + static_cast<size_t>(bh) * p.N * D;
  __nv_bfloat16* dst = p.dst[t] + static_cast<size_t>(bh) * p.N * D;
  const int sub = lane % kTpr, which = lane / kTpr;
  uint4 v[kInsts];
#pragma unroll
  for (int i = 0; i < kInsts; ++i) {
    const int j = i * kRowsPerInst + which;    // row of the warp's 32
    const int sn = __shfl_sync(0xffffffffu, src_n, j);
    if (row0 + j < p.N) v[i] = reinterpret_cast<const uint4*>(src + static_cast<size_t>(sn) * D)[sub];
  }
#pragma unroll
  for (int i = 0; i < kInsts; ++i) {
    const int j = i * kRowsPerInst + which;
    if (row0 + j < p.N) reinterpret_cast<uint4*>(dst + static_cast<size_t>(row0 + j) * D)[sub] = v[i];
  }
}

}  // namespace sa
