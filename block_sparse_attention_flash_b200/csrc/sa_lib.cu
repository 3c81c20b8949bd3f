// sa_lib.cu — host side of the C ABI declared in include/sparse_attn.h.
//
// One translation unit holds every kernel (included below) so that the
// per-device error word is a single __device__ variable.  Host code only
// validates arguments, encodes TMA tensor maps, picks the kernel instance and
// launches it on the caller's stream; all arithmetic runs on the GPU.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "sa_attn_bwd.cuh"
#include "sa_attn_fwd.cuh"
#include "sa_common.cuh"
#include "sa_masks.cuh"
#include "sa_permute.cuh"
#include "sa_pyr_fwd.cuh"
#include "sparse_attn.h"

namespace {

using sa::AttnParams;

constexpr int kMaxDevices = 64;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
int ceil_div(long long a, long long b) { return static_cast<int>((a + b - 1) / b); }
cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

sa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? SA_OK : SA_ERR_CUDA; }

// ---------------------------------------------------------- tensor maps ---
PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// [B*H, rows, D] bf16 viewed as a 3D tensor (D innermost), 64 x 128 x 1 boxes,
// 128-byte swizzle, zero fill outside the tensor.
// [BH][rows][D] fp32, box 32 columns (128 bytes) x box_rows rows, 128-byte swizzle.
bool encode_f32_map(CUtensorMap* map, const void* base, int BH, int rows, int D, int box_rows) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 4, static_cast<cuuint64_t>(rows) * D * 4};
  cuuint32_t box[3] = {32, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_rows_map(CUtensorMap* map, const void* base, int BH, int rows, int D, int box_rows) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows), static_cast<cuuint64_t>(BH)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(rows) * D * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ----------------------------------------------- per-device kernel set-up ---
struct DeviceInit {
  std::once_flag flag;
  cudaError_t err = cudaSuccess;
  int n_sm = 1;
};
DeviceInit g_dev_init[kMaxDevices];

cudaError_t init_device_kernels() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  DeviceInit& di = g_dev_init[dev];
  std::call_once(di.flag, [&di] {
    cudaError_t r = cudaSuccess;
    auto set = [&r](const void* fn, int bytes) {
      if (r == cudaSuccess) r = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    };
    set(reinterpret_cast<const void*>(&sa::attn_fwd_kernel<128, 128, false>), sa::AttnSmem<128>::kAlloc);
    set(reinterpret_cast<const void*>(&sa::attn_fwd_kernel<128, 64, false>), sa::AttnSmem<128>::kAlloc);
    set(reinterpret_cast<const void*>(&sa::attn_fwd_kernel<64, 128, false>), sa::AttnSmem<64>::kAlloc);
    set(reinterpret_cast<const void*>(&sa::attn_fwd_kernel<64, 64, false>), sa::AttnSmem<64>::kAlloc);
    set(reinterpret_cast<const void*>(&sa::attn_fwd_kernel<128, 128, true>), sa::AttnSmem<128>::kAlloc);
    set(reinterpret_cast<const void*>(&sa::attn_fwd_kernel<128, 64, true>), sa::AttnSmem<128>::kAlloc);
    set(reinterpret_cast<const void*>(&sa::attn_fwd_kernel<64, 128, true>), sa::AttnSmem<64>::kAlloc);
    set(reinterpret_cast<const void*>(&sa::attn_fwd_kernel<64, 64, true>), sa::AttnSmem<64>::kAlloc);
    set(reinterpret_cast<const void*>(&sa::pyr_fwd_kernel<128, 128, false>), sa::PyrSmem<128>::kAlloc);
    set(reinterpret_cast<const void*>(&sa::pyr_fwd_kernel<128, 64, false>), sa::PyrSmem<128>::kAlloc);
    set(reinterpret_cast<const void*>(&sa::pyr_fwd_kernel<64, 128, false>), sa::PyrSmem<64>::kAlloc);
    set(reinterpret_cast<const void*>(&sa::pyr_fwd_kernel<64, 64, false>), sa::PyrSmem<64>::kAlloc);
    set(reinterpret_cast<const void*>(&sa::pyr_fwd_kernel<128, 128, true>), sa::PyrSmem<128>::kAlloc);
    set(reinterpret_cast<const void*>(&sa::pyr_fwd_kernel<128, 64, true>), sa::PyrSmem<128>::kAlloc);
    set(reinterpret_cast<const void*>(&sa::pyr_fwd_kernel<64, 128, true>), sa::PyrSmem<64>::kAlloc);
    set(reinterpret_cast<const void*>(&sa::pyr_fwd_kernel<64, 64, true>), sa::PyrSmem<64>::kAlloc);
    set(reinterpret_cast<const void*>(&sa::bwd_dkdv_kernel<128, 128>), sa::BwdSmem<128>::kAlloc);
    set(reinterpret_cast<const void*>(&sa::bwd_dkdv_kernel<128, 64>), sa::BwdSmem<128>::kAlloc);
    set(reinterpret_cast<const void*>(&sa::bwd_dkdv_kernel<64, 128>), sa::BwdSmem<64>::kAlloc);
    set(reinterpret_cast<const void*>(&sa::bwd_dkdv_kernel<64, 64>), sa::BwdSmem<64>::kAlloc);
    set(reinterpret_cast<const void*>(&sa::bwd_dq_kernel<128, 128>), sa::BwdSmem<128>::kAlloc);
    set(reinterpret_cast<const void*>(&sa::bwd_dq_kernel<128, 64>), sa::BwdSmem<128>::kAlloc);
    set(reinterpret_cast<const void*>(&sa::bwd_dq_kernel<64, 128>), sa::BwdSmem<64>::kAlloc);
    set(reinterpret_cast<const void*>(&sa::bwd_dq_kernel<64, 64>), sa::BwdSmem<64>::kAlloc);
    set(reinterpret_cast<const void*>(&sa::block_scores_tc_kernel<128>), sa::kScoresTcSmem + 1024);
    set(reinterpret_cast<const void*>(&sa::block_scores_tc_kernel<64>), sa::kScoresTcSmem + 1024);
    set(reinterpret_cast<const void*>(&sa::block_select_kernel),
        static_cast<int>(sa::select_smem_bytes(sa::kMaxSelect)));
    int dev = 0, n_sm = 0;
    if (r == cudaSuccess) r = cudaGetDevice(&dev);
    if (r == cudaSuccess) r = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    if (r == cudaSuccess && n_sm > 0) di.n_sm = n_sm;
    di.err = r;
  });
  return di.err;
}

// SM count of the current device (valid after init_device_kernels succeeded).
int device_sm_count() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 1;
  return g_dev_init[dev].n_sm;
}

// Number of work units, out of `units` launched one CTA each, to run as two
// CTAs each (one per q-tile of the pair).  The attention kernel allocates all
// 512 TMEM columns, so one CTA per SM is active and a launch runs in waves of
// n_sm CTAs.  When the last wave holds no more than half of the SMs, its units
// are split: twice as many CTAs, each with half the rows, finish that wave
// sooner (each still streams all of its K/V tiles, so a full wave is left
// alone).
long long tail_units_to_split(long long units, int n_sm) {
  if (n_sm <= 0) return 0;
  const long long tail = units % n_sm;
  return (tail > 0 && 2 * tail <= n_sm) ? tail : 0;
}

// Launch with programmatic stream serialization (128 threads a CTA): the
// kernel's CTAs may be scheduled, and run their set-up, while the previous
// kernel on the stream is still finishing.  Only the mask builder's scores
// and warp selections are launched this way; each executes
// griddepcontrol.wait, which returns once the previous kernel has completed
// and its writes are visible, before it touches global memory that a kernel
// before it reads or writes.  A kernel lets its dependents start early
// (griddepcontrol.launch_dependents) only after its own wait, or, for the
// block means (an ordinary launch), at its start: each kernel therefore runs
// ahead of its immediate predecessor only, never of a kernel further back.
template <typename... P, typename... A>
cudaError_t launch_pdl(void (*kern)(P...), dim3 grid, int smem, cudaStream_t s, A... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<P>(args)...);
}

bool valid_dim(int d) { return d == 64 || d == 128; }
bool valid_block(int b) { return b == 64 || b == 128; }

// Cumulative level quota ceil(f * nb) for a fraction passed as fp32.  The fp32
// value of a decimal fraction can sit just above it (0.1f = 0.10000000149),
// which would lift an exact product (0.1 * 1000 = 100) past the integer; a
// product within 1e-3 blocks above an integer is taken as that integer.  The
// representation error is below 2^-24 * nb <= 2.5e-4 blocks for nb <= 4096.
int level_quota(float f, int nb) {
  return static_cast<int>(std::ceil(static_cast<double>(f) * nb - 1e-3));
}

// Host-side checks shared by sa_build_mask and sa_build_mask_noalloc (all but
// the workspace).  *empty is set for a call with no rows (nothing to launch).
sa_status check_build_mask_args(const void* q, const void* k, int B, int H, int N, int d, int block, int mode,
                                float tau, const float* level_frac, const uint8_t* mask_out, const float* scores_out,
                                bool* empty) {
  *empty = false;
  if (B < 0 || H < 0 || N < 0) return SA_ERR_INVALID_ARG;
  if (mode != SA_MASK_TAU && mode != SA_MASK_LEVELS && mode != SA_MASK_GLOBAL) return SA_ERR_INVALID_ARG;
  if ((mode == SA_MASK_TAU || mode == SA_MASK_GLOBAL) && !(tau > 0.f && tau <= 1.f)) return SA_ERR_INVALID_ARG;
  if (B == 0 || H == 0 || N == 0) {
    *empty = true;
    return SA_OK;
  }
  if (!valid_dim(d) || !valid_block(block)) return SA_ERR_UNSUPPORTED;
  if (!q || !k || !mask_out) return SA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k)) return SA_ERR_INVALID_ARG;
  if (scores_out && !aligned16(scores_out)) return SA_ERR_INVALID_ARG;   // rows are stored as float4
  if (ceil_div(N, block) > sa::kMaxSelect) return SA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H > 65535) return SA_ERR_UNSUPPORTED;
  if (mode == SA_MASK_LEVELS) {
    if (!level_frac) return SA_ERR_INVALID_ARG;
    float prev = 0.f;
    for (int i = 0; i < 3; ++i) {
      const float f = level_frac[i];
      if (!(f >= prev && f <= 1.f)) return SA_ERR_INVALID_ARG;
      prev = f;
    }
  }
  return SA_OK;
}

}  // namespace

extern "C" {

const char* sa_status_string(sa_status s) {
  switch (s) {
    case SA_OK: return "SA_OK";
    case SA_ERR_INVALID_ARG: return "SA_ERR_INVALID_ARG";
    case SA_ERR_UNSUPPORTED: return "SA_ERR_UNSUPPORTED";
    case SA_ERR_CUDA: return "SA_ERR_CUDA";
    case SA_ERR_TIMEOUT: return "SA_ERR_TIMEOUT";
  }
  return "SA_ERR_UNKNOWN";
}

int sa_version(void) { return 100; }

sa_status sa_get_device_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(as_stream(stream));
  if (e != cudaSuccess) return SA_ERR_CUDA;
  int word = 0;
  e = cudaMemcpyFromSymbol(&word, sa::g_error_word, sizeof(int));
  if (e != cudaSuccess) return SA_ERR_CUDA;
  if (word != 0) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(sa::g_error_word, &zero, sizeof(int));
    if (e != cudaSuccess) return SA_ERR_CUDA;
  }
  if (word & (1 << SA_ERR_TIMEOUT)) return SA_ERR_TIMEOUT;
  return word ? SA_ERR_CUDA : SA_OK;
}

sa_status sa_self_test_timeout(uint64_t wait_ns, void* stream) {
  if (wait_ns == 0 || wait_ns > 1000000000ull) return SA_ERR_INVALID_ARG;
  sa::self_test_timeout_kernel<<<1, 32, 0, as_stream(stream)>>>(static_cast<unsigned long long>(wait_ns));
  return cuda_status(cudaGetLastError());
}

size_t sa_build_mask_workspace(int B, int H, int N, int d, int block) {
  if (B <= 0 || H <= 0 || N <= 0 || d <= 0 || block <= 0) return 0;
  const size_t nb = static_cast<size_t>(ceil_div(N, block));
  const size_t bh = static_cast<size_t>(B) * H;
  return (4 * bh * nb * d + bh * nb * nb) * sizeof(float);
}

sa_status sa_build_mask(const void* q, const void* k, int B, int H, int N, int d, int block, int mode, float tau,
                        const float* level_frac, uint8_t* mask_out, float* scores_out, void* workspace,
                        size_t workspace_bytes, void* stream) {
  bool empty = false;
  const sa_status st =
      check_build_mask_args(q, k, B, H, N, d, block, mode, tau, level_frac, mask_out, scores_out, &empty);
  if (st != SA_OK || empty) return st;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return SA_ERR_INVALID_ARG;
  if (workspace_bytes < sa_build_mask_workspace(B, H, N, d, block)) return SA_ERR_INVALID_ARG;
  const int nb = ceil_div(N, block);
  int c0 = 0, c1 = 0, c2 = 0;
  if (mode == SA_MASK_LEVELS) {
    c0 = level_quota(level_frac[0], nb);
    c1 = level_quota(level_frac[1], nb);
    c2 = level_quota(level_frac[2], nb);
  }
  cudaError_t e = init_device_kernels();
  if (e != cudaSuccess) return SA_ERR_CUDA;
  const int BH = B * H;
  // the block means as tf32 hi / lo parts, then the scores
  const size_t mean_n = static_cast<size_t>(BH) * nb * d;
  float* qmean = static_cast<float*>(workspace);
  float* qlo = qmean + mean_n;
  float* khi = qlo + mean_n;
  float* klo = khi + mean_n;
  float* scores = scores_out ? scores_out : klo + mean_n;
  cudaStream_t s = as_stream(stream);
  const float scale = 1.0f / std::sqrt(static_cast<float>(d));
  const auto* qb = static_cast<const __nv_bfloat16*>(q);
  const auto* kb = static_cast<const __nv_bfloat16*>(k);
  sa::ScoresMaps smaps;
  if (!encode_f32_map(&smaps.qhi, qmean, BH, nb, d, 128) || !encode_f32_map(&smaps.qlo, qlo, BH, nb, d, 128) ||
      !encode_f32_map(&smaps.khi, khi, BH, nb, d, 256) || !encode_f32_map(&smaps.klo, klo, BH, nb, d, 256))
    return SA_ERR_CUDA;
  dim3 g1(nb, BH, 2), g2(ceil_div(nb, 256), ceil_div(nb, 128), BH);
  constexpr int kScoresSmem = sa::kScoresTcSmem + 1024;
  if (d == 128) {
    sa::block_means_kernel<128><<<g1, 128, 0, s>>>(qb, kb, N, block, nb, qmean, qlo, khi, klo);
    e = launch_pdl(sa::block_scores_tc_kernel<128>, g2, kScoresSmem, s, smaps, nb, scale, scores);
  } else {
    sa::block_means_kernel<64><<<g1, 128, 0, s>>>(qb, kb, N, block, nb, qmean, qlo, khi, klo);
    e = launch_pdl(sa::block_scores_tc_kernel<64>, g2, kScoresSmem, s, smaps, nb, scale, scores);
  }
  if (e != cudaSuccess) return SA_ERR_CUDA;
  const long long nrows = static_cast<long long>(BH) * nb;
  const unsigned warp_grid = static_cast<unsigned>((nrows + 3) / 4);
  if (mode == SA_MASK_GLOBAL) {
    // the block means are no longer needed: their space holds the row
    // statistics, then (Nb > 64) the heads' bins and search state
    float2* stats = reinterpret_cast<float2*>(qmean);
    sa::global_row_stats_kernel<<<warp_grid, 128, 0, s>>>(scores, nb, nrows, stats);
    if (nb <= 64) {
      sa::global_select_kernel<<<BH, sa::kGlobalThreads, 0, s>>>(scores, stats, nb, tau, mask_out);
      return cuda_status(cudaGetLastError());
    }
    const size_t stats_bytes = (static_cast<size_t>(BH) * nb * sizeof(float2) + 255) / 256 * 256;
    float* hist = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(qmean) + stats_bytes);
    auto* state = reinterpret_cast<unsigned long long*>(hist + static_cast<size_t>(BH) * 256);
    const int per_head = std::max(1, std::min(64, (148 * 4 + BH - 1) / BH));
    const dim3 gs(per_head, BH);
    sa::global_init_kernel<<<BH, 256, 0, s>>>(hist, state);
    for (int pass = 0; pass < 8; ++pass) {
      sa::global_hist_kernel<<<gs, sa::kGlobalSliceThreads, 0, s>>>(scores, stats, nb, pass, state, hist);
      sa::global_decide_kernel<<<BH, 256, 0, s>>>(hist, state, nb, tau, pass);
    }
    sa::global_mark_kernel<<<gs, sa::kGlobalSliceThreads, 0, s>>>(scores, stats, nb, state, mask_out);
    return cuda_status(cudaGetLastError());
  }
  const float* cscores = scores;
  auto tau_rows = [&](auto kern) {
    return launch_pdl(kern, dim3(warp_grid), 0, s, cscores, nb, nrows, tau, mask_out);
  };
  auto level_rows = [&](auto kern) {
    return launch_pdl(kern, dim3(warp_grid), 0, s, cscores, nb, nrows, c0, c1, c2, mask_out);
  };
  if (mode == SA_MASK_TAU && nb <= 1024) {
    if (nb <= 32)
      e = tau_rows(sa::tau_select_warp_kernel<1>);
    else if (nb <= 64)
      e = tau_rows(sa::tau_select_warp_kernel<2>);
    else if (nb <= 128)
      e = tau_rows(sa::tau_select_warp_kernel<4>);
    else if (nb <= 256)
      e = tau_rows(sa::tau_select_warp_kernel<8>);
    else if (nb <= 512)
      e = tau_rows(sa::tau_select_warp_kernel<16>);
    else
      e = tau_rows(sa::tau_select_warp_kernel<32>);
    return cuda_status(e != cudaSuccess ? e : cudaGetLastError());
  }
  if (nb <= 32)
    e = level_rows(sa::level_select_warp_kernel<1>);
  else if (nb <= 64)
    e = level_rows(sa::level_select_warp_kernel<2>);
  else if (nb <= 128)
    e = level_rows(sa::level_select_warp_kernel<4>);
  else if (nb <= 256)
    e = level_rows(sa::level_select_warp_kernel<8>);
  else if (nb <= 512)
    e = level_rows(sa::level_select_warp_kernel<16>);
  else if (nb <= 1024)
    e = level_rows(sa::level_select_warp_kernel<32>);
  else
    sa::block_select_kernel<<<static_cast<unsigned>(nrows), sa::kSelectThreads, sa::select_smem_bytes(nb), s>>>(
        scores, nb, mode, tau, c0, c1, c2, mask_out);
  return cuda_status(e != cudaSuccess ? e : cudaGetLastError());
}

sa_status sa_radial_mask(int T, int Hh, int Ww, int block, uint8_t* mask_out, void* stream) {
  if (T < 0 || Hh < 0 || Ww < 0 || block <= 0) return SA_ERR_INVALID_ARG;
  const long long N = static_cast<long long>(T) * Hh * Ww;
  if (N == 0) return SA_OK;
  if (!mask_out) return SA_ERR_INVALID_ARG;
  if (N > (1ll << 30)) return SA_ERR_UNSUPPORTED;
  const int nb = ceil_div(N, block);
  const int F = Hh * Ww;
  const int S = ceil_div(F, block);
  sa::radial_mask_kernel<<<nb, 256, 0, as_stream(stream)>>>(nb, F, block, S, mask_out);
  return cuda_status(cudaGetLastError());
}

sa_status sa_pyramid_pool(const void* k, const void* v, int B, int H, int N, int d, int block, void* const* k_pool,
                          void* const* v_pool, void* stream) {
  if (B < 0 || H < 0 || N < 0) return SA_ERR_INVALID_ARG;
  if (B == 0 || H == 0 || N == 0) return SA_OK;
  if (!valid_dim(d) || !valid_block(block)) return SA_ERR_UNSUPPORTED;
  if (!k || !v || !k_pool || !v_pool) return SA_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v)) return SA_ERR_INVALID_ARG;
  for (int i = 0; i < 3; ++i)
    if (!k_pool[i] || !v_pool[i] || !aligned16(k_pool[i]) || !aligned16(v_pool[i])) return SA_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H > 65535) return SA_ERR_UNSUPPORTED;
  const int BH = B * H;
  auto kp = [&](int i) { return static_cast<__nv_bfloat16*>(k_pool[i]); };
  auto vp = [&](int i) { return static_cast<__nv_bfloat16*>(v_pool[i]); };
  const auto* kb = static_cast<const __nv_bfloat16*>(k);
  const auto* vb = static_cast<const __nv_bfloat16*>(v);
  cudaStream_t s = as_stream(stream);
  if (d == 128) {
    dim3 g(ceil_div(N, 8 * 8), BH, 2);
    sa::pyramid_pool_kernel<128><<<g, 128, 0, s>>>(kb, vb, N, kp(0), kp(1), kp(2), vp(0), vp(1), vp(2));
  } else {
    dim3 g(ceil_div(N, 8 * 16), BH, 2);
    sa::pyramid_pool_kernel<64><<<g, 128, 0, s>>>(kb, vb, N, kp(0), kp(1), kp(2), vp(0), vp(1), vp(2));
  }
  return cuda_status(cudaGetLastError());
}

sa_status sa_sparse_attn_fwd(const void* q, const void* k, const void* v, int B, int H, int N, int d, int block,
                             const uint8_t* mask, int64_t mask_sb, int64_t mask_sh, int64_t mask_si,
                             const uint8_t* skip_in, uint8_t* skip_out, float eps, float scale, int order,
                             int causal, void* o, float* lse, void* stream) {
  if (B < 0 || H < 0 || N < 0) return SA_ERR_INVALID_ARG;
  if (order != SA_ORDER_ASCENDING && order != SA_ORDER_RADIAL) return SA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return SA_ERR_INVALID_ARG;
  if (std::isnan(eps) || eps < 0.f) return SA_ERR_INVALID_ARG;
  if (std::isnan(scale) || scale < 0.f || std::isinf(scale)) return SA_ERR_INVALID_ARG;
  if (B == 0 || H == 0 || N == 0) return SA_OK;
  if (!valid_dim(d) || !valid_block(block)) return SA_ERR_UNSUPPORTED;
  if (!q || !k || !v || !o) return SA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return SA_ERR_INVALID_ARG;
  if (mask && (mask_sb < 0 || mask_sh < 0 || mask_si < 0)) return SA_ERR_INVALID_ARG;
  const int n_kv_tiles = ceil_div(N, sa::kTileN);
  if (n_kv_tiles > sa::kMaxKvTiles) return SA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H > 65535) return SA_ERR_UNSUPPORTED;
  cudaError_t e = init_device_kernels();
  if (e != cudaSuccess) return SA_ERR_CUDA;

  const int BH = B * H;
  CUtensorMap tq, tk, tv;
  if (!encode_rows_map(&tq, q, BH, N, d, sa::kTileM) || !encode_rows_map(&tk, k, BH, N, d, sa::kTileN) ||
      !encode_rows_map(&tv, v, BH, N, d, sa::kTileN))
    return SA_ERR_CUDA;

  if (scale == 0.f) scale = 1.0f / std::sqrt(static_cast<float>(d));
  AttnParams p;
  p.B = B;
  p.H = H;
  p.N = N;
  p.nb = ceil_div(N, block);
  p.n_kv_tiles = n_kv_tiles;
  p.mask = mask;
  p.msb = mask_sb;
  p.msh = mask_sh;
  p.msi = mask_si;
  p.skip_in = skip_in;
  p.skip_out = skip_out;
  p.write_skip = skip_out != nullptr;
  p.carry_skip = skip_out != nullptr && skip_out != skip_in;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.eps_raw = std::isinf(eps) ? INFINITY : eps / scale;
  p.radial = order == SA_ORDER_RADIAL;
  p.causal = causal;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;

  const int n_pairs = ceil_div(ceil_div(N, sa::kTileM), 2);
  const long long units = static_cast<long long>(n_pairs) * BH;
  const long long n_split = tail_units_to_split(units, device_sm_count());
  p.n_pairs = n_pairs;
  p.n_full = static_cast<int>(units - n_split);
  dim3 grid(static_cast<unsigned>(units + n_split));
  cudaStream_t s = as_stream(stream);
#define SA_ATTN_LAUNCH(DD, BB, CC) \
  sa::attn_fwd_kernel<DD, BB, CC><<<grid, sa::kAttnThreads, sa::AttnSmem<DD>::kAlloc, s>>>(tq, tk, tv, p)
  if (d == 128 && block == 128)
    causal ? SA_ATTN_LAUNCH(128, 128, true) : SA_ATTN_LAUNCH(128, 128, false);
  else if (d == 128 && block == 64)
    causal ? SA_ATTN_LAUNCH(128, 64, true) : SA_ATTN_LAUNCH(128, 64, false);
  else if (d == 64 && block == 128)
    causal ? SA_ATTN_LAUNCH(64, 128, true) : SA_ATTN_LAUNCH(64, 128, false);
  else
    causal ? SA_ATTN_LAUNCH(64, 64, true) : SA_ATTN_LAUNCH(64, 64, false);
#undef SA_ATTN_LAUNCH
  return cuda_status(cudaGetLastError());
}

sa_status sa_pyramid_attn_fwd(const void* q, const void* k, const void* v, int B, int H, int N, int d, int block,
                              const uint8_t* levels, int64_t lv_sb, int64_t lv_sh, int64_t lv_si,
                              const void* const* k_pool, const void* const* v_pool, float scale, int causal, void* o,
                              float* lse, void* stream) {
  if (B < 0 || H < 0 || N < 0) return SA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return SA_ERR_INVALID_ARG;
  if (std::isnan(scale) || scale < 0.f || std::isinf(scale)) return SA_ERR_INVALID_ARG;
  if (B == 0 || H == 0 || N == 0) return SA_OK;
  if (!valid_dim(d) || !valid_block(block)) return SA_ERR_UNSUPPORTED;
  if (!q || !k || !v || !o || !levels || !k_pool || !v_pool) return SA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return SA_ERR_INVALID_ARG;
  if (lv_sb < 0 || lv_sh < 0 || lv_si < 0) return SA_ERR_INVALID_ARG;
  for (int i = 0; i < 3; ++i)
    if (!k_pool[i] || !v_pool[i] || !aligned16(k_pool[i]) || !aligned16(v_pool[i])) return SA_ERR_INVALID_ARG;
  const int nb = ceil_div(N, block);
  if (nb > sa::kPyrMaxBlocks) return SA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H > 65535) return SA_ERR_UNSUPPORTED;
  cudaError_t e = init_device_kernels();
  if (e != cudaSuccess) return SA_ERR_CUDA;

  const int BH = B * H;
  CUtensorMap tq;
  sa::PyrMaps maps;
  if (!encode_rows_map(&tq, q, BH, N, d, sa::kTileM)) return SA_ERR_CUDA;
  sa::PyrParams p;
  for (int l = 0; l < 4; ++l) {
    const int rows = ceil_div(N, 1 << l);
    const void* kb = l == 0 ? k : k_pool[l - 1];
    const void* vb = l == 0 ? v : v_pool[l - 1];
    // boxes of at most 64 rows: the kernel fills and releases V by 64-key half
    const int box = std::min(block >> l, 64);
    if (!encode_rows_map(&maps.k[l], kb, BH, rows, d, box) || !encode_rows_map(&maps.v[l], vb, BH, rows, d, box))
      return SA_ERR_CUDA;
  }
  if (scale == 0.f) scale = 1.0f / std::sqrt(static_cast<float>(d));
  p.B = B;
  p.H = H;
  p.N = N;
  p.nb = nb;
  p.levels = levels;
  p.lsb = lv_sb;
  p.lsh = lv_sh;
  p.lsi = lv_si;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  const int n_pairs = ceil_div(ceil_div(N, sa::kTileM), 2);
  const long long units = static_cast<long long>(n_pairs) * BH;
  const long long n_split = tail_units_to_split(units, device_sm_count());
  p.n_pairs = n_pairs;
  p.n_full = static_cast<int>(units - n_split);
  dim3 grid(static_cast<unsigned>(units + n_split));
  cudaStream_t s = as_stream(stream);
#define SA_PYR_LAUNCH(DD, BB, CC) \
  sa::pyr_fwd_kernel<DD, BB, CC><<<grid, sa::kPyrThreads, sa::PyrSmem<DD>::kAlloc, s>>>(tq, maps, p)
  if (d == 128 && block == 128)
    causal ? SA_PYR_LAUNCH(128, 128, true) : SA_PYR_LAUNCH(128, 128, false);
  else if (d == 128 && block == 64)
    causal ? SA_PYR_LAUNCH(128, 64, true) : SA_PYR_LAUNCH(128, 64, false);
  else if (d == 64 && block == 128)
    causal ? SA_PYR_LAUNCH(64, 128, true) : SA_PYR_LAUNCH(64, 128, false);
  else
    causal ? SA_PYR_LAUNCH(64, 64, true) : SA_PYR_LAUNCH(64, 64, false);
#undef SA_PYR_LAUNCH
  return cuda_status(cudaGetLastError());
}

}  // extern "C"

// ===========================================================================
// sa_build_mask_noalloc: sa_build_mask for callers that must not allocate.
//
// Some callers cannot call cudaMalloc at the moment they need a mask:
//   - serving runtimes that reserve all device memory up front in their own
//     pool and do not let a library allocate behind their back (a cudaMalloc
//     there fails, or takes memory the pool has promised elsewhere);
//   - latency-critical denoising loops: cudaMalloc and cudaFree can
//     synchronise the device, which stalls every stream of the process.
// For them this variant takes its scratch (block means and block scores, or
// the global selection's row statistics, histograms and search state) from
// one file-scope device array instead of a caller-provided workspace.  The
// array exists on every GPU that loads the library's device code and stays
// allocated there until the process exits.
//
// Everything that runs on the GPU is the same as in sa_build_mask: this entry
// point checks the arguments, looks up the array's device address and then
// calls sa_build_mask with it as the workspace.
// ===========================================================================
namespace {

// Upper bound of the shared scratch: large enough for the 480p workload
// (12 heads, 32,760 tokens, block 64, d 128 needs 25.2 MB).
constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(32) << 20;  // 32 MiB

}  // namespace

static __device__ __align__(256) unsigned char g_build_mask_scratch[kNoAllocScratchBytes];

namespace {

std::mutex g_scratch_mutex;
void* g_scratch_address[kMaxDevices] = {};

// Device address of g_build_mask_scratch on the current device.  In host code
// the array's name is only a host-side stand-in, so the address has to be
// asked from the runtime, with the device current.  Only a successful lookup
// is kept: a lookup that failed (no context yet, a capture in progress) is
// tried again on the next call.
cudaError_t build_mask_scratch(void** out) {
  *out = nullptr;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_address[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_build_mask_scratch);
    if (e != cudaSuccess) {
      cudaGetLastError();  // reset the last-error state: a later launch check must not see this failure
      return e;
    }
    g_scratch_address[dev] = p;
  }
  *out = g_scratch_address[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" sa_status sa_build_mask_noalloc(const void* q, const void* k, int B, int H, int N, int d, int block,
                                           int mode, float tau, const float* level_frac, uint8_t* mask_out,
                                           float* scores_out, void* stream) {
  bool empty = false;
  const sa_status st =
      check_build_mask_args(q, k, B, H, N, d, block, mode, tau, level_frac, mask_out, scores_out, &empty);
  if (st != SA_OK || empty) return st;
  if (sa_build_mask_workspace(B, H, N, d, block) > kNoAllocScratchBytes) return SA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if (build_mask_scratch(&scratch) != cudaSuccess || scratch == nullptr) return SA_ERR_CUDA;
  return sa_build_mask(q, k, B, H, N, d, block, mode, tau, level_frac, mask_out, scores_out, scratch,
                       kNoAllocScratchBytes, stream);
}

// -------------------------------------------------------- backward pass ---
extern "C" {

size_t sa_sparse_attn_bwd_workspace(int B, int H, int N) {
  if (B <= 0 || H <= 0 || N <= 0) return 0;
  return static_cast<size_t>(B) * H * N * sizeof(float);
}

sa_status sa_sparse_attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                             const float* lse, int B, int H, int N, int d, int block, const uint8_t* mask,
                             int64_t mask_sb, int64_t mask_sh, int64_t mask_si, float scale, int causal, void* dq,
                             void* dk, void* dv, void* workspace, size_t workspace_bytes, void* stream) {
  if (B < 0 || H < 0 || N < 0) return SA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return SA_ERR_INVALID_ARG;
  if (std::isnan(scale) || scale < 0.f || std::isinf(scale)) return SA_ERR_INVALID_ARG;
  if (B == 0 || H == 0 || N == 0) return SA_OK;
  if (!valid_dim(d) || !valid_block(block)) return SA_ERR_UNSUPPORTED;
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv || !workspace) return SA_ERR_INVALID_ARG;
  for (const void* ptr : {q, k, v, o, dout, static_cast<const void*>(dq), static_cast<const void*>(dk),
                          static_cast<const void*>(dv), static_cast<const void*>(workspace)})
    if (!aligned16(ptr)) return SA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(lse) & 3u) != 0) return SA_ERR_INVALID_ARG;
  if (workspace_bytes < sa_sparse_attn_bwd_workspace(B, H, N)) return SA_ERR_INVALID_ARG;
  if (mask && (mask_sb < 0 || mask_sh < 0 || mask_si < 0)) return SA_ERR_INVALID_ARG;
  const int n_tiles = ceil_div(N, sa::kTileN);
  if (n_tiles > sa::kMaxKvTiles) return SA_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H > 65535) return SA_ERR_UNSUPPORTED;
  cudaError_t e = init_device_kernels();
  if (e != cudaSuccess) return SA_ERR_CUDA;

  const int BH = B * H;
  CUtensorMap tq, tk, tv, tdo;
  if (!encode_rows_map(&tq, q, BH, N, d, sa::kTileM) || !encode_rows_map(&tk, k, BH, N, d, sa::kTileN) ||
      !encode_rows_map(&tv, v, BH, N, d, sa::kTileN) || !encode_rows_map(&tdo, dout, BH, N, d, sa::kTileM))
    return SA_ERR_CUDA;

  if (scale == 0.f) scale = 1.0f / std::sqrt(static_cast<float>(d));
  float* delta = static_cast<float*>(workspace);
  sa::BwdParams p;
  p.B = B;
  p.H = H;
  p.N = N;
  p.nb = ceil_div(N, block);
  p.n_tiles = n_tiles;
  p.mask = mask;
  p.msb = mask_sb;
  p.msh = mask_sh;
  p.msi = mask_si;
  p.lse = lse;
  p.delta = delta;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.causal = causal;
  p.dq = static_cast<__nv_bfloat16*>(dq);
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);

  cudaStream_t s = as_stream(stream);
  const long long rows = static_cast<long long>(BH) * N;
  const int rows_per_block = 256 / (d / 8);
  const int grid_d = static_cast<int>(std::min<long long>((rows + rows_per_block - 1) / rows_per_block, 148LL * 16));
  const __nv_bfloat16* ob = static_cast<const __nv_bfloat16*>(o);
  const __nv_bfloat16* gb = static_cast<const __nv_bfloat16*>(dout);
  if (d == 128)
    sa::bwd_delta_kernel<128><<<grid_d, 256, 0, s>>>(ob, gb, delta, rows);
  else
    sa::bwd_delta_kernel<64><<<grid_d, 256, 0, s>>>(ob, gb, delta, rows);
  e = cudaGetLastError();
  if (e != cudaSuccess) return SA_ERR_CUDA;

  const dim3 grid(n_tiles, BH);
  if (d == 128 && block == 128) {
    sa::bwd_dkdv_kernel<128, 128><<<grid, sa::kBwdThreads, sa::BwdSmem<128>::kAlloc, s>>>(tq, tk, tv, tdo, p);
    sa::bwd_dq_kernel<128, 128><<<grid, sa::kBwdThreads, sa::BwdSmem<128>::kAlloc, s>>>(tq, tk, tv, tdo, p);
  } else if (d == 128) {
    sa::bwd_dkdv_kernel<128, 64><<<grid, sa::kBwdThreads, sa::BwdSmem<128>::kAlloc, s>>>(tq, tk, tv, tdo, p);
    sa::bwd_dq_kernel<128, 64><<<grid, sa::kBwdThreads, sa::BwdSmem<128>::kAlloc, s>>>(tq, tk, tv, tdo, p);
  } else if (block == 128) {
    sa::bwd_dkdv_kernel<64, 128><<<grid, sa::kBwdThreads, sa::BwdSmem<64>::kAlloc, s>>>(tq, tk, tv, tdo, p);
    sa::bwd_dq_kernel<64, 128><<<grid, sa::kBwdThreads, sa::BwdSmem<64>::kAlloc, s>>>(tq, tk, tv, tdo, p);
  } else {
    sa::bwd_dkdv_kernel<64, 64><<<grid, sa::kBwdThreads, sa::BwdSmem<64>::kAlloc, s>>>(tq, tk, tv, tdo, p);
    sa::bwd_dq_kernel<64, 64><<<grid, sa::kBwdThreads, sa::BwdSmem<64>::kAlloc, s>>>(tq, tk, tv, tdo, p);
  }
  return cuda_status(cudaGetLastError());
}

}  // extern "C"

// ----------------------------------------------------- token permutation ---
extern "C" {

sa_status sa_token_permute(const void* const* src, void* const* dst, int n_tensors, int B, int H, int T, int Hh,
                           int Ww, int d, int order, const uint8_t* head_order, int ct, int ch, int cw, int inverse,
                           void* stream) {
  if (n_tensors < 1 || n_tensors > sa::kPermMaxTensors || !src || !dst) return SA_ERR_INVALID_ARG;
  if (B < 0 || H < 0 || T < 0 || Hh < 0 || Ww < 0) return SA_ERR_INVALID_ARG;
  if (order < 0 || order > 5 || (inverse != 0 && inverse != 1)) return SA_ERR_INVALID_ARG;
  if (ct < 1 || ch < 1 || cw < 1) return SA_ERR_INVALID_ARG;
  const long long N = static_cast<long long>(T) * Hh * Ww;
  if (B == 0 || H == 0 || N == 0) return SA_OK;
  if (T % ct || Hh % ch || Ww % cw) return SA_ERR_INVALID_ARG;
  if (N > (1LL << 30)) return SA_ERR_UNSUPPORTED;
  if (!valid_dim(d)) return SA_ERR_UNSUPPORTED;
  sa::PermParams p;
  for (int i = 0; i < n_tensors; ++i) {
    if (!src[i] || !dst[i] || !aligned16(src[i]) || !aligned16(dst[i]) || src[i] == dst[i]) return SA_ERR_INVALID_ARG;
    p.src[i] = static_cast<const __nv_bfloat16*>(src[i]);
    p.dst[i] = static_cast<__nv_bfloat16*>(dst[i]);
  }
  for (int i = n_tensors; i < sa::kPermMaxTensors; ++i) {
    p.src[i] = nullptr;
    p.dst[i] = nullptr;
  }
  p.n_tensors = n_tensors;
  p.H = H;
  p.N = static_cast<int>(N);
  p.g[0] = T;
  p.g[1] = Hh;
  p.g[2] = Ww;
  p.c[0] = ct;
  p.c[1] = ch;
  p.c[2] = cw;
  p.order = order;
  p.head_order = head_order;
  p.inverse = inverse;
  if (static_cast<long long>(B) * H > 65535) return SA_ERR_UNSUPPORTED;
  const dim3 grid(static_cast<unsigned>((N + 255) / 256), static_cast<unsigned>(B * H), static_cast<unsigned>(n_tensors));
  cudaStream_t s = as_stream(stream);
  if (d == 128)
    sa::token_permute_kernel<128><<<grid, 256, 0, s>>>(p);
  else
    sa::token_permute_kernel<64><<<grid, 256, 0, s>>>(p);
  return cuda_status(cudaGetLastError());
}

}  // extern "C"

// ------------------------------------------- forward from host buffers ---
// Q, K, V come from host memory and O goes back to it: the (b, h) rows are
// streamed through the device in chunks of `heads_per_chunk` heads, two chunk
// buffers in turn, so that the copy of chunk c + 1 in, the attention of chunk
// c and the copy of chunk c - 1 out run at the same time (host-to-device and
// device-to-host on two streams of their own, the attention on the caller's
// stream).  One cudaMemcpyAsync per tensor and chunk.
namespace {

size_t host_chunk_elems(int N, int d, int hc) { return static_cast<size_t>(hc) * N * d; }

}  // namespace

extern "C" {

size_t sa_sparse_attn_fwd_host_workspace(int N, int d, int heads_per_chunk) {
  if (N <= 0 || d <= 0 || heads_per_chunk <= 0) return 0;
  return 2 * 4 * host_chunk_elems(N, d, heads_per_chunk) * 2;   // 2 buffers x (Q, K, V, O) x bf16
}

sa_status sa_sparse_attn_fwd_host(const void* q, const void* k, const void* v, int B, int H, int N, int d,
                                  int block, const uint8_t* mask, int64_t mask_sb, int64_t mask_sh,
                                  int64_t mask_si, const uint8_t* skip_in, uint8_t* skip_out, float eps,
                                  float scale, int order, int causal, void* o, float* lse, void* workspace,
                                  size_t workspace_bytes, int heads_per_chunk, void* stream) {
  if (B < 0 || H < 0 || N < 0 || heads_per_chunk <= 0) return SA_ERR_INVALID_ARG;
  if (B == 0 || H == 0 || N == 0) return SA_OK;
  if (!q || !k || !v || !o || !workspace) return SA_ERR_INVALID_ARG;
  if (!valid_dim(d) || !valid_block(block)) return SA_ERR_UNSUPPORTED;
  const int hc = std::min(heads_per_chunk, H);
  if (workspace_bytes < sa_sparse_attn_fwd_host_workspace(N, d, hc)) return SA_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return SA_ERR_INVALID_ARG;
  const size_t ce = host_chunk_elems(N, d, hc);
  auto* ws = static_cast<__nv_bfloat16*>(workspace);
  __nv_bfloat16* buf[2][4];
  for (int s = 0; s < 2; ++s)
    for (int t = 0; t < 4; ++t) buf[s][t] = ws + (static_cast<size_t>(s) * 4 + t) * ce;
  const auto* hq = static_cast<const __nv_bfloat16*>(q);
  const auto* hk = static_cast<const __nv_bfloat16*>(k);
  const auto* hv = static_cast<const __nv_bfloat16*>(v);
  auto* ho = static_cast<__nv_bfloat16*>(o);
  const size_t nb = static_cast<size_t>(ceil_div(N, block));
  const size_t head_elems = static_cast<size_t>(N) * d;

  cudaStream_t cs = as_stream(stream);
  cudaStream_t in_s = nullptr, out_s = nullptr;
  cudaEvent_t loaded[2] = {nullptr, nullptr}, computed[2] = {nullptr, nullptr}, stored[2] = {nullptr, nullptr};
  sa_status st = SA_OK;
  auto ok = [&](cudaError_t e) {
    if (e != cudaSuccess && st == SA_OK) st = SA_ERR_CUDA;
    return st == SA_OK;
  };
  ok(cudaStreamCreateWithFlags(&in_s, cudaStreamNonBlocking));
  ok(cudaStreamCreateWithFlags(&out_s, cudaStreamNonBlocking));
  for (int s = 0; s < 2 && st == SA_OK; ++s) {
    ok(cudaEventCreateWithFlags(&loaded[s], cudaEventDisableTiming));
    ok(cudaEventCreateWithFlags(&computed[s], cudaEventDisableTiming));
    ok(cudaEventCreateWithFlags(&stored[s], cudaEventDisableTiming));
  }
  // the copies in must not overtake work the caller queued on its stream before this call
  cudaEvent_t start = nullptr;
  if (ok(cudaEventCreateWithFlags(&start, cudaEventDisableTiming)) && ok(cudaEventRecord(start, cs)))
    ok(cudaStreamWaitEvent(in_s, start, 0));
  int chunk = 0;
  for (int b = 0; b < B && st == SA_OK; ++b) {
    for (int h0 = 0; h0 < H && st == SA_OK; h0 += hc, ++chunk) {
      const int nh = std::min(hc, H - h0);
      const int s = chunk & 1;
      const size_t off = (static_cast<size_t>(b) * H + h0) * head_elems;
      const size_t bytes = static_cast<size_t>(nh) * head_elems * 2;
      // buffer s was last read by chunk - 2's attention and its O copied out
      if (chunk >= 2) {
        ok(cudaStreamWaitEvent(in_s, computed[s], 0));
      }
      ok(cudaMemcpyAsync(buf[s][0], hq + off, bytes, cudaMemcpyHostToDevice, in_s));
      ok(cudaMemcpyAsync(buf[s][1], hk + off, bytes, cudaMemcpyHostToDevice, in_s));
      ok(cudaMemcpyAsync(buf[s][2], hv + off, bytes, cudaMemcpyHostToDevice, in_s));
      ok(cudaEventRecord(loaded[s], in_s));
      ok(cudaStreamWaitEvent(cs, loaded[s], 0));
      if (chunk >= 2) ok(cudaStreamWaitEvent(cs, stored[s], 0));
      if (st != SA_OK) break;
      const uint8_t* mk = mask ? mask + b * mask_sb + static_cast<int64_t>(h0) * mask_sh : nullptr;
      const size_t so = (static_cast<size_t>(b) * H + h0) * nb * nb;
      const sa_status a = sa_sparse_attn_fwd(buf[s][0], buf[s][1], buf[s][2], 1, nh, N, d, block, mk, 0, mask_sh,
                                             mask_si, skip_in ? skip_in + so : nullptr,
                                             skip_out ? skip_out + so : nullptr, eps, scale, order, causal,
                                             buf[s][3], lse ? lse + (static_cast<size_t>(b) * H + h0) * N : nullptr,
                                             stream);
      if (a != SA_OK) {
        st = a;
        break;
      }
      ok(cudaEventRecord(computed[s], cs));
      ok(cudaStreamWaitEvent(out_s, computed[s], 0));
      ok(cudaMemcpyAsync(ho + off, buf[s][3], bytes, cudaMemcpyDeviceToHost, out_s));
      ok(cudaEventRecord(stored[s], out_s));
    }
  }
  // the caller's stream sees every copy out before anything it queues next
  for (int s = 0; s < 2; ++s)
    if (stored[s]) cudaStreamWaitEvent(cs, stored[s], 0);
  for (int s = 0; s < 2; ++s) {
    if (loaded[s]) cudaEventDestroy(loaded[s]);
    if (computed[s]) cudaEventDestroy(computed[s]);
    if (stored[s]) cudaEventDestroy(stored[s]);
  }
  if (start) cudaEventDestroy(start);
  if (in_s) cudaStreamDestroy(in_s);
  if (out_s) cudaStreamDestroy(out_s);
  return st;
}

}  // extern "C"
