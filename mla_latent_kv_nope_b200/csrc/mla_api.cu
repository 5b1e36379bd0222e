// C ABI of the MLA decode library: argument validation, workspace layout and
// kernel launches.  Every check runs before anything is enqueued; no entry
// point allocates, frees or synchronises (except mla_get_device_status).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "../../include/mla.h"
#include "common.cuh"
#include "kernels.h"

namespace mla {

// Per-device status word (one copy per device that loads the library).
__device__ int g_status = MLA_OK;

namespace {

// Device address of g_status for the current device, looked up once per
// device.  Host code may not take the address of a __device__ symbol
// directly; the runtime lookup gives the real device pointer.
int* status_ptr() {
  static int* cache[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (!cache[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return nullptr;
    cache[dev] = static_cast<int*>(p);
  }
  return cache[dev];
}

constexpr int kMaxSplits = 1024;

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

int check_dims(const mla_dims* d) {
  if (!d) return MLA_ERR_INVALID_ARG;
  if (d->B <= 0 || d->H <= 0 || d->d_c <= 0 || d->d_r < 0 || d->d_nope <= 0 || d->d_v <= 0 ||
      d->cache_capacity <= 0)
    return MLA_ERR_INVALID_ARG;
  if (d->B > 65535 || d->H > 65535) return MLA_ERR_UNSUPPORTED;
  if (d->dtype == MLA_BF16) {
    if (d->d_c % 8 || d->d_r % 8 || d->d_nope % 8 || d->d_v % 8) return MLA_ERR_UNSUPPORTED;
  } else if (d->dtype == MLA_F32) {
    if (d->d_c % 4 || d->d_r % 2 || d->d_nope % 4 || d->d_v % 4) return MLA_ERR_UNSUPPORTED;
  } else {
    return MLA_ERR_INVALID_ARG;
  }
  if (d->d_c > 1024 || d->d_r > 256 || d->d_nope > 1024 || d->d_v > 1024)
    return MLA_ERR_UNSUPPORTED;
  return MLA_OK;
}

inline bool decode_uses_tc(const mla_dims* d) { return d->dtype == MLA_BF16; }

// Cycles of the test-only wait injected into the tensor-core decode (0 = none).
uint64_t g_inject_wait_cycles = 0;

cudaError_t launch_decode_any(const mla_dims* d, const void* q_cat, const void* cache,
                              const PageMap& pm, const int32_t* seqlens, float scale, int W,
                              float* o_part, float* lse_part, int* status, cudaStream_t s) {
  if (decode_uses_tc(d))
    return launch_decode_tc(static_cast<const __nv_bfloat16*>(q_cat),
                            static_cast<const __nv_bfloat16*>(cache), pm, seqlens, d->B, d->H,
                            d->cache_capacity, d->d_r, scale, W, o_part, lse_part, status,
                            g_inject_wait_cycles, s);
  return launch_decode_simt<float>(static_cast<const float*>(q_cat),
                                   static_cast<const float*>(cache), pm, seqlens, d->B, d->H,
                                   d->d_c, d->d_r, d->cache_capacity, scale, W, o_part, lse_part,
                                   status, s);
}

PageMap contiguous_map(const mla_dims* d) { return PageMap{nullptr, 0, 0, d->cache_capacity}; }

// Checks of a page table argument: capacity covered by max_blocks pages.
int check_pages(const mla_dims* d, int64_t num_pages, const int32_t* block_table,
                int32_t max_blocks) {
  if (!block_table || num_pages <= 0 || max_blocks <= 0) return MLA_ERR_INVALID_ARG;
  if (d->cache_capacity > int64_t(max_blocks) * kTileKeys) return MLA_ERR_INVALID_ARG;
  if (num_pages * kTileKeys >= (int64_t(1) << 31)) return MLA_ERR_UNSUPPORTED;
  if (!aligned16(block_table)) return MLA_ERR_ALIGNMENT;
  return MLA_OK;
}

// Shapes the decode kernels take.  The tensor-core path addresses cache rows
// with a 32-bit TMA coordinate, so a contiguous cache of 2^31 rows or more
// (B * capacity) is refused here rather than failing at launch.
int decode_shape_supported(const mla_dims* d, bool contiguous) {
  if (d->dtype == MLA_BF16 && (d->d_c != 512 || (d->d_r != 64 && d->d_r != 0)))
    return MLA_ERR_UNSUPPORTED;
  if (d->dtype == MLA_BF16 && contiguous &&
      int64_t(d->B) * d->cache_capacity >= (int64_t(1) << 31))
    return MLA_ERR_UNSUPPORTED;
  return MLA_OK;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

struct WsLayout {
  size_t o_off, lse_off, total;
};

WsLayout ws_layout(const mla_dims* d, int W) {
  const size_t slots = size_t(d->B) + size_t(W) - 1;
  WsLayout l;
  l.o_off = 0;
  l.lse_off = round_up(slots * size_t(d->H) * size_t(d->d_c) * sizeof(float), 256);
  l.total = l.lse_off + round_up(slots * size_t(d->H) * sizeof(float), 256);
  return l;
}

inline int cuda_status(cudaError_t e) { return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA; }

// softmax_scale = 0 selects the pages' scale 1/sqrt(d_h + d_h^R) ([MLA-とは]
// "Decoupled RoPE"): the query/key width per head is d_nope + d_r.
inline float effective_scale(const mla_dims* d, float softmax_scale) {
  return softmax_scale == 0.f ? float(1.0 / sqrt(double(d->d_nope + d->d_r))) : softmax_scale;
}

}  // namespace
}  // namespace mla

using namespace mla;

extern "C" {

int64_t mla_cache_row_elems(int32_t d_c, int32_t d_r) { return int64_t(d_c) + int64_t(d_r); }

const char* mla_status_string(int s) {
  switch (s) {
    case MLA_OK: return "ok";
    case MLA_ERR_INVALID_ARG: return "invalid argument";
    case MLA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case MLA_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case MLA_ERR_WORKSPACE: return "workspace missing or too small";
    case MLA_ERR_CUDA: return "CUDA error";
    case MLA_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case MLA_ERR_BOUNDS: return "device-side bounds check failed";
    default: return "unknown status";
  }
}

int mla_get_device_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MLA_ERR_CUDA;
  int v = MLA_OK;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return MLA_ERR_CUDA;
  const int zero = MLA_OK;
  if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return MLA_ERR_CUDA;
  return v;
}

int mla_debug_inject_wait(uint64_t cycles) {
  g_inject_wait_cycles = cycles;
  return MLA_OK;
}

// ---------------------------------------------------------------------------
namespace {
bool use_tc_gemm(const mla_dims* d) {
  return d->dtype == MLA_BF16 && gemm_tc_supported(d->d_c, d->d_r, d->d_nope, d->d_v);
}
}  // namespace

size_t mla_cache_append_workspace_bytes(const mla_dims* d, int32_t hidden) {
  if (check_dims(d) != MLA_OK || hidden <= 0) return 0;
  const size_t parts = use_tc_gemm(d) ? size_t(append_tc_splits(hidden)) : 1;
  return round_up(parts * size_t(d->B) * size_t(d->d_c + d->d_r) * sizeof(float), 256);
}

namespace {
int cache_append_impl(const mla_dims* d, int32_t hidden, const void* h, const void* W_DKV,
                      const float* gamma, float eps, float rope_base, void* cache,
                      const PageMap& pm, int32_t* seqlens, void* workspace,
                      size_t workspace_bytes, void* stream) {
  int st = check_dims(d);
  if (st) return st;
  if (hidden <= 0 || !h || !W_DKV || !cache || !seqlens) return MLA_ERR_INVALID_ARG;
  if (!(eps >= 0.f) || !(rope_base > 0.f)) return MLA_ERR_INVALID_ARG;
  if (d->dtype == MLA_BF16 ? (hidden % 8) : (hidden % 4)) return MLA_ERR_UNSUPPORTED;
  if (!aligned16(h) || !aligned16(W_DKV) || !aligned16(cache) || !aligned16(seqlens) ||
      (gamma && !aligned16(gamma)) || (workspace && !aligned16(workspace)))
    return MLA_ERR_ALIGNMENT;
  if (!workspace || workspace_bytes < mla_cache_append_workspace_bytes(d, hidden))
    return MLA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* x = static_cast<float*>(workspace);
  if (use_tc_gemm(d)) {
    cudaError_t e = launch_append_proj_tc(static_cast<const __nv_bfloat16*>(h),
                                          static_cast<const __nv_bfloat16*>(W_DKV), d->B,
                                          d->d_c + d->d_r, hidden, x, status_ptr(), s);
    if (e != cudaSuccess) return MLA_ERR_CUDA;
    return cuda_status(launch_append_finalize<__nv_bfloat16>(
        x, append_tc_splits(hidden), gamma, eps, rope_base, d->B, d->d_c, d->d_r,
        d->cache_capacity, static_cast<__nv_bfloat16*>(cache), pm, seqlens, status_ptr(), s));
  }
  if (d->dtype == MLA_BF16)
    return cuda_status(launch_cache_append<__nv_bfloat16>(
        static_cast<const __nv_bfloat16*>(h), static_cast<const __nv_bfloat16*>(W_DKV), gamma,
        eps, rope_base, d->B, d->d_c, d->d_r, hidden, d->cache_capacity,
        static_cast<__nv_bfloat16*>(cache), pm, seqlens, x, status_ptr(), s));
  return cuda_status(launch_cache_append<float>(
      static_cast<const float*>(h), static_cast<const float*>(W_DKV), gamma, eps, rope_base,
      d->B, d->d_c, d->d_r, hidden, d->cache_capacity, static_cast<float*>(cache), pm, seqlens,
      x, status_ptr(), s));
}

int decode_impl(const mla_dims* d, const void* q_cat, const void* cache, const PageMap& pm,
                const int32_t* seqlens, float softmax_scale, int num_splits, void* workspace,
                size_t workspace_bytes, int* splits_used, void* stream);
}  // namespace

int mla_cache_append(const mla_dims* d, int32_t hidden, const void* h, const void* W_DKV,
                     const float* gamma, float eps, float rope_base, void* cache,
                     int32_t* seqlens, void* workspace, size_t workspace_bytes, void* stream) {
  if (check_dims(d)) return check_dims(d);
  return cache_append_impl(d, hidden, h, W_DKV, gamma, eps, rope_base, cache, contiguous_map(d),
                           seqlens, workspace, workspace_bytes, stream);
}

int mla_cache_append_paged(const mla_dims* d, int32_t hidden, const void* h, const void* W_DKV,
                           const float* gamma, float eps, float rope_base, void* cache_pool,
                           int64_t num_pages, const int32_t* block_table, int32_t max_blocks,
                           int32_t* seqlens, void* workspace, size_t workspace_bytes,
                           void* stream) {
  int st = check_dims(d);
  if (st) return st;
  if ((st = check_pages(d, num_pages, block_table, max_blocks))) return st;
  return cache_append_impl(d, hidden, h, W_DKV, gamma, eps, rope_base, cache_pool,
                           PageMap{block_table, max_blocks, num_pages, d->cache_capacity}, seqlens,
                           workspace, workspace_bytes, stream);
}

// ---------------------------------------------------------------------------
int mla_absorb_q(const mla_dims* d, const void* q_nope, const void* q_pe, const void* W_UK,
                 const int32_t* q_pos, float rope_base, void* q_cat, void* stream) {
  int st = check_dims(d);
  if (st) return st;
  if (!q_nope || (d->d_r && !q_pe) || !W_UK || !q_cat) return MLA_ERR_INVALID_ARG;
  if (q_pos && !(rope_base > 0.f)) return MLA_ERR_INVALID_ARG;
  if (!aligned16(q_nope) || (q_pe && !aligned16(q_pe)) || !aligned16(W_UK) ||
      !aligned16(q_cat) || (q_pos && !aligned16(q_pos)))
    return MLA_ERR_ALIGNMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (use_tc_gemm(d))
    return cuda_status(launch_absorb_q_tc(
        static_cast<const __nv_bfloat16*>(q_nope), static_cast<const __nv_bfloat16*>(q_pe),
        static_cast<const __nv_bfloat16*>(W_UK), q_pos, rope_base, d->B, d->H, d->d_r,
        static_cast<__nv_bfloat16*>(q_cat), status_ptr(), s));
  if (d->dtype == MLA_BF16)
    return cuda_status(launch_absorb_q<__nv_bfloat16>(
        static_cast<const __nv_bfloat16*>(q_nope), static_cast<const __nv_bfloat16*>(q_pe),
        static_cast<const __nv_bfloat16*>(W_UK), q_pos, rope_base, d->B, d->H, d->d_c, d->d_r,
        d->d_nope, static_cast<__nv_bfloat16*>(q_cat), s));
  return cuda_status(launch_absorb_q<float>(
      static_cast<const float*>(q_nope), static_cast<const float*>(q_pe),
      static_cast<const float*>(W_UK), q_pos, rope_base, d->B, d->H, d->d_c, d->d_r, d->d_nope,
      static_cast<float*>(q_cat), s));
}

// ---------------------------------------------------------------------------
int mla_decode_default_splits(const mla_dims* d) {
  if (check_dims(d) != MLA_OK) return 0;
  const int sms = sm_count();
  if (sms <= 0) return 0;
  int W;
  if (decode_uses_tc(d)) {
    W = sms / decode_tc_head_groups(d->H);
  } else {
    const int groups = (d->H + 7) / 8;
    W = (2 * sms + groups - 1) / groups;
  }
  if (W < 1) W = 1;
  if (W > kMaxSplits) W = kMaxSplits;
  return W;
}

size_t mla_decode_workspace_bytes(const mla_dims* d, int num_splits) {
  if (check_dims(d) != MLA_OK) return 0;
  const int W = num_splits > 0 ? num_splits : mla_decode_default_splits(d);
  if (W <= 0 || W > kMaxSplits) return 0;
  return ws_layout(d, W).total;
}

namespace {
int decode_impl(const mla_dims* d, const void* q_cat, const void* cache, const PageMap& pm,
                const int32_t* seqlens, float softmax_scale, int num_splits, void* workspace,
                size_t workspace_bytes, int* splits_used, void* stream) {
  int st = check_dims(d);
  if (st) return st;
  if ((st = decode_shape_supported(d, pm.table == nullptr))) return st;
  if (!q_cat || !cache || !seqlens || num_splits < 0 || num_splits > kMaxSplits ||
      !(softmax_scale >= 0.f) || softmax_scale == INFINITY)
    return MLA_ERR_INVALID_ARG;
  softmax_scale = effective_scale(d, softmax_scale);
  if (!aligned16(q_cat) || !aligned16(cache) || !aligned16(seqlens) ||
      (workspace && !aligned16(workspace)))
    return MLA_ERR_ALIGNMENT;
  const int W = num_splits > 0 ? num_splits : mla_decode_default_splits(d);
  if (W <= 0) return MLA_ERR_CUDA;
  const WsLayout l = ws_layout(d, W);
  if (!workspace || workspace_bytes < l.total) return MLA_ERR_WORKSPACE;
  if (splits_used) *splits_used = W;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* o_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + l.o_off);
  float* lse_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + l.lse_off);
  return cuda_status(launch_decode_any(d, q_cat, cache, pm, seqlens, softmax_scale, W, o_part,
                                       lse_part, status_ptr(), s));
}
}  // namespace

int mla_decode(const mla_dims* d, const void* q_cat, const void* cache, const int32_t* seqlens,
               float softmax_scale, int num_splits, void* workspace, size_t workspace_bytes,
               int* splits_used, void* stream) {
  if (check_dims(d)) return check_dims(d);
  return decode_impl(d, q_cat, cache, contiguous_map(d), seqlens, softmax_scale, num_splits,
                     workspace, workspace_bytes, splits_used, stream);
}

int mla_decode_paged(const mla_dims* d, const void* q_cat, const void* cache_pool,
                     int64_t num_pages, const int32_t* block_table, int32_t max_blocks,
                     const int32_t* seqlens, float softmax_scale, int num_splits,
                     void* workspace, size_t workspace_bytes, int* splits_used, void* stream) {
  int st = check_dims(d);
  if (st) return st;
  if ((st = check_pages(d, num_pages, block_table, max_blocks))) return st;
  return decode_impl(d, q_cat, cache_pool,
                     PageMap{block_table, max_blocks, num_pages, d->cache_capacity}, seqlens,
                     softmax_scale, num_splits, workspace, workspace_bytes, splits_used, stream);
}

// ---------------------------------------------------------------------------
// FP8 latent cache: rows [d_c E4M3 codes || d_r bf16 RoPE keys] plus one fp32
// power-of-two scale per row (shape 512 / 64, bf16 weights and queries).
namespace {
bool fp8_shape(const mla_dims* d) {
  return d->dtype == MLA_BF16 && gemm_tc_supported(d->d_c, d->d_r, d->d_nope, d->d_v) &&
         d->d_r == 64;
}
}  // namespace

int64_t mla_cache_fp8_row_bytes(int32_t d_c, int32_t d_r) {
  return int64_t(d_c) + 2 * int64_t(d_r);
}

int mla_cache_append_fp8(const mla_dims* d, int32_t hidden, const void* h, const void* W_DKV,
                         const float* gamma, float eps, float rope_base, void* cache,
                         float* scales, int32_t* seqlens, void* workspace,
                         size_t workspace_bytes, void* stream) {
  int st = check_dims(d);
  if (st) return st;
  if (!fp8_shape(d)) return MLA_ERR_UNSUPPORTED;
  if (hidden <= 0 || !h || !W_DKV || !cache || !scales || !seqlens) return MLA_ERR_INVALID_ARG;
  if (!(eps >= 0.f) || !(rope_base > 0.f)) return MLA_ERR_INVALID_ARG;
  if (hidden % 8) return MLA_ERR_UNSUPPORTED;
  if (!aligned16(h) || !aligned16(W_DKV) || !aligned16(cache) || !aligned16(scales) ||
      !aligned16(seqlens) || (gamma && !aligned16(gamma)) || (workspace && !aligned16(workspace)))
    return MLA_ERR_ALIGNMENT;
  if (!workspace || workspace_bytes < mla_cache_append_workspace_bytes(d, hidden))
    return MLA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* x = static_cast<float*>(workspace);
  cudaError_t e = launch_append_proj_tc(static_cast<const __nv_bfloat16*>(h),
                                        static_cast<const __nv_bfloat16*>(W_DKV), d->B,
                                        d->d_c + d->d_r, hidden, x, status_ptr(), s);
  if (e != cudaSuccess) return MLA_ERR_CUDA;
  return cuda_status(launch_append_finalize_fp8(
      x, append_tc_splits(hidden), gamma, eps, rope_base, d->B, d->d_c, d->d_r,
      d->cache_capacity, static_cast<uint8_t*>(cache), scales, contiguous_map(d), seqlens,
      status_ptr(), s));
}

int mla_decode_fp8(const mla_dims* d, const void* q_cat, const void* cache, const float* scales,
                   const int32_t* seqlens, float softmax_scale, int num_splits, void* workspace,
                   size_t workspace_bytes, int* splits_used, void* stream) {
  int st = check_dims(d);
  if (st) return st;
  if (!fp8_shape(d)) return MLA_ERR_UNSUPPORTED;
  if (int64_t(d->B) * d->cache_capacity >= (int64_t(1) << 31)) return MLA_ERR_UNSUPPORTED;
  if (!q_cat || !cache || !scales || !seqlens || num_splits < 0 || num_splits > kMaxSplits ||
      !(softmax_scale >= 0.f) || softmax_scale == INFINITY)
    return MLA_ERR_INVALID_ARG;
  softmax_scale = effective_scale(d, softmax_scale);
  if (!aligned16(q_cat) || !aligned16(cache) || !aligned16(scales) || !aligned16(seqlens) ||
      (workspace && !aligned16(workspace)))
    return MLA_ERR_ALIGNMENT;
  const int W = num_splits > 0 ? num_splits : mla_decode_default_splits(d);
  if (W <= 0) return MLA_ERR_CUDA;
  const WsLayout l = ws_layout(d, W);
  if (!workspace || workspace_bytes < l.total) return MLA_ERR_WORKSPACE;
  if (splits_used) *splits_used = W;
  float* o_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + l.o_off);
  float* lse_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + l.lse_off);
  return cuda_status(launch_decode_tc_fp8(
      static_cast<const __nv_bfloat16*>(q_cat), static_cast<const uint8_t*>(cache), scales,
      contiguous_map(d), seqlens, d->B, d->H, d->cache_capacity, softmax_scale, W, o_part,
      lse_part, status_ptr(), g_inject_wait_cycles, static_cast<cudaStream_t>(stream)));
}

// ---------------------------------------------------------------------------
// Materialised prefill of one sequence.
namespace {
int check_prefill(const mla_dims* d, int32_t T, int64_t L) {
  if (!d) return MLA_ERR_INVALID_ARG;
  if (d->H <= 0 || T < 0 || L <= 0) return MLA_ERR_INVALID_ARG;
  if (d->dtype != MLA_BF16 || d->d_c != 512 || d->d_nope != 128 || d->d_v != 128 ||
      (d->d_r != 64 && d->d_r != 0) || d->H > 65535)
    return MLA_ERR_UNSUPPORTED;
  // 32-bit TMA row coordinates over [H * L] and [H * T] matrices.
  if (int64_t(d->H) * L >= (int64_t(1) << 31) || int64_t(d->H) * T >= (int64_t(1) << 31))
    return MLA_ERR_UNSUPPORTED;
  return MLA_OK;
}
}  // namespace

size_t mla_prefill_workspace_bytes(const mla_dims* d, int32_t T, int64_t L) {
  if (check_prefill(d, T, L) != MLA_OK) return 0;
  return prefill_workspace_bytes(T, L, d->H, d->d_r);
}

int mla_prefill(const mla_dims* d, int32_t T, int64_t L, const void* q_nope, const void* q_pe,
                const int32_t* q_pos, const void* W_UK, const void* W_UV, const void* rows,
                float softmax_scale, float rope_base, void* out, float* lse, void* workspace,
                size_t workspace_bytes, void* stream) {
  int st = check_prefill(d, T, L);
  if (st) return st;
  if (T == 0) return MLA_OK;
  if (!q_nope || (d->d_r && !q_pe) || !q_pos || !W_UK || !W_UV || !rows || !out)
    return MLA_ERR_INVALID_ARG;
  softmax_scale = effective_scale(d, softmax_scale);
  if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale) || !(rope_base > 0.f))
    return MLA_ERR_INVALID_ARG;
  if (!aligned16(q_nope) || (q_pe && !aligned16(q_pe)) || !aligned16(W_UK) ||
      !aligned16(W_UV) || !aligned16(rows) || !aligned16(out) || (workspace && !aligned16(workspace)))
    return MLA_ERR_ALIGNMENT;
  if (!workspace || workspace_bytes < prefill_workspace_bytes(T, L, d->H, d->d_r))
    return MLA_ERR_WORKSPACE;
  return cuda_status(launch_prefill(
      static_cast<const __nv_bfloat16*>(q_nope), static_cast<const __nv_bfloat16*>(q_pe), q_pos,
      static_cast<const __nv_bfloat16*>(W_UK), static_cast<const __nv_bfloat16*>(W_UV),
      static_cast<const __nv_bfloat16*>(rows), T, L, d->H, d->d_r, softmax_scale, rope_base,
      static_cast<__nv_bfloat16*>(out), lse, workspace, status_ptr(),
      static_cast<cudaStream_t>(stream)));
}

// ---------------------------------------------------------------------------
// W^O folded into the value side.
namespace {
int check_fold(const mla_dims* d, int32_t d_model) {
  int st = check_dims(d);
  if (st) return st;
  if (d->dtype != MLA_BF16 || d->d_c != 512 || d->d_v != 128) return MLA_ERR_UNSUPPORTED;
  if (d_model <= 0) return MLA_ERR_INVALID_ARG;
  return MLA_OK;
}
}  // namespace

int mla_fold_output_weights(const mla_dims* d, int32_t d_model, const void* W_O,
                            const void* W_UV, void* W_fold, void* stream) {
  int st = check_fold(d, d_model);
  if (st) return st;
  if (!W_O || !W_UV || !W_fold) return MLA_ERR_INVALID_ARG;
  if (!aligned16(W_O) || !aligned16(W_UV) || !aligned16(W_fold)) return MLA_ERR_ALIGNMENT;
  return cuda_status(launch_fold_weights(static_cast<const __nv_bfloat16*>(W_O),
                                         static_cast<const __nv_bfloat16*>(W_UV), d_model, d->H,
                                         static_cast<__nv_bfloat16*>(W_fold), status_ptr(),
                                         static_cast<cudaStream_t>(stream)));
}

size_t mla_out_proj_folded_workspace_bytes(const mla_dims* d, int32_t d_model) {
  if (check_fold(d, d_model) != MLA_OK || d->B > kFoldedMaxBatch) return 0;
  return folded_proj_workspace_bytes(d->B, d->H, d_model);
}

int mla_out_proj_folded(const mla_dims* d, int32_t d_model, const float* o_lat, const void* W_fold,
                        void* u, void* workspace, size_t workspace_bytes, void* stream) {
  int st = check_fold(d, d_model);
  if (st) return st;
  if (d->B > kFoldedMaxBatch) return MLA_ERR_UNSUPPORTED;
  if (!o_lat || !W_fold || !u) return MLA_ERR_INVALID_ARG;
  if (!aligned16(o_lat) || !aligned16(W_fold) || !aligned16(u) ||
      (workspace && !aligned16(workspace)))
    return MLA_ERR_ALIGNMENT;
  if (!workspace || workspace_bytes < folded_proj_workspace_bytes(d->B, d->H, d_model))
    return MLA_ERR_WORKSPACE;
  return cuda_status(launch_folded_proj(o_lat, static_cast<const __nv_bfloat16*>(W_fold), d->B,
                                        d->H, d_model, workspace, static_cast<__nv_bfloat16*>(u),
                                        status_ptr(), static_cast<cudaStream_t>(stream)));
}

// ---------------------------------------------------------------------------
int mla_combine(const mla_dims* d, const int32_t* seqlens, const void* workspace,
                size_t workspace_bytes, int splits_used, float* o_lat, float* lse, void* stream) {
  int st = check_dims(d);
  if (st) return st;
  if (!seqlens || !workspace || !o_lat || splits_used <= 0 || splits_used > kMaxSplits)
    return MLA_ERR_INVALID_ARG;
  if (!aligned16(seqlens) || !aligned16(workspace) || !aligned16(o_lat) ||
      (lse && !aligned16(lse)))
    return MLA_ERR_ALIGNMENT;
  const WsLayout l = ws_layout(d, splits_used);
  if (workspace_bytes < l.total) return MLA_ERR_WORKSPACE;
  const char* ws = static_cast<const char*>(workspace);
  return cuda_status(launch_combine(seqlens, d->cache_capacity, d->B, d->H, d->d_c, splits_used,
                                    reinterpret_cast<const float*>(ws + l.o_off),
                                    reinterpret_cast<const float*>(ws + l.lse_off), o_lat, lse,
                                    static_cast<cudaStream_t>(stream)));
}

// ---------------------------------------------------------------------------
int mla_merge_partials(const mla_dims* d, int n_parts, const float* o_parts,
                       const float* lse_parts, float* o_lat, float* lse, void* stream) {
  int st = check_dims(d);
  if (st) return st;
  if (n_parts <= 0 || n_parts > kMaxSplits || !o_parts || !lse_parts || !o_lat)
    return MLA_ERR_INVALID_ARG;
  if (!aligned16(o_parts) || !aligned16(lse_parts) || !aligned16(o_lat) ||
      (lse && !aligned16(lse)))
    return MLA_ERR_ALIGNMENT;
  return cuda_status(launch_merge_partials(int64_t(d->B) * d->H, d->d_c, n_parts, o_parts,
                                           lse_parts, o_lat, lse,
                                           static_cast<cudaStream_t>(stream)));
}

// ---------------------------------------------------------------------------
int mla_out_proj(const mla_dims* d, const float* o_lat, const void* W_UV, void* out,
                 void* stream) {
  int st = check_dims(d);
  if (st) return st;
  if (!o_lat || !W_UV || !out) return MLA_ERR_INVALID_ARG;
  if (!aligned16(o_lat) || !aligned16(W_UV) || !aligned16(out)) return MLA_ERR_ALIGNMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (use_tc_gemm(d))
    return cuda_status(launch_out_proj_tc(o_lat, static_cast<const __nv_bfloat16*>(W_UV), d->B,
                                          d->H, static_cast<__nv_bfloat16*>(out), status_ptr(), s));
  if (d->dtype == MLA_BF16)
    return cuda_status(launch_out_proj<__nv_bfloat16>(o_lat,
                                                      static_cast<const __nv_bfloat16*>(W_UV),
                                                      d->B, d->H, d->d_c, d->d_v,
                                                      static_cast<__nv_bfloat16*>(out), s));
  return cuda_status(launch_out_proj<float>(o_lat, static_cast<const float*>(W_UV), d->B, d->H,
                                            d->d_c, d->d_v, static_cast<float*>(out), s));
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode + combine for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc at all: plugins handed a fixed set of
// buffers by a host framework, or runtimes whose device memory is owned by
// another allocator.  For them the split-KV partials live in the
// file-scope array below instead of a caller-provided workspace.  It is sized
// once (MLA_DECODE_NOALLOC_SCRATCH_BYTES) and every device that loads this
// library holds it until the process exits.
namespace mla {
namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[MLA_DECODE_NOALLOC_SCRATCH_BYTES];

// In host code `g_noalloc_scratch` names a host-side stand-in, not device
// memory, so the kernels get the real device address, looked up once per
// device (with that device current) and cached.
void* noalloc_scratch_ptr() {
  static void* cache[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (!cache[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return nullptr;
    cache[dev] = p;
  }
  return cache[dev];
}

}  // namespace
}  // namespace mla

extern "C" int mla_decode_noalloc(const mla_dims* d, const void* q_cat, const void* cache,
                                  const int32_t* seqlens, float softmax_scale, float* o_lat,
                                  float* lse, void* stream) {
  int st = check_dims(d);
  if (st) return st;
  if ((st = decode_shape_supported(d, true))) return st;
  if (!q_cat || !cache || !seqlens || !o_lat || !(softmax_scale >= 0.f) ||
      softmax_scale == INFINITY)
    return MLA_ERR_INVALID_ARG;
  softmax_scale = effective_scale(d, softmax_scale);
  if (!aligned16(q_cat) || !aligned16(cache) || !aligned16(seqlens) || !aligned16(o_lat) ||
      (lse && !aligned16(lse)))
    return MLA_ERR_ALIGNMENT;
  // Largest split count (up to the default) whose partials fit the array.
  int W = mla_decode_default_splits(d);
  if (W <= 0) return MLA_ERR_CUDA;
  while (W >= 1 && ws_layout(d, W).total > size_t(MLA_DECODE_NOALLOC_SCRATCH_BYTES)) --W;
  if (W < 1) return MLA_ERR_WORKSPACE;  // B * H too large for the fixed scratch
  void* scratch = noalloc_scratch_ptr();
  if (!scratch) return MLA_ERR_CUDA;
  const WsLayout l = ws_layout(d, W);
  float* o_part = reinterpret_cast<float*>(static_cast<char*>(scratch) + l.o_off);
  float* lse_part = reinterpret_cast<float*>(static_cast<char*>(scratch) + l.lse_off);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const cudaError_t e = launch_decode_any(d, q_cat, cache, contiguous_map(d), seqlens,
                                          softmax_scale, W, o_part, lse_part, status_ptr(), s);
  if (e != cudaSuccess) return MLA_ERR_CUDA;
  return cuda_status(launch_combine(seqlens, d->cache_capacity, d->B, d->H, d->d_c, W, o_part,
                                    lse_part, o_lat, lse, s));
}
