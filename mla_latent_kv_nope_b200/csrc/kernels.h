// Internal launch functions (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace mla {

template <typename T>
cudaError_t launch_absorb_q(const T* q_nope, const T* q_pe, const T* W_UK,
                            const int32_t* q_pos, float rope_base, int B, int H, int d_c,
                            int d_r, int d_n, T* q_cat, cudaStream_t stream);

template <typename T>
cudaError_t launch_decode_simt(const T* q_cat, const T* cache, const PageMap& pm,
                               const int32_t* seqlens,
                               int B, int H, int d_c, int d_r, int64_t cap, float scale,
                               int W, float* o_part, float* lse_part, int* status,
                               cudaStream_t stream);
size_t decode_simt_smem_bytes(int d_c, int d_r);

// Tensor-core decode (bf16, d_c = 512, d_r = 64 or 0).  Returns
// cudaErrorNotSupported when the build has no sm_100a kernel.  `inject_wait`
// > 0 adds a wait of that many SM cycles on a barrier nothing arrives on (a
// test of the give-up path).
cudaError_t launch_decode_tc(const __nv_bfloat16* q_cat, const __nv_bfloat16* cache,
                             const PageMap& pm, const int32_t* seqlens, int B, int H, int64_t cap,
                             int d_r, float scale, int W, float* o_part, float* lse_part,
                             int* status, uint64_t inject_wait, cudaStream_t stream);
int decode_tc_head_groups(int H);
// The same over an FP8 latent cache: rows [512 E4M3 codes || 64 bf16 RoPE keys]
// (640 bytes) addressed through `pm`, and one fp32 scale per row (`scales`,
// indexed like the rows).
cudaError_t launch_decode_tc_fp8(const __nv_bfloat16* q_cat, const uint8_t* cache,
                                 const float* scales, const PageMap& pm, const int32_t* seqlens,
                                 int B, int H, int64_t cap, float scale, int W, float* o_part,
                                 float* lse_part, int* status, uint64_t inject_wait,
                                 cudaStream_t stream);
// 2D TMA map over the cache viewed as [rows, 576] bf16: 64 x 64 boxes, 128-byte
// swizzle.  False if the driver entry point is missing or encoding fails.
bool make_cache_rows_map(CUtensorMap* map, const void* base, uint64_t rows);
// The same over rows of R bf16 (R a multiple of 64).
bool make_cache_rows_map_r(CUtensorMap* map, const void* base, uint64_t rows, int R);


cudaError_t launch_combine(const int32_t* seqlens, int64_t cap, int B, int H, int d_c, int W,
                           const float* o_part, const float* lse_part, float* o_lat,
                           float* lse, cudaStream_t stream);
// Log-sum-exp merge of n per-range results: o_parts [n][BH][d_c], lse_parts
// [n][BH] -> o_lat [BH][d_c], lse [BH] (lse may be null).
cudaError_t launch_merge_partials(int64_t BH, int d_c, int n, const float* o_parts,
                                  const float* lse_parts, float* o_lat, float* lse,
                                  cudaStream_t stream);

template <typename T>
cudaError_t launch_out_proj(const float* o_lat, const T* W_UV, int B, int H, int d_c,
                            int d_v, T* out, cudaStream_t stream);

template <typename T>
cudaError_t launch_cache_append(const T* h, const T* W_DKV, const float* gamma, float eps,
                                float rope_base, int B, int d_c, int d_r, int hidden,
                                int64_t cap, T* cache, const PageMap& pm, int32_t* seqlens,
                                float* x_ws, int* status, cudaStream_t stream);
// Finalize only (norm, rotation, store, length bump) over n_parts partial sums
// part[p][b][r] of the projection.
template <typename T>
cudaError_t launch_append_finalize(const float* part, int n_parts, const float* gamma, float eps,
                                   float rope_base, int B, int d_c, int d_r, int64_t cap,
                                   T* cache, const PageMap& pm, int32_t* seqlens, int* status,
                                   cudaStream_t stream);

// Finalize into an FP8 latent cache: rows of [d_c E4M3 codes || d_r bf16 RoPE
// keys] (d_c + 2 d_r bytes) and one fp32 power-of-two scale per row.
cudaError_t launch_append_finalize_fp8(const float* part, int n_parts, const float* gamma,
                                       float eps, float rope_base, int B, int d_c, int d_r,
                                       int64_t cap, uint8_t* cache, float* scales,
                                       const PageMap& pm, int32_t* seqlens, int* status,
                                       cudaStream_t stream);

// Tensor-core kernels for the bf16 step (d_c = 512, d_r = 64 or 0, d_nope = d_v = 128).
bool gemm_tc_supported(int d_c, int d_r, int d_n, int d_v);
cudaError_t launch_out_proj_tc(const float* o_lat, const __nv_bfloat16* W_UV, int B, int H,
                               __nv_bfloat16* out, int* status, cudaStream_t stream);
cudaError_t launch_absorb_q_tc(const __nv_bfloat16* q_nope, const __nv_bfloat16* q_pe,
                               const __nv_bfloat16* W_UK, const int32_t* q_pos, float rope_base,
                               int B, int H, int d_r, __nv_bfloat16* q_cat, int* status,
                               cudaStream_t stream);
int append_tc_splits(int hidden);
cudaError_t launch_append_proj_tc(const __nv_bfloat16* h, const __nv_bfloat16* W_DKV, int B,
                                  int R, int hidden, float* part, int* status,
                                  cudaStream_t stream);

// W^O folded into the value side: W_fold [d_model, H * 512] (bf16) with
// W_fold[m, i*512 + c] = sum_v W_O[m, i*128 + v] W_UV[i, v, c] (d_c = 512,
// d_v = 128), and the per-step u [B, d_model] = W_fold o_lat (o_lat fp32
// [B, H * 512], rounded to bf16 for the MMA; B <= kFoldedMaxBatch).
constexpr int kFoldedMaxBatch = 64;
cudaError_t launch_fold_weights(const __nv_bfloat16* W_O, const __nv_bfloat16* W_UV, int d_model,
                                int H, __nv_bfloat16* w_fold, int* status, cudaStream_t stream);
int folded_proj_splits(int d_model, int H);
size_t folded_proj_workspace_bytes(int B, int H, int d_model);
cudaError_t launch_folded_proj(const float* o_lat, const __nv_bfloat16* w_fold, int B, int H,
                               int d_model, void* workspace, __nv_bfloat16* u, int* status,
                               cudaStream_t stream);

// Materialised prefill of one sequence (bf16, d_c = 512, d_nope = d_v = 128,
// d_r = 64 or 0): q_nope [T, H, 128], q_pe [T, H, d_r], q_pos [T], rows
// [L, 512 + d_r] -> out [T, H, 128] bf16, lse [T, H] fp32 (nullable).  The
// workspace holds the rotated queries and the materialised K^C and V.
size_t prefill_workspace_bytes(int T, int64_t L, int H, int d_r);
cudaError_t launch_prefill(const __nv_bfloat16* q_nope, const __nv_bfloat16* q_pe,
                           const int32_t* q_pos, const __nv_bfloat16* W_UK,
                           const __nv_bfloat16* W_UV, const __nv_bfloat16* rows, int T, int64_t L,
                           int H, int d_r, float scale, float rope_base, __nv_bfloat16* out,
                           float* lse, void* workspace, int* status, cudaStream_t stream);

}  // namespace mla
