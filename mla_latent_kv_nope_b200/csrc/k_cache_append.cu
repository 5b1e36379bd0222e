// Cache append: one new latent row per sequence.
//   x = W_DKV h_b                                  ([MLA-とは] "MLAの発想", c^KV = W^DKV h;
//                                                   "Decoupled RoPE", k^R = R_j W^KR h_j)
//   c = x[0:d_c] / sqrt(mean(x[0:d_c]^2) + eps) * gamma   (latent RMSNorm, 正規化の扱い)
//   k = RoPE(x[d_c:], pos = L_b)
//   cache[b, L_b] = [c || k];  L_b += 1
//
// Two passes.  The projection pass reads W_DKV once: block = 4 rows of W_DKV,
// all sequences (in chunks of 16), every thread striding over the hidden
// dimension, then a block reduction; it writes x to the fp32 workspace.  The
// finalize pass (block per sequence) applies the norm, the rotation and the
// single rounding, checks the capacity, writes row L_b and bumps L_b.
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"

namespace mla {

namespace {

constexpr int kApRows = 4;
constexpr int kApBatch = 16;
constexpr int kApThreads = 256;
constexpr int kFinBatch = 32;       // partial sums loaded together in the finalize

template <typename T>
__global__ void __launch_bounds__(kApThreads)
append_project_kernel(const T* __restrict__ h, const T* __restrict__ W, int B, int R,
                      int hidden, float* __restrict__ x_out) {
  __shared__ float s_red[kApThreads / 32][kApRows * kApBatch];
  const int r0 = blockIdx.x * kApRows;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int b0 = 0; b0 < B; b0 += kApBatch) {
    const int nb = min(kApBatch, B - b0);
    float acc[kApRows][kApBatch];
#pragma unroll
    for (int r = 0; r < kApRows; ++r)
#pragma unroll
      for (int bb = 0; bb < kApBatch; ++bb) acc[r][bb] = 0.f;
    for (int k = threadIdx.x; k < hidden; k += kApThreads) {
      float wv[kApRows];
#pragma unroll
      for (int r = 0; r < kApRows; ++r)
        wv[r] = (r0 + r < R) ? Storage<T>::to_f(W[int64_t(r0 + r) * hidden + k]) : 0.f;
#pragma unroll
      for (int bb = 0; bb < kApBatch; ++bb) {
        if (bb < nb) {
          const float hv = Storage<T>::to_f(h[int64_t(b0 + bb) * hidden + k]);
#pragma unroll
          for (int r = 0; r < kApRows; ++r) acc[r][bb] = fmaf(wv[r], hv, acc[r][bb]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < kApRows; ++r)
#pragma unroll
      for (int bb = 0; bb < kApBatch; ++bb) {
        const float v = warp_sum(acc[r][bb]);
        if (lane == 0) s_red[warp][r * kApBatch + bb] = v;
      }
    __syncthreads();
    if (threadIdx.x < kApRows * kApBatch) {
      const int r = threadIdx.x / kApBatch, bb = threadIdx.x % kApBatch;
      float v = 0.f;
#pragma unroll
      for (int wdx = 0; wdx < kApThreads / 32; ++wdx) v += s_red[wdx][threadIdx.x];
      if (r0 + r < R && bb < nb) x_out[int64_t(b0 + bb) * R + r0 + r] = v;
    }
    __syncthreads();
  }
}

template <typename T>
__global__ void __launch_bounds__(1024)
append_finalize_kernel(const float* __restrict__ part, int n_parts,
                       const float* __restrict__ gamma, float eps, float rope_base, int d_c,
                       int d_r, int64_t cap, T* __restrict__ cache, const PageMap pm,
                       int32_t* __restrict__ seqlens, int* __restrict__ status) {
  pdl_wait();   // the projection sums come from the kernel launched just before
  pdl_trigger();
  const int b = blockIdx.x;
  const int B = gridDim.x;
  const int R = d_c + d_r;
  extern __shared__ float s_x[];  // [R]: the projection, summed over parts in order
  __shared__ float s_part[32];
  __shared__ int32_t s_L;
  if (threadIdx.x == 0) s_L = seqlens[b];
  // The thread's first gain, loaded with the partial sums (one round trip).
  const float g_first = (gamma && int(threadIdx.x) < d_c) ? gamma[threadIdx.x] : 1.f;
  // Sum the partials in a fixed order (deterministic) with up to
  // kFinBatch loads in flight per thread; one column per thread when the
  // block covers the row.
  for (int c = threadIdx.x; c < R; c += blockDim.x) {
    const float* src = part + int64_t(b) * R + c;
    const int64_t stride = int64_t(B) * R;
    float v = 0.f;
    for (int p0 = 0; p0 < n_parts; p0 += kFinBatch) {
      float x[kFinBatch];
#pragma unroll
      for (int j = 0; j < kFinBatch; ++j) x[j] = p0 + j < n_parts ? src[(p0 + j) * stride] : 0.f;
#pragma unroll
      for (int j = 0; j < kFinBatch; ++j) v += x[j];
    }
    s_x[c] = v;
  }
  __syncthreads();
  const float* xb = s_x;
  float ss = 0.f;
  for (int c = threadIdx.x; c < d_c; c += blockDim.x) ss = fmaf(xb[c], xb[c], ss);
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) s_part[threadIdx.x >> 5] = ss;
  __syncthreads();
  const int32_t L = s_L;
  if (L < 0 || int64_t(L) >= cap) {
    if (threadIdx.x == 0) record_status(status, MLA_ERR_BOUNDS);
    return;
  }
  float tot = 0.f;
#pragma unroll
  for (int wdx = 0; wdx < int(blockDim.x / 32); ++wdx) tot += s_part[wdx];
  const float inv = 1.f / sqrtf(tot / float(d_c) + eps);
  const int64_t r = pm.row(b, L);
  if (r < 0) {   // page id outside the pool: nothing written, length unchanged
    if (threadIdx.x == 0) record_status(status, MLA_ERR_BOUNDS);
    return;
  }
  T* row = cache + r * R;
  for (int c = threadIdx.x; c < d_c; c += blockDim.x) {
    const float g = c == int(threadIdx.x) ? g_first : gamma ? gamma[c] : 1.f;
    row[c] = Storage<T>::from_f(xb[c] * inv * g);
  }
  const int half = d_r / 2;
  for (int k = threadIdx.x; k < half; k += blockDim.x) {
    float cs, sn;
    rope_cos_sin(L, k, d_r, rope_base, &cs, &sn);
    const float x1 = xb[d_c + k], x2 = xb[d_c + k + half];
    row[d_c + k] = Storage<T>::from_f(x1 * cs - x2 * sn);
    row[d_c + k + half] = Storage<T>::from_f(x1 * sn + x2 * cs);
  }
  __syncthreads();
  if (threadIdx.x == 0) seqlens[b] = L + 1;
}

// FP8 latent cache row: d_c E4M3 codes (bytes) then d_r bf16 RoPE keys.
// c = RMSNorm(x[0:d_c]) * gamma as above; its scale is the smallest power of
// two 2^k with max|c| / 2^k <= 448 (a zero row gets 1), and each code is
// c / 2^k rounded to nearest (ties to even) in E4M3, saturating at +-448.
__global__ void __launch_bounds__(1024)
append_finalize_fp8_kernel(const float* __restrict__ part, int n_parts,
                           const float* __restrict__ gamma, float eps, float rope_base, int d_c,
                           int d_r, int64_t cap, uint8_t* __restrict__ cache,
                           float* __restrict__ scales, const PageMap pm,
                           int32_t* __restrict__ seqlens, int* __restrict__ status) {
  pdl_wait();   // the projection sums come from the kernel launched just before
  pdl_trigger();
  const int b = blockIdx.x;
  const int B = gridDim.x;
  const int R = d_c + d_r;
  const int row_bytes = d_c + 2 * d_r;
  extern __shared__ float s_x[];  // [R]
  __shared__ float s_part[32];
  __shared__ int32_t s_L;
  if (threadIdx.x == 0) s_L = seqlens[b];
  const float g_first = (gamma && int(threadIdx.x) < d_c) ? gamma[threadIdx.x] : 1.f;
  for (int c = threadIdx.x; c < R; c += blockDim.x) {
    const float* src = part + int64_t(b) * R + c;
    const int64_t stride = int64_t(B) * R;
    float v = 0.f;
    for (int p0 = 0; p0 < n_parts; p0 += kFinBatch) {
      float x[kFinBatch];
#pragma unroll
      for (int j = 0; j < kFinBatch; ++j) x[j] = p0 + j < n_parts ? src[(p0 + j) * stride] : 0.f;
#pragma unroll
      for (int j = 0; j < kFinBatch; ++j) v += x[j];
    }
    s_x[c] = v;
  }
  __syncthreads();
  float ss = 0.f;
  for (int c = threadIdx.x; c < d_c; c += blockDim.x) ss = fmaf(s_x[c], s_x[c], ss);
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) s_part[threadIdx.x >> 5] = ss;
  __syncthreads();
  const int32_t L = s_L;
  if (L < 0 || int64_t(L) >= cap) {
    if (threadIdx.x == 0) record_status(status, MLA_ERR_BOUNDS);
    return;
  }
  float tot = 0.f;
#pragma unroll
  for (int wdx = 0; wdx < int(blockDim.x / 32); ++wdx) tot += s_part[wdx];
  const float inv = 1.f / sqrtf(tot / float(d_c) + eps);
  const int64_t r = pm.row(b, L);
  if (r < 0) {
    if (threadIdx.x == 0) record_status(status, MLA_ERR_BOUNDS);
    return;
  }
  __syncthreads();   // every thread has read s_part before it is reused
  // The normalised latent (fp32) and its largest magnitude.
  float amax = 0.f;
  for (int c = threadIdx.x; c < d_c; c += blockDim.x) {
    const float v = s_x[c] * inv * (c == int(threadIdx.x) ? g_first : gamma ? gamma[c] : 1.f);
    s_x[c] = v;
    amax = fmaxf(amax, fabsf(v));
  }
  amax = warp_max(amax);
  if ((threadIdx.x & 31) == 0) s_part[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = 0.f;
#pragma unroll
  for (int wdx = 0; wdx < int(blockDim.x / 32); ++wdx) amax = fmaxf(amax, s_part[wdx]);
  // amax = f * 2^e with f in [0.5, 1); 448 = 0.875 * 2^9, so the smallest k
  // with amax / 2^k <= 448 is e - 9 when f <= 0.875, else e - 8.
  int k = 0;
  if (amax > 0.f) {
    int e;
    const float f = frexpf(amax, &e);
    k = f <= 0.875f ? e - 9 : e - 8;
  }
  const float inv_scale = ldexpf(1.f, -k);
  uint8_t* row = cache + r * row_bytes;
  for (int c = 2 * threadIdx.x; c < d_c; c += 2 * blockDim.x) {
    const __nv_fp8x2_storage_t q = __nv_cvt_float2_to_fp8x2(
        make_float2(s_x[c] * inv_scale, s_x[c + 1] * inv_scale), __NV_SATFINITE, __NV_E4M3);
    *reinterpret_cast<__nv_fp8x2_storage_t*>(row + c) = q;
  }
  __nv_bfloat16* rope = reinterpret_cast<__nv_bfloat16*>(row + d_c);
  const int half = d_r / 2;
  for (int kk = threadIdx.x; kk < half; kk += blockDim.x) {
    float cs, sn;
    rope_cos_sin(L, kk, d_r, rope_base, &cs, &sn);
    const float x1 = s_x[d_c + kk], x2 = s_x[d_c + kk + half];
    rope[kk] = __float2bfloat16_rn(x1 * cs - x2 * sn);
    rope[kk + half] = __float2bfloat16_rn(x1 * sn + x2 * cs);
  }
  if (threadIdx.x == 0) scales[r] = ldexpf(1.f, k);
  __syncthreads();
  if (threadIdx.x == 0) seqlens[b] = L + 1;
}

}  // namespace

cudaError_t launch_append_finalize_fp8(const float* part, int n_parts, const float* gamma,
                                       float eps, float rope_base, int B, int d_c, int d_r,
                                       int64_t cap, uint8_t* cache, float* scales,
                                       const PageMap& pm, int32_t* seqlens, int* status,
                                       cudaStream_t stream) {
  const size_t smem = sizeof(float) * size_t(d_c + d_r);
  const int threads = min(1024, (d_c + d_r + 31) / 32 * 32);
  return launch_pdl(append_finalize_fp8_kernel, dim3(B), dim3(threads), smem, stream, part,
                    n_parts, gamma, eps, rope_base, d_c, d_r, cap, cache, scales, pm, seqlens,
                    status);
}

template <typename T>
cudaError_t launch_cache_append(const T* h, const T* W_DKV, const float* gamma, float eps,
                                float rope_base, int B, int d_c, int d_r, int hidden,
                                int64_t cap, T* cache, const PageMap& pm, int32_t* seqlens,
                                float* x_ws, int* status, cudaStream_t stream) {
  const int R = d_c + d_r;
  append_project_kernel<T><<<(R + kApRows - 1) / kApRows, kApThreads, 0, stream>>>(
      h, W_DKV, B, R, hidden, x_ws);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_append_finalize<T>(x_ws, 1, gamma, eps, rope_base, B, d_c, d_r, cap, cache, pm,
                                   seqlens, status, stream);
}

template <typename T>
cudaError_t launch_append_finalize(const float* part, int n_parts, const float* gamma, float eps,
                                   float rope_base, int B, int d_c, int d_r, int64_t cap,
                                   T* cache, const PageMap& pm, int32_t* seqlens, int* status,
                                   cudaStream_t stream) {
  const size_t smem = sizeof(float) * size_t(d_c + d_r);
  const int threads = min(1024, (d_c + d_r + 31) / 32 * 32);
  return launch_pdl(append_finalize_kernel<T>, dim3(B), dim3(threads), smem, stream, part,
                    n_parts, gamma, eps, rope_base, d_c, d_r, cap, cache, pm, seqlens, status);
}

template cudaError_t launch_append_finalize<float>(const float*, int, const float*, float, float,
                                                   int, int, int, int64_t, float*,
                                                   const PageMap&, int32_t*, int*, cudaStream_t);
template cudaError_t launch_append_finalize<__nv_bfloat16>(const float*, int, const float*, float,
                                                           float, int, int, int, int64_t,
                                                           __nv_bfloat16*, const PageMap&,
                                                           int32_t*, int*, cudaStream_t);

template cudaError_t launch_cache_append<float>(const float*, const float*, const float*,
                                                float, float, int, int, int, int, int64_t,
                                                float*, const PageMap&, int32_t*, float*, int*,
                                                cudaStream_t);
template cudaError_t launch_cache_append<__nv_bfloat16>(
    const __nv_bfloat16*, const __nv_bfloat16*, const float*, float, float, int, int, int,
    int, int64_t, __nv_bfloat16*, const PageMap&, int32_t*, float*, int*, cudaStream_t);

}  // namespace mla
