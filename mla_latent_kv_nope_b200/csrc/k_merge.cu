// Log-sum-exp merge of per-range decode results (sequence-sharded decode).
//
// When every device holds a contiguous token range of each sequence, each
// range gives a normalised latent output o_k and its log-sum-exp lse_k; the
// attention over the whole sequence is
//   lse = log sum_k exp(lse_k),   o = sum_k exp(lse_k - lse) o_k,
// the same identity that merges split-KV partials (it makes a softmax over
// disjoint key sets equal the softmax over their union).  A range with
// lse_k = -inf holds no keys and contributes nothing; its o_k is not read.
#include "common.cuh"
#include "kernels.h"

namespace mla {

namespace {

constexpr int kMergeWarps = 8;
constexpr int kMergeThreads = 32 * kMergeWarps;

// One warp per (sequence, head) pair: lanes stride over the partials for the
// max and the sum of exponentials, then over the 4-column groups of the row,
// so each partial's row is read as contiguous 512-byte warp loads.
__global__ void __launch_bounds__(kMergeThreads)
merge_partials_kernel(int64_t BH, int d_c, int n, const float* __restrict__ o_parts,
                      const float* __restrict__ lse_parts, float* __restrict__ o_lat,
                      float* __restrict__ lse_out) {
  const int64_t pair = int64_t(blockIdx.x) * kMergeWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (pair >= BH) return;
  float m = -INFINITY;
  for (int k = lane; k < n; k += 32) m = fmaxf(m, lse_parts[int64_t(k) * BH + pair]);
  m = warp_max(m);
  float4* dst = reinterpret_cast<float4*>(o_lat + pair * d_c);
  const int nq = d_c / 4;
  if (m == -INFINITY) {  // no range holds a key of this sequence
    for (int q = lane; q < nq; q += 32) dst[q] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (lse_out && lane == 0) lse_out[pair] = -INFINITY;
    return;
  }
  float z = 0.f;
  for (int k = lane; k < n; k += 32) {
    const float l = lse_parts[int64_t(k) * BH + pair];
    if (l != -INFINITY) z += expf(l - m);
  }
  z = warp_sum(z);
  const float inv_z = 1.f / z;
  for (int q = lane; q < nq; q += 32) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int k = 0; k < n; ++k) {
      const float l = lse_parts[int64_t(k) * BH + pair];
      if (l == -INFINITY) continue;
      const float wk = expf(l - m) * inv_z;
      const float4 v = reinterpret_cast<const float4*>(o_parts + (int64_t(k) * BH + pair) * d_c)[q];
      acc.x = fmaf(wk, v.x, acc.x);
      acc.y = fmaf(wk, v.y, acc.y);
      acc.z = fmaf(wk, v.z, acc.z);
      acc.w = fmaf(wk, v.w, acc.w);
    }
    dst[q] = acc;
  }
  if (lse_out && lane == 0) lse_out[pair] = m + logf(z);
}

}  // namespace

cudaError_t launch_merge_partials(int64_t BH, int d_c, int n, const float* o_parts,
                                  const float* lse_parts, float* o_lat, float* lse,
                                  cudaStream_t stream) {
  const int64_t blocks = (BH + kMergeWarps - 1) / kMergeWarps;
  if (blocks <= 0 || blocks > int64_t(0x7fffffff)) return cudaErrorInvalidValue;
  merge_partials_kernel<<<unsigned(blocks), kMergeThreads, 0, stream>>>(BH, d_c, n, o_parts,
                                                                         lse_parts, o_lat, lse);
  return cudaGetLastError();
}

}  // namespace mla
