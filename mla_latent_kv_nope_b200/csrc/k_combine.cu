// Log-sum-exp merge of the split-KV partials written by the decode kernels.
//
//   lse[b,i]   = log sum_s exp(lse_s)
//   o_lat[b,i] = sum_s exp(lse_s - lse[b,i]) * o_s
//
// The partials of sequence b live in slots (b + w) for every non-empty worker
// w whose tile range meets b's tiles; the block recomputes that set from the
// sequence lengths exactly as the decode kernels dealt the tiles.
// One block per (head, sequence); each thread owns 4 consecutive latent
// columns (float4 loads/stores).
#include "common.cuh"
#include "kernels.h"

namespace mla {

namespace {

constexpr int kCombineThreads = 128;

__global__ void __launch_bounds__(kCombineThreads)
combine_kernel(const int32_t* __restrict__ seqlens, int64_t cap, int B, int H, int d_c, int W,
               const float* __restrict__ o_part, const float* __restrict__ lse_part,
               float* __restrict__ o_lat, float* __restrict__ lse_out) {
  const int i = blockIdx.x, b = blockIdx.y;
  __shared__ int64_t s_T, s_prefix;
  __shared__ float s_w[1024];  // per-worker weights (W <= 1024)
  __shared__ float s_lse;
  if (threadIdx.x == 0) {
    int64_t T = 0, pre = 0;
    for (int bb = 0; bb < B; ++bb) {
      const int64_t nt = tiles_of(clamp_len(seqlens[bb], cap));
      if (bb < b) pre += nt;
      T += nt;
    }
    s_T = T;
    s_prefix = pre;
  }
  __syncthreads();
  const int64_t T = s_T, pre = s_prefix;
  const int64_t nt = tiles_of(clamp_len(seqlens[b], cap));
  float* dst = o_lat + (int64_t(b) * H + i) * d_c;
  if (nt == 0) {
    for (int c = threadIdx.x * 4; c < d_c; c += kCombineThreads * 4)
      *reinterpret_cast<float4*>(dst + c) = make_float4(0.f, 0.f, 0.f, 0.f);
    if (threadIdx.x == 0 && lse_out) lse_out[int64_t(b) * H + i] = -INFINITY;
    return;
  }
  const int w_first = int(worker_of_tile(pre, T, W));
  const int w_last = int(worker_of_tile(pre + nt - 1, T, W));
  const int nw = w_last - w_first + 1;
  if (threadIdx.x == 0) {
    float m = -INFINITY;
    for (int k = 0; k < nw; ++k) {
      const int w = w_first + k;
      const bool empty = worker_tile_begin(w, T, W) == worker_tile_begin(w + 1, T, W);
      const float l = empty ? -INFINITY : lse_part[int64_t(b + w) * H + i];
      s_w[k] = l;
      m = fmaxf(m, l);
    }
    float z = 0.f;
    for (int k = 0; k < nw; ++k) {
      const float e = s_w[k] == -INFINITY ? 0.f : expf(s_w[k] - m);
      s_w[k] = e;
      z += e;
    }
    for (int k = 0; k < nw; ++k) s_w[k] /= z;
    s_lse = m + logf(z);
  }
  __syncthreads();
  for (int c = threadIdx.x * 4; c < d_c; c += kCombineThreads * 4) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int k = 0; k < nw; ++k) {
      const float wk = s_w[k];
      if (wk == 0.f) continue;
      const float4 v = *reinterpret_cast<const float4*>(
          o_part + (int64_t(b + w_first + k) * H + i) * d_c + c);
      acc.x = fmaf(wk, v.x, acc.x);
      acc.y = fmaf(wk, v.y, acc.y);
      acc.z = fmaf(wk, v.z, acc.z);
      acc.w = fmaf(wk, v.w, acc.w);
    }
    *reinterpret_cast<float4*>(dst + c) = acc;
  }
  if (threadIdx.x == 0 && lse_out) lse_out[int64_t(b) * H + i] = s_lse;
}

}  // namespace

cudaError_t launch_combine(const int32_t* seqlens, int64_t cap, int B, int H, int d_c, int W,
                           const float* o_part, const float* lse_part, float* o_lat,
                           float* lse, cudaStream_t stream) {
  dim3 grid(H, B);
  combine_kernel<<<grid, kCombineThreads, 0, stream>>>(seqlens, cap, B, H, d_c, W, o_part,
                                                       lse_part, o_lat, lse);
  return cudaGetLastError();
}

}  // namespace mla
