// Log-sum-exp merge of the split-KV partials written by the decode kernels.
//
//   lse[b,i]   = log sum_s exp(lse_s)
//   o_lat[b,i] = sum_s exp(lse_s - lse[b,i]) * o_s
//
// The partials of sequence b live in slots (b + w) for every non-empty worker
// w whose tile range meets b's tiles; the block recomputes that set from the
// sequence lengths exactly as the decode kernels dealt the tiles.
// (Kernel layout: see combine_kernel.)
#include "common.cuh"
#include "kernels.h"

namespace mla {

namespace {

constexpr int kCombineWarps = 8;   // heads per block (one warp each)
constexpr int kCombineThreads = 32 * kCombineWarps;
constexpr int kMaxDcPerLane = 32;  // d_c <= 1024

// Block = (sequence b, group of 8 heads).  The tile prefix of b and the total
// are reduced by the whole block; then each warp merges one head: its lanes
// read the partials' lse values, reduce max and sum with shuffles, and
// accumulate d_c / 32 columns each over the partials (loads in flight
// together rather than one after another).
__global__ void __launch_bounds__(kCombineThreads)
combine_kernel(const int32_t* __restrict__ seqlens, int64_t cap, int B, int H, int d_c, int W,
               const float* __restrict__ o_part, const float* __restrict__ lse_part,
               float* __restrict__ o_lat, float* __restrict__ lse_out) {
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.y * kCombineWarps + warp;
  __shared__ int64_t s_red[2][kCombineWarps];
  int64_t pre = 0, tot = 0;
  for (int bb = threadIdx.x; bb < B; bb += kCombineThreads) {
    const int64_t nt = tiles_of(clamp_len(seqlens[bb], cap));
    tot += nt;
    if (bb < b) pre += nt;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    pre += __shfl_xor_sync(0xffffffffu, pre, o);
    tot += __shfl_xor_sync(0xffffffffu, tot, o);
  }
  if (lane == 0) {
    s_red[0][warp] = pre;
    s_red[1][warp] = tot;
  }
  __syncthreads();
  pre = 0;
  tot = 0;
#pragma unroll
  for (int k = 0; k < kCombineWarps; ++k) {
    pre += s_red[0][k];
    tot += s_red[1][k];
  }
  if (i >= H) return;
  const int64_t T = tot;
  const int64_t nt = tiles_of(clamp_len(seqlens[b], cap));
  float* dst = o_lat + (int64_t(b) * H + i) * d_c;
  if (nt == 0) {
    for (int c = lane * 4; c < d_c; c += 128)
      *reinterpret_cast<float4*>(dst + c) = make_float4(0.f, 0.f, 0.f, 0.f);
    if (lane == 0 && lse_out) lse_out[int64_t(b) * H + i] = -INFINITY;
    return;
  }
  const int w_first = int(worker_of_tile(pre, T, W));
  const int w_last = int(worker_of_tile(pre + nt - 1, T, W));
  // Weights of the partials: lane k holds partial k's lse (32 at a time).
  const int nw = w_last - w_first + 1;
  float m = -INFINITY;
  for (int k0 = 0; k0 < nw; k0 += 32) {
    const int w = w_first + k0 + lane;
    const bool live = (k0 + lane < nw) &&
                      worker_tile_begin(w, T, W) != worker_tile_begin(w + 1, T, W);
    if (live) m = fmaxf(m, lse_part[int64_t(b + w) * H + i]);
  }
  m = warp_max(m);
  float z = 0.f;
  float my_e = 0.f;  // exp(lse - m) of this lane's partial in the first 32
  for (int k0 = 0; k0 < nw; k0 += 32) {
    const int w = w_first + k0 + lane;
    const bool live = (k0 + lane < nw) &&
                      worker_tile_begin(w, T, W) != worker_tile_begin(w + 1, T, W);
    const float e = live ? expf(lse_part[int64_t(b + w) * H + i] - m) : 0.f;
    if (k0 == 0) my_e = e;
    z += e;
  }
  z = warp_sum(z);
  const float inv_z = 1.f / z;
  float acc[kMaxDcPerLane / 4][4];
#pragma unroll
  for (int q = 0; q < kMaxDcPerLane / 4; ++q) acc[q][0] = acc[q][1] = acc[q][2] = acc[q][3] = 0.f;
  // Partials two at a time so their loads are in flight together.
  for (int k = 0; k < nw; k += 2) {
    const int wa = w_first + k, wb = w_first + k + 1;
    float ea = k < 32 ? __shfl_sync(0xffffffffu, my_e, k) : 0.f;
    float eb = k + 1 < 32 ? __shfl_sync(0xffffffffu, my_e, min(k + 1, 31)) : 0.f;
    if (k >= 32) {
      const bool la = worker_tile_begin(wa, T, W) != worker_tile_begin(wa + 1, T, W);
      ea = la ? expf(lse_part[int64_t(b + wa) * H + i] - m) : 0.f;
    }
    if (k + 1 >= 32 && k + 1 < nw) {
      const bool lb = worker_tile_begin(wb, T, W) != worker_tile_begin(wb + 1, T, W);
      eb = lb ? expf(lse_part[int64_t(b + wb) * H + i] - m) : 0.f;
    }
    if (k + 1 >= nw) eb = 0.f;
    ea *= inv_z;
    eb *= inv_z;
    const float* sa = o_part + (int64_t(b + wa) * H + i) * d_c;
    const float* sb = o_part + (int64_t(b + min(wb, w_last)) * H + i) * d_c;
#pragma unroll
    for (int q = 0; q < kMaxDcPerLane / 4; ++q) {
      const int c = (q * 32 + lane) * 4;
      if (c < d_c) {
        const float4 va = ea != 0.f ? *reinterpret_cast<const float4*>(sa + c)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 vb = eb != 0.f ? *reinterpret_cast<const float4*>(sb + c)
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
        acc[q][0] = fmaf(ea, va.x, fmaf(eb, vb.x, acc[q][0]));
        acc[q][1] = fmaf(ea, va.y, fmaf(eb, vb.y, acc[q][1]));
        acc[q][2] = fmaf(ea, va.z, fmaf(eb, vb.z, acc[q][2]));
        acc[q][3] = fmaf(ea, va.w, fmaf(eb, vb.w, acc[q][3]));
      }
    }
  }
#pragma unroll
  for (int q = 0; q < kMaxDcPerLane / 4; ++q) {
    const int c = (q * 32 + lane) * 4;
    if (c < d_c)
      *reinterpret_cast<float4*>(dst + c) = make_float4(acc[q][0], acc[q][1], acc[q][2], acc[q][3]);
  }
  if (lane == 0 && lse_out) lse_out[int64_t(b) * H + i] = m + logf(z);
}

}  // namespace

cudaError_t launch_combine(const int32_t* seqlens, int64_t cap, int B, int H, int d_c, int W,
                           const float* o_part, const float* lse_part, float* o_lat,
                           float* lse, cudaStream_t stream) {
  dim3 grid(B, (H + kCombineWarps - 1) / kCombineWarps);
  combine_kernel<<<grid, kCombineThreads, 0, stream>>>(seqlens, cap, B, H, d_c, W, o_part,
                                                       lse_part, o_lat, lse);
  return cudaGetLastError();
}

}  // namespace mla
