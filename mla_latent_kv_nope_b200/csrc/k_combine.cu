// Log-sum-exp merge of the split-KV partials written by the decode kernels.
//
//   lse[b,i]   = log sum_s exp(lse_s)
//   o_lat[b,i] = sum_s exp(lse_s - lse[b,i]) * o_s
//
// The partials of sequence b live in slots (b + w) for every non-empty worker
// w whose tile range meets b's tiles; the block recomputes that set from the
// sequence lengths exactly as the decode kernels dealt the tiles.
// Partials are stored as o_part[slot][d_c / 4][H][4] (see combine_kernel).
#include "common.cuh"
#include "kernels.h"

namespace mla {

namespace {

constexpr int kCombineHeads = 32;    // heads per block, one per lane
constexpr int kCombineWarps = 8;
constexpr int kCombineThreads = 32 * kCombineWarps;
constexpr int kQuadsPerWarp = 4;     // 4-column groups per warp
constexpr int kQuadsPerBlock = kCombineWarps * kQuadsPerWarp;   // 128 columns
constexpr int kFastParts = 4;        // partials merged with all loads in one round

// Block = (sequence b, 32 heads, 128 columns).  The partials are stored as
// o_part[slot][d_c / 4][H][4], so a warp load of one 4-column group for 32
// consecutive heads is one contiguous 512-byte read.  Each thread owns one
// head (its lane) and 4 column groups; it reduces the lse values of the
// head's partials (max, then the sum of exponentials) and accumulates its
// columns over the partials, two partials per step (8 loads in flight).  The
// merged block goes through shared memory so o_lat rows are written with
// coalesced stores.
__global__ void __launch_bounds__(kCombineThreads, 4)
combine_kernel(const int32_t* __restrict__ seqlens, int64_t cap, int B, int H, int d_c, int W,
               const float* __restrict__ o_part, const float* __restrict__ lse_part,
               float* __restrict__ o_lat, float* __restrict__ lse_out) {
  __shared__ float4 s_rows[kCombineHeads][kQuadsPerBlock + 1];
  __shared__ int64_t s_red[2][kCombineWarps];
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h0 = blockIdx.y * kCombineHeads;
  const int i = h0 + lane;
  const bool head_ok = i < H;
  const int nq = d_c / 4;
  const int q_base = blockIdx.z * kQuadsPerBlock;
  const int nqb = min(kQuadsPerBlock, nq - q_base);
  const int nh = min(kCombineHeads, H - h0);
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
  const int64_t T = tot;
  const int64_t nt = tiles_of(clamp_len(seqlens[b], cap));
  if (nt == 0) {
    for (int idx = threadIdx.x; idx < nh * nqb; idx += kCombineThreads)
      reinterpret_cast<float4*>(o_lat + (int64_t(b) * H + h0 + idx / nqb) * d_c)[q_base + idx % nqb] =
          make_float4(0.f, 0.f, 0.f, 0.f);
    if (blockIdx.z == 0 && warp == 0 && head_ok && lse_out) lse_out[int64_t(b) * H + i] = -INFINITY;
    return;
  }
  const int w_first = int(worker_of_tile(pre, T, W));
  const int w_last = int(worker_of_tile(pre + nt - 1, T, W));
  auto live = [&](int w) { return worker_tile_begin(w, T, W) != worker_tile_begin(w + 1, T, W); };
  // Column groups of this thread: q_base + warp + 8 j, j < 4.
  const float4* src0 = reinterpret_cast<const float4*>(o_part) + int64_t(q_base + warp) * H + i;
  const int64_t slot_stride = int64_t(nq) * H;   // float4 units
  float4 acc[kQuadsPerWarp];
#pragma unroll
  for (int j = 0; j < kQuadsPerWarp; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
  const int np = w_last - w_first + 1;
  float m = -INFINITY, z = 0.f;
  if (np <= kFastParts) {
    // Common case (up to 4 partials): their lse values in one round of
    // loads, then their column groups in two rounds.
    float lv[kFastParts];
#pragma unroll
    for (int k = 0; k < kFastParts; ++k) {
      const int w = w_first + k;
      lv[k] = (k < np && head_ok && live(w)) ? lse_part[int64_t(b + w) * H + i] : -INFINITY;
    }
#pragma unroll
    for (int k = 0; k < kFastParts; ++k) m = fmaxf(m, lv[k]);
    float e[kFastParts];
#pragma unroll
    for (int k = 0; k < kFastParts; ++k) {
      e[k] = lv[k] == -INFINITY ? 0.f : expf(lv[k] - m);
      z += e[k];
    }
    const float inv_z = head_ok ? 1.f / z : 0.f;
#pragma unroll
    for (int k = 0; k < kFastParts; ++k) e[k] *= inv_z;
    // Two column groups per round keep the live registers low enough for four
    // blocks per SM.
#pragma unroll
    for (int j0 = 0; j0 < kQuadsPerWarp; j0 += 2) {
      float4 v[kFastParts][2];
#pragma unroll
      for (int k = 0; k < kFastParts; ++k) {
        const float4* sk = src0 + int64_t(b + w_first + (k < np ? k : 0)) * slot_stride;
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const int j = j0 + jj;
          const bool in = e[k] != 0.f && warp + kCombineWarps * j < nqb;
          v[k][jj] = in ? sk[int64_t(kCombineWarps * j) * H] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int k = 0; k < kFastParts; ++k)
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const int j = j0 + jj;
          acc[j].x = fmaf(e[k], v[k][jj].x, acc[j].x);
          acc[j].y = fmaf(e[k], v[k][jj].y, acc[j].y);
          acc[j].z = fmaf(e[k], v[k][jj].z, acc[j].z);
          acc[j].w = fmaf(e[k], v[k][jj].w, acc[j].w);
        }
    }
  } else {
    for (int w = w_first; w <= w_last; ++w)
      if (live(w) && head_ok) m = fmaxf(m, lse_part[int64_t(b + w) * H + i]);
    for (int w = w_first; w <= w_last; ++w)
      if (live(w) && head_ok) z += expf(lse_part[int64_t(b + w) * H + i] - m);
    const float inv_z = head_ok ? 1.f / z : 0.f;
    auto weight = [&](int w) {
      return (live(w) && head_ok) ? expf(lse_part[int64_t(b + w) * H + i] - m) * inv_z : 0.f;
    };
    for (int w = w_first; w <= w_last; w += 2) {
      const bool two = w + 1 <= w_last;
      const float ea = weight(w), eb = two ? weight(w + 1) : 0.f;
      const float4* sa = src0 + int64_t(b + w) * slot_stride;
      const float4* sb = src0 + int64_t(b + (two ? w + 1 : w)) * slot_stride;
      float4 va[kQuadsPerWarp], vb[kQuadsPerWarp];
#pragma unroll
      for (int j = 0; j < kQuadsPerWarp; ++j) {
        const bool in = head_ok && warp + kCombineWarps * j < nqb;
        va[j] = (in && ea != 0.f) ? sa[int64_t(kCombineWarps * j) * H] : make_float4(0.f, 0.f, 0.f, 0.f);
        vb[j] = (in && eb != 0.f) ? sb[int64_t(kCombineWarps * j) * H] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int j = 0; j < kQuadsPerWarp; ++j) {
        acc[j].x = fmaf(ea, va[j].x, fmaf(eb, vb[j].x, acc[j].x));
        acc[j].y = fmaf(ea, va[j].y, fmaf(eb, vb[j].y, acc[j].y));
        acc[j].z = fmaf(ea, va[j].z, fmaf(eb, vb[j].z, acc[j].z));
        acc[j].w = fmaf(ea, va[j].w, fmaf(eb, vb[j].w, acc[j].w));
      }
    }
  }
#pragma unroll
  for (int j = 0; j < kQuadsPerWarp; ++j) s_rows[lane][warp + kCombineWarps * j] = acc[j];
  __syncthreads();
  for (int idx = threadIdx.x; idx < nh * nqb; idx += kCombineThreads) {
    const int hh = idx / nqb, q = idx % nqb;
    reinterpret_cast<float4*>(o_lat + (int64_t(b) * H + h0 + hh) * d_c)[q_base + q] = s_rows[hh][q];
  }
  if (blockIdx.z == 0 && warp == 0 && head_ok && lse_out) lse_out[int64_t(b) * H + i] = m + logf(z);
}

}  // namespace

cudaError_t launch_combine(const int32_t* seqlens, int64_t cap, int B, int H, int d_c, int W,
                           const float* o_part, const float* lse_part, float* o_lat,
                           float* lse, cudaStream_t stream) {
  const int nq = d_c / 4;
  dim3 grid(B, (H + kCombineHeads - 1) / kCombineHeads, (nq + kQuadsPerBlock - 1) / kQuadsPerBlock);
  combine_kernel<<<grid, kCombineThreads, 0, stream>>>(seqlens, cap, B, H, d_c, W, o_part,
                                                       lse_part, o_lat, lse);
  return cudaGetLastError();
}

}  // namespace mla
