// Log-sum-exp merge of the split-KV partials written by the decode kernels.
//
//   lse[b,i]   = log sum_s exp(lse_s)
//   o_lat[b,i] = sum_s exp(lse_s - lse[b,i]) * o_s
//
// The partials of sequence b live in slots (b + w) for every non-empty worker
// w whose unit range meets b's tiles; the block recomputes that set from the
// sequence lengths exactly as the decode kernels dealt the work units (each
// sequence's kSwitchUnits start-up units, then its tiles).
// Partials are stored as o_part[slot][d_c / 4][H][4] (see combine_kernel).
#include "common.cuh"
#include "kernels.h"

namespace mla {

namespace {

constexpr int kCombineHeads = 32;    // heads per block, one per lane
constexpr int kCombineWarps = 8;
constexpr int kCombineThreads = 32 * kCombineWarps;
constexpr int kFastParts = 4;        // partials merged with all loads in one round

// Block = (sequence b, 32 heads, 128 columns).  The partials are stored as
// o_part[slot][d_c / 4][H][4], so a warp load of one 4-column group for 32
// consecutive heads is one contiguous 512-byte read.  Each thread owns one
// head (its lane) and 4 column groups; it reduces the lse values of the
// head's partials (max, then the sum of exponentials) and accumulates its
// columns over the partials: up to four partials (the common case of many
// shorter sequences) with all loads in one round, more one at a time.  The
// merged block goes through shared memory so o_lat rows are written with
// coalesced stores.
constexpr int kQuadsPerWarp = 4;
constexpr int kQuadsPerBlock = kCombineWarps * kQuadsPerWarp;   // 128 columns

__global__ void __launch_bounds__(kCombineThreads, 4)
combine_kernel(const int32_t* __restrict__ seqlens, int64_t cap, int B, int H, int d_c, int W,
               const float* __restrict__ o_part, const float* __restrict__ lse_part,
               float* __restrict__ o_lat, float* __restrict__ lse_out) {
  constexpr int kBatch = 1;   // partials per round past the first four
  __shared__ float4 s_rows[kCombineHeads][kQuadsPerBlock + 1];
  __shared__ int64_t s_red[2][kCombineWarps];
  pdl_wait();   // the partials come from the decode launched just before
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
    const int64_t nu = units_of(clamp_len(seqlens[bb], cap));
    tot += nu;
    if (bb < b) pre += nu;
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
  // The sequence's tiles are units [pre + kSwitchUnits, + nt) of the deal.
  const int w_first = int(worker_of_tile(pre + kSwitchUnits, T, W));
  const int w_last = int(worker_of_tile(pre + kSwitchUnits + nt - 1, T, W));
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
    auto lse_of = [&](int w) {
      return (w <= w_last && head_ok && live(w)) ? lse_part[int64_t(b + w) * H + i] : -INFINITY;
    };
    for (int w0 = w_first; w0 <= w_last; w0 += 8) {
      float lv[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) lv[k] = lse_of(w0 + k);
#pragma unroll
      for (int k = 0; k < 8; ++k) m = fmaxf(m, lv[k]);
    }
    for (int w0 = w_first; w0 <= w_last; w0 += 8) {
      float lv[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) lv[k] = lse_of(w0 + k);
#pragma unroll
      for (int k = 0; k < 8; ++k) z += lv[k] == -INFINITY ? 0.f : expf(lv[k] - m);
    }
    const float inv_z = head_ok ? 1.f / z : 0.f;
    for (int w0 = w_first; w0 <= w_last; w0 += kBatch) {
      float e[kBatch];
#pragma unroll
      for (int k = 0; k < kBatch; ++k) {
        const float l = lse_of(w0 + k);
        e[k] = l == -INFINITY ? 0.f : expf(l - m) * inv_z;
      }
      float4 v[kBatch][kQuadsPerWarp];
#pragma unroll
      for (int k = 0; k < kBatch; ++k) {
        const float4* sk = src0 + int64_t(b + (e[k] != 0.f ? w0 + k : w_first)) * slot_stride;
#pragma unroll
        for (int j = 0; j < kQuadsPerWarp; ++j) {
          const bool in = e[k] != 0.f && warp + kCombineWarps * j < nqb;
          v[k][j] = in ? sk[int64_t(kCombineWarps * j) * H] : make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int k = 0; k < kBatch; ++k)
#pragma unroll
        for (int j = 0; j < kQuadsPerWarp; ++j) {
          acc[j].x = fmaf(e[k], v[k][j].x, acc[j].x);
          acc[j].y = fmaf(e[k], v[k][j].y, acc[j].y);
          acc[j].z = fmaf(e[k], v[k][j].z, acc[j].z);
          acc[j].w = fmaf(e[k], v[k][j].w, acc[j].w);
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

// Many partials per sequence (few long sequences dealt over many workers):
// block = (sequence b, 32 heads, 8 four-column groups), and the 8 warps split
// the PARTIALS between them (warp k takes partials k, k + 8, ...) instead of
// the columns, so a sequence with 40 partials costs each thread about 5
// partial loads per column group.  The lse maximum and sum and the weighted
// column sums are then reduced across the warps through shared memory.
constexpr int kManyQuads = 8;

__global__ void __launch_bounds__(kCombineThreads, 2)
combine_many_kernel(const int32_t* __restrict__ seqlens, int64_t cap, int B, int H, int d_c, int W,
                    const float* __restrict__ o_part, const float* __restrict__ lse_part,
                    float* __restrict__ o_lat, float* __restrict__ lse_out) {
  __shared__ float4 s_acc[kCombineWarps][kCombineHeads][kManyQuads];
  __shared__ float s_red[kCombineWarps][kCombineHeads];
  __shared__ int64_t s_pre[2][kCombineWarps];
  pdl_wait();   // the partials come from the decode launched just before
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h0 = blockIdx.y * kCombineHeads;
  const int i = h0 + lane;
  const bool head_ok = i < H;
  const int nq = d_c / 4;
  const int q_base = blockIdx.z * kManyQuads;
  const int nqb = min(kManyQuads, nq - q_base);
  const int nh = min(kCombineHeads, H - h0);
  int64_t pre = 0, tot = 0;
  for (int bb = threadIdx.x; bb < B; bb += kCombineThreads) {
    const int64_t nu = units_of(clamp_len(seqlens[bb], cap));
    tot += nu;
    if (bb < b) pre += nu;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    pre += __shfl_xor_sync(0xffffffffu, pre, o);
    tot += __shfl_xor_sync(0xffffffffu, tot, o);
  }
  if (lane == 0) {
    s_pre[0][warp] = pre;
    s_pre[1][warp] = tot;
  }
  __syncthreads();
  pre = 0;
  tot = 0;
#pragma unroll
  for (int k = 0; k < kCombineWarps; ++k) {
    pre += s_pre[0][k];
    tot += s_pre[1][k];
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
  // The sequence's tiles are units [pre + kSwitchUnits, + nt) of the deal.
  const int w_first = int(worker_of_tile(pre + kSwitchUnits, T, W));
  const int w_last = int(worker_of_tile(pre + kSwitchUnits + nt - 1, T, W));
  // This warp's partials: w_first + warp + 8 j.  Their lse values, up to 8
  // per warp in registers (64 partials per sequence), the rest reloaded.
  auto lse_of = [&](int w) {
    const bool live = worker_tile_begin(w, T, W) != worker_tile_begin(w + 1, T, W);
    return (w <= w_last && head_ok && live) ? lse_part[int64_t(b + w) * H + i] : -INFINITY;
  };
  float lv[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) lv[j] = lse_of(w_first + warp + kCombineWarps * j);
  float m = -INFINITY;
#pragma unroll
  for (int j = 0; j < 8; ++j) m = fmaxf(m, lv[j]);
  for (int w = w_first + warp + 64; w <= w_last; w += kCombineWarps) m = fmaxf(m, lse_of(w));
  s_red[warp][lane] = m;
  __syncthreads();
  m = -INFINITY;
#pragma unroll
  for (int k = 0; k < kCombineWarps; ++k) m = fmaxf(m, s_red[k][lane]);
  float z = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) z += lv[j] == -INFINITY ? 0.f : expf(lv[j] - m);
  for (int w = w_first + warp + 64; w <= w_last; w += kCombineWarps) {
    const float l = lse_of(w);
    z += l == -INFINITY ? 0.f : expf(l - m);
  }
  __syncthreads();   // every warp has read s_red's maxima
  s_red[warp][lane] = z;
  __syncthreads();
  z = 0.f;
#pragma unroll
  for (int k = 0; k < kCombineWarps; ++k) z += s_red[k][lane];
  const float inv_z = head_ok && z > 0.f ? 1.f / z : 0.f;
  // Weighted column sums of this warp's partials, two partials per round.
  float4 acc[kManyQuads];
#pragma unroll
  for (int q = 0; q < kManyQuads; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
  const float4* src0 = reinterpret_cast<const float4*>(o_part) + int64_t(q_base) * H + i;
  const int64_t slot_stride = int64_t(nq) * H;   // float4 units
  for (int j0 = 0; w_first + warp + kCombineWarps * j0 <= w_last; j0 += 2) {
    float e[2];
    float4 v[2][kManyQuads];
#pragma unroll
    for (int jj = 0; jj < 2; ++jj) {
      const int j = j0 + jj;
      const int w = w_first + warp + kCombineWarps * j;
      const float l = j < 8 ? lv[j < 8 ? j : 0] : lse_of(w);
      e[jj] = (w > w_last || l == -INFINITY) ? 0.f : expf(l - m) * inv_z;
      const float4* sw = src0 + int64_t(b + (e[jj] != 0.f ? w : w_first)) * slot_stride;
#pragma unroll
      for (int q = 0; q < kManyQuads; ++q)
        v[jj][q] = (e[jj] != 0.f && q < nqb) ? sw[int64_t(q) * H] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int jj = 0; jj < 2; ++jj)
#pragma unroll
      for (int q = 0; q < kManyQuads; ++q) {
        acc[q].x = fmaf(e[jj], v[jj][q].x, acc[q].x);
        acc[q].y = fmaf(e[jj], v[jj][q].y, acc[q].y);
        acc[q].z = fmaf(e[jj], v[jj][q].z, acc[q].z);
        acc[q].w = fmaf(e[jj], v[jj][q].w, acc[q].w);
      }
  }
#pragma unroll
  for (int q = 0; q < kManyQuads; ++q) s_acc[warp][lane][q] = acc[q];
  __syncthreads();
  // Thread (head hh, group q), q fastest, so 8 threads write 128 contiguous bytes.
  const int hh = threadIdx.x / kManyQuads, q = threadIdx.x % kManyQuads;
  if (hh < nh && q < nqb) {
    float4 r = s_acc[0][hh][q];
#pragma unroll
    for (int k = 1; k < kCombineWarps; ++k) {
      const float4 a = s_acc[k][hh][q];
      r.x += a.x;
      r.y += a.y;
      r.z += a.z;
      r.w += a.w;
    }
    reinterpret_cast<float4*>(o_lat + (int64_t(b) * H + h0 + hh) * d_c)[q_base + q] = r;
  }
  if (blockIdx.z == 0 && warp == 0 && head_ok && lse_out) lse_out[int64_t(b) * H + i] = m + logf(z);
}

}  // namespace

cudaError_t launch_combine(const int32_t* seqlens, int64_t cap, int B, int H, int d_c, int W,
                           const float* o_part, const float* lse_part, float* o_lat,
                           float* lse, cudaStream_t stream) {
  const int nq = d_c / 4;
  const int hb = (H + kCombineHeads - 1) / kCombineHeads;
  // Many partials per sequence on average (few long sequences): the warps
  // split the partials.  Both are launched with programmatic overlap; the
  // decode before them triggers only by finishing, so the combine's launch
  // overlaps the decode's drain and nothing more.
  if (int64_t(B) + W - 1 > int64_t(kFastParts) * B)
    return launch_pdl(combine_many_kernel, dim3(B, hb, (nq + kManyQuads - 1) / kManyQuads),
                      dim3(kCombineThreads), 0, stream, seqlens, cap, B, H, d_c, W, o_part,
                      lse_part, o_lat, lse);
  return launch_pdl(combine_kernel, dim3(B, hb, (nq + kQuadsPerBlock - 1) / kQuadsPerBlock),
                    dim3(kCombineThreads), 0, stream, seqlens, cap, B, H, d_c, W, o_part, lse_part,
                    o_lat, lse);
}

}  // namespace mla
