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
constexpr int kFastParts = 4;        // partials per sequence on average: above, warps split them

// Online log-sum-exp accumulation of a round of up to kRound partials: the
// running maximum m, sum z and unnormalised column sums acc are rescaled when
// the maximum grows, so the lse values and the columns of a round are loaded
// together (one memory round trip per round instead of an lse pass first).
constexpr int kRound = 4;

template <int kQ>
__device__ __forceinline__ void lse_round(const float (&lv)[kRound], const float4 (&v)[kRound][kQ],
                                          float& m, float& z, float4 (&acc)[kQ]) {
  float mb = -INFINITY;
#pragma unroll
  for (int k = 0; k < kRound; ++k) mb = fmaxf(mb, lv[k]);
  const float m_new = fmaxf(m, mb);
  if (m_new == -INFINITY) return;   // nothing live yet
  if (m_new != m) {
    const float sc = m == -INFINITY ? 0.f : expf(m - m_new);
    z *= sc;
#pragma unroll
    for (int q = 0; q < kQ; ++q) {
      acc[q].x *= sc;
      acc[q].y *= sc;
      acc[q].z *= sc;
      acc[q].w *= sc;
    }
    m = m_new;
  }
#pragma unroll
  for (int k = 0; k < kRound; ++k) {
    const float e = lv[k] == -INFINITY ? 0.f : expf(lv[k] - m);
    z += e;
#pragma unroll
    for (int q = 0; q < kQ; ++q) {
      acc[q].x = fmaf(e, v[k][q].x, acc[q].x);
      acc[q].y = fmaf(e, v[k][q].y, acc[q].y);
      acc[q].z = fmaf(e, v[k][q].z, acc[q].z);
      acc[q].w = fmaf(e, v[k][q].w, acc[q].w);
    }
  }
}

// The partials are dead once this kernel has read them: its loads mark their
// L2 lines evict-first (the decode stored them evict-last so that they would
// wait in L2 for this kernel), so they leave L2 before any other data.
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ float4 ld_last_use(const float4* p, uint64_t policy) {
  float4 v;
  asm volatile("ld.global.L2::cache_hint.v4.f32 {%0, %1, %2, %3}, [%4], %5;"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p), "l"(policy));
  return v;
}
__device__ __forceinline__ float ld_last_use(const float* p, uint64_t policy) {
  float v;
  asm volatile("ld.global.L2::cache_hint.f32 %0, [%1], %2;" : "=f"(v) : "l"(p), "l"(policy));
  return v;
}

// Units before sequence b and in the whole batch (every thread of the block
// takes part; one round trip over the lengths).
__device__ __forceinline__ void unit_prefix(const int32_t* seqlens, int64_t cap, int B, int b,
                                            int64_t (&s_red)[2][kCombineWarps], int64_t& pre,
                                            int64_t& tot) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pre = 0;
  tot = 0;
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
}

// Block = (sequence b, 32 heads, 128 columns).  The partials are stored as
// o_part[slot][d_c / 4][H][4], so a warp load of one 4-column group for 32
// consecutive heads is one contiguous 512-byte read.  Each thread owns one
// head (its lane) and 4 column groups; per round it loads the lse values and
// the column groups of up to four partials (for most batches every partial of
// the sequence: one round).  The merged block goes through shared memory so
// o_lat rows are written with coalesced stores.
constexpr int kQuadsPerWarp = 4;
constexpr int kQuadsPerBlock = kCombineWarps * kQuadsPerWarp;   // 128 columns

__global__ void __launch_bounds__(kCombineThreads, 2)
combine_kernel(const int32_t* __restrict__ seqlens, int64_t cap, int B, int H, int d_c, int W,
               const float* __restrict__ o_part, const float* __restrict__ lse_part,
               float* __restrict__ o_lat, float* __restrict__ lse_out) {
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
  int64_t pre, T;
  unit_prefix(seqlens, cap, B, b, s_red, pre, T);
  const int64_t nt = tiles_of(clamp_len(seqlens[b], cap));
  if (nt == 0) {
    for (int idx = threadIdx.x; idx < nh * nqb; idx += kCombineThreads)
      reinterpret_cast<float4*>(o_lat + (int64_t(b) * H + h0 + idx / nqb) * d_c)[q_base + idx % nqb] =
          make_float4(0.f, 0.f, 0.f, 0.f);
    if (blockIdx.z == 0 && warp == 0 && head_ok && lse_out) lse_out[int64_t(b) * H + i] = -INFINITY;
    return;
  }
  // The sequence's tiles are units [pre + kSwitchUnits, + nt) of the deal;
  // a worker with an empty unit range (only when T < W) holds no partial.
  const int w_first = int(worker_of_tile(pre + kSwitchUnits, T, W));
  const int w_last = int(worker_of_tile(pre + kSwitchUnits + nt - 1, T, W));
  auto live = [&](int w) {
    return T >= W || worker_tile_begin(w, T, W) != worker_tile_begin(w + 1, T, W);
  };
  // Column groups of this thread: q_base + warp + 8 j, j < 4.
  const float4* src0 = reinterpret_cast<const float4*>(o_part) + int64_t(q_base + warp) * H + i;
  const int64_t slot_stride = int64_t(nq) * H;   // float4 units
  const uint64_t dead = l2_policy_evict_first();
  float4 acc[kQuadsPerWarp];
#pragma unroll
  for (int j = 0; j < kQuadsPerWarp; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
  float m = -INFINITY, z = 0.f;
  for (int w0 = w_first; w0 <= w_last; w0 += kRound) {
    float lv[kRound];
    float4 v[kRound][kQuadsPerWarp];
#pragma unroll
    for (int k = 0; k < kRound; ++k) {
      const int w = w0 + k;
      const bool use = w <= w_last && head_ok && live(w);
      lv[k] = use ? ld_last_use(lse_part + int64_t(b + w) * H + i, dead) : -INFINITY;
      const float4* sk = src0 + int64_t(b + (use ? w : w_first)) * slot_stride;
#pragma unroll
      for (int j = 0; j < kQuadsPerWarp; ++j)
        v[k][j] = (use && warp + kCombineWarps * j < nqb)
                      ? ld_last_use(sk + int64_t(kCombineWarps * j) * H, dead)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    lse_round(lv, v, m, z, acc);
  }
  const float inv_z = head_ok && z > 0.f ? 1.f / z : 0.f;
#pragma unroll
  for (int j = 0; j < kQuadsPerWarp; ++j)
    s_rows[lane][warp + kCombineWarps * j] =
        make_float4(acc[j].x * inv_z, acc[j].y * inv_z, acc[j].z * inv_z, acc[j].w * inv_z);
  __syncthreads();
  for (int idx = threadIdx.x; idx < nh * nqb; idx += kCombineThreads) {
    const int hh = idx / nqb, q = idx % nqb;
    reinterpret_cast<float4*>(o_lat + (int64_t(b) * H + h0 + hh) * d_c)[q_base + q] = s_rows[hh][q];
  }
  if (blockIdx.z == 0 && warp == 0 && head_ok && lse_out) lse_out[int64_t(b) * H + i] = m + logf(z);
}

// Many partials per sequence (few long sequences dealt over many workers):
// block = (sequence b, 32 heads, 4 four-column groups), and the 8 warps split
// the PARTIALS between them (warp k takes partials k, k + 8, ...) instead of
// the columns, four per round, so a sequence with 40 partials costs each
// thread two rounds of loads.  Each warp keeps its own running maximum, sum
// and column sums; the warps' results are rescaled to the common maximum and
// summed through shared memory.
constexpr int kManyQuads = 4;

__global__ void __launch_bounds__(kCombineThreads, 2)
combine_many_kernel(const int32_t* __restrict__ seqlens, int64_t cap, int B, int H, int d_c, int W,
                    const float* __restrict__ o_part, const float* __restrict__ lse_part,
                    float* __restrict__ o_lat, float* __restrict__ lse_out) {
  __shared__ float4 s_acc[kCombineWarps][kCombineHeads][kManyQuads];
  __shared__ float s_m[kCombineWarps][kCombineHeads];
  __shared__ float s_z[kCombineWarps][kCombineHeads];
  __shared__ int64_t s_red[2][kCombineWarps];
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
  int64_t pre, T;
  unit_prefix(seqlens, cap, B, b, s_red, pre, T);
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
  auto live = [&](int w) {
    return T >= W || worker_tile_begin(w, T, W) != worker_tile_begin(w + 1, T, W);
  };
  const float4* src0 = reinterpret_cast<const float4*>(o_part) + int64_t(q_base) * H + i;
  const int64_t slot_stride = int64_t(nq) * H;   // float4 units
  const uint64_t dead = l2_policy_evict_first();
  float4 acc[kManyQuads];
#pragma unroll
  for (int q = 0; q < kManyQuads; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
  float m = -INFINITY, z = 0.f;
  for (int w0 = w_first + warp; w0 <= w_last; w0 += kRound * kCombineWarps) {
    float lv[kRound];
    float4 v[kRound][kManyQuads];
#pragma unroll
    for (int k = 0; k < kRound; ++k) {
      const int w = w0 + kCombineWarps * k;
      const bool use = w <= w_last && head_ok && live(w);
      lv[k] = use ? ld_last_use(lse_part + int64_t(b + w) * H + i, dead) : -INFINITY;
      const float4* sw = src0 + int64_t(b + (use ? w : w_first)) * slot_stride;
#pragma unroll
      for (int q = 0; q < kManyQuads; ++q)
        v[k][q] = (use && q < nqb) ? ld_last_use(sw + int64_t(q) * H, dead)
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    lse_round(lv, v, m, z, acc);
  }
  s_m[warp][lane] = m;
  s_z[warp][lane] = z;
#pragma unroll
  for (int q = 0; q < kManyQuads; ++q) s_acc[warp][lane][q] = acc[q];
  __syncthreads();
  // Thread (head hh, group q), q fastest, so 4 threads write 64 contiguous bytes.
  const int hh = threadIdx.x / kManyQuads, q = threadIdx.x % kManyQuads;
  if (hh < nh) {
    float mx = -INFINITY;
#pragma unroll
    for (int k = 0; k < kCombineWarps; ++k) mx = fmaxf(mx, s_m[k][hh]);
    float zz = 0.f;
    float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int k = 0; k < kCombineWarps; ++k) {
      const float mk = s_m[k][hh];
      const float sc = mk == -INFINITY ? 0.f : expf(mk - mx);
      zz = fmaf(s_z[k][hh], sc, zz);
      const float4 a = s_acc[k][hh][q];
      r.x = fmaf(a.x, sc, r.x);
      r.y = fmaf(a.y, sc, r.y);
      r.z = fmaf(a.z, sc, r.z);
      r.w = fmaf(a.w, sc, r.w);
    }
    const float inv = zz > 0.f ? 1.f / zz : 0.f;
    if (q < nqb)
      reinterpret_cast<float4*>(o_lat + (int64_t(b) * H + h0 + hh) * d_c)[q_base + q] =
          make_float4(r.x * inv, r.y * inv, r.z * inv, r.w * inv);
    if (blockIdx.z == 0 && q == 0 && lse_out) lse_out[int64_t(b) * H + h0 + hh] = mx + logf(zz);
  }
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
  // overlaps the decode's drain and nothing more.  Early triggers measured
  // slower on B200: in the decode 1.5 us per v3 step; in the combine (so
  // that out_proj could load its weight during the combine's tail) 2.5 us
  // faster on the v3 step but 7.5 us slower on the v2-lite step and 4 us
  // slower per decode + combine pair run back to back.
  if (int64_t(B) + W - 1 > int64_t(kFastParts) * B)
    return launch_pdl(combine_many_kernel, dim3(B, hb, (nq + kManyQuads - 1) / kManyQuads),
                      dim3(kCombineThreads), 0, stream, seqlens, cap, B, H, d_c, W, o_part,
                      lse_part, o_lat, lse);
  return launch_pdl(combine_kernel, dim3(B, hb, (nq + kQuadsPerBlock - 1) / kQuadsPerBlock),
                    dim3(kCombineThreads), 0, stream, seqlens, cap, B, H, d_c, W, o_part, lse_part,
                    o_lat, lse);
}

}  // namespace mla
