// Split-KV latent decode on CUDA cores (fp32 path; any d_c, d_r within the
// header's limits).
//
// Computes, per sequence b and head i, over the keys of one work range:
//   s_j = scale * (q_cat[b,i] . row_j),  online softmax, o = sum_j p_j row_j[0:d_c]
// ([MLA-とは] "実装上のトレードオフ": the absorbed decode is MQA whose shared key
// is the latent row and whose shared value is its first d_c entries.)
//
// Block = (worker w, head group).  One warp per head; the block stages 32 key
// rows at a time in shared memory (fp32, rows padded by one word so that lane j
// reading row j is conflict-free), then every warp scores its head against
// them and folds them into its running (max, sum, accumulator).
#include "common.cuh"
#include "kernels.h"

namespace mla {

namespace {

constexpr int kSimtHeads = 8;   // heads (warps) per block
constexpr int kSimtKeys = 32;   // keys staged per step
constexpr int kMaxAccPerLane = 32;  // d_c <= 1024

template <typename T>
__global__ void __launch_bounds__(kSimtHeads * 32)
decode_simt_kernel(const T* __restrict__ q_cat, const T* __restrict__ cache, const PageMap pm,
                   const int32_t* __restrict__ seqlens, int B, int H, int d_c,
                   int R, int64_t cap, float scale, int W,
                   float* __restrict__ o_part, float* __restrict__ lse_part,
                   int* __restrict__ status) {
  extern __shared__ float smem[];
  const int ldr = R + 1;
  float* s_rows = smem;                          // [kSimtKeys][R+1]
  float* s_q = s_rows + kSimtKeys * ldr;         // [kSimtHeads][R]

  const int w = blockIdx.x;
  const int h0 = blockIdx.y * kSimtHeads;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int head = h0 + warp;

  // Total work units T (tiles plus each sequence's start-up units, as the
  // tensor-core kernels deal them) and this worker's unit range.
  int64_t n_tiles = 0;
  for (int b = 0; b < B; ++b) {
    n_tiles += units_of(clamp_len(seqlens[b], cap));
    if (w == 0 && blockIdx.y == 0 && threadIdx.x == 0 && int64_t(seqlens[b]) > cap)
      record_status(status, MLA_ERR_BOUNDS);
  }
  if (n_tiles == 0) return;
  const int64_t t_begin = worker_tile_begin(w, n_tiles, W);
  const int64_t t_end = worker_tile_begin(w + 1, n_tiles, W);
  if (t_begin >= t_end) return;

  // Walk the sequences whose tiles overlap [t_begin, t_end).
  int64_t prefix = 0;
  for (int b = 0; b < B && prefix < t_end; ++b) {
    const int64_t L = clamp_len(seqlens[b], cap);
    const int64_t nt = tiles_of(L);
    const int64_t r0 = prefix + kSwitchUnits;   // this sequence's first tile
    const int64_t lo_t = max(r0, t_begin), hi_t = min(r0 + nt, t_end);
    if (nt > 0 && lo_t < hi_t) {
      const int64_t key_lo = (lo_t - r0) * kTileKeys;
      const int64_t key_hi = min((hi_t - r0) * int64_t(kTileKeys), L);

      // Stage this block's queries.
      __syncthreads();
      for (int idx = threadIdx.x; idx < kSimtHeads * R; idx += blockDim.x) {
        const int hh = h0 + idx / R;
        s_q[idx] = hh < H ? Storage<T>::to_f(q_cat[(int64_t(b) * H + hh) * R + idx % R]) : 0.f;
      }
      float m = -INFINITY, l = 0.f;
      float acc[kMaxAccPerLane];
#pragma unroll
      for (int k = 0; k < kMaxAccPerLane; ++k) acc[k] = 0.f;

      for (int64_t k0 = key_lo; k0 < key_hi; k0 += kSimtKeys) {
        const int nk = int(min(int64_t(kSimtKeys), key_hi - k0));
        __syncthreads();
        for (int idx = threadIdx.x; idx < nk * R; idx += blockDim.x) {
          const int j = idx / R, c = idx % R;
          const int64_t r = pm.row(b, k0 + j);   // -1: page id outside the pool
          if (r < 0 && c == 0) record_status(status, MLA_ERR_BOUNDS);
          s_rows[j * ldr + c] = r < 0 ? 0.f : Storage<T>::to_f(cache[r * R + c]);
        }
        __syncthreads();
        // Score: lane j takes key j.
        float s = -INFINITY;
        if (lane < nk) {
          const float* q = s_q + warp * R;
          const float* r = s_rows + lane * ldr;
          float a = 0.f;
          for (int c = 0; c < R; ++c) a = fmaf(q[c], r[c], a);
          s = a * scale;
        }
        const float m_new = fmaxf(m, warp_max(s));
        const float p = lane < nk ? expf(s - m_new) : 0.f;
        const float alpha = expf(m - m_new);  // m = -inf on the first step -> 0
        l = l * alpha + warp_sum(p);
        m = m_new;
#pragma unroll
        for (int k = 0; k < kMaxAccPerLane; ++k) acc[k] *= alpha;
        for (int j = 0; j < nk; ++j) {
          const float pj = __shfl_sync(0xffffffffu, p, j);
          const float* r = s_rows + j * ldr;
#pragma unroll
          for (int k = 0; k < kMaxAccPerLane; ++k) {
            const int c = lane + 32 * k;
            if (c < d_c) acc[k] = fmaf(pj, r[c], acc[k]);
          }
        }
      }
      if (head < H) {
        const int slot = b + w;
        const float inv_l = 1.f / l;
        // Partials are o_part[slot][d_c / 4][H][4].
        float* o = o_part + int64_t(slot) * d_c * H + int64_t(head) * 4;
#pragma unroll
        for (int k = 0; k < kMaxAccPerLane; ++k) {
          const int c = lane + 32 * k;
          if (c < d_c) o[int64_t(c >> 2) * H * 4 + (c & 3)] = acc[k] * inv_l;
        }
        if (lane == 0) lse_part[int64_t(slot) * H + head] = m + logf(l);
      }
    }
    prefix += units_of(L);
  }
}

}  // namespace

template <typename T>
cudaError_t launch_decode_simt(const T* q_cat, const T* cache, const PageMap& pm,
                               const int32_t* seqlens,
                               int B, int H, int d_c, int d_r, int64_t cap,
                               float scale, int W, float* o_part, float* lse_part,
                               int* status, cudaStream_t stream) {
  const int R = d_c + d_r;
  const size_t smem = sizeof(float) * (size_t(kSimtKeys) * (R + 1) + size_t(kSimtHeads) * R);
  auto kern = decode_simt_kernel<T>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(W, (H + kSimtHeads - 1) / kSimtHeads);
  kern<<<grid, kSimtHeads * 32, smem, stream>>>(q_cat, cache, pm, seqlens, B, H, d_c, R,
                                                 cap, scale, W, o_part, lse_part, status);
  return cudaGetLastError();
}

template cudaError_t launch_decode_simt<float>(const float*, const float*, const PageMap&,
                                               const int32_t*,
                                               int, int, int, int, int64_t, float, int,
                                               float*, float*, int*, cudaStream_t);
template cudaError_t launch_decode_simt<__nv_bfloat16>(const __nv_bfloat16*,
                                                       const __nv_bfloat16*, const PageMap&,
                                                       const int32_t*,
                                                       int, int, int, int, int64_t, float,
                                                       int, float*, float*, int*,
                                                       cudaStream_t);

size_t decode_simt_smem_bytes(int d_c, int d_r) {
  const int R = d_c + d_r;
  return sizeof(float) * (size_t(kSimtKeys) * (R + 1) + size_t(kSimtHeads) * R);
}

}  // namespace mla
