// Value up-projection applied once, after the latent-space weighted sum:
//   out[b,i,v] = sum_c W_UV[i,v,c] * o_lat[b,i,c]
// ([MLA-とは] "Value側の吸収": o_{t,i} = W^UV_i (sum_j a_{tj,i} c^KV_j).)
//
// Bound by reading W_UV once (H * d_v * d_c elements).  Block = (head i,
// 16-sequence chunk); the chunk's o_lat rows are staged in shared memory, each
// warp takes rows v of W^UV_i, lanes stride over c (coalesced), and the warp
// reduces one fp32 accumulator per sequence.
#include "common.cuh"
#include "kernels.h"

namespace mla {

namespace {

constexpr int kOpWarps = 8;
constexpr int kOpBatch = 16;

template <typename T>
__global__ void __launch_bounds__(kOpWarps * 32)
out_proj_kernel(const float* __restrict__ o_lat, const T* __restrict__ W_UV, int B, int H,
                int d_c, int d_v, T* __restrict__ out) {
  extern __shared__ float s_o[];  // [kOpBatch][d_c]
  const int i = blockIdx.x;
  const int b0 = blockIdx.y * kOpBatch;
  const int nb = min(kOpBatch, B - b0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int idx = threadIdx.x; idx < nb * d_c; idx += blockDim.x) {
    const int bb = idx / d_c, c = idx % d_c;
    s_o[idx] = o_lat[(int64_t(b0 + bb) * H + i) * d_c + c];
  }
  __syncthreads();
  for (int v = warp; v < d_v; v += kOpWarps) {
    const T* w = W_UV + (int64_t(i) * d_v + v) * d_c;
    float acc[kOpBatch];
#pragma unroll
    for (int bb = 0; bb < kOpBatch; ++bb) acc[bb] = 0.f;
    for (int c = lane; c < d_c; c += 32) {
      const float wv = Storage<T>::to_f(w[c]);
#pragma unroll
      for (int bb = 0; bb < kOpBatch; ++bb) acc[bb] = fmaf(wv, s_o[bb * d_c + c], acc[bb]);
    }
#pragma unroll
    for (int bb = 0; bb < kOpBatch; ++bb) {
      const float r = warp_sum(acc[bb]);
      if (lane == 0 && bb < nb)
        out[(int64_t(b0 + bb) * H + i) * d_v + v] = Storage<T>::from_f(r);
    }
  }
}

}  // namespace

template <typename T>
cudaError_t launch_out_proj(const float* o_lat, const T* W_UV, int B, int H, int d_c,
                            int d_v, T* out, cudaStream_t stream) {
  const size_t smem = sizeof(float) * size_t(kOpBatch) * d_c;
  auto kern = out_proj_kernel<T>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(smem));
    if (e != cudaSuccess) return e;
  }
  dim3 grid(H, (B + kOpBatch - 1) / kOpBatch);
  kern<<<grid, kOpWarps * 32, smem, stream>>>(o_lat, W_UV, B, H, d_c, d_v, out);
  return cudaGetLastError();
}

template cudaError_t launch_out_proj<float>(const float*, const float*, int, int, int, int,
                                            float*, cudaStream_t);
template cudaError_t launch_out_proj<__nv_bfloat16>(const float*, const __nv_bfloat16*, int,
                                                    int, int, int, __nv_bfloat16*,
                                                    cudaStream_t);

}  // namespace mla
