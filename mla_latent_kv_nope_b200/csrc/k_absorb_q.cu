// Query absorption: q_cat[b,i] = [ W^UK_i^T q^C_{b,i} ; RoPE(q^R_{b,i}, q_pos[b]) ]
// ([MLA-とは] "行列吸収": q~ := W^UK_i^T q in R^{d_c}, built once per step;
//  "Decoupled RoPE": the decoupled query is rotated at its position.)
//
// The pass is bound by reading W_UK once (H * d_nope * d_c elements).  Block
// = (head i, 128-column slab of d_c, 16-sequence batch chunk): the slab of
// W^UK_i is streamed row by row with one column per thread (coalesced), the
// chunk's q^C rows sit in shared memory, and each thread keeps one fp32
// accumulator per sequence.  The column-slab-0 blocks also write the rotated
// RoPE block.
#include "common.cuh"
#include "kernels.h"

namespace mla {

namespace {

constexpr int kAbsCols = 128;
constexpr int kAbsBatch = 16;

template <typename T>
__global__ void __launch_bounds__(kAbsCols)
absorb_q_kernel(const T* __restrict__ q_nope, const T* __restrict__ q_pe,
                const T* __restrict__ W_UK, const int32_t* __restrict__ q_pos,
                float rope_base, int B, int H, int d_c, int d_r, int d_n,
                T* __restrict__ q_cat) {
  extern __shared__ float s_q[];  // [kAbsBatch][d_n]
  const int i = blockIdx.x;
  const int col = blockIdx.y * kAbsCols + threadIdx.x;
  const int b0 = blockIdx.z * kAbsBatch;
  const int nb = min(kAbsBatch, B - b0);
  const int R = d_c + d_r;

  for (int idx = threadIdx.x; idx < nb * d_n; idx += blockDim.x) {
    const int bb = idx / d_n, r = idx % d_n;
    s_q[idx] = Storage<T>::to_f(q_nope[(int64_t(b0 + bb) * H + i) * d_n + r]);
  }
  __syncthreads();

  if (col < d_c) {
    float acc[kAbsBatch];
#pragma unroll
    for (int bb = 0; bb < kAbsBatch; ++bb) acc[bb] = 0.f;
    const T* w = W_UK + int64_t(i) * d_n * d_c + col;
    for (int r = 0; r < d_n; ++r) {
      const float wv = Storage<T>::to_f(w[int64_t(r) * d_c]);
#pragma unroll
      for (int bb = 0; bb < kAbsBatch; ++bb) acc[bb] = fmaf(s_q[bb * d_n + r], wv, acc[bb]);
    }
#pragma unroll
    for (int bb = 0; bb < kAbsBatch; ++bb)
      if (bb < nb) q_cat[(int64_t(b0 + bb) * H + i) * R + col] = Storage<T>::from_f(acc[bb]);
  }

  if (blockIdx.y == 0) {
    const int half = d_r / 2;
    for (int idx = threadIdx.x; idx < nb * half; idx += blockDim.x) {
      const int bb = idx / half, k = idx % half;
      const int64_t row = (int64_t(b0 + bb) * H + i);
      const float x1 = Storage<T>::to_f(q_pe[row * d_r + k]);
      const float x2 = Storage<T>::to_f(q_pe[row * d_r + k + half]);
      float y1 = x1, y2 = x2;
      if (q_pos) {
        float c, s;
        rope_cos_sin(q_pos[b0 + bb], k, d_r, rope_base, &c, &s);
        y1 = x1 * c - x2 * s;
        y2 = x1 * s + x2 * c;
      }
      q_cat[row * R + d_c + k] = Storage<T>::from_f(y1);
      q_cat[row * R + d_c + k + half] = Storage<T>::from_f(y2);
    }
  }
}

}  // namespace

template <typename T>
cudaError_t launch_absorb_q(const T* q_nope, const T* q_pe, const T* W_UK,
                            const int32_t* q_pos, float rope_base, int B, int H, int d_c,
                            int d_r, int d_n, T* q_cat, cudaStream_t stream) {
  const size_t smem = sizeof(float) * size_t(kAbsBatch) * d_n;
  auto kern = absorb_q_kernel<T>;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(smem));
    if (e != cudaSuccess) return e;
  }
  dim3 grid(H, (d_c + kAbsCols - 1) / kAbsCols, (B + kAbsBatch - 1) / kAbsBatch);
  kern<<<grid, kAbsCols, smem, stream>>>(q_nope, q_pe, W_UK, q_pos, rope_base, B, H, d_c,
                                         d_r, d_n, q_cat);
  return cudaGetLastError();
}

template cudaError_t launch_absorb_q<float>(const float*, const float*, const float*,
                                            const int32_t*, float, int, int, int, int, int,
                                            float*, cudaStream_t);
template cudaError_t launch_absorb_q<__nv_bfloat16>(const __nv_bfloat16*,
                                                    const __nv_bfloat16*,
                                                    const __nv_bfloat16*, const int32_t*,
                                                    float, int, int, int, int, int,
                                                    __nv_bfloat16*, cudaStream_t);

}  // namespace mla
