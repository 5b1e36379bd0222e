// W^O folded into the value side ([MLA-とは] "Value側の吸収": W^UV_i can be
// absorbed into the output projection, B_i = W^O_i W^UV_i, so the latent-space
// weighted sums go straight to the model width: u = sum_i B_i o_lat_i).
//
//   fold      W_fold[m, i d_c + c] = sum_v W_O[m, i d_v + v] W_UV[i, v, c]
//             one CTA per (128 rows of m, head i, 256 columns c): A = W_O rows
//             (K-major, K = d_v = 128), B = W_UV[i] (MN-major), 8 MMAs.
//   folded    u[b, m] = sum_k W_fold[m, k] o_lat[b, k],  k = i d_c + c
//   projection   weight streaming: CTA = (128 rows of m, one of S slices of
//             K), W_fold tiles [128 x 64] and o_lat (bf16) tiles [N x 64]
//             through a TMA ring, the accumulator in tensor memory; each CTA
//             writes an fp32 partial that a second kernel sums in a fixed
//             order (deterministic).
// o_lat is rounded to bf16 once for the tensor-core operand (as out_proj does).
// Every wait is bounded; on give-up a kernel records MLA_ERR_DEVICE_TIMEOUT,
// drains what it issued and skips its stores.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace mla {

namespace {

using namespace sm100;

constexpr int kThr = 128;

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  const __nv_bfloat162 p = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&p);
}

__device__ __forceinline__ bool wait_all(uint64_t* bar, uint32_t parity) {
  volatile int no_abort = 0;
  return mbar_wait(bar, parity, &no_abort, kWaitLimitCycles);
}

// ---------------------------------------------------------------------------
// fold: smem A 2 x [128 x 128 B] (32 KB) | B 4 x [128 (K) x 128 B] (64 KB)
constexpr size_t kFoldSmem = 2 * 16384 + 4 * 16384 + 64 + 1024;

__global__ void __launch_bounds__(kThr, 1)
fold_weights_tc_kernel(const __grid_constant__ CUtensorMap tm_wo,
                       const __grid_constant__ CUtensorMap tm_wuv, int d_model, int H,
                       __nv_bfloat16* __restrict__ w_fold, int* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint8_t* sA = sm;
  uint8_t* sB = sm + 2 * 16384;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + 4 * 16384);
  uint32_t* tbase = reinterpret_cast<uint32_t*>(bars + 2);
  const int m0 = blockIdx.x * 128, i = blockIdx.y, half = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(&bars[0], 6 * 16384);
    for (int kc = 0; kc < 2; ++kc)   // W_O rows m0.., columns of head i (K = d_v)
      tma_load_2d(&tm_wo, &bars[0], sA + kc * 16384, i * 128 + kc * 64, m0);
    for (int c = 0; c < 4; ++c)      // W_UV[i] rows (K), 64 of the 256 output columns each
      tma_load_2d(&tm_wuv, &bars[0], sB + c * 16384, half * 256 + c * 64, i * 128);
  }
  if (warp == 0) {
    tmem_alloc(tbase, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tbase;
  bool ok = wait_all(&bars[0], 0);
  if (warp == 0) ok = __all_sync(0xffffffffu, ok);   // the issuing warp decides as one
  if (warp == 0 && ok) {
    tc_fence_after();
    constexpr uint32_t idesc = idesc_bf16_f32(128, 256, false, true);
    const uint64_t a0 = smem_desc_sw128(smem_u32(sA), 16, 1024);
    const uint64_t b0 = smem_desc_sw128(smem_u32(sB), 16384, 1024);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks)
      mma_bf16_ss_w(tmem, a0 + uint64_t(((ks / 4) * 16384 + (ks % 4) * 32) >> 4),
                    b0 + uint64_t((ks * 2048) >> 4), idesc, ks != 0);
  }
  if (warp == 0) mma_commit_w(&bars[1]);   // no MMA issued: arrives at once
  ok = wait_all(&bars[1], 0) && ok;
  tc_fence_after();
  const int m = m0 + 32 * warp + lane;
  __nv_bfloat16* dst = w_fold + int64_t(m) * H * 512 + int64_t(i) * 512 + half * 256;
#pragma unroll 1
  for (int c0 = 0; c0 < 256; c0 += 32) {
    uint32_t r[32];
    tmem_ld32(tmem + (uint32_t(32 * warp) << 16) + uint32_t(c0), r);
    tmem_wait_ld();
    if (ok && m < d_model) {
#pragma unroll
      for (int e = 0; e < 32; e += 8) {
        uint4 v;
        v.x = pack_bf16x2(__uint_as_float(r[e]), __uint_as_float(r[e + 1]));
        v.y = pack_bf16x2(__uint_as_float(r[e + 2]), __uint_as_float(r[e + 3]));
        v.z = pack_bf16x2(__uint_as_float(r[e + 4]), __uint_as_float(r[e + 5]));
        v.w = pack_bf16x2(__uint_as_float(r[e + 6]), __uint_as_float(r[e + 7]));
        *reinterpret_cast<uint4*>(dst + c0 + e) = v;
      }
    }
  }
  if (!ok && threadIdx.x == 0) {
    record_status(status, MLA_ERR_DEVICE_TIMEOUT);
    wait_all(&bars[0], 0);   // the loads land before the shared memory is released
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ---------------------------------------------------------------------------
// o_lat fp32 -> bf16 (the tensor-core operand of the folded projection).
__global__ void to_bf16_kernel(const float4* __restrict__ x, uint2* __restrict__ y, int64_t n4) {
  for (int64_t k = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; k < n4;
       k += int64_t(gridDim.x) * blockDim.x) {
    const float4 v = x[k];
    y[k] = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
  }
}

// ---------------------------------------------------------------------------
// Folded projection: stage = A [128 x 128 B] (16 KB) + X [Np x 128 B].
constexpr int kFpStages = 4;   // 4 x 24 KB: two CTAs fit on an SM

__host__ __device__ constexpr size_t fp_stage_bytes(int np) { return 16384 + size_t(np) * 128; }

__global__ void __launch_bounds__(kThr, 1)
folded_proj_tc_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                      int d_model, int n, int np, int64_t k_chunks, int splits,
                      float* __restrict__ part, int* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  const size_t stage_bytes = fp_stage_bytes(np);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kFpStages * stage_bytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + kFpStages;
  uint64_t* done = bars + 2 * kFpStages;
  uint32_t* tbase = reinterpret_cast<uint32_t*>(bars + 2 * kFpStages + 1);
  const int m0 = blockIdx.x * 128, split = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t c_begin = (int64_t(split) * k_chunks) / splits;
  const int64_t c_end = (int64_t(split + 1) * k_chunks) / splits;
  const int nc = int(c_end - c_begin);
  uint32_t tcols = 32;
  while (tcols < uint32_t(np)) tcols <<= 1;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kFpStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == 0) {
    tmem_alloc(tbase, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tbase;
  __shared__ int s_abort;
  if (threadIdx.x == 0) s_abort = 0;
  __syncthreads();
  volatile int* abort_flag = &s_abort;
  bool ok = true;
  uint32_t issued = 0;
  if (warp == 1) {
    // producer (one lane)
    if (lane == 0) {
      for (int j = 0; j < nc; ++j) {
        const int s = j % kFpStages;
        if (j >= kFpStages &&
            !(ok = mbar_wait(&empty[s], ((j / kFpStages) - 1) & 1, abort_flag, kWaitLimitCycles)))
          break;
        uint8_t* st = sm + s * stage_bytes;
        mbar_arrive_expect_tx(&full[s], uint32_t(stage_bytes));
        const int32_t kx = int32_t((c_begin + j) * 64);
        tma_load_2d(&tm_w, &full[s], st, kx, m0);
        tma_load_2d(&tm_x, &full[s], st + 16384, kx, 0);
        ++issued;
      }
      if (!ok) *abort_flag = 1;
    }
  } else if (warp == 0) {
    // MMA issuer (the whole warp waits; elect.sync issues)
    const uint32_t idesc = idesc_bf16_f32(128, np, false, false);
    for (int j = 0; j < nc; ++j) {
      const int s = j % kFpStages;
      bool got = mbar_try(&full[s], (j / kFpStages) & 1);
      if (!__all_sync(0xffffffffu, got)) {
        got = mbar_wait(&full[s], (j / kFpStages) & 1, abort_flag, kWaitLimitCycles);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          if (lane == 0) *abort_flag = 1;
          break;
        }
      }
      tc_fence_after();
      const uint32_t st = smem_u32(sm + s * stage_bytes);
      const uint64_t a0 = smem_desc_sw128(st, 16, 1024);
      const uint64_t b0 = smem_desc_sw128(st + 16384, 16, 1024);
#pragma unroll
      for (int k = 0; k < 4; ++k)
        mma_bf16_ss_w(tmem, a0 + uint64_t((k * 32) >> 4), b0 + uint64_t((k * 32) >> 4), idesc,
                      (j | k) != 0);
      mma_commit_w(&empty[s]);
    }
    mma_commit_w(done);
  }
  __syncthreads();
  ok = wait_all(done, 0) && ok && !*abort_flag;
  tc_fence_after();
  // D[m][n]: thread (warp w, lane t) holds row m0 + 32w + t.
  const int m = m0 + 32 * warp + lane;
#pragma unroll 1
  for (int c0 = 0; c0 < np; c0 += 32) {
    uint32_t r[32];
    tmem_ld32(tmem + (uint32_t(32 * warp) << 16) + uint32_t(c0), r);
    tmem_wait_ld();
    if (ok && m < d_model) {
#pragma unroll
      for (int e = 0; e < 32; ++e)
        if (c0 + e < n)
          part[(int64_t(split) * n + c0 + e) * d_model + m] = nc > 0 ? __uint_as_float(r[e]) : 0.f;
    }
  }
  if (!ok && threadIdx.x == 0) record_status(status, MLA_ERR_DEVICE_TIMEOUT);
  // Loads issued but never consumed land before the shared memory is released.
  if (warp == 1 && lane == 0) {
    volatile int no_abort = 0;
    for (uint32_t k = issued > kFpStages ? issued - kFpStages : 0; k < issued; ++k)
      mbar_wait(&full[k % kFpStages], (k / kFpStages) & 1, &no_abort, kWaitLimitCycles);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, tcols);
  }
}

// u[b, m] = sum over splits of part[s][b][m], in split order.
__global__ void reduce_splits_kernel(const float* __restrict__ part, int splits, int64_t nm,
                                     __nv_bfloat16* __restrict__ u) {
  for (int64_t k = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; k < nm;
       k += int64_t(gridDim.x) * blockDim.x) {
    float v = 0.f;
    for (int s = 0; s < splits; ++s) v += part[int64_t(s) * nm + k];
    u[k] = __float2bfloat16_rn(v);
  }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// bf16 [rows, cols] row-major, boxes [box_rows, 64], 128-byte swizzle; rows
// past the end read as zeros.
bool make_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes) {
  static bool done[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (done[dev]) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(bytes));
  if (e == cudaSuccess) done[dev] = true;
  return e;
}

int sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  return n;
}

}  // namespace

cudaError_t launch_fold_weights(const __nv_bfloat16* W_O, const __nv_bfloat16* W_UV, int d_model,
                                int H, __nv_bfloat16* w_fold, int* status, cudaStream_t stream) {
  CUtensorMap tm_wo, tm_wuv;
  if (!make_map(&tm_wo, W_O, uint64_t(d_model), uint64_t(H) * 128, 128) ||
      !make_map(&tm_wuv, W_UV, uint64_t(H) * 128, 512, 128))
    return cudaErrorInvalidValue;
  cudaError_t e = set_smem(fold_weights_tc_kernel, kFoldSmem);
  if (e != cudaSuccess) return e;
  dim3 grid((d_model + 127) / 128, H, 2);
  fold_weights_tc_kernel<<<grid, kThr, kFoldSmem, stream>>>(tm_wo, tm_wuv, d_model, H, w_fold,
                                                            status);
  return cudaGetLastError();
}

int folded_proj_splits(int d_model, int H) {
  const int m_tiles = (d_model + 127) / 128;
  const int64_t k_chunks = int64_t(H) * 512 / 64;
  int s = 2 * sms() / m_tiles;   // one wave of two CTAs per SM
  if (s < 1) s = 1;
  if (s > k_chunks) s = int(k_chunks);
  return s;
}

size_t folded_proj_workspace_bytes(int B, int H, int d_model) {
  const size_t xb = ((size_t(B) * H * 512 * 2) + 255) / 256 * 256;
  const size_t pb = size_t(folded_proj_splits(d_model, H)) * B * d_model * 4;
  return xb + (pb + 255) / 256 * 256;
}

cudaError_t launch_folded_proj(const float* o_lat, const __nv_bfloat16* w_fold, int B, int H,
                               int d_model, void* workspace, __nv_bfloat16* u, int* status,
                               cudaStream_t stream) {
  if (B < 1 || B > kFoldedMaxBatch) return cudaErrorInvalidValue;
  const int64_t K = int64_t(H) * 512;
  __nv_bfloat16* xb = static_cast<__nv_bfloat16*>(workspace);
  float* part = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                         ((size_t(B) * K * 2) + 255) / 256 * 256);
  const int64_t n4 = int64_t(B) * K / 4;
  to_bf16_kernel<<<int((n4 + 255) / 256 < 4096 ? (n4 + 255) / 256 : 4096), 256, 0, stream>>>(
      reinterpret_cast<const float4*>(o_lat), reinterpret_cast<uint2*>(xb), n4);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int np = (B + 15) / 16 * 16;   // the MMA's N: the batch padded to 16 (zero rows)
  CUtensorMap tm_w, tm_x;
  if (!make_map(&tm_w, w_fold, uint64_t(d_model), uint64_t(K), 128) ||
      !make_map(&tm_x, xb, uint64_t(B), uint64_t(K), uint32_t(np)))
    return cudaErrorInvalidValue;
  const size_t smem = kFpStages * fp_stage_bytes(kFoldedMaxBatch) + 8 * (2 * kFpStages + 2) + 1024;
  if ((e = set_smem(folded_proj_tc_kernel, smem)) != cudaSuccess) return e;
  const int splits = folded_proj_splits(d_model, H);
  const size_t used = kFpStages * fp_stage_bytes(np) + 8 * (2 * kFpStages + 2) + 1024;
  dim3 grid((d_model + 127) / 128, splits);
  folded_proj_tc_kernel<<<grid, kThr, used, stream>>>(tm_w, tm_x, d_model, B, np, K / 64, splits,
                                                      part, status);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int64_t nm = int64_t(B) * d_model;
  reduce_splits_kernel<<<int((nm + 255) / 256 < 2048 ? (nm + 255) / 256 : 2048), 256, 0, stream>>>(
      part, splits, nm, u);
  return cudaGetLastError();
}

}  // namespace mla
