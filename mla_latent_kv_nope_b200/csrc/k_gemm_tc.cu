// Tensor-core kernels for the three weight-streaming contractions of the bf16
// decode step.  In each the weight is the long side (M = 128 rows per MMA)
// and the batch of sequences is N, so a CTA streams a weight block once
// through TMA (128-byte swizzle) and multiplies it with every sequence:
//
//   out_proj  out[b,i,:] = W^UV_i o_lat[b,i,:]          ([MLA-とは] "Value側の吸収")
//             A = W_UV[i] (K-major, K = d_c), B = o_lat rows converted to bf16
//   absorb_q  q~[b,i,:]  = W^UK_i^T q^C[b,i,:]          ([MLA-とは] "行列吸収")
//             A = W_UK[i]^T: W_UK[i] is [d_nope, d_c] row-major, i.e. an
//             MN-major A operand with M = d_c; B = q_nope rows (K = d_nope)
//   append    x[b,:]     = W_DKV h[b,:]                  ([MLA-とは] "MLAの発想",
//             A = W_DKV (K-major, K = hidden) split over    "Decoupled RoPE")
//             K across CTAs; each writes an fp32 partial that the finalize
//             kernel sums in a fixed order (deterministic).
// One warp issues the MMAs (elect.sync); accumulators live in TMEM and are
// read back with 32x32b tcgen05.ld (thread t of warp w gets row 32w+t).
// Every wait is bounded; on give-up the kernel records MLA_ERR_DEVICE_TIMEOUT
// and skips its stores.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace mla {

namespace {

using namespace sm100;

constexpr int kThreadsG = 128;
constexpr int kChunk = 64;                  // bf16 elements per 128-byte row

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// Block-wide bounded wait on an mbarrier (every thread polls).
__device__ __forceinline__ bool block_wait(uint64_t* bar, uint32_t parity) {
  volatile int no_abort = 0;
  return mbar_wait(bar, parity, &no_abort, kWaitLimitCycles);
}

// Store bf16 pairs of row `r` (64 elements = 8 16-byte units) into a K-major
// 128-byte-swizzled tile whose rows are 128 bytes apart.
__device__ __forceinline__ void st_sw128_unit(uint8_t* tile, int r, int unit, uint4 v) {
  *reinterpret_cast<uint4*>(tile + r * 128 + ((unit ^ (r & 7)) * 16)) = v;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 p = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&p);
}

// ---------------------------------------------------------------------------
// out_proj: CTA per head; N chunks of up to 64 sequences.
// smem: W 8 x [128 x 128 B] (128 KB) | X 8 x [64 x 128 B] (64 KB) | barriers
constexpr int kOpN = 64;
constexpr size_t kOpSmem = 8 * 16384 + 8 * (kOpN * 128) + 64 + 1024;

__global__ void __launch_bounds__(kThreadsG, 1)
out_proj_tc_kernel(const __grid_constant__ CUtensorMap tm_w, const float* __restrict__ o_lat,
                   int B, int H, __nv_bfloat16* __restrict__ out, int* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint8_t* sW = sm;
  uint8_t* sX = sm + 8 * 16384;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sX + 8 * kOpN * 128);  // [0]=w, [1]=mma
  uint32_t* tbase = reinterpret_cast<uint32_t*>(bars + 2);
  const int i = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // Nothing is read before the kernel in front (the combine) has finished:
  // the weight could have been written by stream work before this call too.
  pdl_wait();
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(&bars[0], 8 * 16384);
    for (int c = 0; c < 8; ++c) tma_load_2d(&tm_w, &bars[0], sW + c * 16384, c * kChunk, i * 128);
  }
  if (warp == 0) {
    tmem_alloc(tbase, kOpN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_trigger();
  const uint32_t tmem = *tbase;
  bool ok = true;
  constexpr uint32_t idesc = idesc_bf16_f32(128, kOpN, false, false);
  int pass = 0;
  for (int n0 = 0; n0 < B; n0 += kOpN, ++pass) {
    const int nc = min(kOpN, B - n0);
    // o_lat rows (fp32) -> bf16, K-major swizzled; rows >= nc are zero.
    // Each thread owns 32 16-byte units; 16 units' loads are issued together.
#pragma unroll 1
    for (int base = 0; base < kOpN * 64; base += 16 * kThreadsG) {
      float4 x[16][2];
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int u = base + j * kThreadsG + threadIdx.x;
        const int r = u / 64, c = (u / 8) % 8, unit = u % 8;
        if (r < nc) {
          const float4* src = reinterpret_cast<const float4*>(
              o_lat + (int64_t(n0 + r) * H + i) * 512 + c * kChunk + unit * 8);
          x[j][0] = src[0];
          x[j][1] = src[1];
        } else {
          x[j][0] = x[j][1] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const int u = base + j * kThreadsG + threadIdx.x;
        const int r = u / 64, c = (u / 8) % 8, unit = u % 8;
        st_sw128_unit(sX + c * (kOpN * 128), r, unit,
                      make_uint4(pack_bf16(x[j][0].x, x[j][0].y), pack_bf16(x[j][0].z, x[j][0].w),
                                 pack_bf16(x[j][1].x, x[j][1].y), pack_bf16(x[j][1].z, x[j][1].w)));
      }
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (pass == 0) ok = block_wait(&bars[0], 0) && ok;
    if (warp == 0) {
      tc_fence_after();
      const uint64_t a0 = smem_desc_sw128(smem_u32(sW), 16, 1024);
      const uint64_t b0 = smem_desc_sw128(smem_u32(sX), 16, 1024);
#pragma unroll
      for (int c = 0; c < 8; ++c)
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_bf16_ss_w(tmem, a0 + uint64_t((c * 16384 + k * 32) >> 4),
                        b0 + uint64_t((c * kOpN * 128 + k * 32) >> 4), idesc, (c | k) != 0);
      mma_commit_w(&bars[1]);
    }
    ok = block_wait(&bars[1], pass & 1) && ok;
    tc_fence_after();
    // D[v][b]: thread (warp w, lane t) holds row v = 32w + t.
    const int v = 32 * warp + lane;
#pragma unroll 1
    for (int c0 = 0; c0 < kOpN; c0 += 32) {
      uint32_t r[32];
      tmem_ld32(tmem + (uint32_t(32 * warp) << 16) + uint32_t(c0), r);
      tmem_wait_ld();
      if (ok) {
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (c0 + e < nc)
            out[(int64_t(n0 + c0 + e) * H + i) * 128 + v] = __float2bfloat16_rn(__uint_as_float(r[e]));
      }
    }
    tc_fence_before();
    __syncthreads();  // X and the accumulator are reused by the next pass
    tc_fence_after();
  }
  if (!ok && threadIdx.x == 0) record_status(status, MLA_ERR_DEVICE_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kOpN);
  }
}

// ---------------------------------------------------------------------------
// absorb_q: grid (head, 4 blocks of 128 output columns); N chunks of up to
// 64 sequences.  Each CTA streams the 32 KB of W_UK[i] its columns need, and
// takes a quarter of the head's RoPE pairs.
// smem: W_UK[i][:, 128m : 128m+128] 2 x [128 (K = r) x 128 B (64 c)] (32 KB) |
//       X 2 x [64 x 128 B] | barriers
constexpr int kAbN = 64;
constexpr int kAbBlocks = 4;                 // d_c = 512 = 4 x 128 output columns
constexpr size_t kAbSmem = 2 * 16384 + 2 * (kAbN * 128) + 64 + 1024;

__global__ void __launch_bounds__(kThreadsG, 1)
absorb_q_tc_kernel(const __grid_constant__ CUtensorMap tm_w, const __nv_bfloat16* __restrict__ q_nope,
                   const __nv_bfloat16* __restrict__ q_pe, const int32_t* __restrict__ q_pos,
                   float rope_base, int B, int H, int d_r, __nv_bfloat16* __restrict__ q_cat,
                   int* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint8_t* sW = sm;
  uint8_t* sX = sm + 2 * 16384;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sX + 2 * kAbN * 128);
  uint32_t* tbase = reinterpret_cast<uint32_t*>(bars + 2);
  const int i = blockIdx.x;
  const int mb = blockIdx.y;                 // output columns [128 mb, 128 mb + 128)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kR = 512 + d_r;   // q_cat row: 512 absorbed columns, then the RoPE block (64 or none)
  // Rotation frequencies of the 32 RoPE pairs, computed once per CTA while
  // the weight block loads.
  __shared__ double s_inv[32];
  if (threadIdx.x < 32) s_inv[threadIdx.x] = rope_inv_freq(threadIdx.x, 64, rope_base);
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(&bars[0], 2 * 16384);
    for (int c = 0; c < 2; ++c)
      tma_load_2d(&tm_w, &bars[0], sW + c * 16384, (2 * mb + c) * kChunk, i * 128);
  }
  if (warp == 0) {
    tmem_alloc(tbase, kAbN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tbase;
  bool ok = true;
  constexpr uint32_t idesc = idesc_bf16_f32(128, kAbN, /*A MN-major*/ true, false);
  int pass = 0;
  for (int n0 = 0; n0 < B; n0 += kAbN, ++pass) {
    const int nc = min(kAbN, B - n0);
    {
      uint4 v[kAbN * 16 / kThreadsG];
#pragma unroll
      for (int j = 0; j < kAbN * 16 / kThreadsG; ++j) {
        const int u = j * kThreadsG + threadIdx.x;
        const int r = u / 16, c = (u / 8) % 2, unit = u % 8;
        v[j] = r < nc ? *reinterpret_cast<const uint4*>(q_nope + (int64_t(n0 + r) * H + i) * 128 +
                                                        c * kChunk + unit * 8)
                      : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int j = 0; j < kAbN * 16 / kThreadsG; ++j) {
        const int u = j * kThreadsG + threadIdx.x;
        st_sw128_unit(sX + (u / 8 % 2) * (kAbN * 128), u / 16, u % 8, v[j]);
      }
    }
    fence_proxy_async_smem();
    __syncthreads();
    if (pass == 0) ok = block_wait(&bars[0], 0) && ok;
    if (warp == 0) {
      tc_fence_after();
      // A for output rows [128 mb, 128 mb + 128): the two loaded c-chunks
      // (LBO = 16 KB between 64-wide c groups), K-step k = rows 16k..16k+15
      // of W_UK[i].
      const uint64_t a0 = smem_desc_sw128(smem_u32(sW), 16384, 1024);
      const uint64_t b0 = smem_desc_sw128(smem_u32(sX), 16, 1024);
#pragma unroll
      for (int k = 0; k < 8; ++k)
        mma_bf16_ss_w(tmem, a0 + uint64_t((k * 2048) >> 4),
                      b0 + uint64_t(((k / 4) * kAbN * 128 + (k % 4) * 32) >> 4), idesc, k != 0);
      mma_commit_w(&bars[1]);
    }
    ok = block_wait(&bars[1], pass & 1) && ok;
    tc_fence_after();
    const int crow = 32 * warp + lane;
#pragma unroll 1
    for (int c0 = 0; c0 < kAbN; c0 += 32) {
      uint32_t r[32];
      tmem_ld32(tmem + (uint32_t(32 * warp) << 16) + uint32_t(c0), r);
      tmem_wait_ld();
      if (ok) {
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (c0 + e < nc)
            q_cat[(int64_t(n0 + c0 + e) * H + i) * kR + mb * 128 + crow] =
                __float2bfloat16_rn(__uint_as_float(r[e]));
      }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }
  // Decoupled RoPE block: rotate q_pe at q_pos (or copy when q_pos is NULL).
  // Pairs (b, k) are taken 8 per thread with every load issued before the
  // first rotation, so the pass costs one memory round trip per 8 pairs.
  constexpr int kRopeBatch = 8;
  const int n_pairs = d_r / 2;   // 32, or 0 without a RoPE block
  const int u_lo = int(int64_t(B) * n_pairs * mb / kAbBlocks);
  const int u_hi = int(int64_t(B) * n_pairs * (mb + 1) / kAbBlocks);
  for (int u0 = u_lo; u0 < u_hi; u0 += kRopeBatch * kThreadsG) {
    float x1[kRopeBatch], x2[kRopeBatch];
    int32_t pos[kRopeBatch];
#pragma unroll
    for (int j = 0; j < kRopeBatch; ++j) {
      const int u = u0 + j * kThreadsG + threadIdx.x;
      const bool in = u < u_hi;
      const int b = in ? u / 32 : 0, k = u % 32;
      const int64_t row = int64_t(b) * H + i;
      x1[j] = __bfloat162float(q_pe[row * 64 + k]);
      x2[j] = __bfloat162float(q_pe[row * 64 + k + 32]);
      pos[j] = q_pos ? q_pos[b] : 0;
    }
#pragma unroll
    for (int j = 0; j < kRopeBatch; ++j) {
      const int u = u0 + j * kThreadsG + threadIdx.x;
      if (u >= u_hi) continue;
      const int b = u / 32, k = u % 32;
      const int64_t row = int64_t(b) * H + i;
      float y1 = x1[j], y2 = x2[j];
      if (q_pos) {
        float c, sn;
        rope_cos_sin_at(pos[j], s_inv[k], &c, &sn);
        y1 = x1[j] * c - x2[j] * sn;
        y2 = x1[j] * sn + x2[j] * c;
      }
      q_cat[row * kR + 512 + k] = __float2bfloat16_rn(y1);
      q_cat[row * kR + 512 + k + 32] = __float2bfloat16_rn(y2);
    }
  }
  if (!ok && threadIdx.x == 0) record_status(status, MLA_ERR_DEVICE_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kAbN);
  }
}

// ---------------------------------------------------------------------------
// append projection: grid (M tiles of 128 rows of W_DKV, K splits of 256,
// N chunks of 64 sequences).  Each CTA writes part[split][b][r] (fp32).
// smem: A 4 x [128 x 128 B] (64 KB) | B 4 x [64 x 128 B] (32 KB) | barriers
constexpr int kApN = 64;
constexpr int kApKc = 256;
constexpr size_t kApSmem = 4 * 16384 + 4 * (kApN * 128) + 64 + 1024;

__global__ void __launch_bounds__(kThreadsG, 1)
append_proj_tc_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_h,
                      int B, int R, float* __restrict__ part, int* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint8_t* sA = sm;
  uint8_t* sB = sm + 4 * 16384;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + 4 * kApN * 128);
  uint32_t* tbase = reinterpret_cast<uint32_t*>(bars + 2);
  const int mt = blockIdx.x, split = blockIdx.y, n0 = blockIdx.z * kApN;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k0 = split * kApKc;
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbar_init();
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(&bars[0], 4 * 16384 + 4 * kApN * 128);
    for (int c = 0; c < 4; ++c) {
      tma_load_2d(&tm_w, &bars[0], sA + c * 16384, k0 + c * kChunk, mt * 128);
      tma_load_2d(&tm_h, &bars[0], sB + c * (kApN * 128), k0 + c * kChunk, n0);
    }
  }
  if (warp == 0) {
    tmem_alloc(tbase, kApN);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_trigger();   // the finalize may be scheduled; it waits for this grid's sums
  const uint32_t tmem = *tbase;
  bool ok = block_wait(&bars[0], 0);
  if (warp == 0) {
    tc_fence_after();
    constexpr uint32_t idesc = idesc_bf16_f32(128, kApN, false, false);
    const uint64_t a0 = smem_desc_sw128(smem_u32(sA), 16, 1024);
    const uint64_t b0 = smem_desc_sw128(smem_u32(sB), 16, 1024);
#pragma unroll
    for (int c = 0; c < 4; ++c)
#pragma unroll
      for (int k = 0; k < 4; ++k)
        mma_bf16_ss_w(tmem, a0 + uint64_t((c * 16384 + k * 32) >> 4),
                      b0 + uint64_t((c * kApN * 128 + k * 32) >> 4), idesc, (c | k) != 0);
    mma_commit_w(&bars[1]);
  }
  ok = block_wait(&bars[1], 0) && ok;
  tc_fence_after();
  const int r = mt * 128 + 32 * warp + lane;
  const int nc = min(kApN, B - n0);
#pragma unroll 1
  for (int c0 = 0; c0 < kApN; c0 += 32) {
    uint32_t v[32];
    tmem_ld32(tmem + (uint32_t(32 * warp) << 16) + uint32_t(c0), v);
    tmem_wait_ld();
    if (ok && r < R) {
#pragma unroll
      for (int e = 0; e < 32; ++e)
        if (c0 + e < nc)
          part[(int64_t(split) * B + n0 + c0 + e) * R + r] = __uint_as_float(v[e]);
    }
  }
  if (!ok && threadIdx.x == 0) record_status(status, MLA_ERR_DEVICE_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kApN);
  }
}

// ---------------------------------------------------------------------------
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

// 2D bf16 map over a row-major [rows, cols] matrix with [box_rows, 64] boxes.
bool make_map(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {uint32_t(kChunk), box_rows};
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

}  // namespace

bool gemm_tc_supported(int d_c, int d_r, int d_n, int d_v) {
  return d_c == 512 && (d_r == 64 || d_r == 0) && d_n == 128 && d_v == 128;
}

cudaError_t launch_out_proj_tc(const float* o_lat, const __nv_bfloat16* W_UV, int B, int H,
                               __nv_bfloat16* out, int* status, cudaStream_t stream) {
  CUtensorMap tm;
  if (!make_map(&tm, W_UV, uint64_t(H) * 128, 512, 128)) return cudaErrorInvalidValue;
  cudaError_t e = set_smem(out_proj_tc_kernel, kOpSmem);
  if (e != cudaSuccess) return e;
  return launch_pdl(out_proj_tc_kernel, dim3(H), dim3(kThreadsG), kOpSmem, stream, tm, o_lat, B,
                    H, out, status);
}

cudaError_t launch_absorb_q_tc(const __nv_bfloat16* q_nope, const __nv_bfloat16* q_pe,
                               const __nv_bfloat16* W_UK, const int32_t* q_pos, float rope_base,
                               int B, int H, int d_r, __nv_bfloat16* q_cat, int* status,
                               cudaStream_t stream) {
  if (d_r != 64 && d_r != 0) return cudaErrorInvalidValue;
  CUtensorMap tm;
  if (!make_map(&tm, W_UK, uint64_t(H) * 128, 512, 128)) return cudaErrorInvalidValue;
  cudaError_t e = set_smem(absorb_q_tc_kernel, kAbSmem);
  if (e != cudaSuccess) return e;
  absorb_q_tc_kernel<<<dim3(H, kAbBlocks), kThreadsG, kAbSmem, stream>>>(tm, q_nope, q_pe, q_pos,
                                                                         rope_base, B, H,
                                                                         d_r, q_cat, status);
  return cudaGetLastError();
}

int append_tc_splits(int hidden) { return (hidden + kApKc - 1) / kApKc; }

cudaError_t launch_append_proj_tc(const __nv_bfloat16* h, const __nv_bfloat16* W_DKV, int B,
                                  int R, int hidden, float* part, int* status,
                                  cudaStream_t stream) {
  CUtensorMap tw, th;
  if (!make_map(&tw, W_DKV, uint64_t(R), uint64_t(hidden), 128) ||
      !make_map(&th, h, uint64_t(B), uint64_t(hidden), kApN))
    return cudaErrorInvalidValue;
  cudaError_t e = set_smem(append_proj_tc_kernel, kApSmem);
  if (e != cudaSuccess) return e;
  dim3 grid((R + 127) / 128, append_tc_splits(hidden), (B + kApN - 1) / kApN);
  append_proj_tc_kernel<<<grid, kThreadsG, kApSmem, stream>>>(tw, th, B, R, part, status);
  return cudaGetLastError();
}

}  // namespace mla
