// Materialised prefill for one sequence ([MLA-とは] "実装上のトレードオフ":
// prefill is compute-bound, so the per-head keys and values are formed
// explicitly and the heads run ordinary causal attention; the absorbed form is
// the decode's).
//
//   prefill_kv_tc_kernel  K^C_i[l] = W^UK_i c_l,  V_i[l] = W^UV_i c_l
//                         -> kc [H, L, 128] fp16, v [H, L, 128] bf16, and
//                         kr [L, d_r] fp16 (the rows' k^R, converted once)
//                         one CTA per (128 rows l, head i): A = latent rows
//                         (K-major, K = d_c = 512), B = [W^UK_i ; W^UV_i]
//                         (256 rows, K-major), D [128 x 256] fp32 in TMEM
//   prefill_attn_tc_kernel  causal softmax attention of head i, 128 queries
//                         per CTA, 128-key tiles; the query row is
//                         Q_i[t] = [q^C[t,i] ; RoPE(q^R[t,i], q_pos[t])], formed
//                         by the CTA straight into tensor memory; the key of
//                         row l is [K^C_i[l] ; k^R_l] (k^R already rotated),
//                         head dim 128 + d_r, value dim 128
//
// The causal rule: query t sees rows l <= q_pos[t] (clamped to L - 1); a
// query with q_pos[t] < 0 sees nothing (out 0, lse -inf).
// Precision: the QK^T operands (queries, K^C, k^R) are fp16 and P, V are
// bf16, all with fp32 accumulation.  Materialising K adds a rounding that the
// absorbed decode does not have, and with a peaked softmax bf16 keys and
// queries alone put the output 3 % off the exact result; fp16's 11-bit
// significand brings that under 0.5 %.  Queries, keys and k^R must lie within
// fp16's range (|x| < 65504).
// Every wait is bounded; on give-up a kernel records MLA_ERR_DEVICE_TIMEOUT,
// drains what it issued and skips its stores.
#include <cuda.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "tensor_map.cuh"

namespace mla {

namespace {

using namespace sm100;

constexpr int kDn = 128;       // d_nope
constexpr int kDv = 128;       // d_v
constexpr int kDcP = 512;      // d_c
constexpr int kTileQ = 128;    // queries per attention CTA
constexpr int kTileK = 128;    // keys per attention tile
constexpr int kBox = 16384;    // one [128 rows x 64] bf16 box, 128-byte swizzle

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  const __nv_bfloat162 p = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&p);
}
__device__ __forceinline__ uint32_t pack_f16x2(float a, float b) {
  const __half2 p = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&p);
}
// 8 bf16 (one 16-byte unit) -> 8 fp16.
__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 u) {
  const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&u);
  uint4 r;
  uint32_t* o = reinterpret_cast<uint32_t*>(&r);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float2 f = __bfloat1622float2(b[j]);
    o[j] = pack_f16x2(f.x, f.y);
  }
  return r;
}

// Block-wide bounded wait (every calling thread polls; no abort flag).
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity) {
  volatile int no_abort = 0;
  return mbar_wait(bar, parity, &no_abort, kWaitLimitCycles);
}

// ---------------------------------------------------------------------------
// RoPE angles of the queries: cs[t][k] = (cos, sin) of q_pos[t] * base^(-2k/d_r)
// for the d_r/2 pairs, formed once per token (every head uses them).
__global__ void prefill_rope_table_kernel(const int32_t* __restrict__ q_pos, int T, int d_r,
                                          float rope_base, float2* __restrict__ cs) {
  pdl_trigger();   // the K/V projection does not read the table: let it start
  const int half = d_r / 2;
  const int64_t n = int64_t(T) * half;
  for (int64_t u = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; u < n;
       u += int64_t(gridDim.x) * blockDim.x) {
    const int t = int(u / half), k = int(u % half);
    const int32_t pos = q_pos[t];
    float c, sn;
    rope_cos_sin(pos < 0 ? 0 : pos, k, d_r, rope_base, &c, &sn);
    cs[u] = make_float2(c, sn);
  }
}

// ---------------------------------------------------------------------------
// K/V materialisation.  smem: 4 stages x (A [128 x 128 B] | B [256 x 128 B])
constexpr int kKvStages = 4;
constexpr int kKvStage = kBox + 2 * kBox;                  // 48 KB
constexpr size_t kKvSmem = size_t(kKvStages) * kKvStage + 8 * (2 * kKvStages + 1) + 16 + 1024;
constexpr int kKvThreads = 128;

__global__ void __launch_bounds__(kKvThreads, 1)
prefill_kv_tc_kernel(const __grid_constant__ CUtensorMap tm_rows,
                     const __grid_constant__ CUtensorMap tm_wuk,
                     const __grid_constant__ CUtensorMap tm_wuv, int64_t L, int H, int d_r,
                     const __nv_bfloat16* __restrict__ rows, __half* __restrict__ kc,
                     __nv_bfloat16* __restrict__ v, __half* __restrict__ kr,
                     int* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + kKvStages * kKvStage);
  uint64_t* empty = full + kKvStages;
  uint64_t* done = empty + kKvStages;
  uint32_t* tbase = reinterpret_cast<uint32_t*>(done + 1);
  __shared__ int s_abort;
  const int64_t l0 = int64_t(blockIdx.x) * 128;
  const int i = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kChunks = kDcP / 64;   // 8
  if (threadIdx.x == 0) {
    for (int s = 0; s < kKvStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    s_abort = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == 0) {
    tmem_alloc(tbase, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_trigger();
  const uint32_t tmem = *tbase;
  volatile int* abort_flag = &s_abort;
  bool ok = true;
  int issued = 0;
  if (warp == 1) {
    if (lane == 0) {
      for (int c = 0; c < kChunks; ++c) {
        const int s = c % kKvStages;
        if (c >= kKvStages &&
            !(ok = mbar_wait(&empty[s], ((c / kKvStages) - 1) & 1, abort_flag, kWaitLimitCycles)))
          break;
        uint8_t* st = sm + s * kKvStage;
        mbar_arrive_expect_tx(&full[s], kKvStage);
        tma_load_2d(&tm_rows, &full[s], st, c * 64, int32_t(l0));
        tma_load_2d(&tm_wuk, &full[s], st + kBox, c * 64, i * 128);
        tma_load_2d(&tm_wuv, &full[s], st + 2 * kBox, c * 64, i * 128);
        ++issued;
      }
      if (!ok) *abort_flag = 1;
    }
  } else if (warp == 0) {
    constexpr uint32_t idesc = idesc_bf16_f32(128, 256, false, false);
    for (int c = 0; c < kChunks; ++c) {
      const int s = c % kKvStages;
      bool got = mbar_try(&full[s], (c / kKvStages) & 1);
      if (!__all_sync(0xffffffffu, got)) {
        got = mbar_wait(&full[s], (c / kKvStages) & 1, abort_flag, kWaitLimitCycles);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          if (lane == 0) *abort_flag = 1;
          break;
        }
      }
      tc_fence_after();
      const uint32_t st = smem_u32(sm + s * kKvStage);
      const uint64_t a0 = smem_desc_sw128(st, 16, 1024);
      const uint64_t b0 = smem_desc_sw128(st + kBox, 16, 1024);
#pragma unroll
      for (int k = 0; k < 4; ++k)
        mma_bf16_ss_w(tmem, a0 + uint64_t((k * 32) >> 4), b0 + uint64_t((k * 32) >> 4), idesc,
                      (c | k) != 0);
      mma_commit_w(&empty[s]);
    }
    mma_commit_w(done);
  }
  __syncthreads();
  ok = wait_bar(done, 0) && ok && !*abort_flag;
  tc_fence_after();
  // D[r][n]: thread (warp w, lane t) holds row l0 + 32w + t; columns 0-127 are
  // K^C, 128-255 are V.
  const int64_t l = l0 + 32 * warp + lane;
#pragma unroll 1
  for (int c0 = 0; c0 < 256; c0 += 32) {
    uint32_t r[32];
    tmem_ld32(tmem + (uint32_t(32 * warp) << 16) + uint32_t(c0), r);
    tmem_wait_ld();
    if (ok && l < L) {
      const int64_t off = (int64_t(i) * L + l) * 128 + (c0 & 127);
      const bool is_k = c0 < 128;                       // K^C fp16, V bf16
      uint4* dst = reinterpret_cast<uint4*>(is_k ? static_cast<void*>(kc + off)
                                                 : static_cast<void*>(v + off));
#pragma unroll
      for (int e = 0; e < 32; e += 8) {
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float a = __uint_as_float(r[e + 2 * j]), b = __uint_as_float(r[e + 2 * j + 1]);
          w[j] = is_k ? pack_f16x2(a, b) : pack_bf16x2(a, b);
        }
        dst[e / 8] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
  // The head-0 CTAs also convert their rows' k^R to fp16 (the QK^T operand).
  if (i == 0 && d_r && ok && l < L) {
    const uint4* src = reinterpret_cast<const uint4*>(rows + l * (kDcP + d_r) + kDcP);
    uint4* dst = reinterpret_cast<uint4*>(kr + l * d_r);
    for (int u = 0; u < d_r / 8; ++u) dst[u] = bf16x8_to_f16x8(src[u]);
  }
  if (!ok && threadIdx.x == 0) record_status(status, MLA_ERR_DEVICE_TIMEOUT);
  // Loads issued but never consumed land before the shared memory is released.
  if (warp == 1 && lane == 0) {
    for (int k = issued > kKvStages ? issued - kKvStages : 0; k < issued; ++k)
      wait_bar(&full[k % kKvStages], (k / kKvStages) & 1);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
  pdl_wait();   // the kernel before (the query angles) has finished too
}

// ---------------------------------------------------------------------------
// Causal attention: one CTA per (128 queries, head).
// Tensor memory (512 columns): O [128 x 128] fp32 at 0; S double buffer
// 2 x 128 at 128, whose first 64 columns receive P (bf16 pairs) once both
// threads of a row have read their S; Q (fp16 pairs: 96 columns, 64 without
// RoPE) at 384, the tensor-memory A operand of QK^T.  Shared memory: a
// 3-stage K ring (K^C boxes and the k^R box of 128 keys) and a 2-stage V ring,
// with separate barriers, so a K stage is refilled as soon as its QK^T is
// done and the load of key tile k + 3 overlaps tiles k + 1 and k + 2.
// Warps 0-7: query rows into tensor memory, softmax, epilogue (warp w: rows
// 32 (w % 4) .., columns 64 (w / 4) .. of S, P and O, so two threads per
// row); warp 8: K loads; warp 9: MMA issue; warp 10: V loads.
constexpr int kKStages = 3;
constexpr int kVStages = 2;
constexpr int kKStage = 3 * kBox;                         // 48 KB
constexpr int kVStage = 2 * kBox;                         // 32 KB
constexpr int kAtSoftmaxThreads = 256;
constexpr int kAtKLoad = 8;
constexpr int kAtMma = 9;
constexpr int kAtVLoad = 10;
constexpr int kAtThreads = 352;
constexpr uint32_t kColO = 0, kColS = 128, kColQ = 384;
constexpr float kRescaleLog2 = 8.f;  // rescale O only when the max grows by > 2^8

struct AttnBars {
  uint64_t k_full[kKStages], k_empty[kKStages];
  uint64_t v_full[kVStages], v_empty[kVStages];
  uint64_t q_ready, s_full[2], p_full[2], pv_done[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int max_vis;
  float row_max[2][2][kTileQ];   // [tile parity][column half][row]: the halves' maxima
  float row_sum[2][kTileQ];      // [column half][row]: the halves' sums, at the end
};
constexpr size_t kAtSmem =
    size_t(kKStages) * kKStage + size_t(kVStages) * kVStage + sizeof(AttnBars) + 1024;
static_assert(kAtSmem <= 232448, "shared memory budget of one CTA");

// Warp-uniform bounded wait that also gives up when another role aborted.
__device__ __forceinline__ bool warp_wait_bar(uint64_t* bar, uint32_t parity,
                                              volatile int* abort_flag) {
  if (__all_sync(0xffffffffu, mbar_try(bar, parity))) return true;
  const bool ok = mbar_wait(bar, parity, abort_flag, kWaitLimitCycles);
  return __all_sync(0xffffffffu, ok);
}

// One arrival per warp on a barrier that counts warps: every lane's tensor-
// memory stores are complete and ordered before lane 0 arrives.
__device__ __forceinline__ void warp_arrive_after_tmem_st(uint64_t* bar) {
  tmem_wait_st();
  tc_fence_before();
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// The query row Q_i[t] = [q^C ; RoPE(q^R, pos)] in fp16 pairs, written to
// tensor memory by the two threads of the row: half 0 takes q^C dims 0-127
// (dims 0-63 without RoPE), half 1 the RoPE block (dims 64-127 of q^C
// without RoPE).  Every global load of a thread is issued before the first
// use, so the row costs one memory round trip.  Rows past T are zero.
__device__ __forceinline__ void nope_to_tmem(const uint4* __restrict__ src, bool valid, int j0,
                                             int j1, uint32_t taddr) {
  uint4 raw[16];
#pragma unroll
  for (int u = 0; u < 16; ++u)
    raw[u] = (valid && u < 4 * (j1 - j0)) ? src[4 * j0 + u] : make_uint4(0, 0, 0, 0);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    if (j >= j1 - j0) break;
    uint32_t v[16];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint4 hq = bf16x8_to_f16x8(raw[4 * j + u]);
      v[4 * u] = hq.x;
      v[4 * u + 1] = hq.y;
      v[4 * u + 2] = hq.z;
      v[4 * u + 3] = hq.w;
    }
    tmem_st16(taddr + uint32_t(16 * (j0 + j)), v);
  }
}

// RoPE block (d_r = 64): y[k] = x[k] c_k - x[k+32] s_k, y[k+32] = x[k] s_k +
// x[k+32] c_k, with (c_k, s_k) from the angle table; 32 packed columns.
__device__ __forceinline__ void rope_to_tmem(const uint4* __restrict__ src,
                                             const float4* __restrict__ cs4, bool valid,
                                             uint32_t taddr) {
  uint4 xr[8];
  float4 a[16];
#pragma unroll
  for (int u = 0; u < 8; ++u) xr[u] = valid ? src[u] : make_uint4(0, 0, 0, 0);
#pragma unroll
  for (int u = 0; u < 16; ++u) a[u] = valid ? cs4[u] : make_float4(1.f, 0.f, 1.f, 0.f);
  float x[64];
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&xr[u]);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 f = __bfloat1622float2(p2[q]);
      x[8 * u + 2 * q] = f.x;
      x[8 * u + 2 * q + 1] = f.y;
    }
  }
  uint32_t v[32];
#pragma unroll
  for (int e = 0; e < 32; e += 2) {
    const float4 c = a[e / 2];                 // (cos, sin) of pairs e and e + 1
    v[e / 2] = pack_f16x2(x[e] * c.x - x[e + 32] * c.y, x[e + 1] * c.z - x[e + 33] * c.w);
    v[16 + e / 2] = pack_f16x2(x[e] * c.y + x[e + 32] * c.x, x[e + 1] * c.w + x[e + 33] * c.z);
  }
  tmem_st32(taddr, v);
}

__global__ void __launch_bounds__(kAtThreads, 1)
prefill_attn_tc_kernel(const __grid_constant__ CUtensorMap tm_kc,
                       const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_kr,
                       const __nv_bfloat16* __restrict__ q_nope,
                       const __nv_bfloat16* __restrict__ q_pe, const float2* __restrict__ cs,
                       const int32_t* __restrict__ q_pos, int T, int64_t L, int H, int d_r,
                       float scale_log2, __nv_bfloat16* __restrict__ out,
                       float* __restrict__ lse, int* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  uint8_t* sK = sm;
  uint8_t* sV = sm + kKStages * kKStage;
  AttnBars* bars = reinterpret_cast<AttnBars*>(sV + kVStages * kVStage);
  // Query tiles vary fastest, so the CTAs in flight share a few heads' K and
  // V through L2; within a head the longest query tiles start first.
  const int i = blockIdx.y;
  const int qt = int(gridDim.x) - 1 - int(blockIdx.x);
  const int q0 = qt * kTileQ;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nq = (kDn + d_r) / 64;                       // 64-wide chunks of the head dim
  volatile int* abort_flag = &bars->abort_flag;
  pdl_wait();   // K^C, V, k^R and the query angles come from the kernels before
  if (threadIdx.x == 0) {
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&bars->k_full[s], 1);
      mbar_init(&bars->k_empty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&bars->v_full[s], 1);
      mbar_init(&bars->v_empty[s], 1);
    }
    mbar_init(&bars->q_ready, kAtSoftmaxThreads / 32);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->s_full[b], 1);
      mbar_init(&bars->p_full[b], kAtSoftmaxThreads / 32);
      mbar_init(&bars->pv_done[b], 1);
    }
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    bars->max_vis = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == kAtMma) {
    tmem_alloc(&bars->tmem_base, 512);
    tmem_relinquish();
  }
  // Rows this CTA's queries may see: vis = min(q_pos + 1, L), 0 past T or
  // for a negative position.
  int64_t vis = 0;
  int32_t pos = 0;
  if (threadIdx.x < kAtSoftmaxThreads) {
    const int t = q0 + (threadIdx.x & (kTileQ - 1));
    pos = t < T ? q_pos[t] : -1;
    vis = pos < 0 ? 0 : (int64_t(pos) + 1 < L ? int64_t(pos) + 1 : L);
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x < kTileQ && vis > 0) atomicMax(&bars->max_vis, int(vis));
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const int n_tiles = int((int64_t(bars->max_vis) + kTileK - 1) / kTileK);
  bool ok = true;

  if (warp == kAtKLoad || warp == kAtVLoad) {
    // ---------------------------------------------------------------- TMA
    const bool is_k = warp == kAtKLoad;
    const int stages = is_k ? kKStages : kVStages;
    uint64_t* full = is_k ? bars->k_full : bars->v_full;
    uint64_t* empty = is_k ? bars->k_empty : bars->v_empty;
    int issued = 0;
    if (lane == 0 && n_tiles > 0) {
      for (int k = 0; k < n_tiles; ++k) {
        const int s = k % stages;
        if (k >= stages &&
            !(ok = mbar_wait(&empty[s], ((k / stages) - 1) & 1, abort_flag, kWaitLimitCycles)))
          break;
        const int32_t row = int32_t(int64_t(i) * L + int64_t(k) * kTileK);
        if (is_k) {
          uint8_t* st = sK + s * kKStage;
          mbar_arrive_expect_tx(&full[s], uint32_t(nq * kBox));
          tma_load_2d(&tm_kc, &full[s], st, 0, row);
          tma_load_2d(&tm_kc, &full[s], st + kBox, 64, row);
          if (d_r) tma_load_2d(&tm_kr, &full[s], st + 2 * kBox, 0, k * kTileK);
        } else {
          uint8_t* st = sV + s * kVStage;
          mbar_arrive_expect_tx(&full[s], uint32_t(2 * kBox));
          tma_load_2d(&tm_v, &full[s], st, 0, row);
          tma_load_2d(&tm_v, &full[s], st + kBox, 64, row);
        }
        ++issued;
      }
      if (!ok) *abort_flag = 1;
      // Every issued load lands before the shared memory is released.
      for (int k = issued > stages ? issued - stages : 0; k < issued; ++k)
        wait_bar(&full[k % stages], (k / stages) & 1);
    }
  } else if (warp == kAtMma) {
    // ---------------------------------------------------------------- MMA
    if (n_tiles > 0) {
      // kind::f16 MMAs: the instruction descriptor names the operand type (fp16 for
      // QK^T, bf16 for P.V).
      constexpr uint32_t idesc_qk = idesc_f16_f32(128, 128, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 128, false, true);
      ok = warp_wait_bar(&bars->q_ready, 0, abort_flag);
      auto issue_pv = [&](int j) -> bool {
        const int b = j & 1, sv = j % kVStages;
        if (!warp_wait_bar(&bars->p_full[b], (j >> 1) & 1, abort_flag)) return false;
        if (!warp_wait_bar(&bars->v_full[sv], (j / kVStages) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint64_t v0 = smem_desc_sw128(smem_u32(sV + sv * kVStage), kBox, 1024);
#pragma unroll
        for (int kk = 0; kk < kTileK / 16; ++kk)
          mma_bf16_ts_w(tmem + kColO, tmem + kColS + uint32_t(b * 128 + kk * 8),
                        v0 + uint64_t((kk * 2048) >> 4), idesc_pv, j > 0 || kk > 0);
        mma_commit_w(&bars->pv_done[b]);
        mma_commit_w(&bars->v_empty[sv]);
        return true;
      };
      for (int k = 0; ok && k < n_tiles; ++k) {
        const int sk = k % kKStages;
        if (!(ok = warp_wait_bar(&bars->k_full[sk], (k / kKStages) & 1, abort_flag))) break;
        tc_fence_after();
        const uint32_t kb = smem_u32(sK + sk * kKStage);
        const uint32_t d = tmem + kColS + uint32_t((k & 1) * 128);
        for (int c = 0; c < nq; ++c) {
          const uint64_t b0 = smem_desc_sw128(kb + uint32_t(c * kBox), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ts_w(d, tmem + kColQ + uint32_t(c * 32 + kk * 8),
                         b0 + uint64_t((kk * 32) >> 4), idesc_qk, (c | kk) != 0);
        }
        mma_commit_w(&bars->s_full[k & 1]);
        mma_commit_w(&bars->k_empty[sk]);
        if (k >= 1 && !(ok = issue_pv(k - 1))) break;
      }
      if (ok) ok = issue_pv(n_tiles - 1);
      if (!ok && lane == 0) *abort_flag = 1;
    }
    // Every product issued has finished before tensor memory is released.
    mma_commit_w(&bars->drain);
    if (lane == 0) wait_bar(&bars->drain, 0);
    __syncwarp();
  } else if (warp < kAtSoftmaxThreads / 32) {
    // ---------------------------------------------------------------- softmax
    // Thread (warp w, lane) owns row r = 32 (w % 4) + lane, columns
    // [64 h, 64 h + 64) with h = w / 4, of S, P and O.  The two halves of a row
    // swap their maxima through shared memory once per tile (a 64-thread named
    // barrier per lane quadrant) and apply the same rescales, so their partial
    // sums add up at the end.
    const int quad = warp & 3, h = warp >> 2;
    const int r = 32 * quad + lane;
    const uint32_t lane_base = uint32_t(32 * quad) << 16;
    const int cb = 64 * h;
    // The query row into tensor memory (see nope_to_tmem / rope_to_tmem).
    {
      const int t = q0 + r;
      const bool valid = t < T;
      const int64_t row = int64_t(valid ? t : 0) * H + i;
      const uint4* src = reinterpret_cast<const uint4*>(q_nope + row * kDn);
      const uint32_t qa = tmem + lane_base + kColQ;
      if (h == 0) {
        nope_to_tmem(src, valid, 0, d_r ? 4 : 2, qa);
      } else if (d_r) {
        rope_to_tmem(reinterpret_cast<const uint4*>(q_pe + row * d_r),
                     reinterpret_cast<const float4*>(cs + int64_t(valid ? t : 0) * (d_r / 2)),
                     valid, qa + 64);
      } else {
        nope_to_tmem(src, valid, 2, 4, qa);
      }
      warp_arrive_after_tmem_st(&bars->q_ready);
    }
    float m_run = -INFINITY, l_run = 0.f;
    // Both halves of a row run every iteration up to the named barrier, even
    // after a give-up (then with no work), so the barrier never waits for a
    // thread that left the loop.
    for (int k = 0; k < n_tiles; ++k) {
      const int b = k & 1;
      if (!ok) bars->abort_flag = 1;   // the other roles stop waiting for this warp
      if (ok) ok = warp_wait_bar(&bars->s_full[b], (k >> 1) & 1, abort_flag);
      const int64_t nv = vis - int64_t(k) * kTileK - cb;   // visible columns of this half
      const int nvalid = nv <= 0 ? 0 : (nv >= 64 ? 64 : int(nv));
      const uint32_t s_addr = tmem + lane_base + kColS + uint32_t(b * 128);
      uint32_t va[32], vb[32];
      float mt = -INFINITY;
      if (ok) {
        tc_fence_after();
        tmem_ld32(s_addr + uint32_t(cb), va);
        tmem_ld32(s_addr + uint32_t(cb + 32), vb);
        tmem_wait_ld();
        if (nvalid == 64) {
#pragma unroll
          for (int e = 0; e < 32; ++e)
            mt = fmaxf(mt, fmaxf(__uint_as_float(va[e]), __uint_as_float(vb[e])));
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            if (e < nvalid) mt = fmaxf(mt, __uint_as_float(va[e]));
            if (e + 32 < nvalid) mt = fmaxf(mt, __uint_as_float(vb[e]));
          }
        }
      }
      bars->row_max[b][h][r] = mt;
      // Both halves have their S in registers past this barrier, so P may
      // overwrite the S columns.
      asm volatile("bar.sync %0, 64;" ::"r"(1 + quad) : "memory");
      if (!ok) continue;
      mt = fmaxf(mt, bars->row_max[b][1 - h][r]);
      const float m_new = fmaxf(m_run, mt * scale_log2);
      const bool rescale = m_run != -INFINITY && m_new > m_run + kRescaleLog2;
      if (__any_sync(0xffffffffu, rescale)) {
        // O holds the products up to tile k - 1: wait for the last of them.
        if (!(ok = warp_wait_bar(&bars->pv_done[(k - 1) & 1], ((k - 1) >> 1) & 1, abort_flag)))
          continue;
        tc_fence_after();
        const float f = rescale ? ex2_approx(m_run - m_new) : 1.f;
#pragma unroll 1
        for (int c0 = 0; c0 < 64; c0 += 32) {
          uint32_t o[32];
          const uint32_t oa = tmem + lane_base + kColO + uint32_t(cb + c0);
          tmem_ld32(oa, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
          tmem_st32(oa, o);
        }
        tmem_wait_st();
        if (rescale) {
          l_run *= f;
          m_run = m_new;
        }
      }
      if (m_run == -INFINITY) m_run = m_new;
      const float mu = m_run == -INFINITY ? 0.f : m_run;
      float sum = 0.f;
      uint32_t pa[16], pb[16];
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        float p0 = ex2_approx(fmaf(__uint_as_float(va[e]), scale_log2, -mu));
        float p1 = ex2_approx(fmaf(__uint_as_float(va[e + 1]), scale_log2, -mu));
        float p2 = ex2_approx(fmaf(__uint_as_float(vb[e]), scale_log2, -mu));
        float p3 = ex2_approx(fmaf(__uint_as_float(vb[e + 1]), scale_log2, -mu));
        if (nvalid < 64) {
          p0 = e < nvalid ? p0 : 0.f;
          p1 = e + 1 < nvalid ? p1 : 0.f;
          p2 = e + 32 < nvalid ? p2 : 0.f;
          p3 = e + 33 < nvalid ? p3 : 0.f;
        }
        sum += (p0 + p1) + (p2 + p3);
        pa[e / 2] = pack_bf16x2(p0, p1);
        pb[e / 2] = pack_bf16x2(p2, p3);
      }
      // P of keys [64 h, 64 h + 64) into columns [32 h, 32 h + 32) of the S buffer.
      tmem_st16(s_addr + uint32_t(cb / 2), pa);
      tmem_st16(s_addr + uint32_t(cb / 2 + 16), pb);
      l_run += sum;
      warp_arrive_after_tmem_st(&bars->p_full[b]);
    }
    if (!ok) {
      bars->abort_flag = 1;
    } else if (n_tiles > 0) {
      ok = warp_wait_bar(&bars->pv_done[(n_tiles - 1) & 1], ((n_tiles - 1) >> 1) & 1, abort_flag);
      tc_fence_after();
    }
    // Row sum of both halves.  Both threads of a row reach this barrier
    // whatever happened above (an abort only skips stores).
    bars->row_sum[h][r] = l_run;
    asm volatile("bar.sync %0, 64;" ::"r"(1 + quad) : "memory");
    const float l_row = bars->row_sum[0][r] + bars->row_sum[1][r];
    const int t = q0 + r;
    const float inv = l_row > 0.f ? 1.f / l_row : 0.f;
#pragma unroll 1
    for (int c0 = 0; c0 < 64; c0 += 32) {
      uint32_t o[32];
      if (n_tiles > 0) {
        tmem_ld32(tmem + lane_base + kColO + uint32_t(cb + c0), o);
        tmem_wait_ld();
      }
      if (ok && t < T) {
        __nv_bfloat16* dst = out + (int64_t(t) * H + i) * kDv + cb + c0;
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          float x[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) x[j] = n_tiles > 0 ? __uint_as_float(o[e + j]) * inv : 0.f;
          *reinterpret_cast<uint4*>(dst + e) =
              make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]),
                         pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7]));
        }
      }
    }
    if (h == 0 && ok && t < T && lse)
      lse[int64_t(t) * H + i] = l_row > 0.f ? (m_run + __log2f(l_row)) * 0.69314718055994531f
                                            : -INFINITY;
  }
  __syncthreads();
  if (threadIdx.x == 0 && bars->abort_flag) record_status(status, MLA_ERR_DEVICE_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == kAtMma) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <typename K>
cudaError_t set_smem_once(K kernel, size_t bytes) {
  static bool done[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (done[dev]) return cudaSuccess;
  const cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(bytes));
  if (e == cudaSuccess) done[dev] = true;
  return e;
}

size_t round1k(size_t x) { return (x + 1023) / 1024 * 1024; }

}  // namespace

size_t prefill_workspace_bytes(int T, int64_t L, int H, int d_r) {
  return 2 * round1k(size_t(H) * L * 128 * 2) + round1k(size_t(L) * d_r * 2) +
         round1k(size_t(T) * (d_r / 2) * 8);
}

cudaError_t launch_prefill(const __nv_bfloat16* q_nope, const __nv_bfloat16* q_pe,
                           const int32_t* q_pos, const __nv_bfloat16* W_UK,
                           const __nv_bfloat16* W_UV, const __nv_bfloat16* rows, int T, int64_t L,
                           int H, int d_r, float scale, float rope_base, __nv_bfloat16* out,
                           float* lse, void* workspace, int* status, cudaStream_t stream) {
  if (T <= 0) return cudaSuccess;
  const int R = kDcP + d_r;
  // Workspace: kc [H, L, 128] fp16 | v [H, L, 128] bf16 | kr [L, d_r] fp16 |
  // cs [T, d_r/2] float2, each rounded up to 1 KB.
  uint8_t* p = static_cast<uint8_t*>(workspace);
  __half* kc = reinterpret_cast<__half*>(p);
  p += round1k(size_t(H) * L * 128 * 2);
  __nv_bfloat16* v = reinterpret_cast<__nv_bfloat16*>(p);
  p += round1k(size_t(H) * L * 128 * 2);
  __half* kr = reinterpret_cast<__half*>(p);
  p += round1k(size_t(L) * d_r * 2);
  float2* cs = reinterpret_cast<float2*>(p);

  CUtensorMap tm_rows, tm_wuk, tm_wuv, tm_kc, tm_v, tm_kr;
  if (!make_map16(&tm_rows, rows, uint64_t(L), uint64_t(R), uint64_t(R), 128) ||
      !make_map16(&tm_wuk, W_UK, uint64_t(H) * 128, kDcP, kDcP, 128) ||
      !make_map16(&tm_wuv, W_UV, uint64_t(H) * 128, kDcP, kDcP, 128) ||
      !make_map16(&tm_kc, kc, uint64_t(H) * L, 128, 128, 128) ||
      !make_map16(&tm_v, v, uint64_t(H) * L, 128, 128, 128))
    return cudaErrorInvalidValue;
  // Without RoPE the k^R map is never read; it is built over kc instead.
  if (!(d_r ? make_map16(&tm_kr, kr, uint64_t(L), uint64_t(d_r), uint64_t(d_r), 128)
            : make_map16(&tm_kr, kc, uint64_t(H) * L, 128, 128, 128)))
    return cudaErrorInvalidValue;

  cudaError_t e;
  if (d_r) {
    const int64_t n = int64_t(T) * (d_r / 2);
    prefill_rope_table_kernel<<<int((n + 255) / 256 < 2048 ? (n + 255) / 256 : 2048), 256, 0,
                                stream>>>(q_pos, T, d_r, rope_base, cs);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  // With RoPE the projection may start beside the angle kernel: that kernel
  // itself started only after all earlier work in the stream, and the
  // projection reads only inputs.  It waits for the angle kernel before it
  // finishes, so the attention kernel, which waits for the projection, sees
  // the table.  Without RoPE it is an ordinary launch.
  if ((e = set_smem_once(prefill_kv_tc_kernel, kKvSmem)) != cudaSuccess) return e;
  const dim3 kv_grid(unsigned((L + 127) / 128), H);
  if (d_r) {
    e = launch_pdl(prefill_kv_tc_kernel, kv_grid, dim3(kKvThreads), kKvSmem, stream, tm_rows,
                   tm_wuk, tm_wuv, L, H, d_r, rows, kc, v, kr, status);
  } else {
    prefill_kv_tc_kernel<<<kv_grid, kKvThreads, kKvSmem, stream>>>(tm_rows, tm_wuk, tm_wuv, L, H,
                                                                   d_r, rows, kc, v, kr, status);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) return e;

  if ((e = set_smem_once(prefill_attn_tc_kernel, kAtSmem)) != cudaSuccess) return e;
  const float scale_log2 = scale * 1.4426950408889634f;
  return launch_pdl(prefill_attn_tc_kernel, dim3(unsigned((T + kTileQ - 1) / kTileQ), H),
                    dim3(kAtThreads), kAtSmem, stream, tm_kc, tm_v, tm_kr, q_nope, q_pe,
                    static_cast<const float2*>(cs), q_pos, T, L, H, d_r, scale_log2, out, lse,
                    status);
}

}  // namespace mla
