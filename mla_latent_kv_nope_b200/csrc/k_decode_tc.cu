// Tensor-core split-KV latent decode for sm_100a (bf16, d_c = 512, d_r = 64).
//
// What it computes ([MLA-とは] "実装上のトレードオフ": after absorption the
// decode is MQA with head dim d_c + d_r = 576 -- one latent row per cached
// token is the key of every head, its first 512 entries the value;
// "Value側の吸収": the weighted sum stays in latent space):
//   S = q_cat[b, heads] . C^T            (M = 64 heads, N = 64 keys, K = 576)
//   online softmax over the keys of one work range
//   O = P . C[:, 0:512]                  (M = 64 heads, N = 512, K = 64 keys)
// The two products are dense because all heads share the same latent rows.
//
// Structure (one CTA = 64 heads of one work range; CTAs of the same range for
// the other head groups are launched next to it so the tile is read from HBM
// once and from L2 after that):
//   warp 4      TMA producer: per tile, 9 boxes of [64 keys x 64 dims] bf16
//               with 128-byte swizzle into a 2-stage ring; the 64-head query
//               block is loaded the same way once per sequence.
//   warp 5      MMA issuer: tcgen05.mma kind::f16 (bf16 in, fp32 in TMEM).
//               QK^T of tile i+1 is issued while the softmax of tile i runs.
//   warps 0-3   softmax + correction + epilogue, reading S from TMEM
//               (tcgen05.ld), writing P as bf16 into the tile's dead RoPE
//               chunk (the swizzled K-major A operand of P.C), rescaling the
//               TMEM accumulator only when the running max grows by more
//               than 2^8, and storing the partial (o, lse).
// TMEM (M = 64 tiles occupy lanes 0-15 of each 32-lane quadrant, or lanes
// 16-31 with a lane offset of 16):
//   lanes +0 : cols [0,256)  O[:, 0:256]      cols [256,384) S double buffer
//   lanes +16: cols [0,256)  O[:, 256:512]
// Every wait is bounded (2 s); on give-up the CTA raises a shared abort flag,
// records MLA_ERR_DEVICE_TIMEOUT, drains its own loads, frees TMEM and exits.
#include <cuda.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace mla {

namespace {

using namespace sm100;

constexpr int kHeadsPerCta = 64;
constexpr int kR = 576;
constexpr int kDc = 512;
constexpr int kChunkElems = 64;                       // one 128-byte swizzle row
constexpr int kChunks = kR / kChunkElems;             // 9 (8 latent + 1 RoPE)
constexpr int kRopeChunk = 8;
constexpr int kChunkBytes = kTileKeys * 128;          // 8192
constexpr int kStageBytes = kChunks * kChunkBytes;    // 73728
constexpr int kStages = 2;
constexpr int kSoftmaxWarps = 4;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kThreads = 32 * (kSoftmaxWarps + 2);    // 192
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 256;
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr float kRescaleThreshold = 8.f;  // log2 units: rescale when the max grows by > 2^8

struct Barriers {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t q_full, q_empty;
  uint64_t s_full[2], s_free[2];
  uint64_t p_full[2];
  uint64_t o_free;
  uint64_t mma_drain;
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t kOffQ = 0;
constexpr size_t kOffStage = kStageBytes;
constexpr size_t kOffBar = kOffStage + size_t(kStages) * kStageBytes;
constexpr size_t kSmemBytes = kOffBar + sizeof(Barriers) + 1024;  // + alignment slack

constexpr uint32_t kIdescQK = idesc_bf16_f32(64, 64, false, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(64, 256, false, true);

__device__ __forceinline__ void raise_abort(Barriers* bars, int* status) {
  bars->abort_flag = 1;
  record_status(status, MLA_ERR_DEVICE_TIMEOUT);
}

// Warp-uniform bounded wait (all 32 lanes poll; lane 0 owns the time limit).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 0;; ++it) {
    const bool ok = mbar_try(bar, parity);
    if (__all_sync(0xffffffffu, ok)) return true;
    if ((it & 63) == 63) {
      int give_up = 0;
      if ((threadIdx.x & 31) == 0)
        give_up = (*abort_flag != 0) || (global_timer_ns() - t0 > kWaitLimitNs);
      if (__shfl_sync(0xffffffffu, give_up, 0)) return false;
    }
  }
}

// Sequences overlapping this worker's tile range are visited in order; the
// callback gets (b, first tile, end tile (both local to b), length).
template <typename F>
__device__ __forceinline__ void for_each_segment(const int32_t* seqlens, int B, int64_t cap,
                                                 int64_t t_begin, int64_t t_end, F&& f) {
  int64_t prefix = 0;
  for (int b = 0; b < B && prefix < t_end; ++b) {
    const int64_t L = clamp_len(seqlens[b], cap);
    const int64_t nt = tiles_of(L);
    const int64_t lo = max(prefix, t_begin), hi = min(prefix + nt, t_end);
    if (lo < hi) {
      if (!f(b, lo - prefix, hi - prefix, L)) return;
    }
    prefix += nt;
  }
}

__global__ void __launch_bounds__(kThreads, 1)
decode_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_c,
                 const int32_t* __restrict__ seqlens, int B, int H, int64_t cap,
                 float scale_log2, int W, float* __restrict__ o_part,
                 float* __restrict__ lse_part, int* __restrict__ status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + kOffQ;
  uint8_t* sStage = smem + kOffStage;
  Barriers* bars = reinterpret_cast<Barriers*>(smem + kOffBar);

  const int g = blockIdx.x;   // head group
  const int w = blockIdx.y;   // worker
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  int64_t n_tiles = 0;
  for (int b = 0; b < B; ++b) n_tiles += tiles_of(clamp_len(seqlens[b], cap));
  if (n_tiles == 0) return;
  const int64_t t_begin = worker_tile_begin(w, n_tiles, W);
  const int64_t t_end = worker_tile_begin(w + 1, n_tiles, W);
  if (t_begin >= t_end) return;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->q_full, 1);
    mbar_init(&bars->q_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->s_full[s], 1);
      mbar_init(&bars->s_free[s], 32 * kSoftmaxWarps);
      mbar_init(&bars->p_full[s], 32 * kSoftmaxWarps);
    }
    mbar_init(&bars->o_free, 32 * kSoftmaxWarps);
    mbar_init(&bars->mma_drain, 1);
    bars->abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_c);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort_flag = &bars->abort_flag;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t i = 0;
      int seg = 0;
      bool ok = true;
      for_each_segment(seqlens, B, cap, t_begin, t_end,
                       [&](int b, int64_t lo, int64_t hi, int64_t) {
        if (seg > 0 && !(ok = mbar_wait(&bars->q_empty, (seg - 1) & 1, abort_flag, kWaitLimitNs)))
          return false;
        ++seg;
        mbar_arrive_expect_tx(&bars->q_full, kStageBytes);
        const int32_t qrow = b * H + g * kHeadsPerCta;
        for (int c = 0; c < kChunks; ++c)
          tma_load_2d(&tm_q, &bars->q_full, sQ + c * kChunkBytes, c * kChunkElems, qrow);
        for (int64_t t = lo; t < hi; ++t, ++i) {
          const int s = i & 1;
          if (i >= 2 && !(ok = mbar_wait(&bars->empty[s], ((i >> 1) - 1) & 1, abort_flag,
                                         kWaitLimitNs)))
            return false;
          mbar_arrive_expect_tx(&bars->full[s], kStageBytes);
          const int32_t crow = int32_t(int64_t(b) * cap + t * kTileKeys);
          uint8_t* dst = sStage + s * kStageBytes;
          for (int c = 0; c < kChunks; ++c)
            tma_load_2d(&tm_c, &bars->full[s], dst + c * kChunkBytes, c * kChunkElems, crow);
        }
        return true;
      });
      if (!ok) {
        raise_abort(bars, status);
        // Drain this CTA's own loads before it may exit: the last load into
        // each stage and the last query block (bounded, ignoring the flag).
        volatile int no_abort = 0;
        for (uint32_t k = (i > 2 ? i - 2 : 0); k < i; ++k)
          mbar_wait(&bars->full[k & 1], (k >> 1) & 1, &no_abort, kWaitLimitNs);
        if (seg > 0) mbar_wait(&bars->q_full, (seg - 1) & 1, &no_abort, kWaitLimitNs);
      }
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t i_qk = 0, i_pv = 0;
      int seg = 0;
      bool ok = true;
      const uint32_t q_base = smem_u32(sQ);
      const uint32_t st_base = smem_u32(sStage);
      for_each_segment(seqlens, B, cap, t_begin, t_end,
                       [&](int, int64_t lo, int64_t hi, int64_t) {
        const uint32_t base = i_pv, end = i_pv + uint32_t(hi - lo);
        if (!(ok = mbar_wait(&bars->q_full, seg & 1, abort_flag, kWaitLimitNs))) return false;
        tc_fence_after();
        uint64_t t_last = global_timer_ns();
        uint32_t spins = 0;
        while (i_pv < end) {
          bool progressed = false;
          if (i_qk < end && i_qk <= i_pv + 1) {
            const int s = i_qk & 1;
            if (mbar_test(&bars->full[s], (i_qk >> 1) & 1) &&
                (i_qk < 2 || mbar_test(&bars->s_free[s], ((i_qk >> 1) - 1) & 1))) {
              tc_fence_after();
              const uint32_t d = tmem + kColS + uint32_t(s) * 64u;
              const uint32_t stage = st_base + uint32_t(s) * kStageBytes;
#pragma unroll 1
              for (int c = 0; c < kChunks; ++c) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  const uint64_t a = smem_desc_sw128(q_base + c * kChunkBytes + k * 32, 16, 1024);
                  const uint64_t bdesc =
                      smem_desc_sw128(stage + c * kChunkBytes + k * 32, 16, 1024);
                  mma_bf16_ss(d, a, bdesc, kIdescQK, (c | k) != 0);
                }
              }
              mma_commit(&bars->s_full[s]);
              ++i_qk;
              if (i_qk == end) mma_commit(&bars->q_empty);
              progressed = true;
            }
          }
          if (!progressed && i_pv < i_qk) {
            const int s = i_pv & 1;
            const bool first = (i_pv == base);
            if (mbar_test(&bars->p_full[s], (i_pv >> 1) & 1) &&
                (!first || seg == 0 || mbar_test(&bars->o_free, (seg - 1) & 1))) {
              tc_fence_after();
              const uint32_t stage = st_base + uint32_t(s) * kStageBytes;
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const uint32_t d = tmem + (h ? (16u << 16) : 0u);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                  const uint64_t a =
                      smem_desc_sw128(stage + kRopeChunk * kChunkBytes + k * 32, 16, 1024);
                  const uint64_t bdesc = smem_desc_sw128(
                      stage + (4 * h) * kChunkBytes + k * 2048, kChunkBytes, 1024);
                  mma_bf16_ss(d, a, bdesc, kIdescPV, !(first && k == 0));
                }
              }
              mma_commit(&bars->empty[s]);
              ++i_pv;
              progressed = true;
            }
          }
          if (progressed) {
            spins = 0;
            t_last = global_timer_ns();
          } else if ((++spins & 255) == 0) {
            if (*abort_flag || global_timer_ns() - t_last > kWaitLimitNs) {
              ok = false;
              return false;
            }
          }
        }
        ++seg;
        return true;
      });
      if (!ok) raise_abort(bars, status);
      // Every MMA issued by this thread has completed before TMEM is freed.
      mma_commit(&bars->mma_drain);
      volatile int no_abort = 0;
      mbar_wait(&bars->mma_drain, 0, &no_abort, kWaitLimitNs);
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int q = warp;                      // TMEM lane quadrant
    const bool lo_half = lane < 16;
    const int row = 16 * q + (lane & 15);    // head row within the CTA
    const int head = g * kHeadsPerCta + row;
    const uint32_t lane_base = uint32_t(32 * q) << 16;
    const int tid = threadIdx.x;             // 0..127
    float m_ref = -INFINITY, l_sum = 0.f;
    uint32_t i = 0;
    bool ok = true;
    for_each_segment(seqlens, B, cap, t_begin, t_end,
                     [&](int b, int64_t lo, int64_t hi, int64_t L) {
      const int slot = b + w;
      for (int64_t t = lo; t < hi; ++t, ++i) {
        const int s = i & 1;
        if (!(ok = warp_wait(&bars->s_full[s], (i >> 1) & 1, abort_flag))) return false;
        tc_fence_after();
        uint32_t sv[64];
        {
          uint32_t (&a)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[0]);
          uint32_t (&c)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[32]);
          tmem_ld32(tmem + lane_base + kColS + uint32_t(s) * 64u, a);
          tmem_ld32(tmem + lane_base + kColS + uint32_t(s) * 64u + 32u, c);
        }
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&bars->s_free[s]);

        const int64_t key0 = t * kTileKeys;
        const int valid = int(min(int64_t(kTileKeys), L - key0));
        uint8_t* stage = sStage + s * kStageBytes;
        if (valid < kTileKeys) {
          // Rows past the sequence end may hold anything: zero them so the
          // P.C product (where their weight is exactly 0) stays finite.
          fence_proxy_async_smem();
          const int nrow = kTileKeys - valid;
          for (int u = tid; u < nrow * 8 * 8; u += 32 * kSoftmaxWarps) {
            const int r = valid + u / 64, c = (u / 8) % 8, v = u % 8;
            *reinterpret_cast<uint4*>(stage + c * kChunkBytes + r * 128 + v * 16) =
                make_uint4(0, 0, 0, 0);
          }
        }
        const bool first = (t == lo);
        float alpha = 1.f;
        int resc = 0;
        if (lo_half) {
          float mt = -INFINITY;
#pragma unroll
          for (int j = 0; j < 64; ++j) {
            const float x = (j < valid) ? __uint_as_float(sv[j]) * scale_log2 : -INFINITY;
            sv[j] = __float_as_uint(x);
            mt = fmaxf(mt, x);
          }
          if (first) {
            m_ref = mt;
            l_sum = 0.f;
          } else if (mt > m_ref + kRescaleThreshold) {
            alpha = exp2f(m_ref - mt);
            m_ref = mt;
            l_sum *= alpha;
            resc = 1;
          }
          float sum = 0.f;
          uint8_t* prow = stage + kRopeChunk * kChunkBytes + row * 128;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float p0 = exp2f(__uint_as_float(sv[8 * u + 2 * e]) - m_ref);
              const float p1 = exp2f(__uint_as_float(sv[8 * u + 2 * e + 1]) - m_ref);
              const __nv_bfloat162 pp = __floats2bfloat162_rn(p0, p1);
              sum += __low2float(pp) + __high2float(pp);
              pk[e] = *reinterpret_cast<const uint32_t*>(&pp);
            }
            *reinterpret_cast<uint4*>(prow + ((u ^ (row & 7)) * 16)) =
                make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
          l_sum += sum;
        }
        alpha = __shfl_sync(0xffffffffu, alpha, lane & 15);
        resc = __shfl_sync(0xffffffffu, resc, lane & 15);
        if (__any_sync(0xffffffffu, resc)) {
          // O holds tile i-1's product once PV(i-1) has completed.
          const uint32_t prev = i - 1;
          if (!(ok = warp_wait(&bars->empty[prev & 1], (prev >> 1) & 1, abort_flag))) return false;
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < 256; c += 32) {
            uint32_t r[32];
            tmem_ld32(tmem + lane_base + uint32_t(c), r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            tmem_st32(tmem + lane_base + uint32_t(c), r);
          }
          tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bars->p_full[s]);
      }
      // Segment epilogue: normalised partial output and log-sum-exp.
      const uint32_t last = i - 1;
      if (!(ok = warp_wait(&bars->empty[last & 1], (last >> 1) & 1, abort_flag))) return false;
      tc_fence_after();
      const float l_row = __shfl_sync(0xffffffffu, l_sum, lane & 15);
      const float inv = 1.f / l_row;
      float* dst = o_part + (int64_t(slot) * H + head) * kDc + (lo_half ? 0 : 256);
#pragma unroll 1
      for (int c = 0; c < 256; c += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_base + uint32_t(c), r);
        tmem_wait_ld();
        if (head < H) {
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dst + c + e) =
                make_float4(__uint_as_float(r[e]) * inv, __uint_as_float(r[e + 1]) * inv,
                            __uint_as_float(r[e + 2]) * inv, __uint_as_float(r[e + 3]) * inv);
        }
      }
      if (lo_half && head < H)
        lse_part[int64_t(slot) * H + head] = (m_ref + log2f(l_sum)) * 0.69314718055994531f;
      tc_fence_before();
      mbar_arrive(&bars->o_free);
      return true;
    });
    if (!ok && lane == 0) raise_abort(bars, status);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
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

// 2D bf16 map over a row-major [rows, 576] matrix, 64 x 64 boxes, 128B swizzle.
bool make_rows_map(CUtensorMap* map, const void* base, uint64_t rows) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cuuint64_t(kR), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(kR) * 2};
  const cuuint32_t box[2] = {cuuint32_t(kChunkElems), cuuint32_t(kTileKeys)};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

int decode_tc_head_groups(int H) { return (H + kHeadsPerCta - 1) / kHeadsPerCta; }

cudaError_t launch_decode_tc(const __nv_bfloat16* q_cat, const __nv_bfloat16* cache,
                             const int32_t* seqlens, int B, int H, int64_t cap, float scale,
                             int W, float* o_part, float* lse_part, int* status,
                             cudaStream_t stream) {
  if (int64_t(B) * cap >= (int64_t(1) << 31) || int64_t(B) * H >= (int64_t(1) << 31))
    return cudaErrorInvalidValue;
  CUtensorMap tm_q, tm_c;
  if (!make_rows_map(&tm_q, q_cat, uint64_t(B) * H) ||
      !make_rows_map(&tm_c, cache, uint64_t(B) * uint64_t(cap)))
    return cudaErrorInvalidValue;
  static bool attr_done[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(kSmemBytes));
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  const float scale_log2 = scale * 1.4426950408889634f;
  dim3 grid(decode_tc_head_groups(H), W);
  decode_tc_kernel<<<grid, kThreads, kSmemBytes, stream>>>(tm_q, tm_c, seqlens, B, H, cap,
                                                           scale_log2, W, o_part, lse_part,
                                                           status);
  return cudaGetLastError();
}

}  // namespace mla
