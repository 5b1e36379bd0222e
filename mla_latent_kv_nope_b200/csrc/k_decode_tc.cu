// Tensor-core split-KV latent decode for sm_100a (bf16, d_c = 512, d_r = 64,
// or d_r = 0 for MLA without the decoupled RoPE part; or an FP8 latent cache,
// widened in shared memory to fp16 operands).
//
// What it computes ([MLA-とは] "実装上のトレードオフ": after absorption the
// decode is MQA with head dim d_c + d_r = 576 -- one latent row per cached
// token is the key of every head, its first 512 entries the value;
// "Value側の吸収": the weighted sum stays in latent space):
//   S = q_cat[b, heads] . C^T            (M = 64 heads, N = 64 keys, K = 512 + d_r)
//   online softmax over the keys of one work range
//   O = P . C[:, 0:512]                  (M = 64 heads, N = 512, K = 64 keys)
// The two products are dense because all heads share the same latent rows.
//
// Structure (one CTA = 64 heads of one work range; CTAs of the same range for
// the other head groups are launched next to it so the tile is read from HBM
// once and from L2 after that):
//   warp 4      TMA producer: per 64-key tile, 9 (or 8 without RoPE) boxes of
//               [64 keys x 64 dims] bf16 with 128-byte swizzle into a 3-stage
//               ring.  A stage always
//               has 9 chunks: the ninth (the RoPE keys, or nothing without
//               RoPE) receives P once S has been computed.
//   warp 5      QK^T issuer: S = Q C^T with Q read from tensor memory (only
//               the cache tile is fetched from shared memory); it runs ahead
//               as far as the stages and the two S buffers allow.
//   warp 6      P.C issuer: O += P C with P and C from shared memory, as soon
//               as a tile's probabilities are written.  Two issuing warps keep
//               a ready P.C from waiting behind a queued QK^T (a warp's next
//               barrier poll waits for its own MMAs to be taken up).
//   warps 0-3   softmax, correction and epilogue.  At each sequence start
//               they write the 64 x 576 query block into tensor memory.
// Tensor memory (an M = 64 tile occupies 16 of the 32 lanes of each
// quadrant; "lo" = lanes 0-15, "hi" = lanes 16-31):
//   lo lanes: cols [0,64) and [64,128) S double buffer; cols [128,416) Q
//             (512 + d_r bf16 packed in pairs)
//   hi lanes: cols [0,256) O[:, 0:256]; cols [256,512) O[:, 256:512]
// All tensor-memory traffic of the softmax warps uses 16-lane accesses, so
// each row is shared by two threads (keys 0-31 / 32-63 of S; columns
// 0-255 / 256-511 of O) and the other lane half is never touched.
// Every wait is bounded (about 2 s of SM cycles); on give-up the CTA raises
// a shared abort flag, records MLA_ERR_DEVICE_TIMEOUT, drains its own loads
// and MMAs, frees TMEM and exits.
#include <cuda.h>
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"
#include "tile_deal.cuh"

namespace mla {

namespace {

using namespace sm100;

constexpr int kHeadsPerCta = 64;
constexpr int kR = 576;                               // row width with RoPE
constexpr int kDc = 512;
constexpr int kChunkElems = 64;                       // one 128-byte swizzle row
constexpr int kChunks = kR / kChunkElems;             // 9 chunks per stage (8 latent + 1)
constexpr int kRopeChunk = 8;                         // RoPE keys, then P
constexpr int kChunkBytes = kTileKeys * 128;          // 8192
constexpr int kStageBytes = kChunks * kChunkBytes;    // 73728
constexpr int kStages = 3;
constexpr int kSoftmaxWarps = 4;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;                           // QK^T; owns the TMEM allocation
constexpr int kPvWarp = 6;                            // P.C
constexpr int kWidenWarp0 = 7;                        // FP8 cache: warps 7-10 widen codes
constexpr int kWidenThreads = 128;
// 224 threads; 352 with the FP8 cache's widen warps.
template <bool kFp8>
struct Threads { static constexpr int n = 32 * (kSoftmaxWarps + 3) + (kFp8 ? kWidenThreads : 0); };
// FP8 cache rows: 512 E4M3 codes then 64 bf16 RoPE keys (640 bytes); a stage
// receives the 4 code boxes [64 rows x 128 codes] in chunks 4-7 and the RoPE
// box in chunk 8.
constexpr int kFp8RowBytes = 512 + 2 * 64;
constexpr uint32_t kFp8LoadBytes = 5 * 8192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;                         // lo lanes, 2 x 64 columns
constexpr uint32_t kColQ = 128;                       // lo lanes, 288 columns
constexpr uint32_t kHiLanes = 16u << 16;              // lane offset of the hi half
constexpr float kRescaleThreshold = 8.f;  // log2 units: rescale when the max grows by > 2^8

struct Barriers {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t q_ready;
  uint64_t s_full[2], s_free[2];
  uint64_t p_full[2];
  uint64_t o_free;
  uint64_t mma_drain, pv_drain;
  uint64_t never;                 // injected test wait: nothing ever arrives on it
  uint64_t widened[kStages];      // FP8 cache: the stage holds fp16 latent rows
  uint64_t wsync[kStages];        // FP8 cache: every widen thread has read its codes
  uint32_t tmem_base;
  int abort_flag;
};

constexpr size_t kOffStage = 0;
constexpr size_t kOffBar = size_t(kStages) * kStageBytes;
constexpr size_t kOffPrefix = kOffBar + ((sizeof(Barriers) + 15) / 16) * 16;
constexpr size_t kSmemBytes = kOffPrefix + kTilePrefixSmemBytes + 1024;
static_assert(kSmemBytes <= 232448, "shared memory budget of one CTA");

constexpr uint32_t kIdescQK = idesc_bf16_f32(64, 64, false, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(64, 256, false, true);
// FP8 cache: both products in fp16 (the widened codes, the query, the scaled
// RoPE keys and P are fp16 operands).
constexpr uint32_t kIdescQK16 = idesc_f16_f32(64, 64, false, false);
constexpr uint32_t kIdescPV16 = idesc_f16_f32(64, 256, false, true);

__device__ __forceinline__ void raise_abort(Barriers* bars, int* status) {
  bars->abort_flag = 1;
  record_status(status, MLA_ERR_DEVICE_TIMEOUT);
}

// Warp-uniform bounded wait (all 32 lanes poll; lane 0 owns the limit).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          uint64_t limit = kWaitLimitCycles) {
  if (__all_sync(0xffffffffu, mbar_try(bar, parity))) return true;
  const uint64_t t0 = sm_cycles();
  for (uint32_t it = 0;; ++it) {
    const bool ok = mbar_try(bar, parity);
    if (__all_sync(0xffffffffu, ok)) return true;
    if ((it & 63) == 63) {
      int give_up = 0;
      if ((threadIdx.x & 31) == 0)
        give_up = (*abort_flag != 0) || (sm_cycles() - t0 > limit);
      if (__shfl_sync(0xffffffffu, give_up, 0)) return false;
    }
  }
}

// 8 E4M3 codes (little-endian in `c`) times the token's power-of-two scale
// (`s2`, the scale as fp16 in both halves), as 8 fp16: the code converts
// exactly (every finite E4M3 value is an fp16 value) and the product is one
// fp16 multiply, exact while it is a normal fp16 (|c| >= 2^-14) and rounded
// once below that.  fp16 holds every latent value of magnitude below 65504
// and every power-of-two scale from 2^-24 to 2^15.
__device__ __forceinline__ uint4 e4m3x8_to_f16(uint2 c, __half2 s2) {
  uint32_t out[4];
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const uint32_t word = p < 2 ? c.x : c.y;
    const __nv_fp8x2_storage_t pair = __nv_fp8x2_storage_t((word >> (16 * (p & 1))) & 0xFFFFu);
    const __half2 v = __hmul2(__half2(__nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3)), s2);
    out[p] = *reinterpret_cast<const uint32_t*>(&v);
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
}

// 8 bf16 as 8 fp16, rounded to nearest (exact for |x| in fp16's normal
// range with at most 11 significant bits, which every bf16 value has).
__device__ __forceinline__ uint4 bf16x8_to_f16(uint4 v) {
  uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const __half2 h = __floats2half2_rn(__uint_as_float(w[p] << 16),
                                        __uint_as_float(w[p] & 0xFFFF0000u));
    w[p] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

template <int kDr, bool kFp8>
__global__ void __launch_bounds__(Threads<kFp8>::n, 1)
decode_tc_kernel(const __grid_constant__ CUtensorMap tm_c, const __grid_constant__ CUtensorMap tm_codes,
                 const __nv_bfloat16* __restrict__ cache, const float* __restrict__ scales,
                 const PageMap pm,
                 const __nv_bfloat16* __restrict__ q_cat,
                 const int32_t* __restrict__ seqlens, int B, int H, int64_t cap,
                 float scale_log2, int W, float* __restrict__ o_part,
                 float* __restrict__ lse_part, int* __restrict__ status, uint64_t inject_wait) {
  static_assert(!kFp8 || kDr == 64, "the FP8 cache carries the 64-wide RoPE keys");
  constexpr int R = kDc + kDr;                    // cache row and q_cat row width
  constexpr int kLoadChunks = R / kChunkElems;    // bf16 chunks the QK^T product reads
  constexpr uint32_t kLoadBytes = kFp8 ? kFp8LoadBytes : kLoadChunks * kChunkBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sStage = smem + kOffStage;
  Barriers* bars = reinterpret_cast<Barriers*>(smem + kOffBar);

  const int g = blockIdx.x;   // head group
  const int w = blockIdx.y;   // worker
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // Tile prefix of the batch (all threads load lengths in parallel; warp 0
  // scans 32 at a time with shuffles).
  pdl_wait();   // lengths, queries and the appended rows come from earlier kernels
  TilePrefix tp;
  const int64_t n_tiles = build_tile_prefix(smem + kOffPrefix, seqlens, B, cap, &tp);
  if (n_tiles == 0) return;
  const int64_t t_begin = worker_tile_begin(w, n_tiles, W);
  const int64_t t_end = worker_tile_begin(w + 1, n_tiles, W);
  if (t_begin >= t_end) return;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->q_ready, 32 * kSoftmaxWarps);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->s_full[s], 1);
      mbar_init(&bars->s_free[s], 32 * kSoftmaxWarps);
      mbar_init(&bars->p_full[s], 32 * kSoftmaxWarps);
    }
    mbar_init(&bars->o_free, 32 * kSoftmaxWarps);
    mbar_init(&bars->mma_drain, 1);
    mbar_init(&bars->pv_drain, 1);
    mbar_init(&bars->never, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->widened[s], kWidenThreads);
      mbar_init(&bars->wsync[s], kWidenThreads);
    }
    bars->abort_flag = 0;
    fence_mbar_init();
    fence_proxy_async_smem();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&tm_c);
    if (kFp8) tma_prefetch_desc(&tm_codes);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort_flag = &bars->abort_flag;
  uint32_t n_issued = 0;   // loads issued by the producer (lane 0 of its warp)

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t i = 0;
      bool ok = true;
      for_each_segment(tp, t_begin, t_end,
                       [&](int b, int64_t lo, int64_t hi, int64_t) {
        // No L2 prefetch ahead of the stage loads: measured on B200 it was
        // neutral with 128 heads and cost 10 % with 64 (prefetched tiles
        // evicted before their loads by the other CTAs' streams).
        for (int64_t t = lo; t < hi; ++t, ++i) {
          const int s = i % kStages;
          // The tile's first row (a page-table read when paged) is looked up
          // before the stage wait so its latency hides behind it.  A page id
          // outside the pool is reported and read as zeros (a row past the
          // tensor map).
          int64_t r = pm.tile_row(b, t);
          if (i >= kStages && !(ok = mbar_wait(&bars->empty[s], ((i / kStages) - 1) & 1,
                                               abort_flag, kWaitLimitCycles)))
            return false;
          if (r < 0) {
            record_status(status, MLA_ERR_BOUNDS);
            r = pm.total_rows(B);
          }
          mbar_arrive_expect_tx(&bars->full[s], kLoadBytes);
          const int32_t crow = int32_t(r);
          uint8_t* dst = sStage + s * kStageBytes;
          if (kFp8) {
            // Codes: 4 boxes [64 rows x 128 bytes] into chunks 4-7 (128-byte
            // swizzle); RoPE keys: bf16 columns 256..319 of the row into chunk 8.
            for (int c = 0; c < 4; ++c)
              tma_load_2d(&tm_codes, &bars->full[s], dst + (4 + c) * kChunkBytes, c * 128, crow);
            tma_load_2d(&tm_c, &bars->full[s], dst + kRopeChunk * kChunkBytes, 256, crow);
          } else {
            for (int c = 0; c < kLoadChunks; ++c)
              tma_load_2d(&tm_c, &bars->full[s], dst + c * kChunkBytes, c * kChunkElems, crow);
          }
        }
        return true;
      });
      if (!ok) raise_abort(bars, status);
      n_issued = i;
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ QK^T issuer
    // The whole warp waits (all lanes poll) and elect.sync issues each
    // instruction from one lane.
    uint32_t i = 0;
    int seg = 0;
    bool ok = true;
    const uint32_t st_base = smem_u32(sStage);
    // Test hook: a wait on a barrier nothing arrives on, so the give-up path runs.
    if (inject_wait) ok = warp_wait(&bars->never, 0, abort_flag, inject_wait);
    if (ok) for_each_segment(tp, t_begin, t_end, [&](int, int64_t lo, int64_t hi, int64_t) {
      // The softmax warps have written this sequence's query block.
      if (!(ok = warp_wait(&bars->q_ready, seg & 1, abort_flag))) return false;
      for (int64_t t = lo; t < hi; ++t, ++i) {
        const int st = i % kStages, sb = i & 1;
        // The stage holds bf16 rows (for the FP8 cache: once widened).
        if (!(ok = warp_wait(kFp8 ? &bars->widened[st] : &bars->full[st], (i / kStages) & 1,
                             abort_flag)))
          return false;
        if (i >= 2 && !(ok = warp_wait(&bars->s_free[sb], ((i >> 1) - 1) & 1, abort_flag)))
          return false;
        tc_fence_after();
        const uint32_t d = tmem + kColS + uint32_t(sb) * 64u;
        // Descriptor and TMEM address bases are formed once; each of the 36
        // MMAs then only adds a compile-time offset (the start address field
        // is the low 14 bits: shared-memory offsets >> 4).
        const uint64_t b0 = smem_desc_sw128(st_base + uint32_t(st) * kStageBytes, 16, 1024);
        const uint32_t a0 = tmem + kColQ;
#pragma unroll
        for (int c = 0; c < kLoadChunks; ++c) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            mma_bf16_ts_w(d, a0 + uint32_t(c * 4 + k) * 8u,
                          b0 + uint64_t((c * kChunkBytes + k * 32) >> 4),
                          kFp8 ? kIdescQK16 : kIdescQK, (c | k) != 0);
        }
        mma_commit_w(&bars->s_full[sb]);
      }
      ++seg;
      return true;
    });
    if (!ok && lane == 0) raise_abort(bars, status);
    // Every MMA issued by this warp has completed before TMEM is freed.
    mma_commit_w(&bars->mma_drain);
    volatile int no_abort = 0;
    warp_wait(&bars->mma_drain, 0, &no_abort);
  } else if (warp == kPvWarp) {
    // ------------------------------------------------------------ P.C issuer
    uint32_t i = 0;
    int seg = 0;
    bool ok = true;
    const uint32_t st_base = smem_u32(sStage);
    for_each_segment(tp, t_begin, t_end, [&](int, int64_t lo, int64_t hi, int64_t) {
      for (int64_t t = lo; t < hi; ++t, ++i) {
        const int st = i % kStages, sb = i & 1;
        const bool first = (t == lo);
        if (!(ok = warp_wait(&bars->p_full[sb], (i >> 1) & 1, abort_flag))) return false;
        // The previous sequence's epilogue has read O before it is overwritten.
        if (first && seg > 0 && !(ok = warp_wait(&bars->o_free, (seg - 1) & 1, abort_flag)))
          return false;
        tc_fence_after();
        const uint32_t stage = st_base + uint32_t(st) * kStageBytes;
        const uint64_t a0 = smem_desc_sw128(stage + kRopeChunk * kChunkBytes, 16, 1024);
        const uint64_t b0 = smem_desc_sw128(stage, kChunkBytes, 1024);
        // The two output halves are independent accumulators: alternate them
        // so consecutive MMAs do not depend on each other.
#pragma unroll
        for (int k = 0; k < 4; ++k) {
#pragma unroll
          for (int h = 0; h < 2; ++h)
            mma_bf16_ss_w(tmem + kHiLanes + uint32_t(h) * 256u, a0 + uint64_t((k * 32) >> 4),
                          b0 + uint64_t((4 * h * kChunkBytes + k * 2048) >> 4),
                          kFp8 ? kIdescPV16 : kIdescPV, !(first && k == 0));
        }
        mma_commit_w(&bars->empty[st]);
      }
      ++seg;
      return true;
    });
    if (!ok && lane == 0) raise_abort(bars, status);
    mma_commit_w(&bars->pv_drain);
    volatile int no_abort = 0;
    warp_wait(&bars->pv_drain, 0, &no_abort);
  } else if (kFp8 && warp >= kWidenWarp0) {
    // ------------------------------------------------------------ widen (FP8 cache)
    // Thread (r, hh) expands row r of code boxes hh and 2 + hh: box c holds
    // latent columns [128c, 128c + 128), i.e. fp16 chunks 2c and 2c + 1.
    // Boxes 0-1 (chunks 4-5) are widened into chunks 0-3; boxes 2-3 are read
    // into registers, every widen thread meets at `wsync` (so chunks 4-7 have
    // been read by all), then written into chunks 4-7.  Both products run in
    // fp16, so the row's RoPE keys (chunk 8, bf16) are rewritten in place as
    // fp16 too.
    const int wt = threadIdx.x - 32 * kWidenWarp0;
    const int r = wt >> 1, hh = wt & 1;
    uint32_t i = 0;
    bool ok = true;
    auto store_units = [&](uint8_t* stage, int box, int v, uint4 lo, uint4 hi_) {
      // 16 codes -> dims [128 box + 16 v, +16): fp16 units 2(v%4), 2(v%4)+1 of
      // chunk 2 box + v / 4, 128-byte swizzled.
      uint8_t* chunk = stage + (2 * box + v / 4) * kChunkBytes + r * 128;
      const int u0 = 2 * (v % 4);
      *reinterpret_cast<uint4*>(chunk + ((u0 ^ (r & 7)) * 16)) = lo;
      *reinterpret_cast<uint4*>(chunk + (((u0 + 1) ^ (r & 7)) * 16)) = hi_;
    };
    // The row's scale for tile t of sequence b; rows past the sequence's
    // length get 0 (their keys are masked and their rows zeroed before P.C;
    // their stored scales may hold anything).
    auto load_scale = [&](int b, int64_t t) {
      if (b < 0) return 0.f;
      const int64_t key = t * kTileKeys + r;
      const int64_t prow = key < tp.len(b) ? pm.row(b, key) : -1;
      return prow >= 0 ? scales[prow] : 0.f;
    };
    // Scales are read one tile ahead of their use (a global load per row
    // would otherwise put its latency on every tile).
    float next_scale = 0.f;
    {
      const int b0 = tp.next_sequence(-1, t_begin, t_end);
      if (b0 >= 0) next_scale = load_scale(b0, max(tp.tile0(b0), t_begin) - tp.tile0(b0));
    }
    for_each_segment(tp, t_begin, t_end, [&](int b, int64_t lo, int64_t hi, int64_t) {
      for (int64_t t = lo; t < hi; ++t, ++i) {
        const int s = i % kStages;
        const float scale = next_scale;
        // The next tile is t + 1 of this sequence, or tile 0 of the next
        // sequence of the range (a range enters later sequences at tile 0).
        if (t + 1 < hi) next_scale = load_scale(b, t + 1);
        else next_scale = load_scale(tp.next_sequence(b, t_begin, t_end), 0);
        if (!(ok = warp_wait(&bars->full[s], (i / kStages) & 1, abort_flag))) return false;
        uint8_t* stage = sStage + s * kStageBytes;
        const __half2 s2 = __float2half2_rn(scale);
        // Code boxes arrive 128-byte swizzled like the bf16 chunks: unit v
        // (16 codes) of row r sits at 16 (v ^ (r % 8)), so the rows a warp
        // reads together fall in different banks.
        auto code_unit = [&](int box, int v) {
          return *reinterpret_cast<const uint4*>(stage + (4 + box) * kChunkBytes + r * 128 +
                                                 ((v ^ (r & 7)) * 16));
        };
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          const uint4 c = code_unit(hh, v);
          store_units(stage, hh, v, e4m3x8_to_f16(make_uint2(c.x, c.y), s2),
                      e4m3x8_to_f16(make_uint2(c.z, c.w), s2));
        }
        uint4 c2[8];
#pragma unroll
        for (int v = 0; v < 8; ++v) c2[v] = code_unit(2 + hh, v);
        mbar_arrive(&bars->wsync[s]);
        if (!(ok = warp_wait(&bars->wsync[s], (i / kStages) & 1, abort_flag))) return false;
#pragma unroll
        for (int v = 0; v < 8; ++v)
          store_units(stage, 2 + hh, v, e4m3x8_to_f16(make_uint2(c2[v].x, c2[v].y), s2),
                      e4m3x8_to_f16(make_uint2(c2[v].z, c2[v].w), s2));
        // RoPE keys: units 4 hh .. 4 hh + 3 of the row, as fp16.
        {
          uint8_t* rrow = stage + kRopeChunk * kChunkBytes + r * 128;
#pragma unroll
          for (int u = 4 * hh; u < 4 * hh + 4; ++u) {
            uint4* unit = reinterpret_cast<uint4*>(rrow + ((u ^ (r & 7)) * 16));
            *unit = bf16x8_to_f16(*unit);
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(&bars->widened[s]);
      }
      return true;
    });
    if (!ok && lane == 0) raise_abort(bars, status);
  } else {
    // ------------------------------------------------------------ softmax
    const int q = warp;                      // TMEM lane quadrant
    const bool lo_half = lane < 16;
    const int row = 16 * q + (lane & 15);    // head row within the CTA
    const int head = g * kHeadsPerCta + row;
    const uint32_t lo_base = tmem + (uint32_t(32 * q) << 16);
    const uint32_t hi_base = lo_base + kHiLanes;
    const int tid = threadIdx.x;             // 0..127
    float m_ref = -INFINITY, l_sum = 0.f;
    uint32_t i = 0;
    bool ok = true;

    // Query block of sequence b into tensor memory (lo lanes, K-major pairs of
    // bf16 per 32-bit column; fp16 with the FP8 cache).  A row is 72 16-byte units; the two half-warps
    // take alternate units of the same 16 rows, so each warp load reads one
    // 32-byte sector per row, and a 16x32bx2 store with a 4-column split puts
    // unit 2j at columns [8j, 8j+4) and unit 2j+1 at [8j+4, 8j+8).  All 36
    // loads of a thread are issued before the first store (one round trip).
    auto write_query = [&](int b) {
      constexpr int kUnits = R / 16;   // 16-byte units per half-warp thread: 36, or 32 without RoPE
      // All loads in one round trip; in three with the FP8 widen warps
      // sharing the register file.
      constexpr int kBatch = kFp8 ? 12 : kUnits;
      const int64_t qrow = int64_t(b) * H + int64_t(g) * kHeadsPerCta + row;
      const bool valid_row = qrow < int64_t(B) * H;
      const uint4* src = reinterpret_cast<const uint4*>(q_cat + (valid_row ? qrow : 0) * R);
#pragma unroll
      for (int j0 = 0; j0 < kUnits; j0 += kBatch) {
        uint4 v[kBatch];
#pragma unroll
        for (int j = 0; j < kBatch; ++j)
          v[j] = (valid_row && j0 + j < kUnits) ? src[2 * (j0 + j) + (lo_half ? 0 : 1)]
                                                : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int j = 0; j < kBatch; ++j)
          if (j0 + j < kUnits)
            tmem_st16x2_4<4>(lo_base + kColQ + uint32_t(8 * (j0 + j)),
                             kFp8 ? bf16x8_to_f16(v[j]) : v[j]);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bars->q_ready);
    };
    // The contiguous 64-row query block of sequence b into L2 ahead of use.
    auto prefetch_query = [&](int b) {
      if (b >= 0 && tid == 0) {
        const int64_t r0 = int64_t(b) * H + int64_t(g) * kHeadsPerCta;
        const int64_t rows = min(int64_t(kHeadsPerCta), int64_t(B) * H - r0);
        if (rows > 0) bulk_prefetch_l2(q_cat + r0 * R, uint32_t(rows * R * 2));
      }
    };

    auto next_sequence = [&](int after) { return tp.next_sequence(after, t_begin, t_end); };

    // The first sequence's query block; each later one is written as soon as
    // the previous sequence's last S has been read (all its QK^T are done),
    // before that sequence's epilogue, so the next QK^T overlaps the stores.
    const int first_b = next_sequence(-1);
    if (first_b >= 0) write_query(first_b);
    for_each_segment(tp, t_begin, t_end,
                     [&](int b, int64_t lo, int64_t hi, int64_t L) {
      const int slot = b + w;
      prefetch_query(next_sequence(b));
      for (int64_t t = lo; t < hi; ++t, ++i) {
        const int st = i % kStages, sb = i & 1;
        if (!(ok = warp_wait(&bars->s_full[sb], (i >> 1) & 1, abort_flag))) return false;
        tc_fence_after();
        uint32_t xs[32];   // keys 0-31 (threads 0-15) or 32-63 (threads 16-31)
        tmem_ld16x2_32<32>(lo_base + kColS + uint32_t(sb) * 64u, xs);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&bars->s_free[sb]);

        const int64_t key0 = t * kTileKeys;
        const int valid = int(min(int64_t(kTileKeys), L - key0));
        uint8_t* stage = sStage + st * kStageBytes;
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
        const int kofs = lo_half ? 0 : 32;
        float mt = -INFINITY;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float x = (kofs + j < valid) ? __uint_as_float(xs[j]) * scale_log2 : -INFINITY;
          xs[j] = __float_as_uint(x);
          mt = fmaxf(mt, x);
        }
        mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
        float alpha = 1.f;
        int resc = 0;
        if (first) {
          m_ref = mt;
          l_sum = 0.f;
        } else if (mt > m_ref + kRescaleThreshold) {
          alpha = ex2_approx(m_ref - mt);
          m_ref = mt;
          l_sum *= alpha;
          resc = 1;
        }
        {
          float sum = 0.f;
          uint8_t* prow = stage + kRopeChunk * kChunkBytes + row * 128;
#pragma unroll
          for (int uu = 0; uu < 4; ++uu) {
            uint32_t pk[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float p0 = ex2_approx(__uint_as_float(xs[8 * uu + 2 * e]) - m_ref);
              const float p1 = ex2_approx(__uint_as_float(xs[8 * uu + 2 * e + 1]) - m_ref);
              if (kFp8) {   // fp16 operands for P.C with the FP8 cache
                const __half2 pp = __floats2half2_rn(p0, p1);
                sum += __low2float(pp) + __high2float(pp);
                pk[e] = *reinterpret_cast<const uint32_t*>(&pp);
              } else {
                const __nv_bfloat162 pp = __floats2bfloat162_rn(p0, p1);
                sum += __low2float(pp) + __high2float(pp);
                pk[e] = *reinterpret_cast<const uint32_t*>(&pp);
              }
            }
            const int u = (kofs >> 3) + uu;
            *reinterpret_cast<uint4*>(prow + ((u ^ (row & 7)) * 16)) =
                make_uint4(pk[0], pk[1], pk[2], pk[3]);
          }
          l_sum += sum;
        }
        if (__any_sync(0xffffffffu, resc)) {
          // O holds tile i-1's product once PV(i-1) has completed.
          const uint32_t prev = i - 1;
          if (!(ok = warp_wait(&bars->empty[prev % kStages], (prev / kStages) & 1, abort_flag)))
            return false;
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < 256; c += 32) {
            uint32_t r[32];
            tmem_ld16x2_32<256>(hi_base + uint32_t(c), r);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            tmem_st16x2_32<256>(hi_base + uint32_t(c), r);
          }
          tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bars->p_full[sb]);
      }
      // Every QK^T of this sequence has been read back: load the next query.
      const int nb = next_sequence(b);
      if (nb >= 0) write_query(nb);
      // Segment epilogue: normalised partial output and log-sum-exp.
      const uint32_t last = i - 1;
      if (!(ok = warp_wait(&bars->empty[last % kStages], (last / kStages) & 1, abort_flag)))
        return false;
      tc_fence_after();
      const float l_row = l_sum + __shfl_xor_sync(0xffffffffu, l_sum, 16);
      const float inv = 1.f / l_row;
      // Partials are o_part[slot][d_c / 4][H][4]: lanes 0-15 store 16
      // consecutive heads of one 4-column group (256 contiguous bytes), lanes
      // 16-31 the same heads 64 groups further on.
      // The combine reads them right after this kernel: they are stored
      // evict-last so that the cache rows streaming through L2 behind them
      // do not push them out to HBM first.
      float* dst = o_part + ((int64_t(slot) * (kDc / 4) + (lo_half ? 0 : 64)) * H + head) * 4;
      const uint64_t keep = l2_policy_evict_last();
#pragma unroll 1
      for (int c = 0; c < 256; c += 32) {
        uint32_t r[32];
        tmem_ld16x2_32<256>(hi_base + uint32_t(c), r);
        tmem_wait_ld();
        if (head < H) {
#pragma unroll
          for (int e = 0; e < 8; ++e)
            st_global_f4_hint(
                dst + int64_t(c / 4 + e) * H * 4,
                make_float4(__uint_as_float(r[4 * e]) * inv, __uint_as_float(r[4 * e + 1]) * inv,
                            __uint_as_float(r[4 * e + 2]) * inv, __uint_as_float(r[4 * e + 3]) * inv),
                keep);
        }
      }
      if (lo_half && head < H)
        lse_part[int64_t(slot) * H + head] = (m_ref + log2f(l_row)) * 0.69314718055994531f;
      tc_fence_before();
      mbar_arrive(&bars->o_free);
      return true;
    });
    if (!ok && lane == 0) raise_abort(bars, status);
  }

  tc_fence_before();
  __syncthreads();
  // Every role has stopped.  Each load the producer issued lands before the
  // shared memory is released: after a give-up some were never waited for
  // (the last load into each stage; on the normal path these waits return at
  // once).
  if (warp == kProducerWarp && lane == 0) {
    volatile int no_abort = 0;
    for (uint32_t k = (n_issued > kStages ? n_issued - kStages : 0); k < n_issued; ++k)
      mbar_wait(&bars->full[k % kStages], (k / kStages) & 1, &no_abort, kWaitLimitCycles);
  }
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_tiled() {
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

bool make_cache_rows_map(CUtensorMap* map, const void* base, uint64_t rows) {
  return make_cache_rows_map_r(map, base, rows, kR);
}

bool make_cache_rows_map_r(CUtensorMap* map, const void* base, uint64_t rows, int R) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cuuint64_t(R), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(R) * 2};
  const cuuint32_t box[2] = {cuuint32_t(kChunkElems), cuuint32_t(kTileKeys)};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int decode_tc_head_groups(int H) { return (H + kHeadsPerCta - 1) / kHeadsPerCta; }

namespace {
template <int kDr, bool kFp8>
cudaError_t launch_decode_tc_t(const CUtensorMap& tm_c, const CUtensorMap& tm_codes,
                               const __nv_bfloat16* q_cat, const void* cache, const float* scales,
                               const PageMap& pm, const int32_t* seqlens, int B, int H, int64_t cap,
                               float scale, int W, float* o_part, float* lse_part, int* status,
                               uint64_t inject_wait, cudaStream_t stream) {
  static bool attr_done[64] = {false};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(decode_tc_kernel<kDr, kFp8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(kSmemBytes));
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  const float scale_log2 = scale * 1.4426950408889634f;
  dim3 grid(decode_tc_head_groups(H), W);
  return launch_pdl(decode_tc_kernel<kDr, kFp8>, grid, dim3(Threads<kFp8>::n), kSmemBytes, stream,
                    tm_c, tm_codes, static_cast<const __nv_bfloat16*>(cache), scales, pm, q_cat,
                    seqlens, B, H, cap, scale_log2, W, o_part, lse_part, status, inject_wait);
}

// Byte map over FP8 cache rows [rows, 640]: boxes of 128 codes x 64 rows,
// 128-byte swizzled.
bool make_code_rows_map(CUtensorMap* map, const void* base, uint64_t rows) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cuuint64_t(kFp8RowBytes), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(kFp8RowBytes)};
  const cuuint32_t box[2] = {128, cuuint32_t(kTileKeys)};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
}  // namespace

cudaError_t launch_decode_tc(const __nv_bfloat16* q_cat, const __nv_bfloat16* cache,
                             const PageMap& pm, const int32_t* seqlens, int B, int H, int64_t cap,
                             int d_r, float scale, int W, float* o_part, float* lse_part,
                             int* status, uint64_t inject_wait, cudaStream_t stream) {
  if (d_r != 64 && d_r != 0) return cudaErrorInvalidValue;
  if (pm.total_rows(B) >= (int64_t(1) << 31) || int64_t(B) * H >= (int64_t(1) << 31))
    return cudaErrorInvalidValue;
  CUtensorMap tm_c;
  if (!make_cache_rows_map_r(&tm_c, cache, uint64_t(pm.total_rows(B)), kDc + d_r))
    return cudaErrorInvalidValue;
  return d_r == 64 ? launch_decode_tc_t<64, false>(tm_c, tm_c, q_cat, cache, nullptr, pm, seqlens,
                                                   B, H, cap, scale, W, o_part, lse_part, status,
                                                   inject_wait, stream)
                   : launch_decode_tc_t<0, false>(tm_c, tm_c, q_cat, cache, nullptr, pm, seqlens,
                                                  B, H, cap, scale, W, o_part, lse_part, status,
                                                  inject_wait, stream);
}

cudaError_t launch_decode_tc_fp8(const __nv_bfloat16* q_cat, const uint8_t* cache,
                                 const float* scales, const PageMap& pm, const int32_t* seqlens,
                                 int B, int H, int64_t cap, float scale, int W, float* o_part,
                                 float* lse_part, int* status, uint64_t inject_wait,
                                 cudaStream_t stream) {
  if (pm.total_rows(B) >= (int64_t(1) << 31) || int64_t(B) * H >= (int64_t(1) << 31))
    return cudaErrorInvalidValue;
  // The same rows viewed as bf16 [rows, 320] for the RoPE keys (columns 256..319).
  CUtensorMap tm_rope, tm_codes;
  if (!make_cache_rows_map_r(&tm_rope, cache, uint64_t(pm.total_rows(B)), kFp8RowBytes / 2) ||
      !make_code_rows_map(&tm_codes, cache, uint64_t(pm.total_rows(B))))
    return cudaErrorInvalidValue;
  return launch_decode_tc_t<64, true>(tm_rope, tm_codes, q_cat, cache, scales, pm, seqlens, B, H,
                                      cap, scale, W, o_part, lse_part, status, inject_wait,
                                      stream);
}

}  // namespace mla
