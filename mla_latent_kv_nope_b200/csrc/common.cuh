// Shared device helpers for the MLA decode library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/mla.h"

namespace mla {

// Keys per work tile.  The split-KV work list, the combine and every decode
// kernel agree on this unit.
constexpr int kTileKeys = 64;

// Programmatic dependent launch.  A kernel launched with launch_pdl may start
// while the previous kernel in its stream is still running; pdl_wait() blocks
// until that kernel has finished and its writes are visible, so every read of
// a predecessor's output comes after it (without the launch attribute it
// returns at once).  pdl_trigger() lets the next kernel be scheduled; it is
// issued after the caller's own tensor-memory allocation, so a dependent
// that holds tensor memory never waits on a primary that still needs some.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

// Device code records the first error it meets (bounds, timeout) in the
// per-device status word whose address the host passes to the kernel;
// mla_get_device_status reads and clears it.
__device__ __forceinline__ void record_status(int* status, int code) {
  if (status) atomicCAS(status, MLA_OK, code);
}

template <typename T> struct Storage;
template <> struct Storage<float> {
  static __device__ __forceinline__ float load(const float* p) { return *p; }
  static __device__ __forceinline__ float to_f(float v) { return v; }
  static __device__ __forceinline__ float from_f(float v) { return v; }
};
template <> struct Storage<__nv_bfloat16> {
  static __device__ __forceinline__ float load(const __nv_bfloat16* p) {
    return __bfloat162float(*p);
  }
  static __device__ __forceinline__ float to_f(__nv_bfloat16 v) {
    return __bfloat162float(v);
  }
  static __device__ __forceinline__ __nv_bfloat16 from_f(float v) {
    return __float2bfloat16_rn(v);
  }
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Usable length of a sequence: the stored length clamped to [0, capacity], so
// that a corrupt length can never index past the cache.
__device__ __forceinline__ int64_t clamp_len(int32_t L, int64_t cap) {
  return L <= 0 ? 0 : (int64_t(L) > cap ? cap : int64_t(L));
}

// Number of 64-key tiles of a sequence of (clamped) length L.
__device__ __forceinline__ int64_t tiles_of(int64_t L) {
  return L > 0 ? (L + kTileKeys - 1) / kTileKeys : 0;
}

// Work units of a sequence in the split-KV deal: kSwitchUnits units that stand
// for the fixed cost a worker pays to start a sequence (its query block and
// its partial's epilogue: about 5 us, against 1.38 us per tile, measured on
// B200), then its tiles.  A worker that crosses into a new sequence is thus
// given that many fewer tiles.  A sequence without tiles has no units.
constexpr int kSwitchUnits = 4;
__device__ __forceinline__ int64_t units_of(int64_t L) {
  const int64_t nt = tiles_of(L);
  return nt > 0 ? nt + kSwitchUnits : 0;
}

// Where the cached rows of a sequence live.  Contiguous: sequence b owns rows
// [b*cap, (b+1)*cap) of the cache viewed as [rows, d_c + d_r].  Paged: the
// cache is a pool of pages of kTileKeys rows and key j of sequence b is row
// j % kTileKeys of page table[b*max_blocks + j / kTileKeys] (a page holds
// exactly one work tile).
struct PageMap {
  const int32_t* table;   // [B][max_blocks] page ids, or nullptr (contiguous)
  int32_t max_blocks;
  int64_t num_pages;
  int64_t cap;

  // First row of tile t of sequence b; -1 for a page id outside the pool.
  __device__ __forceinline__ int64_t tile_row(int b, int64_t t) const {
    if (!table) return int64_t(b) * cap + t * kTileKeys;
    const int32_t pg = table[int64_t(b) * max_blocks + t];
    return (pg < 0 || int64_t(pg) >= num_pages) ? -1 : int64_t(pg) * kTileKeys;
  }
  // Row of key j of sequence b; -1 for a page id outside the pool.
  __device__ __forceinline__ int64_t row(int b, int64_t j) const {
    const int64_t r = tile_row(b, j / kTileKeys);
    return r < 0 ? -1 : r + j % kTileKeys;
  }
  // Rows addressed by the map (the extent of the cache tensor).
  __host__ __device__ int64_t total_rows(int B) const {
    return table ? num_pages * kTileKeys : int64_t(B) * cap;
  }
};

// First tile owned by worker w of W over T tiles: floor(w*T/W).
__device__ __forceinline__ int64_t worker_tile_begin(int64_t w, int64_t T, int64_t W) {
  return (w * T) / W;
}
// Worker owning tile t: the largest w with floor(w*T/W) <= t.
__device__ __forceinline__ int64_t worker_of_tile(int64_t t, int64_t T, int64_t W) {
  return ((t + 1) * W - 1) / T;
}

// RoPE angle pair for element pair k of a d-wide rotary block at position pos:
// theta = pos * base^(-2k/d).  The frequency and the product are formed in
// double and theta is reduced to [-pi, pi] in double (Cody-Waite style with a
// two-part 2*pi), so the single-precision sincos only ever sees a small,
// exact-enough argument even at positions ~1e5.
__device__ __forceinline__ double rope_inv_freq(int k, int d, float base) {
  return exp2(-2.0 * double(k) / double(d) * log2(double(base)));
}
__device__ __forceinline__ void rope_cos_sin_at(int64_t pos, double inv, float* c, float* s) {
  const double th = double(pos) * inv;
  const double kTwoPiHi = 6.283185307179586232;      // 2*pi rounded to double
  const double kTwoPiLo = 2.4492935982947064e-16;    // 2*pi - kTwoPiHi
  const double n = rint(th * 0.15915494309189535);   // th / (2*pi)
  const double r = fma(-n, kTwoPiLo, fma(-n, kTwoPiHi, th));
  sincosf(float(r), s, c);
}
__device__ __forceinline__ void rope_cos_sin(int64_t pos, int k, int d, float base,
                                             float* c, float* s) {
  rope_cos_sin_at(pos, rope_inv_freq(k, d, base), c, s);
}

}  // namespace mla
