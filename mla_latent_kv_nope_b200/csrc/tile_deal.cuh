// The split-KV work list shared by the tensor-core decode kernels.
//
// The key space of all sequences, cut into tiles of kTileKeys rows, is laid
// out in batch order as work units: each sequence with tiles takes
// kSwitchUnits units (its start-up cost) and then one unit per tile (T units
// in all).  The units are dealt into W contiguous ranges: worker w takes
// units [floor(wT/W), floor((w+1)T/W)) and walks the sequences whose tiles
// overlap its range ("segments").  Every role of a CTA walks the same
// segments in the same order, so their barrier phases agree.
#pragma once

#include "common.cuh"

namespace mla {

// Exclusive prefix of per-sequence tile counts, built once per CTA so that no
// role walks the length array through global memory (a chain of dependent
// loads).  Batches with more sequences fall back to walking global memory.
constexpr int kMaxSeqSmem = 1024;
constexpr size_t kTilePrefixSmemBytes = sizeof(int32_t) * (2 * kMaxSeqSmem + 1);

// Unit prefix of the batch: at(b) = sum of the units of sequences < b, from
// shared memory when the batch fits, else recomputed from the lengths; the
// tiles of b are units [tile0(b), tile0(b) + tiles).
struct TilePrefix {
  const int32_t* sp;       // shared prefix [B + 1] or nullptr
  const int32_t* sl;       // shared clamped lengths [B] or nullptr
  const int32_t* seqlens;
  int B;
  int64_t cap;
  __device__ int64_t at(int b) const {
    if (sp) return sp[b];
    int64_t p = 0;
    for (int k = 0; k < b; ++k) p += units_of(clamp_len(seqlens[k], cap));
    return p;
  }
  __device__ int64_t tile0(int b) const { return at(b) + kSwitchUnits; }
  __device__ int64_t len(int b) const { return sl ? sl[b] : clamp_len(seqlens[b], cap); }
  // First sequence whose units end after unit t (binary search on the prefix).
  __device__ int first_after(int64_t t) const {
    if (!sp) {
      int64_t p = 0;
      for (int b = 0; b < B; ++b) {
        p += units_of(len(b));
        if (p > t) return b;
      }
      return B;
    }
    int lo = 0, hi = B;  // smallest b with sp[b + 1] > t
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (sp[mid + 1] > t) hi = mid; else lo = mid + 1;
    }
    return lo;
  }
  // The sequence with tiles in the unit range [t_begin, t_end) that follows
  // sequence `after` (-1 for the first), or -1 if there is none.
  __device__ int next_sequence(int after, int64_t t_begin, int64_t t_end) const {
    for (int bb = (after < 0 ? first_after(t_begin) : after + 1); bb < B; ++bb) {
      const int64_t pre = at(bb);
      if (pre >= t_end) return -1;
      const int64_t nt = tiles_of(len(bb));
      const int64_t r0 = pre + kSwitchUnits;
      if (nt > 0 && max(r0, t_begin) < min(r0 + nt, t_end)) return bb;
    }
    return -1;
  }
};

// Builds the shared prefix (all threads of the block take part; two block
// barriers) and returns the total unit count.  `smem` holds
// kTilePrefixSmemBytes.
__device__ __forceinline__ int64_t build_tile_prefix(uint8_t* smem, const int32_t* seqlens,
                                                     int B, int64_t cap, TilePrefix* tp) {
  int32_t* s_prefix = reinterpret_cast<int32_t*>(smem);
  int32_t* s_lens = s_prefix + (kMaxSeqSmem + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool in_smem = B <= kMaxSeqSmem;
  int64_t n_tiles = 0;
  if (in_smem) {
    for (int b = threadIdx.x; b < B; b += blockDim.x) {
      const int64_t L = clamp_len(seqlens[b], cap);
      s_lens[b] = int32_t(L);
      s_prefix[b + 1] = int32_t(units_of(L));
    }
    __syncthreads();
    if (warp == 0) {
      int32_t carry = 0;
      for (int b0 = 0; b0 < B; b0 += 32) {
        int32_t v = (b0 + lane < B) ? s_prefix[b0 + lane + 1] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int32_t u = __shfl_up_sync(0xffffffffu, v, o);
          if (lane >= o) v += u;
        }
        if (b0 + lane < B) s_prefix[b0 + lane + 1] = carry + v;
        carry += __shfl_sync(0xffffffffu, v, 31);
      }
      if (lane == 0) s_prefix[0] = 0;
    }
    __syncthreads();
    n_tiles = s_prefix[B];
  } else {
    for (int b = 0; b < B; ++b) n_tiles += units_of(clamp_len(seqlens[b], cap));
  }
  *tp = TilePrefix{in_smem ? s_prefix : nullptr, in_smem ? s_lens : nullptr, seqlens, B, cap};
  return n_tiles;
}

// Sequences whose tiles overlap the unit range [t_begin, t_end) are visited
// in order; the callback gets (b, first tile, end tile (both local to b),
// length) and returns false to stop.
template <typename F>
__device__ __forceinline__ void for_each_segment(const TilePrefix& tp, int64_t t_begin,
                                                 int64_t t_end, F&& f) {
  for (int b = tp.first_after(t_begin); b < tp.B; ++b) {
    const int64_t pre = tp.at(b);
    if (pre >= t_end) return;
    const int64_t L = tp.len(b);
    const int64_t nt = tiles_of(L);
    const int64_t r0 = pre + kSwitchUnits;
    const int64_t lo = max(r0, t_begin), hi = min(r0 + nt, t_end);
    if (lo < hi && !f(b, lo - r0, hi - r0, L)) return;
  }
}

}  // namespace mla
