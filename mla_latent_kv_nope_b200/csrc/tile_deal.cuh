// The split-KV work list shared by the tensor-core decode kernels.
//
// The key space of all sequences, cut into tiles of kTileKeys rows and
// concatenated in batch order (T tiles), is dealt into W contiguous ranges;
// worker w takes tiles [floor(wT/W), floor((w+1)T/W)) and walks the
// sequences that overlap its range ("segments").  Every role of a CTA walks
// the same segments in the same order, so their barrier phases agree.
#pragma once

#include "common.cuh"

namespace mla {

// Exclusive prefix of per-sequence tile counts, built once per CTA so that no
// role walks the length array through global memory (a chain of dependent
// loads).  Batches with more sequences fall back to walking global memory.
constexpr int kMaxSeqSmem = 1024;
constexpr size_t kTilePrefixSmemBytes = sizeof(int32_t) * (2 * kMaxSeqSmem + 1);

// Tile prefix of the batch: prefix(b) = sum of tiles of sequences < b, from
// shared memory when the batch fits, else recomputed from the lengths.
struct TilePrefix {
  const int32_t* sp;       // shared prefix [B + 1] or nullptr
  const int32_t* sl;       // shared clamped lengths [B] or nullptr
  const int32_t* seqlens;
  int B;
  int64_t cap;
  __device__ int64_t at(int b) const {
    if (sp) return sp[b];
    int64_t p = 0;
    for (int k = 0; k < b; ++k) p += tiles_of(clamp_len(seqlens[k], cap));
    return p;
  }
  __device__ int64_t len(int b) const { return sl ? sl[b] : clamp_len(seqlens[b], cap); }
  // First sequence whose tiles end after tile t (binary search on the prefix).
  __device__ int first_after(int64_t t) const {
    if (!sp) {
      int64_t p = 0;
      for (int b = 0; b < B; ++b) {
        p += tiles_of(len(b));
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
  // The sequence of the range [t_begin, t_end) that follows sequence `after`
  // (-1 for the first), or -1 if there is none.
  __device__ int next_sequence(int after, int64_t t_begin, int64_t t_end) const {
    for (int bb = (after < 0 ? first_after(t_begin) : after + 1); bb < B; ++bb) {
      const int64_t pre = at(bb);
      if (pre >= t_end) return -1;
      const int64_t nt = tiles_of(len(bb));
      if (nt > 0 && pre + nt > t_begin) return bb;
    }
    return -1;
  }
};

// Builds the shared prefix (all threads of the block take part; two block
// barriers) and returns the total tile count.  `smem` holds
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
      s_prefix[b + 1] = int32_t(tiles_of(L));
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
    for (int b = 0; b < B; ++b) n_tiles += tiles_of(clamp_len(seqlens[b], cap));
  }
  *tp = TilePrefix{in_smem ? s_prefix : nullptr, in_smem ? s_lens : nullptr, seqlens, B, cap};
  return n_tiles;
}

// Sequences overlapping the tile range [t_begin, t_end) are visited in
// order; the callback gets (b, first tile, end tile (both local to b),
// length) and returns false to stop.
template <typename F>
__device__ __forceinline__ void for_each_segment(const TilePrefix& tp, int64_t t_begin,
                                                 int64_t t_end, F&& f) {
  for (int b = tp.first_after(t_begin); b < tp.B; ++b) {
    const int64_t pre = tp.at(b);
    if (pre >= t_end) return;
    const int64_t L = tp.len(b);
    const int64_t nt = tiles_of(L);
    const int64_t lo = max(pre, t_begin), hi = min(pre + nt, t_end);
    if (lo < hi && !f(b, lo - pre, hi - pre, L)) return;
  }
}

}  // namespace mla
