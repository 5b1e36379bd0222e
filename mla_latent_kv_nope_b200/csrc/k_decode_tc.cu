// Tensor-core split-KV decode (bf16, d_c = 512, d_r = 64).
#include "common.cuh"
#include "kernels.h"

namespace mla {

int decode_tc_head_groups(int H) { return (H + 63) / 64; }

cudaError_t launch_decode_tc(const __nv_bfloat16* q_cat, const __nv_bfloat16* cache,
                             const int32_t* seqlens, int B, int H, int64_t cap, float scale,
                             int W, float* o_part, float* lse_part, int* status,
                             cudaStream_t stream) {
  return launch_decode_simt<__nv_bfloat16>(q_cat, cache, seqlens, B, H, 512, 64, cap, scale, W,
                                           o_part, lse_part, status, stream);
}

}  // namespace mla
