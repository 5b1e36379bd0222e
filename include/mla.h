/*
 * mla.h -- C ABI of the B200 (sm_100a) library for single-token Multi-head
 * Latent Attention (MLA) decode over the compressed latent KV cache.
 *
 * What the library computes (citations are to the pages that define MLA):
 *   [MLA-とは]  "Multi-head Latent Attention（MLA）とは？KVキャッシュを圧縮する
 *              DeepSeekの注意機構を完全解説" (disassemble-channel.com)
 *
 * One decode step for a batch of B sequences, each with L_b cached tokens:
 *   1. mla_cache_append  writes the new token's latent row
 *                        [RMSNorm(W^DKV h) * gamma || RoPE(W^KR h, pos = L_b)]
 *                        at row L_b and increments L_b.
 *   2. mla_absorb_q      q_cat = [W^UK_i^T q^C ; RoPE(q^R, q_pos)] per head
 *                        (W^UK absorbed into the query).
 *   3. mla_decode        split-KV attention of q_cat over the latent rows:
 *                        the latent row is the one key shared by all heads,
 *                        its first d_c entries the shared value (MQA with head
 *                        dim d_c + d_r).  Writes partial results.
 *   4. mla_combine       merges the partials by log-sum-exp into
 *                        o_lat = sum_j softmax_j c_j and lse.
 *   5. mla_out_proj      out = W^UV_i o_lat (W^UV applied once, after the sum).
 * K and V are never materialised.
 *
 * Conventions for every entry point
 *   - All tensor arguments are caller-owned DEVICE pointers (e.g. a torch
 *     tensor's data_ptr()), row-major and contiguous, 16-byte aligned.  The
 *     library never allocates, frees or retains memory.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls only
 *     enqueue work and return; nothing synchronises except
 *     mla_get_device_status.
 *   - Argument, shape, alignment and workspace errors return a non-zero
 *     status BEFORE anything is launched.  A failed launch returns
 *     MLA_ERR_CUDA.  Errors found on the device (a sequence already at
 *     capacity, a wait that gave up) are recorded in a per-device status word
 *     read by mla_get_device_status.  No exception crosses the ABI.
 *   - dtype MLA_BF16: bf16 tensors, fp32 accumulation; decode requires
 *     d_c = 512 and d_r = 64, or d_r = 0 (NoPE: rows are c^KV alone) -- the
 *     tensor-core kernels' tile shapes.
 *     dtype MLA_F32: fp32 tensors throughout; d_c, d_nope, d_v multiples of 4,
 *     d_r even, d_c <= 1024, d_r <= 256.
 *   - o_lat and lse are fp32 in both dtypes.
 */
#ifndef MLA_H_
#define MLA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MLA_API __attribute__((visibility("default")))
#else
#define MLA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { MLA_BF16 = 0, MLA_F32 = 1 } mla_dtype;

/* Problem shape.  Names follow [MLA-とは]: H = n_h, d_nope = d_h (content
 * query/key width per head), d_r = d_h^R (decoupled RoPE width), d_c = latent
 * width (kv_lora_rank), d_v = value width per head. */
typedef struct {
  int32_t B;              /* sequences; one query token each */
  int32_t H;              /* attention heads */
  int32_t d_c;            /* latent width */
  int32_t d_r;            /* decoupled RoPE width */
  int32_t d_nope;         /* per-head content width of q and k */
  int32_t d_v;            /* per-head value width */
  int64_t cache_capacity; /* rows allocated per sequence in the cache */
  int32_t dtype;          /* mla_dtype */
} mla_dims;

enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1,    /* null pointer, non-positive or inconsistent size */
  MLA_ERR_UNSUPPORTED = 2,    /* shape/dtype the library has no kernel for */
  MLA_ERR_ALIGNMENT = 3,      /* a pointer is not 16-byte aligned */
  MLA_ERR_WORKSPACE = 4,      /* workspace missing or smaller than required */
  MLA_ERR_CUDA = 5,           /* a CUDA runtime call or launch failed */
  MLA_ERR_DEVICE_TIMEOUT = 6, /* a bounded device-side wait gave up */
  MLA_ERR_BOUNDS = 7          /* device-side index check failed (e.g. cache full) */
};

/* Elements of one latent cache row per token per layer: d_c + d_r
 * ([MLA-とは] "KVキャッシュ容量の比較": MLA caches (d_c + d_h^R) per layer). */
MLA_API int64_t mla_cache_row_elems(int32_t d_c, int32_t d_r);

/* --- 1. cache append ------------------------------------------------------
 * [MLA-とは] "MLAの発想" (c^KV_t = W^DKV h_t), "Decoupled RoPE"
 * (k^R_j = R_j W^KR h_j, cached already rotated), "実装上のトレードオフ"
 * (the normalised latent is cached).  For each sequence b:
 *   x = W_DKV h_b (fp32 accumulation);  c = x[0:d_c] / sqrt(mean(x[0:d_c]^2) + eps) * gamma
 *   k = RoPE(x[d_c:d_c+d_r], pos = L_b) (half-split pairs, theta_k = pos * base^(-2k/d_r))
 *   cache[b, L_b, :] = [c || k] rounded once to the cache dtype;  seqlens[b] = L_b + 1
 * h       [B, hidden]                 dtype
 * W_DKV   [d_c + d_r, hidden]         dtype; rows 0..d_c-1 = W^DKV, the rest = W^KR
 * gamma   [d_c] fp32, or NULL for ones
 * cache   [B, cache_capacity, d_c + d_r] dtype, written at row L_b only
 * seqlens [B] int32, read then incremented on the device
 * workspace  >= mla_cache_append_workspace_bytes(dims, hidden) bytes of device scratch
 *             (partial sums of the projection; contents need not be initialised)
 * A sequence already at capacity is left untouched and sets MLA_ERR_BOUNDS in
 * the device status word. */
MLA_API size_t mla_cache_append_workspace_bytes(const mla_dims* dims, int32_t hidden);
MLA_API int mla_cache_append(const mla_dims* dims, int32_t hidden, const void* h,
                     const void* W_DKV, const float* gamma, float eps,
                     float rope_base, void* cache, int32_t* seqlens,
                     void* workspace, size_t workspace_bytes, void* stream);

/* --- 2. query absorption --------------------------------------------------
 * [MLA-とは] "行列吸収": q~_{t,i} = W^UK_i^T q_{t,i} in R^{d_c};
 * "Decoupled RoPE": q^R rotated at the query position.
 *   q_cat[b,i,0:d_c]      = sum_r q_nope[b,i,r] W_UK[i,r,:]
 *   q_cat[b,i,d_c:d_c+d_r] = RoPE(q_pe[b,i], q_pos[b])   (q_pos == NULL: copied as given)
 * q_nope [B,H,d_nope], q_pe [B,H,d_r], W_UK [H,d_nope,d_c] (dtype);
 * q_pos [B] int32 or NULL; q_cat [B,H,d_c+d_r] (dtype, rounded once). */
MLA_API int mla_absorb_q(const mla_dims* dims, const void* q_nope, const void* q_pe,
                 const void* W_UK, const int32_t* q_pos, float rope_base,
                 void* q_cat, void* stream);

/* --- 3. split-KV latent decode --------------------------------------------
 * [MLA-とは] "実装上のトレードオフ" (absorbed form = MQA with head dim
 * d_c + d_r), "Value側の吸収" (weighted sum in latent space), "Decoupled
 * RoPE" (softmax scale 1/sqrt(d_h + d_h^R)).
 * For sequence b, head i and cached rows j < L_b:
 *   s_j = softmax_scale * (q_cat[b,i] . cache[b,j,:])
 * softmax_scale = 0 selects the pages' scale 1/sqrt(d_nope + d_r); a
 * negative, infinite or NaN scale is MLA_ERR_INVALID_ARG.
 * The key space of all sequences, cut into tiles of 64 rows, is dealt into
 * `num_splits` contiguous ranges (worker w takes tiles [w*T/W, (w+1)*T/W) of
 * the concatenated per-sequence tile lists, T = sum_b ceil(L_b/64)).  Worker w
 * writes, for each sequence b it touches, partial slot (b + w):
 *   o_part[b+w][i][:] = sum_{j in range} e^{s_j - lse_part} c_j,   lse_part[b+w][i] = log sum e^{s_j}
 * Workspace layout (fp32): o_part [B + W - 1][d_c / 4][H][4] (column c of
 * head i at [slot][c / 4][i][c % 4], so 4-column groups of consecutive heads
 * are contiguous), then, 256-byte aligned, lse_part [B + W - 1][H].
 * Rows j >= L_b never influence the result (they may hold anything).
 * num_splits = 0 picks the default for the current device; the number used is
 * returned through splits_used (may be NULL).
 * MLA_ERR_UNSUPPORTED: bf16 needs d_c = 512 and d_r = 64 or 0, and a contiguous
 * bf16 cache must hold fewer than 2^31 rows (B * cache_capacity), the range
 * of the tensor-copy row coordinate. */
MLA_API int mla_decode_default_splits(const mla_dims* dims);
MLA_API size_t mla_decode_workspace_bytes(const mla_dims* dims, int num_splits);
MLA_API int mla_decode(const mla_dims* dims, const void* q_cat, const void* cache,
               const int32_t* seqlens, float softmax_scale, int num_splits,
               void* workspace, size_t workspace_bytes, int* splits_used,
               void* stream);

/* --- 4. log-sum-exp combine ------------------------------------------------
 * Merges the partials of mla_decode (same dims, seqlens and splits_used):
 *   lse[b,i] = log sum_s exp(lse_part_s),  o_lat[b,i] = sum_s exp(lse_part_s - lse[b,i]) o_part_s
 * An empty sequence (L_b = 0) gives o_lat = 0 and lse = -inf.
 * o_lat [B,H,d_c] fp32; lse [B,H] fp32 (may be NULL). */
MLA_API int mla_combine(const mla_dims* dims, const int32_t* seqlens,
                const void* workspace, size_t workspace_bytes, int splits_used,
                float* o_lat, float* lse, void* stream);

/* --- sequence-sharded decode: merge of per-range results -----------------------
 * No counterpart on the pages: a long context can be split by tokens across
 * devices, each holding a contiguous token range of every sequence and
 * running mla_decode + mla_combine on it.  The n range results, gathered into
 * one array, are merged here with the same log-sum-exp identity as the
 * split-KV partials:
 *   lse[b,i] = log sum_k exp(lse_k[b,i]),  o_lat[b,i] = sum_k exp(lse_k[b,i] - lse[b,i]) o_k[b,i]
 * A result with lse_k = -inf (a range holding no key of sequence b) adds
 * nothing and its o_k is not read; if every lse_k is -inf, o_lat = 0 and
 * lse = -inf.
 * o_parts [n_parts][B][H][d_c] fp32 and lse_parts [n_parts][B][H] fp32 are
 * the stacked mla_combine outputs; o_lat [B][H][d_c] fp32; lse [B][H] fp32
 * (may be NULL).  MLA_ERR_INVALID_ARG: n_parts outside [1, 1024] or a NULL
 * array. */
MLA_API int mla_merge_partials(const mla_dims* dims, int n_parts, const float* o_parts,
                               const float* lse_parts, float* o_lat, float* lse, void* stream);

/* --- 5. value up-projection -------------------------------------------------
 * [MLA-とは] "Value側の吸収": o_{t,i} = W^UV_i (sum_j a_{tj,i} c^KV_j).
 *   out[b,i,v] = sum_c W_UV[i,v,c] o_lat[b,i,c]
 * o_lat [B,H,d_c] fp32; W_UV [H,d_v,d_c] dtype; out [B,H,d_v] dtype. */
MLA_API int mla_out_proj(const mla_dims* dims, const float* o_lat, const void* W_UV,
                 void* out, void* stream);

/* --- materialised prefill of one sequence -----------------------------------------
 * [MLA-とは] "実装上のトレードオフ": prefill processes many query tokens at
 * once and is compute-bound, so the per-head keys and values are formed
 * explicitly (k^C_i = W^UK_i c_l, v^C_i = W^UV_i c_l for every latent row l)
 * and the heads run ordinary causal softmax attention with head dim
 * d_nope + d_r (the key's RoPE part is the row's shared, already rotated k^R)
 * and value dim d_v:
 *   q_t,i  = [q_nope[t,i] ; RoPE(q_pe[t,i], q_pos[t])]
 *   s_tl   = softmax_scale * (q_t,i . [W^UK_i c_l ; k^R_l]),   l <= q_pos[t]
 *   out[t,i] = sum_l softmax(s_t)_l W^UV_i c_l,   lse[t,i] = log sum_l exp(s_tl)
 * One sequence per call: rows [L, d_c + d_r] bf16 are its latent cache rows
 * (the prompt's own rows already appended, e.g. by mla_cache_append, so a
 * query attends to itself), q_nope [T, H, d_nope], q_pe [T, H, d_r] bf16,
 * q_pos [T] int32 device positions (any order); query t sees rows
 * 0 .. min(q_pos[t], L - 1), and nothing if q_pos[t] < 0 (out 0, lse -inf).
 * out [T, H, d_v] bf16; lse [T, H] fp32 or NULL.  softmax_scale = 0 selects
 * 1/sqrt(d_nope + d_r); it must be positive.  Only dims->H, d_c, d_r, d_nope,
 * d_v and dtype are read.  Shape: bf16, d_c = 512, d_nope = d_v = 128, d_r =
 * 64 or 0, H * L and H * T below 2^31, L >= 1 (T = 0 does nothing).  The
 * workspace (mla_prefill_workspace_bytes, no initialisation needed) holds the
 * materialised K^C and V and a 16-bit copy of k^R: about 4 * H * L * 128 +
 * 2 * L * d_r bytes.  Precision: the QK^T operands (queries, K^C, k^R) are
 * rounded to fp16 and P, V to bf16, with fp32 accumulation, so queries and
 * keys must lie within fp16's range (|x| < 65504). */
MLA_API size_t mla_prefill_workspace_bytes(const mla_dims* dims, int32_t T, int64_t L);
MLA_API int mla_prefill(const mla_dims* dims, int32_t T, int64_t L, const void* q_nope,
                        const void* q_pe, const int32_t* q_pos, const void* W_UK,
                        const void* W_UV, const void* rows, float softmax_scale,
                        float rope_base, void* out, float* lse, void* workspace,
                        size_t workspace_bytes, void* stream);

/* --- W^O folded into the value side ---------------------------------------------
 * [MLA-とは] "Value側の吸収": W^UV_i can be absorbed into the output
 * projection, B_i = W^O_i W^UV_i in R^{d x d_c}, so the latent-space weighted
 * sums o_lat go straight to the model width:
 *   u[b] = sum_i B_i o_lat[b,i]   (= sum_i W^O_i W^UV_i o_lat[b,i])
 * W_O [d_model, H * d_v] bf16 (column convention: u = W^O o over the heads'
 * concatenated d_v-wide outputs); W_UV [H, d_v, d_c] bf16 as in mla_out_proj.
 * mla_fold_output_weights writes W_fold [d_model, H * d_c] bf16 with
 * W_fold[m, i*d_c + c] = (B_i)[m, c] (fp32 accumulation, rounded once); it
 * runs once, when the weights are loaded.  mla_out_proj_folded reads o_lat
 * [B, H, d_c] fp32 (rounded to bf16 for the tensor cores, as in
 * mla_out_proj) and writes u [B, d_model] bf16, using
 * mla_out_proj_folded_workspace_bytes(dims, d_model) bytes of scratch (no
 * initialisation needed).  Shape: bf16, d_c = 512, d_v = 128; the folded
 * projection needs B <= 64 (MLA_ERR_UNSUPPORTED otherwise).  Per call the
 * folded weight is H * d * d_c bf16 against H * d_v * (d_c + d) for W^UV and
 * W^O unfolded: fewer bytes only when d * (d_c - d_v) < d_v * d_c (d < 171 at
 * d_c = 512, d_v = 128). */
MLA_API int mla_fold_output_weights(const mla_dims* dims, int32_t d_model, const void* W_O,
                                    const void* W_UV, void* W_fold, void* stream);
MLA_API size_t mla_out_proj_folded_workspace_bytes(const mla_dims* dims, int32_t d_model);
MLA_API int mla_out_proj_folded(const mla_dims* dims, int32_t d_model, const float* o_lat,
                                const void* W_fold, void* u, void* workspace,
                                size_t workspace_bytes, void* stream);

/* --- FP8 latent cache ------------------------------------------------------------
 * [abeam] "モデル全体でも推論効率が大きく改善した" names KV-cache quantisation as
 * part of the system's serving efficiency, and [yuuk] "未解決の問い" leaves FP8
 * for MLA open; the format is this library's (the pages fix none).  A cached
 * token is a row of mla_cache_fp8_row_bytes(d_c, d_r) = d_c + 2 d_r bytes:
 * d_c E4M3 codes (OCP E4M3, finite-only: largest 448, no infinities) of the
 * normalised latent, then the d_r RoPE keys in bf16, plus one fp32 scale per
 * token in a separate plane scales [B, cache_capacity]:
 *   c~_j = E4M3(code_j) * scale,  scale = the smallest power of two 2^k with
 *   max_j |c_j| / 2^k <= 448 (a row of zeros gets 1),
 *   code_j = c_j / scale rounded to nearest E4M3 (ties to even), saturating.
 * Shape: bf16, d_c = 512, d_r = 64, d_nope = d_v = 128; contiguous cache only.
 * mla_cache_append_fp8 is mla_cache_append (same h, W_DKV, gamma, eps,
 * rope_base, seqlens, workspace) writing row L_b of cache [B, capacity,
 * 640 bytes] and scales[b, L_b].  mla_decode_fp8 is mla_decode over the
 * dequantised rows [c~ || k^R] (same q_cat, seqlens, scale, splits,
 * workspace, partial layout; mla_combine merges as usual).  Rows past L_b
 * (codes and scales) may hold anything.
 * Precision: its tensor-core products take fp16 operands (fp32 accumulation):
 * c~ (the code times its power-of-two scale), the query and k^R (converted
 * from bf16) and the probabilities.  Each is exact in fp16 for magnitudes in
 * [2^-14, 65504); smaller ones keep fp16's subnormal resolution of 2^-24.
 * So c~, q_cat and k^R must stay below 65504 in magnitude (as for
 * mla_prefill's fp16 scores); every row the append writes from a normalised
 * latent does. */
MLA_API int64_t mla_cache_fp8_row_bytes(int32_t d_c, int32_t d_r);
MLA_API int mla_cache_append_fp8(const mla_dims* dims, int32_t hidden, const void* h,
                                 const void* W_DKV, const float* gamma, float eps,
                                 float rope_base, void* cache_fp8, float* scales,
                                 int32_t* seqlens, void* workspace, size_t workspace_bytes,
                                 void* stream);
MLA_API int mla_decode_fp8(const mla_dims* dims, const void* q_cat, const void* cache_fp8,
                           const float* scales, const int32_t* seqlens, float softmax_scale,
                           int num_splits, void* workspace, size_t workspace_bytes,
                           int* splits_used, void* stream);

/* --- paged latent cache --------------------------------------------------------
 * No counterpart on the pages beyond the name: [MLA-とは] names PagedAttention
 * as the serving-side cache organisation this method fits; the page size is
 * fixed here at 64 rows, one decode work tile.
 * The cache is a pool of num_pages pages, cache_pool [num_pages, 64, d_c + d_r]
 * (dtype), and block_table [B, max_blocks] int32 maps sequence b's key j to
 * row j % 64 of page block_table[b, j / 64].  dims->cache_capacity is the
 * longest sequence allowed and must be <= 64 * max_blocks; entries for tiles
 * at or beyond a sequence's length are never read.  Otherwise these calls are
 * mla_decode and mla_cache_append with the same inputs, outputs, workspace,
 * partial layout and errors (mla_combine merges the partials as usual).  A
 * page id outside [0, num_pages) is not dereferenced: it is recorded as
 * MLA_ERR_BOUNDS in the device status word (decode reads its rows as zeros;
 * append writes nothing and leaves L_b unchanged). */
MLA_API int mla_decode_paged(const mla_dims* dims, const void* q_cat, const void* cache_pool,
                             int64_t num_pages, const int32_t* block_table, int32_t max_blocks,
                             const int32_t* seqlens, float softmax_scale, int num_splits,
                             void* workspace, size_t workspace_bytes, int* splits_used,
                             void* stream);
MLA_API int mla_cache_append_paged(const mla_dims* dims, int32_t hidden, const void* h,
                                   const void* W_DKV, const float* gamma, float eps,
                                   float rope_base, void* cache_pool, int64_t num_pages,
                                   const int32_t* block_table, int32_t max_blocks,
                                   int32_t* seqlens, void* workspace, size_t workspace_bytes,
                                   void* stream);

/* --- 3+4 without a workspace -------------------------------------------------
 * No counterpart on the pages: this is a convenience of this library.
 * For callers that cannot allocate device memory (plugins that only receive
 * fixed buffers from a host framework, runtimes whose device memory is owned
 * by another allocator), this runs mla_decode and mla_combine with the
 * split-KV partials kept in a fixed array inside the library instead of a
 * caller workspace.  Inputs and outputs are as for
 * mla_decode + mla_combine (q_cat, cache, seqlens in; o_lat [B,H,d_c] fp32 and
 * lse [B,H] fp32 (may be NULL) out); nothing is allocated or freed.
 *   - The array holds MLA_DECODE_NOALLOC_SCRATCH_BYTES on every device that
 *     loads the library, until the process exits.  The split count W is the
 *     device default, lowered until the partials (mla_decode's workspace for
 *     W splits) fit:
 *       round_up((B + W - 1) * H * d_c * 4, 256) + round_up((B + W - 1) * H * 4, 256)
 *         <= MLA_DECODE_NOALLOC_SCRATCH_BYTES
 *     if even W = 1 does not fit the call returns MLA_ERR_WORKSPACE and
 *     launches nothing.
 *   - The first call on a device looks up the array's device address with
 *     that device current; make that first call before any stream capture.
 *   - All calls share the one array and it keeps the previous call's
 *     contents (every partial read in a call is written earlier in the same
 *     call).  Calls that overlap on the GPU (different streams, or several
 *     host threads) race on it: serialise them. */
#define MLA_DECODE_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
MLA_API int mla_decode_noalloc(const mla_dims* dims, const void* q_cat, const void* cache,
                               const int32_t* seqlens, float softmax_scale, float* o_lat,
                               float* lse, void* stream);

/* --- failure-detection test hook ------------------------------------------------
 * No counterpart on the pages.  Every wait inside the tensor-core kernels is
 * bounded: a wait that runs out sets MLA_ERR_DEVICE_TIMEOUT in the device
 * status word, the kernel drains its own copies and products and returns, and
 * the context stays usable.  This hook lets a test exercise that path without
 * any fault: with cycles > 0, every later bf16 mla_decode / mla_decode_paged /
 * mla_decode_noalloc launch first waits `cycles` SM cycles on a barrier that
 * nothing ever arrives on, then gives up; its outputs are then undefined.
 * cycles = 0 (the default) turns it off.  Process-wide; not for production
 * use. */
MLA_API int mla_debug_inject_wait(uint64_t cycles);

/* --- status ------------------------------------------------------------------
 * Synchronises `stream`, then returns and clears the current device's status
 * word (MLA_OK if no device-side error was recorded since the last call).
 * Returns MLA_ERR_CUDA if the synchronisation itself failed. */
MLA_API int mla_get_device_status(void* stream);
MLA_API const char* mla_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* MLA_H_ */
