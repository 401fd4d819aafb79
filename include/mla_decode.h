/*
 * mla_decode.h -- C ABI of the B200 (sm_100a) absorbed-form MLA decode library.
 *
 * The operation.  Multi-head latent attention decode over a paged latent KV
 * cache, in absorbed form: each query head is a 576-wide row (512 latent +
 * 64 rope columns); each cached token is one 576-wide bf16 row whose first
 * 512 columns also serve as its value row.  For sequence b, query position
 * i < s_q and head h:
 *     n_i  = seqlen_b - s_q + 1 + i            (tokens visible to query i)
 *     s_j  = softmax_scale * <q[b,i,h,:], k_j>  over j < n_i
 *     out[b,i,h,:] = sum_j softmax(s)_j * k_j[0:512]          (bf16)
 *     lse[b,i,h]   = ln(sum_j exp(s_j))                       (fp32)
 * with out = 0 and lse = -inf when n_i = 0.  This is attention
 * softmax(Q K^T) V as the FlashMLA-ETAP explainer (gist.science) states it
 * in its technical summary ("Methodology / core mechanism"), computed the way
 * that section prescribes: transposed, S^T = K Q^T and O = (V^T P^T)^T, so
 * that the long KV length fills the matrix-multiply M dimension.  The regime
 * (1-2 query tokens, 16 heads, 576-wide heads, contexts up to 64K) is the
 * explainer's "Problem statement" and "Limitations".  The split of the KV
 * range over many CTAs and the merge through log-sum-exp are the online
 * softmax of "FlashMLA: compressing the KV cache" (jsqmd.com), "compute
 * flow", step 4, applied across CTAs instead of across tiles.
 *
 * Calls, in the order a decode step makes them:
 *     mla_decode_metadata   split-KV schedule from the sequence lengths
 *                           (once per step; reusable by every layer);
 *     mla_decode            the attention kernel, then the combine kernel;
 *     mla_decode_attention  the attention kernel alone;
 *     mla_decode_combine    the combine kernel alone (mla_decode already
 *                           launches it; exported for tests and timing);
 *     mla_merge_states      context-parallel decode: merges the results of
 *                           W ranks that each attended over their own range
 *                           of every sequence's pages;
 *     mla_decode_fp8        the decode over an FP8 (e4m3, per-token scale)
 *                           cache (mla_decode_attention_fp8: attention only).
 *
 * Conventions for every call.
 *   - Pointers marked "device" are CUDA device pointers of the current
 *     device; the caller allocates and owns every buffer.  The library makes
 *     no device allocation.  The one piece of device memory it holds is the
 *     fixed MLA_STATIC_WORKSPACE_BYTES array behind
 *     mla_decode_static_workspace, resident on every device that loads the
 *     library and shared by every call of that entry point (see there).
 *     Between calls it keeps only host-side state: encoded tensor maps,
 *     cached by pointer and shape, and the test hook of mla_debug_stall_cta.
 *   - `stream` is a cudaStream_t (0 = the legacy default stream).  All
 *     launches are asynchronous on it; no call synchronises except
 *     mla_get_device_error.
 *   - bf16 tensors are passed as uint16_t bit patterns (IEEE binary32 top
 *     halves).  Every tensor is dense and row-major with the shape given.
 *   - Argument errors are detected on the host and returned before anything
 *     is launched.  A launch failure returns MLA_ERR_CUDA.  Bad data that only
 *     the device can see (a page-table entry outside the cache, a length past
 *     the page table, a schedule built for other shapes, a wait that timed
 *     out) never traps: the kernel records an MLA_DEVERR_* bit in word 0 of
 *     sched_meta, skips or substitutes the access, and finishes; read it back
 *     with mla_get_device_error.
 *
 * Supported shapes: s_q in {1, 2, 4, 8}; H in {16, 32, 64, 128}; page size 64;
 * head widths 576 / 512; 1 <= B <= 4096; 1 <= num_sms <= 4096 and at least
 * the number of head groups, max(1, s_q * H / 64).  Query position i of an
 * s_q-token query sees the first seqlen - s_q + 1 + i cached tokens (none
 * when that is <= 0).
 */
#ifndef MLA_DECODE_H
#define MLA_DECODE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MLA_D_QK 576  /* query / key row width: 512 latent + 64 rope     */
#define MLA_D_V 512   /* value width: the first 512 columns of a key row  */
#define MLA_PAGE 64   /* tokens per page of the cache                    */
#define MLA_TILE 128  /* tokens per attention tile (two pages)           */

typedef enum {
    MLA_OK = 0,
    MLA_ERR_INVALID_ARG = 1,         /* null pointer, negative size, bad scale */
    MLA_ERR_MISALIGNED = 2,          /* a pointer breaks its alignment rule    */
    MLA_ERR_UNSUPPORTED_SHAPE = 3,   /* s_q / H / num_sms outside the set      */
    MLA_ERR_WORKSPACE_TOO_SMALL = 4, /* workspace_bytes < the required size    */
    MLA_ERR_CUDA = 5,                /* a CUDA runtime/driver call failed      */
    MLA_ERR_DEVICE_CHECK = 6         /* mla_get_device_error found a bit set   */
} mla_status_t;

/* Bits of the device error word (word 0 of sched_meta). */
#define MLA_DEVERR_BLOCK_TABLE 1   /* page-table entry outside [0, num_blocks)   */
#define MLA_DEVERR_SEQLEN 2        /* seqlen < 0 or > max_blocks * 64            */
#define MLA_DEVERR_SCHEDULE 4      /* sched_meta for other shapes, or malformed  */
#define MLA_DEVERR_TIMEOUT 8       /* a bounded device-side wait ran out         */

/* Length, in int32 words, of the sched_meta buffer for `num_sms` CTAs. */
size_t mla_sched_meta_ints(int num_sms);

/* Bytes of workspace mla_decode needs for this shape: fp32 partial outputs and
 * partial lse of the split-KV pieces.  Returns 0 for an unsupported shape. */
size_t mla_decode_workspace_size(int B, int s_q, int H, int num_sms);

/* Split-KV scheduling metadata.
 *   cache_seqlens  device int32 [B], tokens cached per sequence.
 *   num_sms        CTAs the decode will run (normally the SM count, 148 on
 *                  B200); must equal the value later passed to mla_decode.
 *   sched_meta     device int32 [mla_sched_meta_ints(num_sms)], written:
 *                  word 0 = device error word (cleared here), a header
 *                  describing the shape, then one work range per CTA group.
 *   num_splits     device int32 [B + 1], written: the prefix sum of the
 *                  number of pieces each sequence's KV range is cut into
 *                  (sequence b owns pieces num_splits[b] .. num_splits[b+1]-1).
 * The KV tiles (128 tokens) of all sequences are laid end to end and cut into
 * equal contiguous ranges, one per CTA group, so variable lengths balance
 * across SMs.  Reads the lengths on the device; no host synchronisation. */
mla_status_t mla_decode_metadata(const int32_t *cache_seqlens, int B, int s_q, int H,
                                 int num_sms, int32_t *sched_meta, int32_t *num_splits,
                                 void *stream);

/* The decode.
 *   q              device bf16 [B, s_q, H, 576], 16-byte aligned.
 *   kv_cache       device bf16 [num_blocks, 64, 576], 16-byte aligned.
 *   block_table    device int32 [B, max_blocks]: page p of sequence b lives in
 *                  kv_cache[block_table[b, p]]; entries past a sequence's
 *                  last page are never used (those in the same 32-page
 *                  window may be loaded, always inside [B, max_blocks]).
 *   cache_seqlens  device int32 [B] (the same buffer given to the metadata).
 *   softmax_scale  finite; applied in fp32 to the scores.
 *   num_sms, sched_meta, num_splits: exactly as produced by
 *                  mla_decode_metadata for the same B, s_q, H, lengths.
 *   workspace      device, 256-byte aligned, workspace_bytes >=
 *                  mla_decode_workspace_size(B, s_q, H, num_sms).  Scratch
 *                  only; its contents need no initialisation.
 *   out            device bf16 [B, s_q, H, 512], 8-byte aligned (written).
 *   lse            device fp32 [B, s_q, H] (written; natural log).
 * Launches the attention kernel and then the combine kernel on `stream`. */
mla_status_t mla_decode(const uint16_t *q, const uint16_t *kv_cache,
                        const int32_t *block_table, const int32_t *cache_seqlens,
                        int B, int s_q, int H, int64_t num_blocks, int max_blocks,
                        float softmax_scale, int num_sms,
                        const int32_t *sched_meta, const int32_t *num_splits,
                        void *workspace, size_t workspace_bytes,
                        uint16_t *out, float *lse, void *stream);

/* The attention kernel alone (mla_decode without its combine step), for
 * callers that schedule the combine themselves or time the kernels apart.
 * Same arguments and checks as mla_decode.  Rows of one-piece sequences are
 * final when it returns; the other rows need mla_decode_combine. */
mla_status_t mla_decode_attention(const uint16_t *q, const uint16_t *kv_cache,
                                  const int32_t *block_table, const int32_t *cache_seqlens,
                                  int B, int s_q, int H, int64_t num_blocks, int max_blocks,
                                  float softmax_scale, int num_sms,
                                  const int32_t *sched_meta, const int32_t *num_splits,
                                  void *workspace, size_t workspace_bytes,
                                  uint16_t *out, float *lse, void *stream);

/* The combine kernel alone: for every (b, i, h) whose sequence was cut into
 * more than one piece, merges the pieces' fp32 partials from the workspace:
 *     lse = M + ln(sum_k exp(lse_k - M)),  out = sum_k exp(lse_k - lse) * O_k
 * and writes out (bf16) and lse; rows of sequences with no tokens get
 * out = 0, lse = -inf; rows of one-piece sequences are left as the decode
 * wrote them.  Arguments as for mla_decode. */
mla_status_t mla_decode_combine(const int32_t *num_splits, const int32_t *sched_meta,
                                const void *workspace, size_t workspace_bytes,
                                int B, int s_q, int H, int num_sms,
                                uint16_t *out, float *lse, void *stream);

/* Size of the workspace built into the library for mla_decode_static_workspace. */
#define MLA_STATIC_WORKSPACE_BYTES (8u << 20)

/* mla_decode without a caller-supplied workspace, for callers that cannot
 * allocate device memory: code that runs where device allocation is not
 * permitted or not wanted -- a host application whose device memory is
 * reserved up front by its own pool, or a plugin inside a framework that owns
 * every allocation -- and so cannot obtain the scratch buffer mla_decode
 * expects.  The scratch is a fixed device array compiled into the library
 * (MLA_STATIC_WORKSPACE_BYTES, 8 MiB); every GPU that loads the library holds
 * it until the process exits.  The paper has no counterpart: this is a
 * packaging convenience, not part of the method.
 *
 * Arguments, layouts and results are those of mla_decode without `workspace`
 * and `workspace_bytes`; the caller still passes every input and output.  This
 * call makes no device allocation and frees nothing.
 *   - Returns MLA_ERR_WORKSPACE_TOO_SMALL, without launching, when the shape
 *     needs more than MLA_STATIC_WORKSPACE_BYTES
 *     (mla_decode_workspace_size(B, s_q, H, num_sms) tells); the message is in
 *     mla_last_error_message.  With 148 CTAs the three s_q = 1, 16-head
 *     workloads of up to 16 sequences fit (4.9 to 5.4 MB); B = 32 at s_q = 2
 *     (about 11.8 MB) and B = 64 at 128 heads (about 36 MB) are refused.
 *   - The first call on a device looks up the array's device address for that
 *     device (once; no allocation).  Make that first call before capturing any
 *     stream.  The address is kept for the life of the process: after a
 *     cudaDeviceReset, or with another context made current on that device,
 *     it is stale, so do not use this entry point across either.
 *   - All calls share the one array and it keeps the last call's contents.
 *     Nothing in it needs to start at zero (every value read is written first
 *     by the same call), but calls whose kernels overlap on the GPU -- on two
 *     streams, or from two host threads -- race on it: serialise them. */
mla_status_t mla_decode_static_workspace(const uint16_t *q, const uint16_t *kv_cache,
                                         const int32_t *block_table, const int32_t *cache_seqlens,
                                         int B, int s_q, int H, int64_t num_blocks, int max_blocks,
                                         float softmax_scale, int num_sms,
                                         const int32_t *sched_meta, const int32_t *num_splits,
                                         uint16_t *out, float *lse, void *stream);

/* FP8 cache.  The same decode over a cache of e4m3 codes with one fp32 scale
 * per cached token: token j's row is e4m3(kv_codes[blk][j % 64][:]) *
 * kv_scale[blk][j % 64] (the juejin.cn "FlashMLA" post, section 5, says
 * FlashMLA runs in mixed precision such as FP8 and BF16; it fixes no format,
 * and this per-token-scale layout is the reading taken).  The tensor cores
 * read the codes as they lie in the cache (tcgen05.mma kind::f8f6f4): each
 * query row is written as two e4m3 terms whose sum is the bf16 row times a
 * per-row power of two (exact but for values below 2^-10 of the row's
 * largest), and each token's softmax weight, multiplied by its scale, as two
 * e4m3 terms (8 significant bits, as a bf16 weight).  Scores, the softmax
 * sums and the outputs are accumulated in fp32 as in mla_decode.  The two
 * e4m3 NaN patterns (s.1111.111) are NaN.
 *   kv_codes   device uint8 [num_blocks, 64, 576] (e4m3 bit patterns, OCP E4M3
 *              as __nv_fp8_e4m3 holds them), 16-byte aligned.
 *   kv_scale   device fp32 [num_blocks, 64], 16-byte aligned.
 *   Every other argument as for mla_decode (same metadata, same workspace).
 * Supported shapes: 16 or 32 query columns per CTA -- H = 16 with s_q = 1 or
 * 2, H = 32 with s_q = 1; others return MLA_ERR_UNSUPPORTED_SHAPE.  mla_decode_attention_fp8 launches the
 * attention kernel alone, mla_decode_fp8 the attention and combine kernels. */
mla_status_t mla_decode_attention_fp8(const uint16_t *q, const uint8_t *kv_codes, const float *kv_scale,
                                      const int32_t *block_table, const int32_t *cache_seqlens, int B, int s_q,
                                      int H, int64_t num_blocks, int max_blocks, float softmax_scale, int num_sms,
                                      const int32_t *sched_meta, const int32_t *num_splits, void *workspace,
                                      size_t workspace_bytes, uint16_t *out, float *lse, void *stream);
mla_status_t mla_decode_fp8(const uint16_t *q, const uint8_t *kv_codes, const float *kv_scale,
                            const int32_t *block_table, const int32_t *cache_seqlens, int B, int s_q, int H,
                            int64_t num_blocks, int max_blocks, float softmax_scale, int num_sms,
                            const int32_t *sched_meta, const int32_t *num_splits, void *workspace,
                            size_t workspace_bytes, uint16_t *out, float *lse, void *stream);

/* Non-absorbed form.  The same latent cache, but each head attends with its
 * own 192-wide keys and 128-wide values, decompressed from the latent rows
 * tile by tile as "FlashMLA: compressing the KV cache to one eighth"
 * (jsqmd.com), "FlashMLA compute flow", steps 1-5, describes (K_tile =
 * C_KV_tile W_UK, V_tile = C_KV_tile W_UV, then S = Q K^T, online softmax,
 * O += softmax(S) V).  For sequence b, query position i and head h, over
 * the same visible tokens j as mla_decode (C_j = the 512 latent columns of
 * token j's row, rope_j = its last 64 columns, cached already rotated and
 * shared by every head):
 *     k_j = [ W_UK[h] C_j (128) ,  rope_j (64) ],   v_j = W_UV[h] C_j (128)
 *     out[b,i,h,:] = sum_j softmax(softmax_scale * <q[b,i,h,:], k_j>)_j v_j
 *     lse[b,i,h]   = ln(sum_j exp(softmax_scale * <q[b,i,h,:], k_j>))
 * The up-projections run on the tensor cores per 128-token tile (fp32
 * accumulation); scores, softmax and the value sum stay in fp32.
 *   q            device bf16 [B, s_q, H, 192]: 128 key columns, then 64 rope.
 *   kv_cache, block_table, cache_seqlens, num_blocks, max_blocks,
 *   softmax_scale: as for mla_decode (no schedule: each CTA takes one
 *                sequence, one head and a fixed share of the tiles).
 *   w_uk, w_uv   device bf16 [H, 128, 512], 16-byte aligned: row e of head h
 *                holds the latent coefficients of key / value dimension e.
 *   num_sms      SMs to size the split of each sequence for (148 on B200).
 *   workspace    device, 256-byte aligned, workspace_bytes >=
 *                mla_decode_naive_workspace_size(B, s_q, H, max_blocks,
 *                num_sms); scratch for the splits' fp32 partial results.
 *   error_word   device int32 [1], zeroed by the caller; the kernel ORs in
 *                MLA_DEVERR_* bits (bad page-table entries, bad lengths,
 *                timed-out waits) and never traps.
 *   out          device bf16 [B, s_q, H, 128], 8-byte aligned (written).
 *   lse          device fp32 [B, s_q, H] (written; natural log).
 * Supported: s_q in {1, 2}; 1 <= H <= 128; 1 <= B <= 4096.  Launches the
 * attention kernel and then its merge kernel on `stream`. */
#define MLA_NAIVE_D 128   /* decompressed key / value width per head */
size_t mla_decode_naive_workspace_size(int B, int s_q, int H, int max_blocks, int num_sms);
mla_status_t mla_decode_naive(const uint16_t *q, const uint16_t *kv_cache, const uint16_t *w_uk,
                              const uint16_t *w_uv, const int32_t *block_table, const int32_t *cache_seqlens,
                              int B, int s_q, int H, int64_t num_blocks, int max_blocks, float softmax_scale,
                              int num_sms, void *workspace, size_t workspace_bytes, int32_t *error_word,
                              uint16_t *out, float *lse, void *stream);

/* Merge of W partial attention states of the same output rows, each computed
 * over a disjoint range of the tokens -- in context-parallel decode, the
 * (out, lse) of W ranks that each hold a contiguous range of every sequence's
 * pages and run mla_decode on it.  The same log-sum-exp merge as the combine
 * (the online softmax of "FlashMLA: compressing the KV cache", jsqmd.com,
 * "compute flow", step 4, applied to whole partial results):
 *     M = max_w lse_w,   lse = M + ln sum_w exp(lse_w - M),
 *     out = sum_w exp(lse_w - lse) * out_w        (fp32, rounded once to bf16)
 * with out = 0 and lse = -inf for a row whose states are all empty
 * (lse_w = -inf, as mla_decode writes for a rank that holds no visible token).
 *   out_parts   device bf16 [W, rows, 512], 16-byte aligned.
 *   lse_parts   device fp32 [W, rows] (natural log), 4-byte aligned.
 *   W           1 <= W <= 64.
 *   rows        number of output rows, 1 <= rows <= 2^31 - 1 (B * s_q * H
 *               for decode results).
 *   out         device bf16 [rows, 512], 16-byte aligned (written).
 *   lse         device fp32 [rows], 4-byte aligned (written).
 * Inputs and outputs must not overlap.  Argument errors return before any
 * launch; asynchronous on `stream`. */
mla_status_t mla_merge_states(const uint16_t *out_parts, const float *lse_parts, int W, int64_t rows,
                              uint16_t *out, float *lse, void *stream);

/* Waits for `stream`, copies word 0 of sched_meta to *host_code, and returns
 * MLA_ERR_DEVICE_CHECK if any bit is set (MLA_OK otherwise). */
mla_status_t mla_get_device_error(const int32_t *sched_meta, int32_t *host_code, void *stream);

/* Static, human-readable name of a status code. */
const char *mla_status_string(mla_status_t status);

/* Text explaining the last error status of a call on the calling thread: the
 * failing CUDA call and its error string for MLA_ERR_CUDA, and the sizes for
 * the MLA_ERR_WORKSPACE_TOO_SMALL of mla_decode_static_workspace.  Every
 * entry point clears it when called, so it never outlives the next call; ""
 * if the last call set none.  Owned by the library. */
const char *mla_last_error_message(void);

/* Test hook for the failure path of the bounded device waits: from the next
 * decode launch on, CTA `cta` announces its first cache load without issuing
 * it, so its waits run out after their time limit (about 2 s), set
 * MLA_DEVERR_TIMEOUT and end; -1 turns the hook off (the default).
 * Process-wide; not for use in production. */
void mla_debug_stall_cta(int cta);

#ifdef __cplusplus
}
#endif

#endif /* MLA_DECODE_H */
