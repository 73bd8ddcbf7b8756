/*
 * attn.h -- C ABI of libattn_b200.so, the B200 (sm_100a) online-softmax
 * ("flash") attention forward:
 *
 *     out = softmax(softmax_scale * Q K^T + additive_mask) V
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor pointers are DEVICE pointers owned by the caller. The library
 *    never frees them and never keeps them after the call returns. The library
 *    makes no allocation call: besides the caller's buffers it only uses
 *    static __device__ memory reserved when the library is loaded (one
 *    per-device status word, and the scratch array of
 *    attn_gqa_decode_noalloc) and kernel parameters.
 *  - bf16 tensors are passed as `const uint16_t*` holding bf16 bit patterns
 *    (1 sign, 8 exponent, 7 mantissa bits). FP8 caches are `const uint8_t*`
 *    holding E4M3FN codes. All tensors are dense, row-major, contiguous in the
 *    layouts stated per function, and every tensor base address must be
 *    16-byte aligned (it is read by the Tensor Memory Accelerator).
 *  - `stream` is a `cudaStream_t` passed as `void*` (NULL = legacy default
 *    stream). Every function only validates its arguments on the host and
 *    enqueues work: it returns before the GPU has finished.
 *  - Return value: ATTN_OK or a negative attn_status. A host-side validation
 *    failure enqueues nothing. Errors the device detects (an out-of-range block
 *    table entry, a bad sequence descriptor, a bounded wait that ran out) are
 *    recorded in the per-device status word and reported by attn_check().
 *  - softmax_scale must be finite and > 0. Rows whose every key is masked
 *    produce an all-zero output row.
 *  - Nothing here falls back to another implementation: an unsupported shape
 *    is an error.
 */
#ifndef ATTN_B200_H
#define ATTN_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ATTN_API __attribute__((visibility("default")))
#else
#define ATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum attn_status {
    ATTN_OK = 0,
    ATTN_ERR_NULL = -1,           /* a required pointer is NULL                      */
    ATTN_ERR_SHAPE = -2,          /* inconsistent or out-of-range sizes / scale      */
    ATTN_ERR_UNSUPPORTED = -3,    /* valid attention, but a shape this build rejects */
    ATTN_ERR_ALIGN = -4,          /* a base address is not 16-byte aligned           */
    ATTN_ERR_WORKSPACE = -5,      /* workspace missing or too small                  */
    ATTN_ERR_CUDA = -6,           /* a CUDA runtime / driver call failed             */
    ATTN_ERR_DEVICE_TIMEOUT = -7, /* a kernel's bounded wait ran out (device side)   */
    ATTN_ERR_BLOCK_TABLE = -8,    /* a block-table entry is outside the pool (device)*/
    ATTN_ERR_SEQUENCE = -9        /* a sequence descriptor is out of range (device)  */
} attn_status;

/*
 * attn_encoder_fwd -- non-causal multi-head encoder attention.
 *
 * Defined by: "V-JEPA2 ViT-L Encoder NKI Kernels for AWS Trainium2" (the K2
 * attention inner, "Repository layout"), "vit-encoder-neuron-kernels"
 * ("Supported shapes and limits": bidirectional self-attention, head_dim 64 or
 * 128) and "gte-encoder-neuron-kernels" ("Constraints": right padding with a
 * 0/1 attention_mask, here generalised to an additive per-key bias).
 *
 *   q, k, v, out : [B, H, S, D] bf16. out may not alias q, k or v.
 *   B, H >= 1; S >= 1; D in {64, 128}.
 *   softmax_scale: finite, > 0 (1/sqrt(D) for the ViT encoders).
 *   key_bias     : NULL, or [B, S] fp32 additive bias added to every query's
 *                  score for key j of batch entry b (0 keep, -inf drop; any
 *                  finite value, -FLT_MAX included, keeps the key). The 128-key
 *                  tiles after the last kept key of an entry are never read (so
 *                  their K and V may hold anything); a dropped key inside a tile
 *                  that holds a kept key has weight 0, but its V row is still
 *                  multiplied by it and must be finite.
 *
 * Every query row attends to all S keys (no causal mask). Accumulation is fp32;
 * out is rounded to bf16 (round-to-nearest-even).
 * Errors: ATTN_ERR_NULL, ATTN_ERR_SHAPE, ATTN_ERR_UNSUPPORTED (D), ATTN_ERR_ALIGN,
 * ATTN_ERR_CUDA.
 */
ATTN_API int attn_encoder_fwd(const uint16_t* q, const uint16_t* k, const uint16_t* v, uint16_t* out,
                     int B, int H, int S, int D, float softmax_scale,
                     const float* key_bias, void* stream);

/*
 * attn_gqa_decode_workspace_size -- bytes of device workspace attn_gqa_decode
 * needs for these sizes: the per-batch lists of live 8-key sub-tiles with their
 * mask values, and the partial results of the key-sequence split (one per warp
 * and (batch, kv head) pair it covers). 0 for invalid sizes.
 */
ATTN_API size_t attn_gqa_decode_workspace_size(int B, int Hq, int Hkv, int S_ctx, int D);

/*
 * attn_gqa_decode -- single-token (S_q = 1) GQA flash-decode.
 *
 * Defined by: "head_dim>128 (256/512) GQA Flash-Decode NKI Kernel for AWS
 * Trainium", sections "Input contract" and "Supported shapes (the eligibility
 * gate)"; the key-sequence split with a log-sum-exp combine is the page's
 * "Future performance follow-on" (multi-program dispatch).
 *
 *   q         : [B, Hq, 1, D] bf16
 *   k, v      : [B, Hkv, S_ctx, D] bf16
 *   attn_mask : NULL (no mask), or [B, 1, 1, S_ctx] fp32 additive (0 keep,
 *               -inf drop). A -inf entry removes the key whatever its K and V
 *               rows hold (even NaN); any finite value, -FLT_MAX included,
 *               keeps the key with that additive score.
 *   out       : [B, Hq, 1, D] bf16
 *   Hq == Hkv * num_kv_groups; query head h reads kv head h / num_kv_groups.
 *   D in {128, 256, 512}; S_ctx >= 1 (no multiple-of-128 requirement).
 *   num_kv_groups in {1, 2, 4, 8}; D == 512 allows at most 4 (else
 *   ATTN_ERR_UNSUPPORTED). B * Hkv <= 65535 and B * Hkv * ceil(S_ctx / 8) < 2^30
 *   (else ATTN_ERR_UNSUPPORTED).
 *   workspace : device buffer of at least attn_gqa_decode_workspace_size(...)
 *               bytes, 16-byte aligned, owned by the caller; its contents on
 *               entry do not matter. Calls that share one workspace must not
 *               overlap on the GPU.
 * Errors: ATTN_ERR_NULL, ATTN_ERR_SHAPE, ATTN_ERR_UNSUPPORTED (D), ATTN_ERR_ALIGN,
 * ATTN_ERR_WORKSPACE, ATTN_ERR_CUDA.
 */
ATTN_API int attn_gqa_decode(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                    const float* attn_mask, uint16_t* out,
                    int B, int Hq, int Hkv, int num_kv_groups, int S_ctx, int D,
                    float softmax_scale, void* workspace, size_t workspace_bytes,
                    void* stream);

/*
 * attn_gqa_decode_noalloc -- attn_gqa_decode for callers that cannot allocate
 * device memory.
 *
 * The pages have no counterpart of this function; it exists for deployment.
 * Some hosts own the whole device-memory budget and forbid allocations after
 * start-up (plugin and embedded runtimes), and some latency-critical loops
 * cannot afford cudaMalloc, which may synchronise the whole device. Such
 * callers cannot provide the workspace attn_gqa_decode needs. This entry point
 * computes exactly what attn_gqa_decode computes (same kernels, same results)
 * but keeps the split-KV partials in a scratch array that the library reserves
 * statically on every device that loads it (ATTN_NOALLOC_SCRATCH_BYTES, held
 * until the process exits). It calls no allocator.
 *
 *   Arguments: as attn_gqa_decode, without the workspace pair. The caller
 *   still owns q, k, v, attn_mask and out.
 *   Limit: attn_gqa_decode_workspace_size(B, Hq, Hkv, S_ctx, D) must not
 *   exceed ATTN_NOALLOC_SCRATCH_BYTES; larger problems are rejected with
 *   ATTN_ERR_WORKSPACE before anything is enqueued.
 *   Set-up: the first call on a device looks up the scratch array's device
 *   address on the current device (once per device; again only if the device's
 *   context was re-created, e.g. after cudaDeviceReset). Make that first call
 *   outside any stream capture.
 *   Sharing: all calls on a device use the same scratch array, which keeps the
 *   previous call's contents (nothing in it needs to start at zero). Calls that
 *   may run at the same time on the GPU (different streams without ordering)
 *   race on it: order them on one stream, or use attn_gqa_decode with separate
 *   workspaces.
 * Errors: as attn_gqa_decode; ATTN_ERR_WORKSPACE when the sizes exceed the
 * scratch; ATTN_ERR_CUDA if the address look-up fails.
 */
#define ATTN_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
ATTN_API int attn_gqa_decode_noalloc(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                     const float* attn_mask, uint16_t* out,
                                     int B, int Hq, int Hkv, int num_kv_groups, int S_ctx, int D,
                                     float softmax_scale, void* stream);

/*
 * attn_paged_history -- history-only attention over a paged FP8 KV cache.
 *
 * Defined by: "Prefill Context-Parallel Attention POC for Trainium2",
 * sections "Layout" (Q [Hq, q_len, D], K/V [blocks, Hkv, block_size, D],
 * O [Hq, q_len, D]), the history-only rule under the target configuration,
 * the runtime additive bias from actual_history_len, and "Current POC
 * constraints" (head_dim multiple of 128, block_size <= 512 and a multiple of
 * 128, Q bf16, K/V FP8 E4M3FN, fp32 max/sum). On one GPU the page's ring of
 * ranks becomes a loop over the blocks named by the block table.
 *
 *   q            : [Hq, Sq, D] bf16
 *   k_cache      : [num_phys_blocks, Hkv, block_size, D] E4M3FN codes
 *   v_cache      : same layout as k_cache
 *   block_table  : [n_table] int32, logical block i -> physical block
 *                  block_table[i]; logical position t lives in logical block
 *                  t / block_size at offset t % block_size.
 *   actual_history_len : 0 <= len <= n_table * block_size. Positions >= len
 *                  are ignored (a partial last block is allowed); blocks
 *                  wholly beyond len are never read.
 *   k_scale, v_scale   : per-tensor dequantisation scales (value = code * scale);
 *                  k_scale finite and > 0, v_scale finite
 *   out          : [Hq, Sq, D] bf16
 *   Hq == Hkv * num_kv_groups; D == 256; block_size in {128, 256, 384, 512}.
 *   Every query attends to every history position < len (no causal mask).
 * Table entries are checked on the device: an entry outside
 * [0, num_phys_blocks) is skipped and recorded as ATTN_ERR_BLOCK_TABLE.
 * Cache rows past len inside the last block read are multiplied by a zero
 * probability, so they must hold finite codes (any value; E4M3FN quantisation
 * never writes the two NaN codes).
 * Errors: ATTN_ERR_NULL, ATTN_ERR_SHAPE, ATTN_ERR_UNSUPPORTED, ATTN_ERR_ALIGN,
 * ATTN_ERR_CUDA.
 */
ATTN_API int attn_paged_history(const uint16_t* q, const uint8_t* k_cache, const uint8_t* v_cache,
                       const int32_t* block_table, int n_table, int num_phys_blocks,
                       int block_size, int actual_history_len,
                       float k_scale, float v_scale, float softmax_scale,
                       int Hq, int Hkv, int num_kv_groups, int Sq, int D,
                       uint16_t* out, void* stream);

/*
 * attn_paged_prefill -- prefill attention over a paged FP8 KV cache: each
 * sequence's current tokens attend to its history and, causally, to each other.
 *
 * Defined by: "Prefill Context-Parallel Attention POC for Trainium2" (layout and
 * constraints as attn_paged_history), completing its "current tokens do not
 * attend to one another yet": the current tokens' K/V are written into the cache
 * after the history first (as E4M3FN codes, like the history), then
 *     out[h, q0 + i] = softmax_t(scale * q[h, q0 + i] . K_t) V_t,
 *     t over logical positions 0 .. hist + i of the sequence's block table,
 * for query i of a sequence whose rows start at q0 and whose history has hist
 * tokens. Several sequences per call.
 *
 *   q           : [Hq, total_q, D] bf16, the sequences' current tokens packed
 *   k_cache, v_cache : [num_phys_blocks, Hkv, block_size, D] E4M3FN codes
 *   block_tables: [num_seqs, table_stride] int32 (device); row s maps sequence
 *                 s's logical blocks to physical blocks
 *   q_start     : [num_seqs + 1] int32 (device), non-decreasing row offsets,
 *                 q_start[0] = 0, q_start[num_seqs] = total_q
 *   hist_lens   : [num_seqs] int32 (device), >= 0, with hist + q_len <=
 *                 table_stride * block_size
 *   max_q_len   : host bound on every q_len (sizes the grid)
 *   k_scale, v_scale, softmax_scale, Hq, Hkv, num_kv_groups, D, block_size:
 *                 as attn_paged_history (D == 256)
 *   out         : [Hq, total_q, D] bf16
 * Cache rows past a sequence's last position inside its last block must hold
 * finite codes, as for attn_paged_history.
 * num_seqs <= 65535. The device checks every sequence descriptor (a bad one
 * writes nothing for that sequence and records ATTN_ERR_SEQUENCE) and every
 * table entry it reads (ATTN_ERR_BLOCK_TABLE). Only blocks up to each tile's
 * last visible position are read.
 * Errors: ATTN_ERR_NULL, ATTN_ERR_SHAPE, ATTN_ERR_UNSUPPORTED, ATTN_ERR_ALIGN,
 * ATTN_ERR_CUDA.
 */
ATTN_API int attn_paged_prefill(const uint16_t* q, const uint8_t* k_cache, const uint8_t* v_cache,
                                const int32_t* block_tables, int table_stride, int num_phys_blocks,
                                int block_size, const int32_t* q_start, const int32_t* hist_lens,
                                int num_seqs, int total_q, int max_q_len,
                                float k_scale, float v_scale, float softmax_scale,
                                int Hq, int Hkv, int num_kv_groups, int D,
                                uint16_t* out, void* stream);

/*
 * attn_rope_qk -- rotary position embedding of the query and key rows.
 *
 * Defined by: "vit-encoder-neuron-kernels", section "Kernels" (the encoder
 * attention takes per-token rotation tables; two pairings of head-dim lanes).
 * For every row (b, h, s) of q and of k and every pair j < D/2, with lanes
 * (ia, ib) = (j, j + D/2) when interleaved == 0 ("half": DINOv3, EVA-02, Llama)
 * or (2j, 2j + 1) when interleaved == 1 (V-JEPA2):
 *     out[ia] = x[ia] cos[s][j] - x[ib] sin[s][j]
 *     out[ib] = x[ia] sin[s][j] + x[ib] cos[s][j]
 * computed in fp32 and rounded to bf16 (round-to-nearest-even). Apply it to Q and
 * K before attn_encoder_fwd.
 *
 *   q, k          : [B, H, S, D] bf16 (device).
 *   q_out, k_out  : [B, H, S, D] bf16 (device); may equal q / k (in place), must
 *                   not otherwise overlap them or each other.
 *   cos_table, sin_table : [S, D/2] fp32 (device), row s for token position s
 *                   (any position grid: 1-D, or 2-D / 3-D patch grids flattened).
 *   B, H, S >= 1; D a multiple of 16, 16 <= D <= 512.
 * All pointers 16-byte aligned. Runs one kernel on `stream`; the caller owns all
 * buffers.
 * Errors: ATTN_ERR_NULL, ATTN_ERR_SHAPE (sizes, interleaved not 0 / 1, partial
 * overlap), ATTN_ERR_UNSUPPORTED (D), ATTN_ERR_ALIGN, ATTN_ERR_CUDA.
 */
ATTN_API int attn_rope_qk(const uint16_t* q, const uint16_t* k, uint16_t* q_out, uint16_t* k_out,
                          const float* cos_table, const float* sin_table,
                          int B, int H, int S, int D, int interleaved, void* stream);

/*
 * attn_qkv_rope_proj -- the QKV projection in front of the encoder attention,
 * with RoPE applied to Q and K in the same kernel.
 *
 * Defined by: "V-JEPA2 ViT-L Encoder NKI Kernels for AWS Trainium2", section
 * "Repository layout" (the attention block K2: QKV projection + RoPE, then the
 * attention inner, then the output projection; LayerNorm affines are folded into
 * the weights, so the projection is a plain affine map) and
 * "vit-encoder-neuron-kernels", section "Kernels" (both RoPE lane pairings):
 *     t = x W_qkv^T + b_qkv,   t [B, S, 3 H D]
 * column block 0 of t is Q, block 1 K, block 2 V; column h D + d of a block is
 * head h, lane d. Q and K are then rotated exactly as attn_rope_qk rotates them
 * (in fp32, before the single rounding to bf16); V is not rotated.
 *
 *   x          : [B, S, C] bf16 (the block's normalised input)
 *   w_qkv      : [3 H D, C] bf16 (a torch.nn.Linear weight: out x in)
 *   b_qkv      : NULL or [3 H D] fp32
 *   cos_table, sin_table : NULL (no rotation) or [S, D/2] fp32 each, row s for
 *                token s; interleaved selects the pairing as in attn_rope_qk
 *   q, k, v    : [B, H, S, D] bf16 outputs, ready for attn_encoder_fwd
 *   B, S, H >= 1; D in {64, 128}; C a multiple of 64; H * D a multiple of 128.
 * fp32 accumulation on the tensor cores. All pointers 16-byte aligned; the
 * caller owns every buffer.
 * Errors: ATTN_ERR_NULL (a table without the other), ATTN_ERR_SHAPE,
 * ATTN_ERR_UNSUPPORTED, ATTN_ERR_ALIGN, ATTN_ERR_CUDA.
 */
ATTN_API int attn_qkv_rope_proj(const uint16_t* x, const uint16_t* w_qkv, const float* b_qkv,
                                const float* cos_table, const float* sin_table, int interleaved,
                                int B, int S, int C, int H, int D,
                                uint16_t* q, uint16_t* k, uint16_t* v, void* stream);

/*
 * attn_out_proj -- the output projection behind the encoder attention.
 *
 * Defined by: "V-JEPA2 ViT-L Encoder NKI Kernels for AWS Trainium2", section
 * "Repository layout" (K2 outer: the out-projection of the attention block):
 *     y[b, s, :] = a[b, s, :] W_o^T + b_o,   a[b, s, h D + d] = o[b, h, s, d]
 * (the heads side by side, read straight from the attention layout).
 *
 *   o     : [B, H, S, D] bf16 (attn_encoder_fwd's output)
 *   w_o   : [C_out, H D] bf16 (a torch.nn.Linear weight)
 *   b_o   : NULL or [C_out] fp32
 *   y     : [B, S, C_out] fp32 (kept in fp32: it is added to the fp32 residual
 *           stream)
 *   B, S, H >= 1; D in {64, 128}; C_out a multiple of 128.
 * All pointers 16-byte aligned; the caller owns every buffer.
 * Errors: ATTN_ERR_NULL, ATTN_ERR_SHAPE, ATTN_ERR_UNSUPPORTED, ATTN_ERR_ALIGN,
 * ATTN_ERR_CUDA.
 */
ATTN_API int attn_out_proj(const uint16_t* o, const uint16_t* w_o, const float* b_o,
                           int B, int S, int H, int D, int C_out, float* y, void* stream);

/*
 * attn_check -- synchronise `stream`, then return and clear the first error the
 * device recorded on the current device since the last check (ATTN_OK if
 * none). Returns ATTN_ERR_CUDA if the synchronisation itself fails.
 */
ATTN_API int attn_check(void* stream);

/* attn_status_string -- static, human-readable name of a status code. */
ATTN_API const char* attn_status_string(int status);

/* attn_version -- library ABI version (major * 10000 + minor * 100 + patch). */
ATTN_API int attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_H */
