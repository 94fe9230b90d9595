/*
 * tq.h -- C ABI of the TQ4/4 KV-cache library for NVIDIA B200 (sm_100a).
 *
 * TQ4/4 keeps 4-bit keys and 4-bit values ("TurboQuant 在 AMD GPU 上把長上下文
 * 延遲壓下來", summary table and section 2):
 *   key   : rotated by the normalised Walsh-Hadamard transform over head_dim
 *           (section 4 of that page), stored as an fp16 L2 norm plus a 4-bit
 *           index per element into a 16-entry centroid table (the Lloyd-Max
 *           table, or one re-fitted on ~20 rotated vectors: "UltraQuant：4-bit
 *           KV 快取加速長代理", section 「方法怎麼做，白話講」);
 *   value : asymmetric uniform 4-bit codes with one fp16 scale and one fp16
 *           zero point per group of 32 elements (section 2: "standard
 *           uniform quantization").
 * Both live in a paged cache of 16-token blocks.
 *
 * Conventions for every call below:
 *   - Pointers marked (device) are CUDA device pointers owned by the caller;
 *     the library never allocates, frees or synchronises inside a hot call.
 *     Pointers marked (host) are ordinary host memory.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream); work is
 *     enqueued asynchronously on it.
 *   - Return value: TQ_OK, or a TQ_ERR_* code after which nothing was
 *     enqueued; tq_last_error() then gives a message (per calling thread).
 *   - `status` (device, may be NULL) is one int32 that kernels OR TQ_STATUS_*
 *     bits into when they meet bad data they cannot check on the host (a
 *     block id out of range, ...).  The caller zeroes it and reads it back
 *     whenever it likes.  Kernels never trap; a flagged element is skipped.
 *   - bf16/fp16 arrays are raw 16-bit IEEE patterns; all arrays are dense,
 *     row-major, with the shapes given.
 *
 * Cache record: one per (physical block, kv head), 16 tokens, 16-byte
 * aligned fields, little-endian; code byte j holds element 2j in its low
 * nibble and element 2j+1 in its high nibble:
 *   [0,      8d)        key codes    [16][d/2] bytes, byte j at row offset j
 *   [8d,     8d+32)     key norms    [16] fp16
 *   [8d+32,  16d+32)    value codes, 8d bytes: byte j = 8m + r of token t at
 *                       (8 (t/2) + r) (d/8) + 4 (m/2) + 2 (t%2) + (m%2)
 *   [16d+32, 17d+32)    value scales fp16: token t, group G at byte
 *                       2 (4 (c (d/32) + G) + u), c = (t%8)/2, u = 2 (t/8) + t%2
 *   [17d+32, 18d+32)    value zeros fp16, same placement
 * (the value placement puts each decode thread's tensor-core operands in
 * contiguous 8- or 16-byte runs)
 * = 2336 bytes at d = 128, 1184 bytes at d = 64.  The cache is
 * [num_blocks][num_kv_heads][record].
 */
#ifndef TQ_H
#define TQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define TQ_API __attribute__((visibility("default")))
#else
#define TQ_API
#endif

#define TQ_BLOCK_TOKENS 16
#define TQ_VALUE_GROUP 32

enum {
    TQ_OK = 0,
    TQ_ERR_INVALID_ARG = 1, /* null pointer, negative size, inconsistent shape */
    TQ_ERR_UNSUPPORTED = 2, /* head_dim not 64/128, H_q % H_kv != 0, too many splits */
    TQ_ERR_ALIGNMENT = 3,   /* a pointer misses its required alignment */
    TQ_ERR_CUDA = 4,        /* a CUDA runtime call failed (message has the CUDA error) */
    TQ_ERR_WORKSPACE = 5    /* workspace pointer NULL or smaller than required */
};

/* device status bits */
enum {
    TQ_STATUS_BAD_SLOT = 1,  /* append: slot or logical slot outside the cache / table */
    TQ_STATUS_BAD_BLOCK = 2, /* a block-table entry outside [0, num_blocks) */
    TQ_STATUS_RANGE = 4,     /* a key norm or value scale/zero overflowed fp16 */
    TQ_STATUS_BAD_LEN = 8,   /* seq_len < 0 or > max_blocks * 16 (treated as 0) */
    TQ_STATUS_TIMEOUT = 16,  /* a kernel gave up waiting (~1 s) for its own copy: the
                                call's output is incomplete; never expected */
    TQ_STATUS_INTERNAL = 32  /* the decode kernel's shared-memory plan did not fit its
                                allocation: nothing was computed; never expected */
};

/* Cache flags.  TQ_CACHE_UNROTATED: the keys are quantised without the
 * Walsh-Hadamard rotation (y = k / ||k|| goes to the table directly).  The
 * pages prefer the rotation because it spreads outlier channels evenly before
 * the quantiser ("TurboQuant 在 AMD GPU 上把長上下文延遲壓下來", section 4); the
 * unrotated cache is the baseline that shows what it buys.  Every call below
 * honours the flag (the decode and prefill skip the query rotation), and a
 * cache must be read with the flags it was written with. */
enum { TQ_CACHE_UNROTATED = 1 };

/* TQ_CACHE_BF16: a full-precision cache for the layers a model keeps unquantised.
 * "TurboQuant 在 AMD GPU 上把長上下文延遲壓下來", section 3: for full-attention
 * models, leaving the first and last layers unquantised recovers accuracy, since
 * those boundary layers are the most sensitive to KV quantisation.  Its record
 * of one (block, kv head) is the 16 tokens' bf16 key rows [16][d] followed by
 * their bf16 value rows [16][d] (64 d bytes; within row r = token (keys) or
 * 16 + token (values), the 16-byte chunk j is stored at position j ^ (r mod 8),
 * so that one copy of a record lands in shared memory ready for conflict-free
 * tensor-core loads).  tq_quantize_append stores the rows
 * as they are (no key tables: k_tables must be NULL), and the decode calls and
 * tq_dequantize read them (the decode's default split count is its own, within the
 * num_splits = 0 workspace); tq_prefill_attention returns TQ_ERR_UNSUPPORTED for
 * it.  Not combinable with TQ_CACHE_UNROTATED. */
enum { TQ_CACHE_BF16 = 2 };

typedef struct {
    int32_t num_blocks;   /* physical 16-token blocks */
    int32_t num_kv_heads; /* H_kv */
    int32_t head_dim;     /* d: 64 or 128 */
    int32_t flags;        /* 0, TQ_CACHE_UNROTATED or TQ_CACHE_BF16 (else TQ_ERR_INVALID_ARG) */
    void* data;           /* (device) [num_blocks][num_kv_heads][record], 16-byte aligned */
} tq_cache_t;

/* Bytes of one (block, kv head) record (2336 at d=128, 1184 at d=64); 0 if d unsupported. */
TQ_API size_t tq_record_bytes(int head_dim);
/* Bytes of a whole cache; 0 on an unsupported shape. */
TQ_API size_t tq_cache_bytes(int num_blocks, int num_kv_heads, int head_dim);
/* Bytes of one record of a cache with these flags (64 d for TQ_CACHE_BF16, else
 * tq_record_bytes(d)); 0 on an unsupported head_dim or flag combination. */
TQ_API size_t tq_cache_record_bytes(int head_dim, int flags);

/* Key tables are 16 fp16 values (raw bit patterns), strictly ascending, so that
 * every centroid is an exact fp16 tensor-core operand.
 *
 * (host) Default key table for head_dim d: the 16-level Lloyd-Max quantiser of
 * N(0,1) scaled by 1/sqrt(d) (the rotated unit vector has coordinates of
 * variance 1/d), rounded to nearest fp16, ascending.  "UltraQuant：4-bit KV
 * 快取加速長代理", 「方法怎麼做，白話講」: the theoretical Lloyd-Max table. */
TQ_API int tq_lloyd_max_table(int head_dim, uint16_t out16[16]);

/* (host) Re-fit a 16-entry key table on n calibration key vectors (bf16
 * [n][head_dim], host): rotate each unit-normalised vector, then run 1-D
 * k-means (Lloyd) from init16 for at most max_iter rounds; empty cells keep
 * their level; the result is sorted and rounded to fp16.  Same page and
 * section: centroids re-fitted on about 20 rotated vectors.  Returns the
 * iteration count (>= 0) or -TQ_ERR_*. */
TQ_API int tq_fit_k_table(const uint16_t* keys_bf16, int n, int head_dim,
                          const uint16_t init16[16], int max_iter, uint16_t out16[16]);

/* Quantise T new tokens and write them into the cache (the TQ4/4 write path):
 * keys by Walsh-Hadamard rotation and the 16-entry look-up table, values by
 * uniform 4-bit codes ("TurboQuant 在 AMD GPU 上把長上下文延遲壓下來", section 2,
 * TQ4/4, and section 4, Walsh-Hadamard rotation); the call follows the write
 * step tq_quantize_append(K, V, block_table, slot_mapping) of the TQ4/4 cache.
 *   K, V        (device) bf16 [T][H_kv][d], 16-byte aligned
 *   block_table (device, may be NULL) int32 [num_seqs][max_blocks]
 *   slot_mapping(device) int32 [T]:
 *       block_table == NULL: physical slot = block * 16 + offset;
 *       block_table != NULL: logical slot = seq * (max_blocks * 16) + position,
 *                            mapped to block_table[seq][position / 16];
 *       -1 skips the token.
 *   k_tables    (device, may be NULL) fp16 [H_kv][16] strictly ascending
 *               per-head key tables; NULL = tq_lloyd_max_table(d) for all heads.
 * Slots outside the cache set TQ_STATUS_BAD_SLOT / _BAD_BLOCK and are skipped.
 * Two tokens mapped to one slot race (last writer wins, per field). */
TQ_API int tq_quantize_append(const void* K, const void* V, const int32_t* block_table, int num_seqs,
                       int max_blocks, const int32_t* slot_mapping, int T,
                       const tq_cache_t* cache, const uint16_t* k_tables, int32_t* status,
                       void* stream);

/* Number of context splits tq_decode_attention uses when num_splits == 0.  It
 * returns 0: the default plan has no fixed split count, it cuts the space of
 * (sequence, kv head, block) records evenly over the whole GPU, so an item is
 * split only where a cut falls inside it.  The arguments are kept for callers
 * that size their own plans from them. */
TQ_API int tq_decode_default_splits(int B, int H_kv, int max_seq_len);
/* Workspace bytes for tq_decode_attention with this many splits (fp32 partial
 * outputs and softmax statistics per (sequence, query head, split)); with
 * num_splits = 0, enough for the default plan of either kind of cache. */
TQ_API size_t tq_decode_workspace_bytes(int B, int H_q, int head_dim, int num_splits);

/* Decode attention over the compressed cache, one query per sequence -- the
 * fused attention over 4-bit keys and values that the TurboQuant kernels run
 * ("TurboQuant 在 AMD GPU 上把長上下文延遲壓下來", summary table and section 2:
 * rotation + LUT keys, uniform values, dequantised inside the attention):
 *   out[b][h] = sum_t softmax_t(scale * <q[b][h], k_hat_t>) * v_hat_t,
 * t < seq_lens[b], with the keys/values the cache holds for kv head
 * h / (H_q / H_kv).  The query is rotated by the same Hadamard transform
 * once, so scores are computed in the rotated domain against the stored
 * centroids; K and V are dequantised in registers and never written out.
 *   q            (device) bf16 [B][H_q][d]; H_q a multiple of H_kv, at most 64 query
 *                heads per kv head (TQ_ERR_UNSUPPORTED otherwise)
 *   block_tables (device) int32 [B][max_blocks]
 *   seq_lens     (device) int32 [B], each in [0, max_blocks*16]
 *   max_seq_len  (host)   upper bound of seq_lens (sizes the split grid); a
 *                         longer seq_len sets TQ_STATUS_BAD_LEN and is cut
 *   out          (device) fp32 [B][H_q][d], 8-byte aligned; a sequence of length 0
 *                gets 0
 *   workspace    (device) >= tq_decode_workspace_bytes(...), 16-byte aligned
 * q, block_tables, seq_lens, k_tables and status must be 4-byte aligned (a
 * pointer that misses its alignment: TQ_ERR_ALIGNMENT, nothing enqueued).
 *   num_splits   0 = tq_decode_default_splits(...), else 1..1024
 * Splits of one sequence are merged by a log-sum-exp combine kernel. */
TQ_API int tq_decode_attention(const void* q, const tq_cache_t* cache, const uint16_t* k_tables,
                        const int32_t* block_tables, int max_blocks, const int32_t* seq_lens,
                        int B, int H_q, int max_seq_len, float scale, float* out,
                        void* workspace, size_t ws_bytes, int num_splits, int32_t* status,
                        void* stream);

/* Decode attention without a caller workspace.  No page describes this call;
 * it exists for callers that cannot allocate device memory at all -- an
 * operator or plugin hosted by another runtime usually receives only the
 * tensors of the call while the host runtime owns (and pools) every other
 * byte of device memory, so it has no way to hand over a workspace.
 * Same arguments, result and checks as tq_decode_attention minus workspace /
 * ws_bytes (those checks run first, with the same error codes); the split
 * partials go to a fixed array compiled into the library
 * (tq_decode_static_scratch_bytes() bytes, 8 MiB, present on every GPU that
 * loads the library until the process exits).  The call allocates and frees
 * nothing.  A split plan whose partials exceed the array is rejected with
 * TQ_ERR_WORKSPACE before anything is enqueued (tq_decode_workspace_bytes
 * bounds a plan's partials from above); pass fewer splits (1 needs none) or
 * use tq_decode_attention.
 * The first call on a device that needs partials looks the array's address
 * up (cudaGetSymbolAddress) and caches it; make that first call before any
 * stream capture.  A device reset (cudaDeviceReset) makes the cached address
 * stale: do not use this call on a device after resetting it.  All calls
 * share the one array and it keeps the last
 * call's contents (nothing in it needs to start at zero): calls that overlap
 * on the GPU -- on different streams, or from different threads -- race on
 * it and must be ordered by the caller. */
TQ_API int tq_decode_attention_static(const void* q, const tq_cache_t* cache,
                                      const uint16_t* k_tables, const int32_t* block_tables,
                                      int max_blocks, const int32_t* seq_lens, int B, int H_q,
                                      int max_seq_len, float scale, float* out, int num_splits,
                                      int32_t* status, void* stream);
/* Size in bytes of the fixed array tq_decode_attention_static uses. */
TQ_API size_t tq_decode_static_scratch_bytes(void);

/* Chunked-prefill attention over the compressed cache: the prompt chunks of
 * multi-turn serving, whose reuse of a cached prefix the pages measure
 * ("TurboQuant 在 AMD GPU 上把長上下文延遲壓下來", summary table: prefix-cache
 * hit rate; "UltraQuant：4-bit KV 快取加速長代理", 「它實際證明了什麼」: late-round
 * TTFT comes from cache residency).  The chunk is appended first
 * (tq_quantize_append), as for the decode: sequence b's chunk is its last
 * q_len = q_start[b+1] - q_start[b] of seq_lens[b] cached tokens, and chunk
 * token i attends to positions 0 .. seq_lens[b] - q_len + i (causal):
 *   out[q_start[b] + i][h] = sum_t softmax_t(scale <q, k_hat_t>) v_hat_t.
 *   q            (device) bf16 [T][H_q][d], 16-byte aligned
 *   block_tables (device) int32 [B][max_blocks]
 *   seq_lens     (device) int32 [B]; seq_lens[b] < q_len or > max_blocks*16 sets
 *                TQ_STATUS_BAD_LEN and that sequence's rows get 0
 *   q_start      (device) int32 [B+1]: chunk b is rows q_start[b] .. q_start[b+1]-1
 *                of q and out; a chunk outside [0, T) sets TQ_STATUS_BAD_LEN and is
 *                skipped (nothing read or written)
 *   T            (host)   rows of q and out
 *   max_q_len    (host)   the largest q_len (sizes the grid); a longer chunk sets
 *                TQ_STATUS_BAD_LEN and only its first max_q_len rows are written
 *   out          (device) fp32 [T][H_q][d], 16-byte aligned
 * Runs on the tcgen05 tensor cores: tiles of 128 (chunk token, query head)
 * rows of one kv head; scores and the output accumulate in tensor memory. */
TQ_API int tq_prefill_attention(const void* q, const tq_cache_t* cache, const uint16_t* k_tables,
                                const int32_t* block_tables, int max_blocks, const int32_t* seq_lens,
                                const int32_t* q_start, int B, int H_q, int T, int max_q_len,
                                float scale, float* out, int32_t* status, void* stream);

/* Dequantise every valid token (checks only; the inverse of the section 2
 * encodings of "TurboQuant 在 AMD GPU 上把長上下文延遲壓下來"): K_hat and V_hat (device) fp32
 * [B][max_len][H_kv][d] in the original (unrotated) domain,
 * k_hat = fp16 norm * H * C[idx] (fp16 norm * C[idx] for a TQ_CACHE_UNROTATED
 * cache),  v_hat = code * scale + zero;
 * rows at or past seq_lens[b] are written as 0.  K_hat and V_hat must be
 * 16-byte aligned, block_tables, seq_lens, k_tables and status 4-byte aligned
 * (else TQ_ERR_ALIGNMENT, nothing enqueued). */
TQ_API int tq_dequantize(const tq_cache_t* cache, const uint16_t* k_tables, const int32_t* block_tables,
                  int max_blocks, const int32_t* seq_lens, int B, int max_len, float* K_hat,
                  float* V_hat, int32_t* status, void* stream);

/* Message of the last failing call on this thread ("" if none). */
TQ_API const char* tq_last_error(void);

#ifdef __cplusplus
}
#endif
#endif
