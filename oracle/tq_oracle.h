/*
 * tq_oracle.h -- plain, slow, fp64 CPU oracle for TQ4/4 KV-cache compression
 * and attention over the compressed cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, includes
 * or calls this code; only the tests, the smoke check and the CPU-baseline
 * leg of the benchmark do.  It shares no source with the CUDA path.
 *
 * What it follows:
 *   - "TurboQuant 在 AMD GPU 上把長上下文延遲壓下來", section 2 (TQ4/4: keys
 *     get a rotation followed by a look-up-table quantiser, values get plain
 *     uniform quantisation) and section 4 (the rotation is a Walsh-Hadamard
 *     transform rather than a dense random one).
 *   - "UltraQuant：4-bit KV 快取加速長代理", section 「方法怎麼做，白話講」
 *     (Walsh-Hadamard rotation, no QJL stage, keys and values treated
 *     asymmetrically, a 16-entry centroid table that is the theoretical
 *     Lloyd-Max one or is re-fitted on about 20 rotated vectors).
 *   The record format (fp16 key norm, group-of-32 value scale/zero, 16-token
 *   blocks) is the TQ4/4 cache format this repository defines; it is written
 *   out field by field in tq_oracle.c.
 *
 * Conventions: all floating point is IEEE binary64 unless a field is stored
 * as fp16/fp32 by the format.  bf16/fp16 values are passed as their raw
 * uint16 bit patterns.  Every function returns 0 on success and a negative
 * number on a bad argument.
 */
#ifndef TQ_ORACLE_H
#define TQ_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define ORC_BLOCK 16     /* tokens per cache block */
#define ORC_VGROUP 32    /* value elements per scale/zero group */

/* scalar conversions */
double orc_bf16_to_double(uint16_t bits);
double orc_fp16_to_double(uint16_t bits);
/* mode: 0 = round to nearest, ties to even; -1 = toward -inf; +1 = toward +inf */
uint16_t orc_fp16_from_double(double x, int mode);
float orc_fp32_from_double(double x); /* round to nearest even */

/* Lloyd-Max 16-level quantiser of the standard normal N(0,1). */
int orc_lloyd_max_gaussian16(double c[16], double tol, int max_iter, int *iters_used);
/* Default key table for head_dim d: fp16(c_j / sqrt(d)) bit patterns, ascending.
 * Every key table is 16 fp16 values (bit patterns), strictly ascending. */
int orc_default_table(int d, uint16_t out[16]);

/* Dense normalised Sylvester Hadamard matrix, H[i*d+j] = (-1)^popcount(i&j)/sqrt(d). */
int orc_hadamard(int d, double *H);

/* Key encode: n = ||k||, u = k/n, y = H u, idx_i = argmin_c |y_i - C[c]| (ties: lower c).
 * y_out (may be NULL) receives the rotated unit coordinates. */
int orc_encode_k(const uint16_t *k_bf16, int d, const uint16_t *table, uint8_t *idx,
                 uint16_t *norm16, double *y_out);
/* Key decode to the original domain: k_hat = fp16(n) * H * C[idx]. */
int orc_decode_k(const uint8_t *idx, uint16_t norm16, int d, const uint16_t *table, double *k_hat);

/* The same without the rotation (the baseline an unrotated cache holds):
 * y_i = k_i / n, idx_i = argmin_c |y_i - C[c]|;  k_hat = fp16(n) * C[idx]. */
int orc_encode_k_unrotated(const uint16_t *k_bf16, int d, const uint16_t *table, uint8_t *idx,
                           uint16_t *norm16, double *y_out);
int orc_decode_k_unrotated(const uint8_t *idx, uint16_t norm16, int d, const uint16_t *table,
                           double *k_hat);

/* Value encode per group of 32: z = fp16 down(min), s = fp16 up((max - z)/15),
 * q = clamp(round_half_even((v - z)/s), 0, 15) (q = 0 when s = 0).
 * r_out (may be NULL) receives (v - z)/s in fp64 (0 when s = 0). */
int orc_encode_v(const uint16_t *v_bf16, int d, uint8_t *q, uint16_t *scale16,
                 uint16_t *zero16, double *r_out);
int orc_decode_v(const uint8_t *q, const uint16_t *scale16, const uint16_t *zero16, int d,
                 double *v_hat);

/* Record format of one (block, kv-head) entry of the paged cache. */
size_t orc_record_bytes(int d);
int orc_pack_token(uint8_t *record, int d, int offset, const uint8_t *kidx, uint16_t knorm,
                   const uint8_t *vq, const uint16_t *vscale, const uint16_t *vzero);
int orc_unpack_token(const uint8_t *record, int d, int offset, uint8_t *kidx, uint16_t *knorm,
                     uint8_t *vq, uint16_t *vscale, uint16_t *vzero);

/* Quantise-append T tokens (K, V bf16 [T][Hkv][d]) into the cache
 * (uint8 [num_blocks][Hkv][record]).
 *   block_table == NULL: slots[t] is a physical slot (block*16 + offset), -1 skips.
 *   block_table != NULL ([num_seqs][max_blocks]): slots[t] is a logical slot
 *     seq*(max_blocks*16) + position, mapped through the table; -1 skips.
 * tables: NULL = default table for every head, else [Hkv][16] fp16 bits.
 * ky/vr (may be NULL): [T][Hkv][d] rotated unit key coordinates and (v-z)/s. */
int orc_quantize_append(const uint16_t *K, const uint16_t *V, int T, int Hkv, int d,
                        const int32_t *block_table, int num_seqs, int max_blocks,
                        const int32_t *slots, const uint16_t *tables, uint8_t *cache,
                        int num_blocks, double *ky, double *vr);
/* rotate = 0: keys by orc_encode_k_unrotated (an unrotated cache); 1: as above. */
int orc_quantize_append_ex(const uint16_t *K, const uint16_t *V, int T, int Hkv, int d,
                           const int32_t *block_table, int num_seqs, int max_blocks,
                           const int32_t *slots, const uint16_t *tables, uint8_t *cache,
                           int num_blocks, double *ky, double *vr, int rotate);

/* Gather + dequantise every valid token of every sequence into
 * Khat, Vhat fp64 [B][max_len][Hkv][d] (original domain); rows past seq_len are 0. */
int orc_dequantize(const uint8_t *cache, int num_blocks, int Hkv, int d, const uint16_t *tables,
                   const int32_t *block_tables, int max_blocks, const int32_t *seq_lens, int B,
                   int max_len, double *Khat, double *Vhat);
/* rotate = 0: keys by orc_decode_k_unrotated. */
int orc_dequantize_ex(const uint8_t *cache, int num_blocks, int Hkv, int d, const uint16_t *tables,
                      const int32_t *block_tables, int max_blocks, const int32_t *seq_lens, int B,
                      int max_len, double *Khat, double *Vhat, int rotate);

/* Exact softmax attention in fp64 over dequantised K/V.
 * q bf16 [B][Hq][d]; query head h reads kv head h / (Hq/Hkv); out fp64 [B][Hq][d]. */
int orc_attention(const uint16_t *q, int B, int Hq, int Hkv, int d, const double *Khat,
                  const double *Vhat, int max_len, const int32_t *seq_lens, double scale,
                  double *out);

/* Chunked-prefill attention over dequantised K/V: the last q_len = q_start[b+1] -
 * q_start[b] of sequence b's seq_lens[b] cached tokens are the chunk, and chunk
 * token i attends to positions 0 .. seq_lens[b] - q_len + i (causal within the
 * chunk).  q bf16 [q_start[B]][Hq][d]; out fp64 [q_start[B]][Hq][d]. */
int orc_prefill_attention(const uint16_t *q, const int32_t *q_start, int B, int Hq, int Hkv, int d,
                          const double *Khat, const double *Vhat, int max_len,
                          const int32_t *seq_lens, double scale, double *out);

/* 1-D k-means (Lloyd) refit of a 16-entry table on n scalar samples, starting
 * from init; empty clusters keep their centroid; the result is sorted and
 * rounded to fp16.  Returns the number of iterations run (>= 0). */
int orc_kmeans_table(const double *samples, int n, const uint16_t *init, int max_iter, uint16_t out[16]);
/* The calibration samples of one head: unit-normalised, rotated key vectors. */
int orc_rotated_unit_samples(const uint16_t *k_bf16, int n_vec, int d, double *out);

#ifdef __cplusplus
}
#endif
#endif
