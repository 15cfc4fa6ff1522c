/*
 * kv4_oracle.h -- plain CPU oracle for the INT4 KV cache (append + decode attention).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link or call
 * this code; only the tests, the smoke check and the benchmark's CPU-baseline leg do.
 * It shares no header, helper, table or constant with the CUDA library.
 *
 * What it computes follows the method pages:
 *   - KV4-RL (ai.info summary), "Methodology in Plain English" para. 2: one affine INT4 group
 *     per token-head vector with an FP16 scale and offset, keys stored in a Hadamard-rotated
 *     basis and queries rotated to match, 4 + 32/128 = 4.25 bits per element.
 *   - KV4-RL, "Key Contributions" item 4 and "Methodology" para. 3: an INT8 side cache for the
 *     first s (sink) and last w (recent) positions, attended as disjoint regions and merged
 *     with per-region softmax statistics.
 *   - SAW-INT4 (gist.science summary), section 2: token-wise INT4 and a block-diagonal
 *     Hadamard rotation with block size h, fused with quantisation.
 * Where the pages are silent (rounding modes, nibble order, INT8 format, byte layout),
 * the reading used here is stated beside each function.
 *
 * Precision: append is an encoding, restated step by step in fp32 with exactly the
 * operations listed (compile with -ffp-contract=off, SSE arithmetic).  Decode attention is
 * computed in fp64 on the dequantised cache.
 */
#ifndef KV4_ORACLE_H
#define KV4_ORACLE_H
#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { ORC_RN = 0, ORC_RD = 1, ORC_RU = 2 };          /* fp16 rounding modes   */
enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_F16 = 2 };       /* input element types   */
enum { ORC_REGIONAL = 0, ORC_SINGLE = 1 };             /* decode evaluation mode */

typedef struct {
  int num_q_heads;     /* Hq                                           */
  int num_kv_heads;    /* Hkv, Hq % Hkv == 0                           */
  int head_dim;        /* D, multiple of 32                            */
  int page_size;       /* P, multiple of 16                            */
  int num_sinks;       /* s                                            */
  int recent_window;   /* w                                            */
  int hadamard_block;  /* h, power of two dividing D (1 = no rotation) */
  int max_seqs;        /* rows of the INT8 side cache                  */
  uint32_t sign_bits[4]; /* randomised-sign rotation: bit d (word d / 32) negates dim d of the
                            key and of the query before the Hadamard; all zero = plain H    */
  int rotate_values;     /* values stored rotated like the keys (H diag(s)); outputs rotated
                            back as diag(s) H o / h                                          */
  int value_format;      /* 0: INT4 values (INT8 in the side cache); 1: values stored as bf16 in
                            the pages and the side cache (keys as in format 0); with 1,
                            rotate_values must be 0                                          */
} orc_config;

/* fp16 helpers (IEEE binary16), written from the format definition. */
uint16_t orc_f32_to_f16(float x, int mode);
float    orc_f16_to_f32(uint16_t h);
float    orc_bf16_to_f32(uint16_t b);
uint16_t orc_f32_to_bf16(float x);  /* nearest, ties to even */

/* Block-diagonal Sylvester Hadamard, unnormalised, fp32 butterfly in ascending stride order. */
void orc_fwht_f32(float* x, int D, int h);
/* Same transform in fp64 (used for the query rotation). */
void orc_fwht_f64(double* x, int D, int h);
/* The key rotation of the append: H diag(s) x, the configured signs, then orc_fwht_f32 (also the
 * value rotation when rotate_values is set). */
void orc_rotate_key(const orc_config* c, float* x);

/* Per-vector quantisers.  codes4 holds one code (0..15) per element, unpacked.  Both return 1
 * when a parameter is not a finite fp16 (the codes are then all zero), else 0. */
int orc_quant_int4(const float* x, int D, uint8_t* codes4, uint16_t* scale, uint16_t* zero);
int orc_quant_int8(const float* x, int D, int8_t* codes8, uint16_t* scale);

/* Storage sizes. */
size_t orc_page_bytes(const orc_config* c);          /* one page, all KV heads             */
size_t orc_side_slot_bytes(const orc_config* c);     /* one sequence slot, all KV heads    */
int    orc_side_tiles(const orc_config* c);          /* 16-row tiles per (slot, head)      */

/* Byte offsets inside one layer's page pool / side cache (exposed for the layout pins). */
size_t orc_k4_byte(const orc_config* c, int page, int g, int pos_in_page, int elem);
/* 1 when element elem of the K codes at pos_in_page is the high nibble of its byte (rows 8-15
 * of a tile), else 0.  V codes: the high nibble holds the odd elements (elem & 1). */
int    orc_k4_high(const orc_config* c, int pos_in_page, int elem);
size_t orc_v4_byte(const orc_config* c, int page, int g, int pos_in_page, int elem);
size_t orc_p4_byte(const orc_config* c, int page, int g, int pos_in_page, int is_v);
size_t orc_k8_byte(const orc_config* c, int slot, int g, int row, int elem);
size_t orc_v8_byte(const orc_config* c, int slot, int g, int row, int elem);
size_t orc_s8_byte(const orc_config* c, int slot, int g, int row, int is_v);
/* value_format 1: byte of the bf16 value element elem (2 bytes, little-endian) in a page tile /
 * in a side-cache row.  orc_p4_byte then names the K parameters only (is_v ignored). */
size_t orc_vb_byte(const orc_config* c, int page, int g, int pos_in_page, int elem);
size_t orc_vb8_byte(const orc_config* c, int slot, int g, int row, int elem);

/* Append T tokens (K, V [T][Hkv][D], element type k_dtype / v_dtype) into host copies of
 * one layer's page pool and side cache.  Returns 0, ORC_APPEND_RANGE when some vector's fp16
 * scale or offset was not finite (stored with zero codes), or a negative error code. */
enum { ORC_APPEND_RANGE = 1 };
int orc_append(const orc_config* c, uint8_t* pool, uint8_t* side, int T,
               const void* K, int k_dtype, const void* V, int v_dtype,
               const int32_t* seq_slot, const int32_t* pos, const int32_t* lens_after,
               const int32_t* page_table, int stride);

/* Dense fp64 dequantised cache of one (sequence b, kv head g), logical order [0, L):
 * khat/vhat [L][D] (keys in the rotated basis), region[L] = 0 sink, 1 INT4, 2 recent. */
int orc_dequant_seq(const orc_config* c, const uint8_t* pool, const uint8_t* side,
                    const int32_t* page_row, int slot, int L, int g,
                    double* khat, double* vhat, int32_t* region);

/* Decode attention for B sequences (row b of the batch is slot b).
 * q [B][Hq][D] of type q_dtype; out [B][Hq][D] fp64; lse [B][Hq] fp64 (natural log).
 * mode ORC_REGIONAL: per-region (m, l, o) merged; the INT4 region is further cut into
 *   chunks of chunk_tokens positions (0 = one chunk) visited in reverse order when
 *   reverse != 0 (split-invariance pins).  mode ORC_SINGLE: one softmax over [0, L).
 * nthreads > 1 runs independent (b, kv head) pairs on OpenMP threads. */
int orc_decode(const orc_config* c, const uint8_t* pool, const uint8_t* side, int B,
               const void* q, int q_dtype, const int32_t* page_table, int stride,
               const int32_t* lens, double* out, double* lse, int mode, int chunk_tokens,
               int reverse, int nthreads);

#ifdef __cplusplus
}
#endif
#endif
