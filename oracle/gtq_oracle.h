/*
 * gtq_oracle.h -- plain CPU oracle for the mixed bit-width key cache (RoPE-aware block bit
 * allocation) and its decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link or call this code;
 * only the tests, the smoke check and the benchmark's CPU-baseline leg do.  It shares no
 * header, helper, table or constant with the CUDA library.
 *
 * Source: "RoPE-Aware Bit Allocation for KV-Cache Quantization" (searcharxiv abstract).  Under
 * RoPE a key's contribution to a later attention logit is a position-dependent sum over its
 * two-dimensional frequency blocks, so key quantisation becomes a per-block bit-allocation
 * problem: blocks of high energy are the sensitive ones and get more bits.  For every layer
 * and KV head a label-free energy score is computed per RoPE block and integer bit widths are
 * handed out greedily by marginal gain, under a fixed K bit budget; the cache is stored packed
 * (the abstract's K3V3 serving path).
 *
 * Readings where the abstract is silent (each one is a convention of this library):
 *   G1 RoPE blocks: the rotate-half pairing of the Qwen and Llama models, block b of a head of
 *      dimension D is the coordinate pair (b, b + D/2), b in [0, D/2).
 *   G2 energy score of block b of KV head g: the sum over the scored keys of
 *      k[b]^2 + k[b + D/2]^2, in fp64, keys in order (label-free: keys only, no queries or
 *      labels).  The same score gives the block's scale sigma_b = sqrt(E_b / (2 T)) rounded to
 *      fp32 (the root mean square of one coordinate of the block over the T scored keys; 1 when
 *      E_b = 0), so that a block's quantisation error scales with its energy.
 *   G3 marginal gain: the distortion of a block at w bits is modelled as E * 4^-w (the error of
 *      a w-bit scalar quantiser on a coordinate of energy E, up to a common constant), so one
 *      more bit gains (3/4) E 4^-w.  Greedy: starting from 0 bits everywhere, give one bit at a
 *      time to the block of largest E 4^-w among blocks below 8 bits, ties to the lowest block
 *      index, until the blocks hold key_bits * D / 2 bits (both coordinates of a block share
 *      its width, so the budget is exactly key_bits bits per dimension).
 *   G4 key quantiser (the abstract's TQ-MSE codebook is not given): every coordinate is
 *      standardised by its block's scale, the token gets one fp16 scale
 *      s = rounded up of max |x_j| / sigma_j over its coded coordinates (width >= 1), and a
 *      coordinate of width w gets the mid-rise uniform code of t = x_j / (sigma_j s) on
 *      [-1, 1]: code = clamp(floor((t + 1) 2^(w-1)), 0, 2^w - 1), every step one fp32 operation;
 *      it is reconstructed as s sigma_j ((2 code + 1) 2^-w - 1).  A coordinate of width 0
 *      stores nothing and is reconstructed as 0.  A non-finite s gives all-zero codes and is
 *      reported.
 *   G5 value quantiser: the per-token affine form of the INT4 cache at value_bits bits: zero =
 *      fp16 rounded down of the min, range = fp16 rounded up of (max - zero) (fp32 subtraction),
 *      code = clamp(rint((x - zero) / (range / (2^b - 1))), 0, 2^b - 1), reconstructed as
 *      zero + code * range / (2^b - 1); a zero range gives all-zero codes; a non-finite zero or
 *      range gives all-zero codes and is reported.
 *   G6 packing: the codes of one vector in coordinate order, each in its width, least
 *      significant bit first, as one little-endian bit stream (bit n of the stream is bit n & 7
 *      of byte n >> 3): key_bits * D / 8 bytes per key, value_bits * D / 8 per value.
 *   G7 page tile of one (page, KV head), P positions (P a multiple of 16): P/16 slices of 16
 *      positions, each holding its 16 key rows, then its 16 value rows, then 16 parameter records
 *      of four fp16 (key scale, a zero pad, value zero, value range); tiles ordered (page, head).
 *      A slice is one contiguous block whatever P is.  No rotation, no side cache: the
 *      abstract's method needs neither.
 *   G8 attention: as for the INT4 cache, q head j reads KV head j / (Hq/Hkv), softmax scale
 *      1/sqrt(D), one softmax over [0, L), in fp64 on the dequantised cache.
 */
#ifndef GTQ_ORACLE_H
#define GTQ_ORACLE_H
#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
  int num_q_heads;   /* Hq                                   */
  int num_kv_heads;  /* Hkv, Hq % Hkv == 0                   */
  int head_dim;      /* D, even, D * key_bits % 8 == 0 ...   */
  int page_size;     /* P, a multiple of 16                  */
  int key_bits;      /* average key bits per dimension, 1..8 */
  int value_bits;    /* value bits per dimension, 1..8       */
} orc_gtq_config;

/* G2: energy[g][b] for K [T][Hkv][D] of element type k_dtype (ORC_F32 / ORC_BF16 / ORC_F16). */
void orc_gtq_energy(int T, int Hkv, int D, const void* K, int k_dtype, double* energy);

/* G2: block scales sigma[b] of nblocks blocks scored over T keys. */
void orc_gtq_scales(const double* energy, int nblocks, int T, float* sigma);

/* G3: greedy widths of nblocks blocks under key_bits per dimension.  Returns 0, or -1 when the
 * budget exceeds 8 bits per dimension. */
int orc_gtq_allocate(const double* energy, int nblocks, int key_bits, uint8_t* widths);

/* The model distortion sum_b E_b 4^-w_b of an allocation (the greedy's objective). */
double orc_gtq_objective(const double* energy, int nblocks, const uint8_t* widths);

/* G4: quantise one key with per-coordinate widths wc[D] and scales sc[D].  Returns 1 when the
 * token scale is not a finite fp16 (codes all zero), else 0. */
int orc_gtq_quant_key(const float* x, int D, const uint8_t* wc, const float* sc, uint8_t* codes, uint16_t* scale);
double orc_gtq_dequant_key(uint16_t scale, float sigma, int w, int code);

/* G5: quantise one value at bits bits per coordinate; same return convention. */
int orc_gtq_quant_value(const float* x, int D, int bits, uint8_t* codes, uint16_t* zero, uint16_t* range);
double orc_gtq_dequant_value(uint16_t zero, uint16_t range, int bits, int code);

/* G6: pack / unpack D codes of widths wc into / from a bit stream of sum(wc) bits. */
void orc_gtq_pack(const uint8_t* codes, const uint8_t* wc, int D, uint8_t* row);
void orc_gtq_unpack(const uint8_t* row, const uint8_t* wc, int D, uint8_t* codes);

/* G7: sizes and byte offsets. */
size_t orc_gtq_key_row_bytes(const orc_gtq_config* c);
size_t orc_gtq_value_row_bytes(const orc_gtq_config* c);
size_t orc_gtq_tile_bytes(const orc_gtq_config* c);
size_t orc_gtq_page_bytes(const orc_gtq_config* c);
size_t orc_gtq_key_row(const orc_gtq_config* c, int page, int g, int pp);
size_t orc_gtq_value_row(const orc_gtq_config* c, int page, int g, int pp);
size_t orc_gtq_param(const orc_gtq_config* c, int page, int g, int pp);

/* Append T tokens (K, V [T][Hkv][D]) into a host copy of one layer's page pool, with the layer's
 * block widths widths[Hkv][D/2] and block scales sigma[Hkv][D/2].  Returns 0, 1 when some vector
 * was out of the fp16 range (stored with zero codes), or a negative error code. */
int orc_gtq_append(const orc_gtq_config* c, const uint8_t* widths, const float* sigma, uint8_t* pool, int T, const void* K,
                   int k_dtype, const void* V, int v_dtype, const int32_t* seq_slot, const int32_t* pos,
                   const int32_t* page_table, int stride);

/* Dense fp64 dequantised keys / values [L][D] of one (sequence row, KV head g). */
int orc_gtq_dequant_seq(const orc_gtq_config* c, const uint8_t* widths, const float* sigma, const uint8_t* pool,
                        const int32_t* page_row, int L, int g, double* khat, double* vhat);

/* G8: decode attention of B sequences; out [B][Hq][D], lse [B][Hq] (natural log). */
int orc_gtq_decode(const orc_gtq_config* c, const uint8_t* widths, const float* sigma, const uint8_t* pool, int B, const void* q,
                   int q_dtype, const int32_t* page_table, int stride, const int32_t* lens, double* out,
                   double* lse, int nthreads);

#ifdef __cplusplus
}
#endif
#endif
