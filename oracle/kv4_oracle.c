/*
 * kv4_oracle.c -- plain, slow, obviously-correct CPU oracle for the INT4 KV cache.
 *
 * TEST INFRASTRUCTURE ONLY: used by the tests, the smoke check and the benchmark's CPU
 * baseline; never by the product path.  It shares no code with the CUDA library.
 *
 * Build: gcc -O2 -std=c11 -fPIC -shared -ffp-contract=off -fno-fast-math -fopenmp
 * (x86-64 SSE arithmetic, so every float operation below is one IEEE binary32 operation).
 *
 * Sources (page title, section):
 *   [KV4-RL Meth.2]  KV4-RL (ai.info summary), "Methodology in Plain English", paragraph 2:
 *                    one affine INT4 group per token-head vector, FP16 scale and offset applied
 *                    after the dot-product reduction, keys Hadamard-rotated with queries rotated
 *                    to match, packed codes read directly, 4 + 32/128 = 4.25 bits per element.
 *   [KV4-RL Meth.3]  same page, paragraph 3, and "Key Contributions" item 4: INT8 side cache for
 *                    the first s and the most recent w positions; disjoint INT4/INT8 regions
 *                    combined through regional softmax statistics.
 *   [SAW-INT4 s2]    SAW-INT4 (gist.science summary), section 2: token-wise INT4, block-diagonal
 *                    Hadamard rotation in blocks of size h, rotation fused with quantisation.
 *
 * Readings where the pages are silent (each one is a convention of this library):
 *   R1 Hadamard: Sylvester H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]], natural order, not
 *      normalised, on contiguous blocks of h elements; butterfly strides 1, 2, ..., h/2.
 *   R2 keys are stored rotated and unnormalised; the query uses (H q) / h, so the product of
 *      rotated query and rotated key equals q . k.  Values are not rotated.
 *   R3 INT4: zero = fp16 rounded down of min, scale = fp16 rounded up of (max - zero)/15,
 *      code = clamp(rint((x - zero)/scale), 0, 15) in fp32; scale 0 gives all-zero codes; a
 *      non-finite zero or scale (values beyond the fp16 range) gives all-zero codes and is
 *      reported by the append.
 *   R4 INT8: symmetric, scale = fp16 rounded up of max|x|/127, code = clamp(rint(x/scale), +-127);
 *      a non-finite scale is treated as in R3.
 *   R5 routing: every token gets INT4 codes; in addition pos < s goes to sink row pos, and
 *      pos >= s with pos >= lens_after - w goes to ring row s + (pos mod w).
 *   R6 byte layout of pages and of the side cache: see the orc_*_byte functions.
 *   R8 bf16 values (value_format 1, the K-INT4 / V-BF16 precision variant): keys exactly as
 *      above; values are not quantised but stored as bf16 (nearest-even from fp32, the input
 *      itself for bf16 inputs) in the pages and, for sink/recent positions, in the side cache,
 *      beside the INT8 keys.
 *   R7 attention: q head j reads kv head j / (Hq/Hkv); softmax scale 1/sqrt(D); regions are
 *      sinks [0, min(s,L)), INT4 [s, max(s, L-w)), recent [max(s, L-w), L).
 */
#include "kv4_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ fp16 / bf16 */

/* Round a binary32 value to binary16 (IEEE 754-2008, binary16: 1 sign, 5 exponent bits with
 * bias 15, 10 fraction bits, subnormal quantum 2^-24, largest finite 65504).  Every step is
 * exact in double: |x| is split into an integer multiple of the target quantum plus a
 * fraction, and the multiple is rounded according to the mode. */
uint16_t orc_f32_to_f16(float x, int mode) {
  uint32_t u;
  memcpy(&u, &x, 4);
  const uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
  const int neg = sign != 0;
  if ((u & 0x7F800000u) == 0x7F800000u) return (u & 0x007FFFFFu) ? (uint16_t)(sign | 0x7E00u) : (uint16_t)(sign | 0x7C00u);
  const double a = fabs((double)x);
  if (a == 0.0) return sign;
  int e2;
  (void)frexp(a, &e2);              /* a = f * 2^e2 with f in [0.5, 1) */
  int E = e2 - 1;                   /* floor(log2 a)                     */
  if (E < -14) E = -14;             /* subnormals share the quantum 2^-24 */
  const double quantum = ldexp(1.0, E - 10);
  const double t = a / quantum;     /* exact (power-of-two divisor)      */
  double n = floor(t);
  const double frac = t - n;        /* exact                             */
  int up;
  if (mode == ORC_RN)
    up = frac > 0.5 || (frac == 0.5 && fmod(n, 2.0) == 1.0);
  else if (mode == ORC_RD)
    up = neg && frac > 0.0;         /* toward -inf: magnitude grows only for negatives */
  else
    up = !neg && frac > 0.0;        /* toward +inf */
  if (up) n += 1.0;
  const double m = n * quantum;
  if (m > 65504.0) {
    if (mode == ORC_RN) return (uint16_t)(sign | 0x7C00u);
    if (mode == ORC_RD) return neg ? (uint16_t)(sign | 0x7C00u) : (uint16_t)0x7BFFu;
    return neg ? (uint16_t)(sign | 0x7BFFu) : (uint16_t)0x7C00u;
  }
  uint16_t bits;
  if (m < ldexp(1.0, -14)) {
    bits = (uint16_t)n;             /* subnormal: quantum is 2^-24, n < 1024 */
  } else {
    int f2;
    (void)frexp(m, &f2);
    const int Em = f2 - 1;          /* -14 .. 15 */
    const double mant = m / ldexp(1.0, Em - 10) - 1024.0;
    bits = (uint16_t)(((Em + 15) << 10) | (int)mant);
  }
  return (uint16_t)(sign | bits);
}

float orc_f16_to_f32(uint16_t h) {
  const int s = h >> 15, e = (h >> 10) & 31, m = h & 1023;
  double v;
  if (e == 0)
    v = ldexp((double)m, -24);
  else if (e == 31)
    v = m ? NAN : INFINITY;
  else
    v = ldexp((double)(m + 1024), e - 25);
  return (float)(s ? -v : v);
}

float orc_bf16_to_f32(uint16_t b) {
  const uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* Round a binary32 value to bfloat16 (8 exponent bits, 7 fraction bits: the upper half of the
 * binary32 pattern), nearest with ties to even, from the format definition: the dropped 16 bits
 * are compared with half of the kept quantum.  Finite inputs only (the library's precondition). */
uint16_t orc_f32_to_bf16(float x) {
  uint32_t u;
  memcpy(&u, &x, 4);
  const uint32_t hi = u >> 16, lo = u & 0xFFFFu;
  const uint32_t up = lo > 0x8000u || (lo == 0x8000u && (hi & 1u));
  return (uint16_t)(hi + up);
}

static double load_elem(const void* base, int dtype, size_t i) {
  if (dtype == ORC_F32) return (double)((const float*)base)[i];
  if (dtype == ORC_BF16) return (double)orc_bf16_to_f32(((const uint16_t*)base)[i]);
  return (double)orc_f16_to_f32(((const uint16_t*)base)[i]);
}

/* ------------------------------------------------------------------ Hadamard (R1) */

/* [SAW-INT4 s2]: the vector is cut into blocks of h and each block gets a local Hadamard
 * transform.  Stage by stage, pairs (j, j + st) inside a block become (a + b, a - b). */
void orc_fwht_f32(float* x, int D, int h) {
  for (int b0 = 0; b0 < D; b0 += h)
    for (int st = 1; st < h; st <<= 1)
      for (int j = b0; j < b0 + h; ++j)
        if (((j - b0) & st) == 0) {
          const float a = x[j], b = x[j + st];
          x[j] = a + b;
          x[j + st] = a - b;
        }
}

/* Randomised-sign variant (a precision variant of the rotation; signs all zero by default): the
 * sign of dimension d is flipped first, so the stored basis is H diag(s). */
static int orc_sign(const orc_config* c, int d) { return (int)((c->sign_bits[d >> 5] >> (d & 31)) & 1u); }

void orc_rotate_key(const orc_config* c, float* x) {
  for (int e = 0; e < c->head_dim; ++e)
    if (orc_sign(c, e)) x[e] = -x[e];
  orc_fwht_f32(x, c->head_dim, c->hadamard_block);
}

void orc_fwht_f64(double* x, int D, int h) {
  for (int b0 = 0; b0 < D; b0 += h)
    for (int st = 1; st < h; st <<= 1)
      for (int j = b0; j < b0 + h; ++j)
        if (((j - b0) & st) == 0) {
          const double a = x[j], b = x[j + st];
          x[j] = a + b;
          x[j + st] = a - b;
        }
}

/* ------------------------------------------------------------------ quantisers (R3, R4) */

/* [KV4-RL Meth.2]: one affine INT4 group per token-head vector with an FP16 scale and
 * offset; x is reconstructed as zero + scale * code.  Minimum and maximum are taken as
 * values (a zero result is +0). */
int orc_quant_int4(const float* x, int D, uint8_t* codes4, uint16_t* scale, uint16_t* zero) {
  float mn = x[0], mx = x[0];
  for (int i = 1; i < D; ++i) {
    if (x[i] < mn) mn = x[i];
    if (x[i] > mx) mx = x[i];
  }
  mn = mn + 0.0f;
  mx = mx + 0.0f;
  const uint16_t zb = orc_f32_to_f16(mn, ORC_RD);
  const float zf = orc_f16_to_f32(zb);
  const float r = mx - zf;
  const float sq = r / 15.0f;
  const uint16_t sb = orc_f32_to_f16(sq, ORC_RU);
  const float sf = orc_f16_to_f32(sb);
  /* R3 range: a vector whose offset or scale is not a finite fp16 (its values reach beyond the
   * fp16 range) keeps its non-finite parameters and all-zero codes, and is reported. */
  const int out_of_range = !isfinite(zf) || !isfinite(sf);
  for (int i = 0; i < D; ++i) {
    int c = 0;
    if (sf != 0.0f && !out_of_range) {
      const float t = (x[i] - zf) / sf;
      const float rq = rintf(t);    /* default rounding mode: nearest, ties to even */
      c = (int)rq;
      if (c < 0) c = 0;
      if (c > 15) c = 15;
    }
    codes4[i] = (uint8_t)c;
  }
  *scale = sb;
  *zero = zb;
  return out_of_range;
}

/* INT8 side-cache format (R4): the pages name INT8 only; symmetric per vector. */
int orc_quant_int8(const float* x, int D, int8_t* codes8, uint16_t* scale) {
  float a = 0.0f;
  for (int i = 0; i < D; ++i) {
    const float ax = fabsf(x[i]);
    if (ax > a) a = ax;
  }
  const uint16_t sb = orc_f32_to_f16(a / 127.0f, ORC_RU);
  const float sf = orc_f16_to_f32(sb);
  const int out_of_range = !isfinite(sf); /* as for INT4: zero codes, reported */
  for (int i = 0; i < D; ++i) {
    int c = 0;
    if (sf != 0.0f && !out_of_range) {
      c = (int)rintf(x[i] / sf);
      if (c < -127) c = -127;
      if (c > 127) c = 127;
    }
    codes8[i] = (int8_t)c;
  }
  *scale = sb;
  return out_of_range;
}

/* ------------------------------------------------------------------ layout (R6) */
/*
 * Page pool of one layer: pages of P positions; a page holds Hkv head blocks of P*(D+8)
 * bytes; a head block holds P/16 tile blocks of 16*(D+8) bytes, one per 16 positions:
 *   [0, 8D)          K codes in 8 pair-rows of D bytes: pair-row p holds rows p (low nibbles)
 *                    and p + 8 (high nibbles), one byte per element.  In a pair-row, element e
 *                    is in 8-byte group e/8, byte (e%8)/2 for even e and 4 + (e%8)/2 for odd e;
 *                    for D >= 128 the two 16-byte halves of every 32 bytes are swapped in odd
 *                    pair-rows.
 *   [8D, 16D)        V codes in 16-bit chunks: chunk (r, Q) holds elements 4Q..4Q+3 of row r
 *                    (element 4Q+k in byte k/2, low nibble for even k); the chunks of rows
 *                    2p and 2p+1 sit side by side in one 32-bit word, and words are grouped
 *                    so that each reader fetches 4*(D/32) contiguous bytes.
 *   [16D, 16D+64)    K (scale, zero) fp16 pairs, row r at 4r.
 *   [16D+64, 16D+128) V (scale, zero) pairs.
 * Side cache of one layer: max_seqs slots x Hkv heads x ceil((s+w)/16) tile blocks of
 * 16*(2D+4) bytes; side row R lives in tile R/16, row r = R % 16:
 *   [0, 16D)         K int8 codes, row r at r*D, 16-byte unit u stored at unit u ^ (r & 1).
 *   [16D, 16D+32)    K fp16 scales, row r at 2r.
 *   [16D+32, 32D+32) V int8 codes, rows 2p and 2p+1 interleaved byte by byte per pair of
 *                    elements, grouped like the INT4 V codes (16-byte halves swapped for odd
 *                    groups when a group is 32 bytes).
 *   [32D+32, 32D+64) V fp16 scales, row r at 2r.
 *   (so a tile is two equal halves, K then V, of 16D + 32 bytes each)
 * The pages leave the layout free ("token-wise INT4 ... without changing the tensor layout"
 * in [SAW-INT4 s2] refers to the paged buffers, which stay paged here).
 */
/* Bytes of one position of one KV head in a page: INT4 values D/2 + 4 (K codes, V codes, two
 * (scale, zero) pairs); bf16 values (value_format 1) D/2 + 4 + 2D (K codes and parameters, V as
 * bf16).  In the side cache: INT8 values 2D + 4 (K and V codes, two scales); bf16 values 3D + 2
 * (K codes and scale, V as bf16). */
static size_t pos4_bytes(const orc_config* c) {
  const size_t D = (size_t)c->head_dim;
  return c->value_format ? D / 2 + 4 + 2 * D : D + 8;
}

static size_t pos8_bytes(const orc_config* c) {
  const size_t D = (size_t)c->head_dim;
  return c->value_format ? 3 * D + 2 : 2 * D + 4;
}

size_t orc_page_bytes(const orc_config* c) {
  return (size_t)c->num_kv_heads * (size_t)c->page_size * pos4_bytes(c);
}

int orc_side_tiles(const orc_config* c) { return (c->num_sinks + c->recent_window + 15) / 16; }

size_t orc_side_slot_bytes(const orc_config* c) {
  return (size_t)c->num_kv_heads * (size_t)orc_side_tiles(c) * 16u * pos8_bytes(c);
}

static size_t tile4_base(const orc_config* c, int page, int g, int pp) {
  const size_t P = (size_t)c->page_size, pb = pos4_bytes(c);
  return (size_t)page * orc_page_bytes(c) + (size_t)g * P * pb + (size_t)(pp / 16) * 16u * pb;
}

size_t orc_k4_byte(const orc_config* c, int page, int g, int pp, int e) {
  const int D = c->head_dim, pr = (pp % 16) & 7;
  const int b = 8 * (e / 8) + (e % 2) * 4 + (e % 8) / 2;  /* byte within the pair-row */
  const int unit = (b / 16) ^ (D >= 128 ? (pr & 1) : 0);
  return tile4_base(c, page, g, pp) + (size_t)pr * (size_t)D + (size_t)(16 * unit + b % 16);
}

int orc_k4_high(const orc_config* c, int pp, int e) {
  (void)c;
  (void)e;
  return (pp % 16) >> 3;
}

size_t orc_v4_byte(const orc_config* c, int page, int g, int pp, int e) {
  const int D = c->head_dim, r = pp % 16;
  const int Q = e / 4, k = e % 4;
  const int wpc = D / 32, ch = 4 * wpc;
  const int p = r >> 1, half = p >> 2, pl = p & 3;
  const int gq = Q / wpc, j = Q % wpc;
  const size_t off = (size_t)(((half * 8 + gq) * 4 + pl) * ch + 4 * j + 2 * (r & 1) + (k >> 1));
  return tile4_base(c, page, g, pp) + (size_t)(8 * D) + off;
}

size_t orc_p4_byte(const orc_config* c, int page, int g, int pp, int is_v) {
  const int D = c->head_dim, r = pp % 16;
  if (c->value_format) return tile4_base(c, page, g, pp) + (size_t)(8 * D + 4 * r); /* K only */
  return tile4_base(c, page, g, pp) + (size_t)(16 * D + 64 * is_v + 4 * r);
}

/* bf16 values (value_format 1): a 16-row block of V in the order the PV tensor-core fragments
 * read it.  Rows 2p and 2p+1 are a pair; elements are grouped in D/8 groups of D/8; for pair p
 * (half = p / 4) and group gq a chunk of D/2 bytes at ((half*8 + gq)*4 + p%4) * D/2 holds the
 * words (V[2p][e], V[2p+1][e]) for the elements e of the group in order, and the 16-byte units of
 * the chunk are permuted by u -> u ^ swz (swz = (p%4 & 2) | (gq & 1) when a chunk has 4 units,
 * gq & 1 when it has 2, 0 when it has 1). */
static size_t vbf_off(int D, int r, int e) {
  const int p = r >> 1, half = p >> 2, pl = p & 3;
  const int dg = D / 8, gq = e / dg, m = e % dg;
  const int units = D / 32;
  const int swz = units >= 4 ? ((pl & 2) | (gq & 1)) : (units >= 2 ? (gq & 1) : 0);
  const int u = (m * 4) / 16, within = (m * 4) % 16;
  return (size_t)(((half * 8 + gq) * 4 + pl) * (D / 2) + 16 * (u ^ swz) + within + 2 * (r & 1));
}

size_t orc_vb_byte(const orc_config* c, int page, int g, int pp, int e) {
  const int D = c->head_dim;
  return tile4_base(c, page, g, pp) + (size_t)(8 * D + 64) + vbf_off(D, pp % 16, e);
}

static size_t tile8_base(const orc_config* c, int slot, int g, int row) {
  const size_t t8 = 16u * pos8_bytes(c);
  return (size_t)slot * orc_side_slot_bytes(c) + (size_t)g * (size_t)orc_side_tiles(c) * t8 +
         (size_t)(row / 16) * t8;
}

size_t orc_k8_byte(const orc_config* c, int slot, int g, int row, int e) {
  const int D = c->head_dim, r = row % 16;
  return tile8_base(c, slot, g, row) + (size_t)(r * D + 16 * ((e / 16) ^ (r & 1)) + e % 16);
}

size_t orc_v8_byte(const orc_config* c, int slot, int g, int row, int e) {
  const int D = c->head_dim, r = row % 16;
  const int p = r >> 1, half = p >> 2, pl = p & 3;
  const int dg = D / 8, ch8 = D / 4;
  const int gq = e / dg, dd = e % dg;
  int b = (dd / 2) * 4 + (dd % 2) * 2 + (r & 1);
  if (ch8 >= 32) b ^= 16 * (gq & 1);
  return tile8_base(c, slot, g, row) + (size_t)(16 * D + 32 + ((half * 8 + gq) * 4 + pl) * ch8 + b);
}

size_t orc_s8_byte(const orc_config* c, int slot, int g, int row, int is_v) {
  const int D = c->head_dim, r = row % 16;
  return tile8_base(c, slot, g, row) + (size_t)(16 * D + is_v * (16 * D + 32) + 2 * r);
}

size_t orc_vb8_byte(const orc_config* c, int slot, int g, int row, int e) {
  const int D = c->head_dim;
  return tile8_base(c, slot, g, row) + (size_t)(16 * D + 32) + vbf_off(D, row % 16, e);
}

static int config_ok(const orc_config* c) {
  const int D = c->head_dim, h = c->hadamard_block;
  if (c->num_kv_heads <= 0 || c->num_q_heads <= 0 || c->num_q_heads % c->num_kv_heads) return 0;
  if (D <= 0 || D % 32) return 0;
  if (c->page_size <= 0 || c->page_size % 16) return 0;
  if (c->num_sinks < 0 || c->recent_window < 0 || c->max_seqs <= 0) return 0;
  if (h <= 0 || (h & (h - 1)) || D % h) return 0;
  if (c->value_format != 0 && c->value_format != 1) return 0;
  if (c->value_format && c->rotate_values) return 0; /* bf16 values are stored as given */
  return 1;
}

static void put_u16(uint8_t* buf, size_t off, uint16_t v) {
  buf[off] = (uint8_t)(v & 0xFF);
  buf[off + 1] = (uint8_t)(v >> 8);
}

static uint16_t get_u16(const uint8_t* buf, size_t off) {
  return (uint16_t)(buf[off] | (buf[off + 1] << 8));
}

static void put_nibble(uint8_t* buf, size_t off, int high, uint8_t code) {
  if (high)
    buf[off] = (uint8_t)((buf[off] & 0x0F) | (code << 4));
  else
    buf[off] = (uint8_t)((buf[off] & 0xF0) | code);
}

static int get_nibble(const uint8_t* buf, size_t off, int high) {
  return high ? (buf[off] >> 4) : (buf[off] & 0x0F);
}

/* ------------------------------------------------------------------ append */

/* [KV4-RL Meth.2] every new K/V vector is quantised on the fly; [SAW-INT4 s2] the key is
 * rotated (blocks of h) before quantisation; [KV4-RL Meth.3] sink and recent positions also
 * go to the INT8 side cache (R5). */
int orc_append(const orc_config* c, uint8_t* pool, uint8_t* side, int T, const void* K, int k_dtype,
               const void* V, int v_dtype, const int32_t* seq_slot, const int32_t* pos,
               const int32_t* lens_after, const int32_t* page_table, int stride) {
  if (!config_ok(c)) return -1;
  const int D = c->head_dim, Hkv = c->num_kv_heads, P = c->page_size;
  const int s = c->num_sinks, w = c->recent_window;
  float* kf = (float*)malloc(sizeof(float) * (size_t)D);
  float* vf = (float*)malloc(sizeof(float) * (size_t)D);
  uint8_t* c4 = (uint8_t*)malloc((size_t)D);
  int8_t* c8 = (int8_t*)malloc((size_t)D);
  if (!kf || !vf || !c4 || !c8) return -2;
  int range = 0;
  for (int t = 0; t < T; ++t) {
    const int b = seq_slot[t], p = pos[t];
    const int page = page_table[(size_t)b * (size_t)stride + (size_t)(p / P)];
    const int pp = p % P;
    for (int g = 0; g < Hkv; ++g) {
      const size_t in0 = ((size_t)t * (size_t)Hkv + (size_t)g) * (size_t)D;
      for (int e = 0; e < D; ++e) {
        kf[e] = (float)load_elem(K, k_dtype, in0 + (size_t)e);
        vf[e] = (float)load_elem(V, v_dtype, in0 + (size_t)e);
      }
      orc_rotate_key(c, kf);
      if (c->rotate_values) orc_rotate_key(c, vf);
      uint16_t sc, zr;
      range |= orc_quant_int4(kf, D, c4, &sc, &zr);
      for (int e = 0; e < D; ++e) put_nibble(pool, orc_k4_byte(c, page, g, pp, e), orc_k4_high(c, pp, e), c4[e]);
      put_u16(pool, orc_p4_byte(c, page, g, pp, 0), sc);
      put_u16(pool, orc_p4_byte(c, page, g, pp, 0) + 2, zr);
      if (c->value_format) {
        /* bf16 values: the value itself, rounded to bf16 (exact for bf16 inputs) */
        for (int e = 0; e < D; ++e) put_u16(pool, orc_vb_byte(c, page, g, pp, e), orc_f32_to_bf16(vf[e]));
      } else {
        range |= orc_quant_int4(vf, D, c4, &sc, &zr);
        for (int e = 0; e < D; ++e) put_nibble(pool, orc_v4_byte(c, page, g, pp, e), e & 1, c4[e]);
        put_u16(pool, orc_p4_byte(c, page, g, pp, 1), sc);
        put_u16(pool, orc_p4_byte(c, page, g, pp, 1) + 2, zr);
      }

      int row = -1;
      if (p < s)
        row = p;
      else if (w > 0 && p >= lens_after[b] - w)
        row = s + p % w;
      if (row >= 0) {
        uint16_t s8;
        range |= orc_quant_int8(kf, D, c8, &s8);
        for (int e = 0; e < D; ++e) side[orc_k8_byte(c, b, g, row, e)] = (uint8_t)c8[e];
        put_u16(side, orc_s8_byte(c, b, g, row, 0), s8);
        if (c->value_format) {
          for (int e = 0; e < D; ++e) put_u16(side, orc_vb8_byte(c, b, g, row, e), orc_f32_to_bf16(vf[e]));
        } else {
          range |= orc_quant_int8(vf, D, c8, &s8);
          for (int e = 0; e < D; ++e) side[orc_v8_byte(c, b, g, row, e)] = (uint8_t)c8[e];
          put_u16(side, orc_s8_byte(c, b, g, row, 1), s8);
        }
      }
    }
  }
  free(kf);
  free(vf);
  free(c4);
  free(c8);
  return range ? ORC_APPEND_RANGE : 0;
}

/* ------------------------------------------------------------------ dequantise */

int orc_dequant_seq(const orc_config* c, const uint8_t* pool, const uint8_t* side, const int32_t* page_row,
                    int slot, int L, int g, double* khat, double* vhat, int32_t* region) {
  if (!config_ok(c)) return -1;
  const int D = c->head_dim, P = c->page_size, s = c->num_sinks, w = c->recent_window;
  const int s_end = L < s ? L : s;
  const int r_begin = (L - w) > s ? (L - w) : s;
  for (int j = 0; j < L; ++j) {
    double* kr = khat + (size_t)j * (size_t)D;
    double* vr = vhat + (size_t)j * (size_t)D;
    if (j < s_end || j >= r_begin) {
      region[j] = j < s_end ? 0 : 2;
      const int row = j < s ? j : s + j % w;
      const double ks = (double)orc_f16_to_f32(get_u16(side, orc_s8_byte(c, slot, g, row, 0)));
      for (int e = 0; e < D; ++e) kr[e] = ks * (double)(int8_t)side[orc_k8_byte(c, slot, g, row, e)];
      if (c->value_format) {
        for (int e = 0; e < D; ++e) vr[e] = (double)orc_bf16_to_f32(get_u16(side, orc_vb8_byte(c, slot, g, row, e)));
      } else {
        const double vs = (double)orc_f16_to_f32(get_u16(side, orc_s8_byte(c, slot, g, row, 1)));
        for (int e = 0; e < D; ++e) vr[e] = vs * (double)(int8_t)side[orc_v8_byte(c, slot, g, row, e)];
      }
    } else {
      region[j] = 1;
      const int page = page_row[j / P], pp = j % P;
      const size_t kp = orc_p4_byte(c, page, g, pp, 0);
      const double ks = (double)orc_f16_to_f32(get_u16(pool, kp));
      const double kz = (double)orc_f16_to_f32(get_u16(pool, kp + 2));
      for (int e = 0; e < D; ++e)
        kr[e] = kz + ks * (double)get_nibble(pool, orc_k4_byte(c, page, g, pp, e), orc_k4_high(c, pp, e));
      if (c->value_format) {
        for (int e = 0; e < D; ++e) vr[e] = (double)orc_bf16_to_f32(get_u16(pool, orc_vb_byte(c, page, g, pp, e)));
      } else {
        const size_t vp = orc_p4_byte(c, page, g, pp, 1);
        const double vs = (double)orc_f16_to_f32(get_u16(pool, vp));
        const double vz = (double)orc_f16_to_f32(get_u16(pool, vp + 2));
        for (int e = 0; e < D; ++e) vr[e] = vz + vs * (double)get_nibble(pool, orc_v4_byte(c, page, g, pp, e), e & 1);
      }
    }
  }
  return 0;
}

/* ------------------------------------------------------------------ decode attention */

typedef struct {
  double m, l;
  double* o;
} part_stats;

/* softmax statistics of one region [a, b): running max m, sum l, unnormalised o. */
static void region_stats(const double* logit, const double* vhat, int D, int a, int b, part_stats* ps) {
  ps->m = -INFINITY;
  ps->l = 0.0;
  for (int e = 0; e < D; ++e) ps->o[e] = 0.0;
  if (b <= a) return;
  for (int j = a; j < b; ++j)
    if (logit[j] > ps->m) ps->m = logit[j];
  for (int j = a; j < b; ++j) {
    const double p = exp(logit[j] - ps->m);
    ps->l += p;
    for (int e = 0; e < D; ++e) ps->o[e] += p * vhat[(size_t)j * (size_t)D + (size_t)e];
  }
}

/* [KV4-RL Meth.3]: regions attended as disjoint sets, merged with their softmax statistics:
 * m = max m_r, l = sum l_r exp(m_r - m), o = sum o_r exp(m_r - m) / l; empty regions skipped. */
static void merge_parts(const part_stats* parts, int n, int D, double* out, double* lse) {
  double m = -INFINITY;
  for (int i = 0; i < n; ++i)
    if (parts[i].l > 0.0 && parts[i].m > m) m = parts[i].m;
  double l = 0.0;
  for (int e = 0; e < D; ++e) out[e] = 0.0;
  if (m == -INFINITY) {
    *lse = -INFINITY;
    return;
  }
  for (int i = 0; i < n; ++i) {
    if (parts[i].l <= 0.0) continue;
    const double f = exp(parts[i].m - m);
    l += parts[i].l * f;
    for (int e = 0; e < D; ++e) out[e] += parts[i].o[e] * f;
  }
  for (int e = 0; e < D; ++e) out[e] /= l;
  *lse = m + log(l);
}

int orc_decode(const orc_config* c, const uint8_t* pool, const uint8_t* side, int B, const void* q, int q_dtype,
               const int32_t* page_table, int stride, const int32_t* lens, double* out, double* lse, int mode,
               int chunk_tokens, int reverse, int nthreads) {
  if (!config_ok(c)) return -1;
  const int D = c->head_dim, Hq = c->num_q_heads, Hkv = c->num_kv_heads, G = Hq / Hkv;
  const int s = c->num_sinks, w = c->recent_window, h = c->hadamard_block;
  const double tau = 1.0 / sqrt((double)D);
  int err = 0;
  if (nthreads < 1) nthreads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
  for (int bg = 0; bg < B * Hkv; ++bg) {
    const int b = bg / Hkv, g = bg % Hkv;
    const int L = lens[b];
    if (L <= 0) {
      for (int i = 0; i < G; ++i) {
        const size_t qh = (size_t)b * (size_t)Hq + (size_t)(g * G + i);
        for (int e = 0; e < D; ++e) out[qh * (size_t)D + (size_t)e] = 0.0;
        if (lse) lse[qh] = -INFINITY;
      }
      continue;
    }
    double* khat = (double*)malloc(sizeof(double) * (size_t)L * (size_t)D);
    double* vhat = (double*)malloc(sizeof(double) * (size_t)L * (size_t)D);
    int32_t* region = (int32_t*)malloc(sizeof(int32_t) * (size_t)L);
    double* logit = (double*)malloc(sizeof(double) * (size_t)L);
    double* qr = (double*)malloc(sizeof(double) * (size_t)D);
    const int max_parts = 3 + (chunk_tokens > 0 ? L / chunk_tokens + 1 : 1);
    part_stats* parts = (part_stats*)malloc(sizeof(part_stats) * (size_t)max_parts);
    double* pbuf = (double*)malloc(sizeof(double) * (size_t)max_parts * (size_t)D);
    if (!khat || !vhat || !region || !logit || !qr || !parts || !pbuf) {
#pragma omp atomic write
      err = -2;
    } else {
      orc_dequant_seq(c, pool, side, page_table + (size_t)b * (size_t)stride, b, L, g, khat, vhat, region);
      for (int i = 0; i < G; ++i) {
        const size_t qh = (size_t)b * (size_t)Hq + (size_t)(g * G + i);
        /* [KV4-RL Meth.2] queries rotated to match the stored key basis: (H q) / h. */
        for (int e = 0; e < D; ++e) qr[e] = load_elem(q, q_dtype, qh * (size_t)D + (size_t)e);
        for (int e = 0; e < D; ++e)
          if (orc_sign(c, e)) qr[e] = -qr[e];
        orc_fwht_f64(qr, D, h);
        for (int e = 0; e < D; ++e) qr[e] *= 1.0 / (double)h;
        for (int j = 0; j < L; ++j) {
          double acc = 0.0;
          for (int e = 0; e < D; ++e) acc += qr[e] * khat[(size_t)j * (size_t)D + (size_t)e];
          logit[j] = tau * acc;
        }
        double* o = out + qh * (size_t)D;
        double lse_v;
        for (int k = 0; k < max_parts; ++k) parts[k].o = pbuf + (size_t)k * (size_t)D;
        int np = 0;
        if (mode == ORC_SINGLE) {
          region_stats(logit, vhat, D, 0, L, &parts[np++]);
        } else {
          const int s_end = L < s ? L : s;
          const int m_begin = s, m_end = (L - w) > s ? (L - w) : s;
          region_stats(logit, vhat, D, 0, s_end, &parts[np++]);
          if (m_end > m_begin) {
            const int ct = chunk_tokens > 0 ? chunk_tokens : (m_end - m_begin);
            const int nchunks = (m_end - m_begin + ct - 1) / ct;
            for (int k = 0; k < nchunks; ++k) {
              const int kk = reverse ? nchunks - 1 - k : k;
              const int a = m_begin + kk * ct;
              const int z = a + ct < m_end ? a + ct : m_end;
              region_stats(logit, vhat, D, a, z, &parts[np++]);
            }
          }
          region_stats(logit, vhat, D, m_end > s_end ? m_end : s_end, L, &parts[np++]);
        }
        merge_parts(parts, np, D, o, &lse_v);
        if (c->rotate_values) {
          /* the values were stored as H diag(s) v: back to the original basis, diag(s) H o / h */
          orc_fwht_f64(o, D, h);
          for (int e = 0; e < D; ++e) o[e] = (orc_sign(c, e) ? -o[e] : o[e]) / (double)h;
        }
        if (lse) lse[qh] = lse_v;
      }
    }
    free(khat);
    free(vhat);
    free(region);
    free(logit);
    free(qr);
    free(parts);
    free(pbuf);
  }
  return err;
}
