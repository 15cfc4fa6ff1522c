/*
 * gtq_oracle.c -- plain, slow, obviously-correct CPU oracle for the mixed bit-width key cache.
 *
 * TEST INFRASTRUCTURE ONLY: used by the tests, the smoke check and the benchmark's CPU
 * baseline; never by the product path.  It shares no code with the CUDA library.  It is
 * compiled into the same library as kv4_oracle.c and uses that file's fp16 helpers.
 *
 * Source: "RoPE-Aware Bit Allocation for KV-Cache Quantization" (searcharxiv abstract): a
 * label-free energy score per RoPE block of every (layer, KV head), integer bit widths handed
 * out greedily by marginal gain under the K budget, a packed cache.  The readings G1-G8 where
 * the abstract is silent are listed in gtq_oracle.h.
 *
 * Precision: the energy score is an fp64 sum in key order; the allocation compares fp64 values
 * scaled by exact powers of four; the quantiser is restated in fp32, one IEEE operation per
 * step (compile with -ffp-contract=off, SSE arithmetic); attention is fp64.
 */
#include "gtq_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#include "kv4_oracle.h"

static double gtq_load(const void* base, int dtype, size_t i) {
  if (dtype == ORC_F32) return (double)((const float*)base)[i];
  if (dtype == ORC_BF16) return (double)orc_bf16_to_f32(((const uint16_t*)base)[i]);
  return (double)orc_f16_to_f32(((const uint16_t*)base)[i]);
}

/* ------------------------------------------------------------------ energy and allocation */

/* G1 + G2: block b is the pair (b, b + D/2); its score is the sum of the squared pair norms. */
void orc_gtq_energy(int T, int Hkv, int D, const void* K, int k_dtype, double* energy) {
  const int nb = D / 2;
  for (int g = 0; g < Hkv; ++g)
    for (int b = 0; b < nb; ++b) {
      double e = 0.0;
      for (int t = 0; t < T; ++t) {
        const size_t row = ((size_t)t * (size_t)Hkv + (size_t)g) * (size_t)D;
        const double x0 = gtq_load(K, k_dtype, row + (size_t)b);
        const double x1 = gtq_load(K, k_dtype, row + (size_t)(b + nb));
        e = e + (x0 * x0 + x1 * x1);
      }
      energy[(size_t)g * (size_t)nb + (size_t)b] = e;
    }
}

/* G2: the root mean square of one coordinate of the block over the T scored keys. */
void orc_gtq_scales(const double* energy, int nblocks, int T, float* sigma) {
  for (int b = 0; b < nblocks; ++b)
    sigma[b] = (energy[b] > 0.0 && T > 0) ? (float)sqrt(energy[b] / (2.0 * (double)T)) : 1.0f;
}

/* G3: one bit at a time to the block whose next bit removes the most modelled distortion. */
int orc_gtq_allocate(const double* energy, int nblocks, int key_bits, uint8_t* widths) {
  if (key_bits < 0 || key_bits > 8) return -1;
  for (int b = 0; b < nblocks; ++b) widths[b] = 0;
  const int steps = key_bits * nblocks;
  for (int s = 0; s < steps; ++s) {
    int best = -1;
    double best_gain = 0.0;
    for (int b = 0; b < nblocks; ++b) {
      if (widths[b] >= 8) continue;
      const double gain = ldexp(energy[b], -2 * (int)widths[b]); /* E * 4^-w, exact */
      if (best < 0 || gain > best_gain) {
        best = b;
        best_gain = gain;
      }
    }
    widths[best] += 1;
  }
  return 0;
}

double orc_gtq_objective(const double* energy, int nblocks, const uint8_t* widths) {
  double d = 0.0;
  for (int b = 0; b < nblocks; ++b) d += ldexp(energy[b], -2 * (int)widths[b]);
  return d;
}

/* ------------------------------------------------------------------ quantisers (G4, G5) */

int orc_gtq_quant_key(const float* x, int D, const uint8_t* wc, const float* sc, uint8_t* codes, uint16_t* scale) {
  float m = 0.0f;
  for (int i = 0; i < D; ++i)
    if (wc[i] > 0) {
      const float a = fabsf(x[i]) / sc[i];
      if (a > m) m = a;
    }
  const uint16_t sb = orc_f32_to_f16(m, ORC_RU);
  const float sf = orc_f16_to_f32(sb);
  const int out_of_range = !isfinite(sf);
  for (int i = 0; i < D; ++i) {
    int c = 0;
    const int w = wc[i];
    if (w > 0 && sf != 0.0f && !out_of_range) {
      const int top = (1 << w) - 1;
      const float d = sc[i] * sf;
      const float t = x[i] / d;
      const float u = (t + 1.0f) * (float)(1 << (w - 1)); /* exact power-of-two product */
      const float f = floorf(u);
      c = f < 0.0f ? 0 : (f > (float)top ? top : (int)f);
    }
    codes[i] = (uint8_t)c;
  }
  *scale = sb;
  return out_of_range;
}

double orc_gtq_dequant_key(uint16_t scale, float sigma, int w, int code) {
  if (w == 0) return 0.0;
  const double s = (double)orc_f16_to_f32(scale);
  return s * (double)sigma * (ldexp(2.0 * code + 1.0, -w) - 1.0);
}

int orc_gtq_quant_value(const float* x, int D, int bits, uint8_t* codes, uint16_t* zero, uint16_t* range) {
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
  const uint16_t rb = orc_f32_to_f16(r, ORC_RU);
  const float rf = orc_f16_to_f32(rb);
  const int out_of_range = !isfinite(zf) || !isfinite(rf);
  const int top = (1 << bits) - 1;
  for (int i = 0; i < D; ++i) {
    int c = 0;
    if (rf != 0.0f && !out_of_range) {
      const float step = rf / (float)top;
      const float t = (x[i] - zf) / step;
      const float rq = rintf(t); /* nearest, ties to even */
      c = rq < 0.0f ? 0 : (rq > (float)top ? top : (int)rq);
    }
    codes[i] = (uint8_t)c;
  }
  *zero = zb;
  *range = rb;
  return out_of_range;
}

double orc_gtq_dequant_value(uint16_t zero, uint16_t range, int bits, int code) {
  const double z = (double)orc_f16_to_f32(zero), r = (double)orc_f16_to_f32(range);
  return z + (double)code * (r / (double)((1 << bits) - 1));
}

/* ------------------------------------------------------------------ packing (G6) */

void orc_gtq_pack(const uint8_t* codes, const uint8_t* wc, int D, uint8_t* row) {
  int nbits = 0;
  for (int i = 0; i < D; ++i) nbits += wc[i];
  memset(row, 0, (size_t)((nbits + 7) / 8));
  int n = 0;
  for (int i = 0; i < D; ++i)
    for (int k = 0; k < wc[i]; ++k, ++n)
      if ((codes[i] >> k) & 1) row[n >> 3] |= (uint8_t)(1u << (n & 7));
}

void orc_gtq_unpack(const uint8_t* row, const uint8_t* wc, int D, uint8_t* codes) {
  int n = 0;
  for (int i = 0; i < D; ++i) {
    int c = 0;
    for (int k = 0; k < wc[i]; ++k, ++n) c |= ((row[n >> 3] >> (n & 7)) & 1) << k;
    codes[i] = (uint8_t)c;
  }
}

/* ------------------------------------------------------------------ layout (G7) */

size_t orc_gtq_key_row_bytes(const orc_gtq_config* c) { return (size_t)c->key_bits * (size_t)c->head_dim / 8; }
size_t orc_gtq_value_row_bytes(const orc_gtq_config* c) { return (size_t)c->value_bits * (size_t)c->head_dim / 8; }
size_t orc_gtq_tile_bytes(const orc_gtq_config* c) {
  return (size_t)c->page_size * (orc_gtq_key_row_bytes(c) + orc_gtq_value_row_bytes(c) + 8);
}
size_t orc_gtq_page_bytes(const orc_gtq_config* c) { return (size_t)c->num_kv_heads * orc_gtq_tile_bytes(c); }
static size_t tile_base(const orc_gtq_config* c, int page, int g) {
  return ((size_t)page * (size_t)c->num_kv_heads + (size_t)g) * orc_gtq_tile_bytes(c);
}
/* the 16-position slice of position pp: its 16 key rows, 16 value rows and 16 records */
static size_t slice_base(const orc_gtq_config* c, int page, int g, int pp) {
  return tile_base(c, page, g) +
         (size_t)(pp / 16) * 16u * (orc_gtq_key_row_bytes(c) + orc_gtq_value_row_bytes(c) + 8u);
}
size_t orc_gtq_key_row(const orc_gtq_config* c, int page, int g, int pp) {
  return slice_base(c, page, g, pp) + (size_t)(pp % 16) * orc_gtq_key_row_bytes(c);
}
size_t orc_gtq_value_row(const orc_gtq_config* c, int page, int g, int pp) {
  return slice_base(c, page, g, pp) + 16u * orc_gtq_key_row_bytes(c) + (size_t)(pp % 16) * orc_gtq_value_row_bytes(c);
}
size_t orc_gtq_param(const orc_gtq_config* c, int page, int g, int pp) {
  return slice_base(c, page, g, pp) + 16u * (orc_gtq_key_row_bytes(c) + orc_gtq_value_row_bytes(c)) + (size_t)(pp % 16) * 8u;
}

static int gtq_config_ok(const orc_gtq_config* c) {
  return c->num_kv_heads > 0 && c->num_q_heads % c->num_kv_heads == 0 && c->head_dim > 0 &&
         c->head_dim % 2 == 0 && c->page_size > 0 && c->page_size % 16 == 0 && c->key_bits >= 1 && c->key_bits <= 8 &&
         c->value_bits >= 1 && c->value_bits <= 8 && (c->key_bits * c->head_dim) % 8 == 0 &&
         (c->value_bits * c->head_dim) % 8 == 0;
}

/* widths and scales of the D coordinates of head g: coordinate i belongs to block i mod D/2 (G1) */
static void coord_params(const orc_gtq_config* c, const uint8_t* widths, const float* sigma, int g, uint8_t* wc,
                         float* sc) {
  const int D = c->head_dim, nb = D / 2;
  for (int i = 0; i < D; ++i) {
    wc[i] = widths[(size_t)g * (size_t)nb + (size_t)(i % nb)];
    sc[i] = sigma[(size_t)g * (size_t)nb + (size_t)(i % nb)];
  }
}

static void put16(uint8_t* p, uint16_t v) {
  p[0] = (uint8_t)(v & 0xFF);
  p[1] = (uint8_t)(v >> 8);
}
static uint16_t get16(const uint8_t* p) { return (uint16_t)(p[0] | (p[1] << 8)); }

int orc_gtq_append(const orc_gtq_config* c, const uint8_t* widths, const float* sigma, uint8_t* pool, int T, const void* K,
                   int k_dtype, const void* V, int v_dtype, const int32_t* seq_slot, const int32_t* pos,
                   const int32_t* page_table, int stride) {
  if (!gtq_config_ok(c)) return -1;
  const int D = c->head_dim, Hkv = c->num_kv_heads, P = c->page_size, nb = D / 2;
  for (int g = 0; g < Hkv; ++g) {
    int sum = 0;
    for (int b = 0; b < nb; ++b) {
      if (widths[(size_t)g * (size_t)nb + (size_t)b] > 8) return -1;
      sum += widths[(size_t)g * (size_t)nb + (size_t)b];
    }
    if (2 * sum != c->key_bits * D) return -1;
  }
  float* kf = (float*)malloc(sizeof(float) * (size_t)D);
  float* vf = (float*)malloc(sizeof(float) * (size_t)D);
  uint8_t* wc = (uint8_t*)malloc((size_t)D);
  uint8_t* wv = (uint8_t*)malloc((size_t)D);
  uint8_t* codes = (uint8_t*)malloc((size_t)D);
  float* sc = (float*)malloc(sizeof(float) * (size_t)D);
  if (!kf || !vf || !wc || !wv || !codes || !sc) {
    free(kf), free(vf), free(wc), free(wv), free(codes), free(sc);
    return -2;
  }
  for (int i = 0; i < D; ++i) wv[i] = (uint8_t)c->value_bits;
  int range = 0;
  for (int t = 0; t < T; ++t) {
    const int b = seq_slot[t], p = pos[t];
    const int page = page_table[(size_t)b * (size_t)stride + (size_t)(p / P)], pp = p % P;
    for (int g = 0; g < Hkv; ++g) {
      const size_t in0 = ((size_t)t * (size_t)Hkv + (size_t)g) * (size_t)D;
      for (int e = 0; e < D; ++e) {
        kf[e] = (float)gtq_load(K, k_dtype, in0 + (size_t)e);
        vf[e] = (float)gtq_load(V, v_dtype, in0 + (size_t)e);
      }
      uint16_t ks, z, r;
      coord_params(c, widths, sigma, g, wc, sc);
      range |= orc_gtq_quant_key(kf, D, wc, sc, codes, &ks);
      orc_gtq_pack(codes, wc, D, pool + orc_gtq_key_row(c, page, g, pp));
      put16(pool + orc_gtq_param(c, page, g, pp), ks);
      put16(pool + orc_gtq_param(c, page, g, pp) + 2, 0);
      range |= orc_gtq_quant_value(vf, D, c->value_bits, codes, &z, &r);
      orc_gtq_pack(codes, wv, D, pool + orc_gtq_value_row(c, page, g, pp));
      put16(pool + orc_gtq_param(c, page, g, pp) + 4, z);
      put16(pool + orc_gtq_param(c, page, g, pp) + 6, r);
    }
  }
  free(kf), free(vf), free(wc), free(wv), free(codes), free(sc);
  return range;
}

int orc_gtq_dequant_seq(const orc_gtq_config* c, const uint8_t* widths, const float* sigma, const uint8_t* pool,
                        const int32_t* page_row, int L, int g, double* khat, double* vhat) {
  if (!gtq_config_ok(c)) return -1;
  const int D = c->head_dim, P = c->page_size;
  uint8_t wc[512], codes[512];
  float sc[512];
  if (D > 512) return -1;
  coord_params(c, widths, sigma, g, wc, sc);
  uint8_t wv[512];
  for (int i = 0; i < D; ++i) wv[i] = (uint8_t)c->value_bits;
  for (int p = 0; p < L; ++p) {
    const int page = page_row[p / P], pp = p % P;
    const uint8_t* prm = pool + orc_gtq_param(c, page, g, pp);
    orc_gtq_unpack(pool + orc_gtq_key_row(c, page, g, pp), wc, D, codes);
    for (int e = 0; e < D; ++e) khat[(size_t)p * (size_t)D + (size_t)e] = orc_gtq_dequant_key(get16(prm), sc[e], wc[e], codes[e]);
    orc_gtq_unpack(pool + orc_gtq_value_row(c, page, g, pp), wv, D, codes);
    for (int e = 0; e < D; ++e) vhat[(size_t)p * (size_t)D + (size_t)e] = orc_gtq_dequant_value(get16(prm + 4), get16(prm + 6), c->value_bits, codes[e]);
  }
  return 0;
}

/* ------------------------------------------------------------------ decode attention (G8) */

int orc_gtq_decode(const orc_gtq_config* c, const uint8_t* widths, const float* sigma, const uint8_t* pool, int B, const void* q,
                   int q_dtype, const int32_t* page_table, int stride, const int32_t* lens, double* out,
                   double* lse, int nthreads) {
  if (!gtq_config_ok(c)) return -1;
  const int D = c->head_dim, Hq = c->num_q_heads, Hkv = c->num_kv_heads, G = Hq / Hkv;
  const double tau = 1.0 / sqrt((double)D);
  int err = 0;
  if (nthreads < 1) nthreads = 1;
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
  for (int bg = 0; bg < B * Hkv; ++bg) {
    const int b = bg / Hkv, g = bg % Hkv, L = lens[b];
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
    double* logit = (double*)malloc(sizeof(double) * (size_t)L);
    if (!khat || !vhat || !logit) {
#pragma omp atomic write
      err = -2;
    } else {
      orc_gtq_dequant_seq(c, widths, sigma, pool, page_table + (size_t)b * (size_t)stride, L, g, khat, vhat);
      for (int i = 0; i < G; ++i) {
        const size_t qh = (size_t)b * (size_t)Hq + (size_t)(g * G + i);
        double m = -INFINITY;
        for (int j = 0; j < L; ++j) {
          double acc = 0.0;
          for (int e = 0; e < D; ++e)
            acc += gtq_load(q, q_dtype, qh * (size_t)D + (size_t)e) * khat[(size_t)j * (size_t)D + (size_t)e];
          logit[j] = tau * acc;
          if (logit[j] > m) m = logit[j];
        }
        double l = 0.0;
        double* o = out + qh * (size_t)D;
        for (int e = 0; e < D; ++e) o[e] = 0.0;
        for (int j = 0; j < L; ++j) {
          const double p = exp(logit[j] - m);
          l += p;
          for (int e = 0; e < D; ++e) o[e] += p * vhat[(size_t)j * (size_t)D + (size_t)e];
        }
        for (int e = 0; e < D; ++e) o[e] /= l;
        if (lse) lse[qh] = m + log(l);
      }
    }
    free(khat);
    free(vhat);
    free(logit);
  }
  return err;
}
