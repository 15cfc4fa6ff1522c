// kv4_mixed.cu -- the mixed bit-width key cache: RoPE-block energy scoring and greedy bit
// allocation, the fused append (block-scaled key codes and affine value codes, bit-packed into
// the page slot), and decode attention over the packed pages.
//
// Method: "RoPE-Aware Bit Allocation for KV-Cache Quantization" (searcharxiv abstract).  Under
// RoPE a key's share of a later logit is a sum over its two-dimensional frequency blocks, so the
// key budget is split per block: for every layer and KV head a label-free energy score is taken
// per RoPE block and integer bit widths are handed out greedily by marginal gain; the cache is
// served from packed pages (the abstract's K3V3 serving path).  Conventions the abstract leaves
// open (identical in the test oracle):
//   - block b of a head is the rotate-half coordinate pair (b, b + D/2); its score is the fp64 sum
//     over the scored keys of k[b]^2 + k[b + D/2]^2 in key order; its scale sigma_b is
//     sqrt(score / 2T) rounded to fp32 (1 for a zero score);
//   - one more bit for a block of score E at w bits gains E 4^-w; bits go one at a time to the
//     largest gain (lowest block on ties), at most 8 per block, key_bits * D / 2 in all;
//   - a key gets one fp16 scale s = rounded up of max |x_j| / sigma_j over coordinates with
//     bits, and coordinate j of width w the mid-rise code floor((x_j / (sigma_j s) + 1) 2^(w-1))
//     clamped to [0, 2^w - 1], reconstructed as s sigma_j ((2 code + 1) 2^-w - 1) (0 for w = 0);
//   - a value gets the per-token affine code of the INT4 cache at value_bits bits: fp16 zero
//     rounded down, fp16 range rounded up, code = rint((x - zero) / (range / (2^b - 1)));
//   - codes are packed in coordinate order, least significant bit first, as one little-endian
//     bit stream per vector; a page tile of one KV head is P/16 slices of 16 positions, each
//     holding its 16 key rows, 16 value rows and 16 8-byte records (key scale, 0, value zero,
//     value range), so that a slice is one contiguous block; tiles ordered (page, head).
//
// Decode: the same flattened split-K as the BF16 baseline (16-position tiles of one (sequence, KV
// head) copied into a per-warp ring, LSE merge).  QK^T runs on m16n8k16 fp16 MMAs: the integer
// codes enter as exact subnormal fp16 A operands (placed at the top of the mantissa field), the
// query as q_j sigma_j in hi/lo fp16 halves (columns 2h, 2h+1 of the 8 N columns) with the
// remaining power of two in the logit scale, and the code-independent part
// sum_j q_j sigma_j (2^-w_j - 1) is added per head.  The MMA's k index is permuted so that the
// four lanes of a key row read neighbouring windows of its bit stream; key rows that would put
// the row lanes on the same shared-memory banks are padded in shared memory.  PV multiplies the
// value codes (subnormal fp16 likewise) by p * step in hi/lo halves and adds sum_t p_t zero_t.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>
#include <cstring>
#include <math.h>

#include <type_traits>

#include "kv4_device.cuh"
#include "kv4_internal.h"
#include "kv4_layout.cuh"
#include "kv4_splitk.cuh"

namespace kv4 {
namespace {

constexpr unsigned FULL = 0xffffffffu;
constexpr float kNegInf = -__builtin_huge_valf();
constexpr int kAppendThreads = 256;

__device__ __forceinline__ float load_elem(const void* base, int dtype, size_t i) {
  if (dtype == KV4_F32) return reinterpret_cast<const float*>(base)[i];
  if (dtype == KV4_BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[i]);
  return __half2float(reinterpret_cast<const __half*>(base)[i]);
}

template <int D>
__device__ __forceinline__ const float* rec_sigma(const uint8_t* alloc, int g) {
  return reinterpret_cast<const float*>(alloc + static_cast<size_t>(g) * mixed_alloc_record_bytes(D));
}
template <int D>
__device__ __forceinline__ const uint8_t* rec_width(const uint8_t* alloc, int g) {
  return alloc + static_cast<size_t>(g) * mixed_alloc_record_bytes(D) + (D / 2) * 4;
}

// ------------------------------------------------------------------ scoring + allocation

// One block per KV head, one thread per RoPE block: the fp64 score in key order (so the
// allocation, an integer decision, is the oracle's bit for bit), the block scale, then the greedy.
template <int D>
__global__ void __launch_bounds__(D / 2) mixed_score_kernel(ScoreArgs a) {
  constexpr int NB = D / 2;
  __shared__ double energy[NB];
  const int g = blockIdx.x, b = threadIdx.x;
  double e = 0.0;
  for (int t = 0; t < a.T; ++t) {
    const size_t row = (static_cast<size_t>(t) * a.Hkv + g) * D;
    const double x0 = static_cast<double>(load_elem(a.K, a.k_dtype, row + b));
    const double x1 = static_cast<double>(load_elem(a.K, a.k_dtype, row + b + NB));
    e = __dadd_rn(e, __dadd_rn(__dmul_rn(x0, x0), __dmul_rn(x1, x1)));
  }
  energy[b] = e;
  float* sigma = reinterpret_cast<float*>(a.alloc + static_cast<size_t>(g) * mixed_alloc_record_bytes(D));
  uint8_t* width = a.alloc + static_cast<size_t>(g) * mixed_alloc_record_bytes(D) + NB * 4;
  sigma[b] = (e > 0.0 && a.T > 0) ? __double2float_rn(__dsqrt_rn(__ddiv_rn(e, 2.0 * static_cast<double>(a.T)))) : 1.0f;
  __syncthreads();
  if (b == 0) {
    uint8_t w[NB];
    for (int i = 0; i < NB; ++i) w[i] = 0;
    const int steps = a.kbits * NB;
    for (int s = 0; s < steps; ++s) {
      int best = -1;
      double best_gain = 0.0;
      for (int i = 0; i < NB; ++i) {
        if (w[i] >= 8) continue;
        const double gain = scalbn(energy[i], -2 * static_cast<int>(w[i]));  // E 4^-w, exact
        if (best < 0 || gain > best_gain) {
          best = i;
          best_gain = gain;
        }
      }
      w[best] += 1;
    }
    for (int i = 0; i < NB; ++i) width[i] = w[i];
  }
}

// ------------------------------------------------------------------ append

// Add `code` (w bits) at bit `o` of a row held as 32-bit words in shared memory.
__device__ __forceinline__ void put_bits(uint32_t* row, int o, uint32_t code, int w) {
  if (w == 0) return;
  const int wi = o >> 5, sh = o & 31;
  atomicOr(&row[wi], code << sh);
  if (sh + w > 32) atomicOr(&row[wi + 1], code >> (32 - sh));
}

// One warp per (token, KV head); lane l holds coordinates l + 32 i.  Row buffers: per warp two
// rows of up to D bytes (8 bits per coordinate) plus a guard word.
template <int D>
__global__ void __launch_bounds__(kAppendThreads) append_mixed_kernel(AppendArgs a) {
  constexpr int NB = D / 2, NI = D / 32, RW = D / 4 + 1;
  __shared__ uint32_t rows[kAppendThreads / 32][2][RW];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gw = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  if (gw >= a.T * a.Hkv) return;
  const int t = gw / a.Hkv, g = gw - t * a.Hkv;
  const int b = a.seq_slot[t], pos = a.pos[t];
  if (b < 0 || b >= a.max_seqs || pos < 0 || pos / a.P >= a.stride) {
    if (lane == 0) atomicOr(a.err, KV4_DEVERR_LENGTH);
    return;
  }
  const int page = a.page_table[static_cast<size_t>(b) * a.stride + pos / a.P];
  if (page < 0 || page >= a.max_pages) {
    if (lane == 0) atomicOr(a.err, KV4_DEVERR_PAGE_RANGE);
    return;
  }
  const float* sig = rec_sigma<D>(a.alloc, g);
  const uint8_t* wid = rec_width<D>(a.alloc, g);
  float k[NI], v[NI], sg[NI];
  int w[NI];
  const size_t in0 = (static_cast<size_t>(t) * a.Hkv + g) * D;
#pragma unroll
  for (int i = 0; i < NI; ++i) {
    const int j = lane + 32 * i;
    k[i] = load_elem(a.K, a.k_dtype, in0 + j);
    v[i] = load_elem(a.V, a.v_dtype, in0 + j);
    sg[i] = sig[j % NB];
    w[i] = wid[j % NB];
  }
  uint32_t* krow = rows[warp][0];
  uint32_t* vrow = rows[warp][1];
  for (int i = lane; i < RW; i += 32) krow[i] = vrow[i] = 0u;

  // bit offsets of the lane's coordinates: exclusive prefix of the block widths (coordinate j is
  // block j mod D/2; the second half of the row starts after key_bits * D / 2 bits)
  int pre[NI];
  {
    int run = 0;
#pragma unroll
    for (int c = 0; c < NB / 32; ++c) {
      int x = w[c];  // block lane + 32 c is coordinate lane + 32 c
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(FULL, x, o);
        if (lane >= o) x += y;
      }
      pre[c] = run + x - w[c];
      run += __shfl_sync(FULL, x, 31);
    }
#pragma unroll
    for (int i = NB / 32; i < NI; ++i) pre[i] = run + pre[i - NB / 32];
  }

  // key: one fp16 scale over the block-standardised coordinates that have bits
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < NI; ++i)
    if (w[i] > 0) m = fmaxf(m, __fdiv_rn(fabsf(k[i]), sg[i]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, o));
  const __half ksh = __float2half_ru(m);
  const float sf = __half2float(ksh);
  const bool kbad = !isfinite(sf);
  __syncwarp();
#pragma unroll
  for (int i = 0; i < NI; ++i) {
    uint32_t c = 0u;
    if (w[i] > 0 && sf != 0.f && !kbad) {
      const int top = (1 << w[i]) - 1;
      const float d = __fmul_rn(sg[i], sf);
      const float tq = __fdiv_rn(k[i], d);
      const float u = __fmul_rn(__fadd_rn(tq, 1.0f), static_cast<float>(1 << (w[i] - 1)));
      const float f = floorf(u);
      c = f < 0.f ? 0u : (f > static_cast<float>(top) ? static_cast<uint32_t>(top) : static_cast<uint32_t>(f));
    }
    put_bits(krow, pre[i], c, w[i]);
  }

  // value: per-token affine code at vbits
  float mn = v[0], mx = v[0];
#pragma unroll
  for (int i = 1; i < NI; ++i) {
    mn = fminf(mn, v[i]);
    mx = fmaxf(mx, v[i]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(FULL, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, o));
  }
  mn = mn + 0.0f;
  mx = mx + 0.0f;
  const __half vzh = __float2half_rd(mn);
  const float zf = __half2float(vzh);
  const __half vrh = __float2half_ru(__fsub_rn(mx, zf));
  const float rf = __half2float(vrh);
  const bool vbad = !isfinite(zf) || !isfinite(rf);
  const int vtop = (1 << a.vbits) - 1;
#pragma unroll
  for (int i = 0; i < NI; ++i) {
    uint32_t c = 0u;
    if (rf != 0.f && !vbad) {
      const float step = __fdiv_rn(rf, static_cast<float>(vtop));
      const float r = rintf(__fdiv_rn(__fsub_rn(v[i], zf), step));
      c = r < 0.f ? 0u : (r > static_cast<float>(vtop) ? static_cast<uint32_t>(vtop) : static_cast<uint32_t>(r));
    }
    put_bits(vrow, (lane + 32 * i) * a.vbits, c, a.vbits);
  }
  if (lane == 0 && (kbad || vbad)) atomicOr(a.err, KV4_DEVERR_RANGE);
  __syncwarp();

  const int KR = a.kbits * D / 8, VR = a.vbits * D / 8, pp = pos % a.P, rr = pp & 15;
  // the position's 16-position slice: 16 key rows, 16 value rows, 16 records
  uint8_t* slice = a.pool + static_cast<size_t>(page) * a.page_bytes +
                   static_cast<size_t>(g) * static_cast<size_t>(a.P) * (KR + VR + 8) +
                   static_cast<size_t>(pp >> 4) * 16 * (KR + VR + 8);
  uint32_t* kdst = reinterpret_cast<uint32_t*>(slice + static_cast<size_t>(rr) * KR);
  uint32_t* vdst = reinterpret_cast<uint32_t*>(slice + 16 * static_cast<size_t>(KR) + static_cast<size_t>(rr) * VR);
  for (int i = lane; i < KR / 4; i += 32) kdst[i] = krow[i];
  for (int i = lane; i < VR / 4; i += 32) vdst[i] = vrow[i];
  if (lane == 0) {
    const unsigned long long rec =
        static_cast<unsigned long long>(__half_as_ushort(ksh)) |
        (static_cast<unsigned long long>(__half_as_ushort(vzh)) << 32) |
        (static_cast<unsigned long long>(__half_as_ushort(vrh)) << 48);
    *reinterpret_cast<unsigned long long*>(slice + 16 * static_cast<size_t>(KR + VR) + static_cast<size_t>(rr) * 8) = rec;
  }
}

// ------------------------------------------------------------------ decode

constexpr int kWarps = 8;
constexpr int kStages = 4;

template <int D, int VB>
struct MixedGeo {
  static constexpr int NK = D / 16;              // k steps of QK^T, m blocks of PV
  static constexpr int VR = VB * D / 8;          // value row bytes
  static constexpr int DPL = D / 8;              // value dims per lane (PV rows gq, gq + 8)
  static constexpr int WIN = DPL * VB;           // value bits per lane and token
  static constexpr int NWA = (WIN + 31) / 32;    // aligned window words
};

// A 16-position slice of a (page, KV head) tile in the page's own layout: 16 key rows of KR bytes,
// 16 value rows of VR bytes, 16 records of 8 bytes.
__host__ __device__ inline int mixed_slice_bytes(int KR, int VR) { return 16 * (KR + VR) + 128; }

// The 8 lanes of one lane group read the same word offset of 8 key rows at once.  Rows of KR bytes
// with KR / 4 a multiple of 16 words put those reads on two banks' worth of offsets (4-way
// conflicts at 4-bit keys for D = 128).  In shared memory such rows get 16 more bytes, which
// spreads the 8 rows over the banks.  The padded rows arrive by one tensor copy whose box starts
// 16 bytes before each row (the tensor's fill value, no memory traffic); the others by a bulk
// copy.  Two-way conflicts (KR / 4 = 8 mod 16) cost less than the row-by-row tensor copy and stay.
__host__ __device__ inline int mixed_key_pad(int KR) { return (KR / 4) % 16 == 0 ? 16 : 0; }

// A ring stage: [16 bytes][16 key rows of KRP = KR + pad bytes][16 value rows][16 records]; with
// padded rows it is rounded up to 128 bytes (the tensor copy's destination is 128-byte aligned).
// A key window may start up to 10 bits before its row (see the extraction table), so row 0 reads
// the word before it: the first 16 bytes keep that read inside the stage, off the previous one,
// whose copy may still be landing; with padded rows they are row 0's pad.  The bits read there
// are masked off.
constexpr int kStageLead = 16;
__host__ __device__ inline int mixed_stage_bytes_padded(int KR, int VR, int pad) {
  const int b = kStageLead + 16 * (KR + pad) + 16 * VR + 128;
  return pad ? (b + 127) & ~127 : b;
}
__host__ __device__ inline int mixed_stage_bytes(int KR, int VR) {
  return mixed_stage_bytes_padded(KR, VR, mixed_key_pad(KR));
}

// One 4-D tensor copy global -> shared (box of the tensor map at coordinates x..w); completion is
// signalled on `bar` as the box's bytes.  Never multicast.
__device__ __forceinline__ void tensor_g2s_4d(void* dst, const CUtensorMap* map, int x, int y, int z, int w,
                                              uint64_t* bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_u32(bar)), "l"(pol)
      : "memory");
}

template <int D, int G>
struct SmemMixedFixed {
  float qbuf[kWarps][G][D];
  // key extraction table per (k step kb, lane group tig).  The four codes c0..c3 (widths w0..w3,
  // sum W <= 32) of coordinates 16 kb + 4 tig + (0..3) follow each other in the bit stream from
  // bit off0.  The 32-bit window x starts t0 = min(10 - w0, 32 - W) bits before off0, so c0 sits
  // at the top of a mantissa field, or at most two bits below it when the four are wide.  Then
  // (x & M0) | (x 2^(26 - w1 - t0 - w0) & M1) is the subnormal pair (c0, c1) with M0 = (2^w0 - 1)
  // << t0 and M1 = (2^w1 - 1) << (26 - w1); z = x >> (t0 + w0 + w1 - 10 + w2) puts c2 at the top
  // of the low field and c3 at bit 10, and (z & M2) | (z 2^(16 - w3) & M3) is (c2, c3).  Words:
  // M0, M1, 2^(26 - w1 - t0 - w0), off0 - t0 (may be negative), the shift of z, M2, M3,
  // 2^(16 - w3).  The shifts into the high half are multiplies, which run on the FMA pipe.
  uint32_t ktab[kWarps][D / 16][4][8];
  uint32_t stage_ok[kWarps][kStages];  // 1 when the stage's page id was inside the pool
  uint64_t bar[kWarps][kStages];
  uint64_t stall[kWarps];  // never arrived on (the wait-limit test hook)
};

// the per-warp rings follow the fixed part, sized at launch from the row widths
template <int D, int G>
constexpr size_t kMixedFixedBytes = (sizeof(SmemMixedFixed<D, G>) + 127) & ~static_cast<size_t>(127);

template <int D, int G>
size_t mixed_smem_bytes(int KR, int VR) {
  return kMixedFixedBytes<D, G> + static_cast<size_t>(kWarps) * kStages * mixed_stage_bytes(KR, VR);
}

__device__ __forceinline__ float exp2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// the fp16 in the low half of a word, as a float
__device__ __forceinline__ float low_half(uint32_t w) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(w & 0xffffu)));
}

// fp16 pair (x0, x1) or the pair of their fp16 rounding remainders
__device__ __forceinline__ uint32_t split_h2(float x0, float x1, bool lo) {
  const __half h0 = __float2half_rn(x0), h1 = __float2half_rn(x1);
  __half r0 = h0, r1 = h1;
  if (lo) {
    r0 = __float2half_rn(x0 - __half2float(h0));
    r1 = __float2half_rn(x1 - __half2float(h1));
  }
  return static_cast<uint32_t>(__half_as_ushort(r0)) | (static_cast<uint32_t>(__half_as_ushort(r1)) << 16);
}

// Integer codes enter the fp16 MMAs as subnormal halves.  A w-bit code c placed at the top of the
// 10-bit mantissa field, bit pattern c 2^(10 - w), is the half c 2^(10 - w) 2^-24 exactly, and a
// pair of them is built from the packed bits with shifts (or multiplies) and masks alone.  The
// tensor cores take subnormal operands, but a product keeps fewer low bits the more leading zeros
// its subnormal operand has; at the top of the field the sums come out as those of the same codes
// given as normal halves.  The constant 2^(10 - w - 24) goes into the query weights (keys) and
// the partial's scale (values).
constexpr int kSubTop = 10;

// x shifted left by n bits (right by -n when n < 0); n is compile-time after unrolling
__device__ __forceinline__ uint32_t shift_to(uint32_t x, int n) { return n >= 0 ? x << n : x >> -n; }

// value codes c0, c1 (< 2^VB) -> the subnormal pair (c0 2^(10 - VB), c1 2^(10 - VB))
template <int VB>
__device__ __forceinline__ uint32_t codes_h2(uint32_t c0, uint32_t c1) {
  return prmt(c0, c1, 0x5410u) << (kSubTop - VB);
}

// bits [p, p + w) of a bit array held in words aw (p and w compile-time after unrolling)
template <int NW>
__device__ __forceinline__ uint32_t take_bits(const uint32_t (&aw)[NW], int p, int w) {
  const int wi = p >> 5, sh = p & 31;
  uint32_t x = aw[wi] >> sh;
  if (sh + w > 32 && wi + 1 < NW) x |= aw[wi + 1] << (32 - sh);
  return x & ((1u << w) - 1u);
}

// Value widths whose fields never straddle a byte: the PV operands are cut out with byte
// permutes and masks.
template <int VB>
constexpr bool kSwarV = VB == 2 || VB == 4 || VB == 8;

// Bit position of the value field of lane dim d within its half once it is cut out.  A field at bit
// s of its byte whose top bit is at bit 7 (two leading zeros in the mantissa field at most) stays
// where it is; a lower one is lifted to the top of the field.  Odd widths always go to the top.
template <int VB>
__host__ __device__ constexpr int value_field_pos(int d) {
  return !kSwarV<VB> ? kSubTop - VB : (((d * VB) & 7) + VB >= 8 ? (d * VB) & 7 : kSubTop - VB);
}

// the value codes of lane dim d entered the MMAs as c 2^(value_field_pos(d) - 24)
template <int VB>
__host__ __device__ constexpr float value_unscale(int d) {
  return static_cast<float>(1 << (24 - value_field_pos<VB>(d)));
}

// (code of dim d of token t0, same of t1) as a subnormal pair, byte-aligned widths: one permute
// puts the field's byte of both tokens into the two halves, a low field is shifted up, one mask
// keeps both fields
template <int VB, int NW>
__device__ __forceinline__ uint32_t swar_pair(const uint32_t (&w0)[NW], const uint32_t (&w1)[NW], int d) {
  const int byte = (d * VB) >> 3, sh = (d * VB) & 7, pos = value_field_pos<VB>(d);
  const uint32_t sel = static_cast<uint32_t>((byte & 3) | ((4 + (byte & 3)) << 8));
  const uint32_t x = prmt(w0[byte >> 2], w1[byte >> 2], sel);
  const uint32_t m = ((1u << VB) - 1u) << pos;
  return (pos > sh ? x << (pos - sh) : x) & (m | (m << 16));
}

// The 16-bit chunk an odd-width value field is cut from: the lowest byte b whose bits
// [8 b, 8 b + 16) hold the field, with bytes b and b + 1 in one word (b % 4 <= 2); -1 when there is
// none (a field across two words).
template <int VB>
__host__ __device__ constexpr int field_chunk(int d) {
  for (int b = 0; 8 * b <= d * VB; ++b)
    if (b % 4 <= 2 && d * VB + VB <= 8 * b + 16) return b;
  return -1;
}

// (code of dim d of token t0, same of t1) as a subnormal pair, any value width.  One byte permute
// puts the field's 16-bit chunk of both tokens into the two halves (shared by every field of that
// chunk), one shift takes both fields to the top of their mantissa fields, one mask keeps them:
// bits that cross between the halves land outside the mask (a field ends at most at bit 16 of its
// chunk).  A field across two words goes through take_bits.
template <int VB, int NW>
__device__ __forceinline__ uint32_t field_pair(const uint32_t (&w0)[NW], const uint32_t (&w1)[NW], int d) {
  const int b = field_chunk<VB>(d);
  if (b < 0) return codes_h2<VB>(take_bits(w0, d * VB, VB), take_bits(w1, d * VB, VB));
  const uint32_t s = static_cast<uint32_t>(b & 3);
  const uint32_t x = prmt(w0[b >> 2], w1[b >> 2], s | ((s + 1u) << 4) | ((s + 4u) << 8) | ((s + 5u) << 12));
  const uint32_t m = ((1u << VB) - 1u) << (kSubTop - VB);
  return shift_to(x, kSubTop - VB - (d * VB - 8 * b)) & (m | (m << 16));
}

// Key rows (KMODE): 0, unpadded, the slice in one bulk copy; 1, padded rows by one tensor copy
// through kmap (the layer's key rows as the tensor [pages][Hkv P / 16 slices][16 rows][KR bytes]);
// 2, padded rows by one bulk copy per row (16 lanes), for when the tensor map cannot be had.  The
// tensor copy's destination is 128-byte aligned: the dynamic shared memory is declared so, and the
// kernel has no static shared memory.
template <int D, int G, int VB, int KMODE>
__global__ void __launch_bounds__(kWarps * 32, 2)
    decode_mixed_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap kmap) {
  using MG = MixedGeo<D, VB>;
  constexpr int NK = MG::NK, NB = D / 2;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  SmemMixedFixed<D, G>& sm = *reinterpret_cast<SmemMixedFixed<D, G>*>(smem_raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, tig = lane & 3;
  const int wid = blockIdx.x * kWarps + warp;
  const int cap = a.stride * a.P;
  const int KR = a.kbits * D / 8;
  constexpr bool PAD = KMODE != 0;
  constexpr int kpad = PAD ? 16 : 0;
  const int KRP = KR + kpad;  // key row stride in shared memory
  const int SB = mixed_stage_bytes_padded(KR, MG::VR, kpad), SL = mixed_slice_bytes(KR, MG::VR);
  const int VO = kStageLead + 16 * KRP, PO = VO + 16 * MG::VR;
  uint8_t* const ring = smem_raw + kMixedFixedBytes<D, G> + static_cast<size_t>(warp) * kStages * SB;
  const size_t tile_bytes = static_cast<size_t>(a.P) * (KR + MG::VR + 8);
  uint64_t* bars = sm.bar[warp];
  if (lane == 0) {
    for (int i = 0; i < kStages; ++i) mbar_init(&bars[i], 1);
    mbar_init(&sm.stall[warp], 1);
    fence_mbar_init();
  }
  __syncwarp();

  const long long total = splitk::prefix_cost(a, cap, lane, a.B);
  const long long Q = splitk::quota(total, a.W);
  const long long c0 = static_cast<long long>(wid) * Q;
  if (c0 >= total) return;
  const long long c1 = c0 + Q < total ? c0 + Q : total;
  splitk::Cur cons = splitk::cursor_at(a, cap, lane, c0);
  splitk::Cur prod = cons;
  const long long nslots = c1 - c0;
  // the tensor copy delivers the padded rows (fill included), the other copies the rows' bytes
  const uint32_t stage_tx = static_cast<uint32_t>(16 * (KMODE == 1 ? KRP : KR) + 16 * MG::VR + 128);

  // Lane 0 arms the stage's barrier, records whether the page is valid and starts the copies of
  // the 16-position slice: unpadded, the whole slice in one bulk copy (it lands in the stage's
  // layout); padded, the key rows by the tensor copy and the value rows with the records by one
  // bulk copy.  In mode 2 the first 16 lanes copy a key row each.  Called by the whole warp.
  auto issue = [&](const splitk::Cur& c, int st) {
    constexpr bool one_lane = KMODE != 2;
    if (one_lane && lane != 0) return;
    // the page of slice c.i, and the slice within it (a shift when P / 16 is a power of two)
    const int lp = a.tp_shift >= 0 ? c.i >> a.tp_shift : (c.i * 16) / a.P;
    int page = 0;
    if (lane == 0) {
      page = a.page_table[static_cast<size_t>(c.b) * a.stride + lp];
      const bool ok = page >= 0 && page < a.max_pages;
      sm.stage_ok[warp][st] = ok ? 1u : 0u;
      if (!ok) atomicOr(a.err, KV4_DEVERR_PAGE_RANGE);
      mbar_arrive_expect_tx(&bars[st], ok ? stage_tx : 0u);
    }
    if constexpr (!one_lane) page = __shfl_sync(FULL, page, 0);
    if (page < 0 || page >= a.max_pages) return;
    const int r0 = c.i * 16 - lp * a.P;
    const uint8_t* src = a.pool + static_cast<size_t>(page) * a.page_bytes + static_cast<size_t>(c.g) * tile_bytes +
                         static_cast<size_t>(r0 >> 4) * SL;
    uint8_t* dst = ring + st * SB;
    const uint64_t pol = l2_policy_evict_first();
    if constexpr (!PAD) {
      bulk_g2s_hint(dst + kStageLead, src, static_cast<uint32_t>(SL), &bars[st], pol);
    } else {
      if constexpr (KMODE == 1) {
        // box from x = -16: each row lands as [16 bytes of fill][KR bytes]
        tensor_g2s_4d(dst, &kmap, -16, 0, c.g * (a.P >> 4) + (r0 >> 4), page, &bars[st], pol);
      } else if (lane < 16) {
        bulk_g2s_hint(dst + kStageLead + lane * KRP, src + lane * KR, static_cast<uint32_t>(KR), &bars[st], pol);
      }
      if (lane == 0) bulk_g2s_hint(dst + VO, src + 16 * KR, static_cast<uint32_t>(16 * MG::VR + 128), &bars[st], pol);
    }
  };

  // Per (sequence, KV head): the key bit table, the scaled query fragments and the constant part
  // of each head's logit.
  uint32_t qf[NK][2];
  float cst = 0.f, inv_scale = 1.f;
  float* qb = &sm.qbuf[warp][0][0];
  uint32_t* ktab = &sm.ktab[warp][0][0][0];  // [kb][tig][8]
  auto load_query = [&](int b, int g) {
    const float* sig = rec_sigma<D>(a.alloc, g);
    const uint8_t* wid8 = rec_width<D>(a.alloc, g);
    // exclusive prefix of the block widths; coordinate j >= D/2 starts after kbits * D/2 bits
    int wv[NB / 32], pre[NB / 32];
    int run = 0;
#pragma unroll
    for (int c = 0; c < NB / 32; ++c) {
      wv[c] = wid8[lane + 32 * c];
      int x = wv[c];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(FULL, x, o);
        if (lane >= o) x += y;
      }
      pre[c] = run + x - wv[c];
      run += __shfl_sync(FULL, x, 31);
    }
    float csum[G];
#pragma unroll
    for (int h = 0; h < G; ++h) csum[h] = 0.f;
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < D / 32; ++i) {
      const int j = lane + 32 * i, c = (j % NB) / 32;
      const int w = wv[c];
      const int off = (j >= NB ? run : 0) + pre[c];
      // the group of four coordinates is four consecutive lanes
      const int g0 = lane & ~3;
      const int off0 = __shfl_sync(FULL, off, g0);
      const int w0 = __shfl_sync(FULL, w, g0), w1 = __shfl_sync(FULL, w, g0 + 1);
      const int w2 = __shfl_sync(FULL, w, g0 + 2), w3 = __shfl_sync(FULL, w, g0 + 3);
      // the code's field sits at bit 10 - w of its half, except c0 of a wide group, which sits at t0
      float lift = 1.f;
      {
        const int e = j & 3;
        uint32_t* ent = ktab + (j >> 2) * 8;  // entry (kb, tig = (j / 4) % 4)
        const int t0 = min(kSubTop - w0, 32 - (w0 + w1 + w2 + w3));
        const uint32_t m = (1u << w) - 1u;
        if (e == 0) {
          lift = static_cast<float>(1 << (kSubTop - w0 - t0));
          ent[0] = m << t0;
          ent[3] = static_cast<uint32_t>(off0 - t0);
        } else if (e == 1) {
          ent[1] = m << (kSubTop + 16 - w);
          ent[2] = 1u << (kSubTop + 16 - w - t0 - w0);
        } else if (e == 2) {
          ent[4] = static_cast<uint32_t>(t0 + w0 + w1 - (kSubTop - w));
          ent[5] = m << (kSubTop - w);
        } else {
          ent[6] = m << (kSubTop + 16 - w);
          ent[7] = 1u << (16 - w);
        }
      }
      const float sgm = sig[j % NB];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const size_t qi = (static_cast<size_t>(b) * a.Hq + static_cast<size_t>(g) * G + h) * D + j;
        const float qs = load_elem(a.q, a.q_dtype, qi) * sgm * a.qscale;
        // the weight of code c is qs 2^(1 - w); the code enters as c 2^(10 - w - 24) / lift, and
        // the remaining 2^(1 - w) / 2^(10 - w - 24) = 2^15 is in inv_scale
        const float qq = w > 0 ? qs * lift : 0.f;
        if (w > 0) csum[h] += qs * (__int_as_float((127 - w) << 23) - 1.0f);      // qs (2^-w - 1)
        qb[h * D + j] = qq;
        amax = fmaxf(amax, fabsf(qq));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, o));
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) csum[h] += __shfl_xor_sync(FULL, csum[h], o);
    cst = 0.f;
#pragma unroll
    for (int h = 0; h < G; ++h)
      if (tig == h) cst = csum[h];
    // a power of two that brings the largest query weight near 2^8 (fp16 hi/lo keep ~22 bits)
    int ex = 0;
    if (amax > 0.f) frexpf(amax, &ex);
    const float scale = ldexpf(1.f, 8 - ex);
    inv_scale = ldexpf(1.f, ex - 8 + 15);
    __syncwarp();
    const int hh = gq >> 1;
    const bool lo = gq & 1;
#pragma unroll
    for (int kb = 0; kb < NK; ++kb) {
      const int j0 = 16 * kb + 4 * tig;
      if (hh < G) {
        const float* qh = qb + hh * D;
        qf[kb][0] = split_h2(qh[j0] * scale, qh[j0 + 1] * scale, lo);
        qf[kb][1] = split_h2(qh[j0 + 2] * scale, qh[j0 + 3] * scale, lo);
      } else {
        qf[kb][0] = qf[kb][1] = 0u;
      }
    }
    __syncwarp();
  };

  float oacc[NK][4];
  float m_run, l_part, pz;
  auto reset = [&]() {
#pragma unroll
    for (int mb = 0; mb < NK; ++mb) oacc[mb][0] = oacc[mb][1] = oacc[mb][2] = oacc[mb][3] = 0.f;
    m_run = kNegInf;
    l_part = 0.f;
    pz = 0.f;
  };
  auto flush = [&](const splitk::Cur& c) {
    float l = l_part, z = pz;
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      l += __shfl_xor_sync(FULL, l, o);
      z += __shfl_xor_sync(FULL, z, o);
    }
    if (tig < G) {
      const long long sid = static_cast<long long>(c.b) * a.Hkv + c.g;
      float* p = a.part + (static_cast<size_t>(wid + sid) * G + tig) * kPartRow<D>;
#pragma unroll
      for (int mb = 0; mb < NK; ++mb) {
        const int d = MG::DPL * gq + 2 * mb;
        const float f0 = value_unscale<VB>(2 * mb), f1 = value_unscale<VB>(2 * mb + 1);
        *reinterpret_cast<float2*>(p + d) =
            make_float2(fmaf(oacc[mb][0] + oacc[mb][1], f0, z), fmaf(oacc[mb][2] + oacc[mb][3], f1, z));
      }
      if (gq == 0) *reinterpret_cast<float2*>(p + D) = make_float2(m_run, l);
    }
  };

  int issued = 0;  // warp-uniform
  for (int k = 0; k < kStages - 1 && k < nslots; ++k) {
    issue(prod, k);
    ++prod.i;
    splitk::settle(a, cap, prod);
    ++issued;
  }
  reset();
  load_query(cons.b, cons.g);
  int Lseg = splitk::clamp_len(a.lens[cons.b], cap);  // length of the consumer's sequence
  // the wait-limit test hook: a first wait on a barrier nothing arrives on, which runs out
  bool failed = a.stall_test && !mbar_wait_bounded(&sm.stall[warp], 0u, a.err, a.wait_ns);
  long long k = 0;
  for (; !failed && k < nslots; ++k) {
    if (issued < nslots) {
      fence_proxy_async_smem();
      issue(prod, static_cast<int>((k + kStages - 1) % kStages));
      ++prod.i;
      splitk::settle(a, cap, prod);
      ++issued;
    }
    const int st = static_cast<int>(k % kStages);
    const bool ok = mbar_wait_bounded(&bars[st], static_cast<uint32_t>((k / kStages) & 1), a.err, a.wait_ns);
    if (__any_sync(FULL, !ok)) {
      failed = true;
      break;
    }
    const uint8_t* buf = ring + st * SB;
    const bool page_ok = sm.stage_ok[warp][st] != 0u;
    const int L = Lseg;
    const int i0 = cons.i * 16;
    const bool v0 = page_ok && tig < G && i0 + gq < L, v1 = page_ok && tig < G && i0 + gq + 8 < L;

    // QK^T.  k index (2 tig, 2 tig + 1, 2 tig + 8, 2 tig + 9) of step kb is coordinate 16 kb +
    // 4 tig + (0, 1, 2, 3), and the query fragments use the same map: the four lanes of a row read
    // neighbouring windows of one 16-coordinate stretch, so with row strides of 4 words mod 8 the
    // 32 lanes fall into distinct banks (or share a word).
    const uint32_t* r0w = reinterpret_cast<const uint32_t*>(buf + kStageLead + gq * KRP);
    const uint32_t* r1w = reinterpret_cast<const uint32_t*>(buf + kStageLead + (gq + 8) * KRP);
    float S[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kb = 0; kb < NK; ++kb) {
      const uint32_t* ent = ktab + (kb * 4 + tig) * 8;
      const uint4 E0 = *reinterpret_cast<const uint4*>(ent);      // M0, M1, multiplier of c1, window start
      const uint4 E1 = *reinterpret_cast<const uint4*>(ent + 4);  // shift of z, M2, M3, multiplier of c3
      // word of the window start (-1: the stage's lead bytes); the funnel shift takes the start
      // mod 32 itself
      const int wi = static_cast<int>(E0.w) >> 5;
      const uint32_t x0 = __funnelshift_r(r0w[wi], r0w[wi + 1], E0.w);
      const uint32_t x1 = __funnelshift_r(r1w[wi], r1w[wi + 1], E0.w);
      const uint32_t z0 = x0 >> E1.x, z1 = x1 >> E1.x;
      mma_f16(S, (x0 & E0.x) | ((x0 * E0.z) & E0.y), (x1 & E0.x) | ((x1 * E0.z) & E0.y),
              (z0 & E1.y) | ((z0 * E1.w) & E1.z), (z1 & E1.y) | ((z1 * E1.w) & E1.z), qf[kb][0], qf[kb][1]);
    }
    const __half* prm = reinterpret_cast<const __half*>(buf + PO);
    // records (key scale, 0, value zero, value range) of rows gq and gq + 8, 8 bytes each
    const uint2 rec0 = *reinterpret_cast<const uint2*>(prm + 4 * gq);
    const uint2 rec1 = *reinterpret_cast<const uint2*>(prm + 4 * (gq + 8));
    const float s0 = v0 ? low_half(rec0.x) : 0.f, s1 = v1 ? low_half(rec1.x) : 0.f;
    const float lg0 = v0 ? s0 * fmaf(S[0] + S[1], inv_scale, cst) : kNegInf;
    const float lg1 = v1 ? s1 * fmaf(S[2] + S[3], inv_scale, cst) : kNegInf;

    float tm = fmaxf(lg0, lg1);
    tm = fmaxf(tm, __shfl_xor_sync(FULL, tm, 4));
    tm = fmaxf(tm, __shfl_xor_sync(FULL, tm, 8));
    tm = fmaxf(tm, __shfl_xor_sync(FULL, tm, 16));
    const float mn = fmaxf(m_run, tm);
    const bool grow = mn > m_run;
    if (__any_sync(FULL, grow)) {
      const float alpha = grow ? (m_run == kNegInf ? 0.f : exp2_fast(m_run - mn)) : 1.f;
#pragma unroll
      for (int mb = 0; mb < NK; ++mb) {
        oacc[mb][0] *= alpha;
        oacc[mb][1] *= alpha;
        oacc[mb][2] *= alpha;
        oacc[mb][3] *= alpha;
      }
      l_part *= alpha;
      pz *= alpha;
      m_run = mn;
    }
    const float mu = m_run == kNegInf ? 0.f : m_run;
    const float p0 = v0 ? exp2_fast(lg0 - mu) : 0.f, p1 = v1 ? exp2_fast(lg1 - mu) : 0.f;
    l_part += p0 + p1;
    if (v0) pz = fmaf(p0, low_half(rec0.y), pz);
    if (v1) pz = fmaf(p1, low_half(rec1.y), pz);

    // PV.  B: p * step of tokens (2 tig, 2 tig + 1, 2 tig + 8, 2 tig + 9) for column gq = (head
    // gq / 2, hi or lo half); A: value codes of dims gq * D/8 + [0, D/8) (rows gq and gq + 8 of
    // m block mb are dims gq * D/8 + 2 mb and + 1) for the same tokens.
    const int hh = gq >> 1;
    const bool lo = gq & 1;
    const int src0 = 8 * tig + hh, src1 = src0 + 4;
    const float x0 = __shfl_sync(FULL, p0, src0), x1 = __shfl_sync(FULL, p0, src1);
    const float x2 = __shfl_sync(FULL, p1, src0), x3 = __shfl_sync(FULL, p1, src1);
    const int tk[4] = {2 * tig, 2 * tig + 1, 2 * tig + 8, 2 * tig + 9};
    const float vstep = 1.0f / static_cast<float>((1 << VB) - 1);
    float ps[4];
    const float xs[4] = {x0, x1, x2, x3};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const bool vt = page_ok && i0 + tk[u] < L;
      ps[u] = vt ? xs[u] * (__half2float(prm[4 * tk[u] + 3]) * vstep) : 0.f;
    }
    uint32_t b0 = 0u, b1 = 0u;
    if (hh < G) {
      b0 = split_h2(ps[0], ps[1], lo);
      b1 = split_h2(ps[2], ps[3], lo);
    }
    // the lane's value bits (dims gq * D/8 + [0, D/8)) of its four tokens, aligned to bit 0
    uint32_t aw[4][MG::NWA];
    const int bit0 = gq * MG::WIN;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t* vr = reinterpret_cast<const uint32_t*>(buf + VO + tk[u] * MG::VR);
      uint32_t raw[MG::NWA + 1];
#pragma unroll
      for (int x = 0; x <= MG::NWA; ++x) raw[x] = vr[(bit0 >> 5) + x];
#pragma unroll
      for (int x = 0; x < MG::NWA; ++x) aw[u][x] = __funnelshift_r(raw[x], raw[x + 1], bit0 & 31);
    }
    // Slots past L (or of a bad page) hold arbitrary bytes, but their codes are finite integers
    // and their B entries are exactly zero, so they add nothing.
#pragma unroll
    for (int mb = 0; mb < NK; ++mb) {
      if constexpr (kSwarV<VB>) {
        mma_f16(oacc[mb], swar_pair<VB>(aw[0], aw[1], 2 * mb), swar_pair<VB>(aw[0], aw[1], 2 * mb + 1),
                swar_pair<VB>(aw[2], aw[3], 2 * mb), swar_pair<VB>(aw[2], aw[3], 2 * mb + 1), b0, b1);
      } else {
        mma_f16(oacc[mb], field_pair<VB>(aw[0], aw[1], 2 * mb), field_pair<VB>(aw[0], aw[1], 2 * mb + 1),
                field_pair<VB>(aw[2], aw[3], 2 * mb), field_pair<VB>(aw[2], aw[3], 2 * mb + 1), b0, b1);
      }
    }
    __syncwarp();

    splitk::Cur nxt = cons;
    ++nxt.i;
    splitk::settle(a, cap, nxt);
    const bool more = k + 1 < nslots;
    if (!more || nxt.b != cons.b || nxt.g != cons.g) {
      flush(cons);
      reset();
      if (more) {
        load_query(nxt.b, nxt.g);
        if (nxt.b != cons.b) Lseg = splitk::clamp_len(a.lens[nxt.b], cap);
      }
    }
    cons = nxt;
  }
  if (failed) {
    for (long long j = k; j < issued; ++j)
      mbar_wait_bounded(&bars[j % kStages], static_cast<uint32_t>((j / kStages) & 1), a.err, a.wait_ns);
  }
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link against the driver
// library); null when it cannot be had
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

// The layer's key rows as the 4-D byte tensor [max_pages][Hkv P / 16][16][KR] (strides KR, the slice
// bytes, the page bytes) with a box of one slice's 16 rows, KR + 16 bytes wide.  False when the
// encoder is missing or refuses; the decode then copies unpadded rows.
bool encode_key_map(CUtensorMap* m, const DecodeArgs& a, int KR, int VR) {
  const PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (enc == nullptr) return false;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(KR), 16u, static_cast<cuuint64_t>(a.Hkv) * (a.P / 16),
                              static_cast<cuuint64_t>(a.max_pages)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(KR), static_cast<cuuint64_t>(mixed_slice_bytes(KR, VR)),
                                 static_cast<cuuint64_t>(a.page_bytes)};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(KR + 16), 16u, 1u, 1u};
  const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<uint8_t*>(a.pool), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int G, int VB>
cudaError_t launch_dgv(const DecodeArgs& a, int ctas, cudaStream_t st, bool row_copies) {
  const int KR = a.kbits * D / 8;
  CUtensorMap kmap;
  memset(&kmap, 0, sizeof(kmap));
  const bool pad = mixed_key_pad(KR) != 0;
  const int kmode = pad ? (!row_copies && encode_key_map(&kmap, a, KR, VB * D / 8) ? 1 : 2) : 0;
  const int smem = static_cast<int>(mixed_smem_bytes<D, G>(KR, VB * D / 8));
  // the attribute is raised once per kernel, to the size of the widest key rows (8 bits per dimension)
  const int smem_max = static_cast<int>(mixed_smem_bytes<D, G>(D, VB * D / 8));
  static std::atomic<uint64_t> done0, done1, done2;
  cudaError_t e = kmode == 1   ? ensure_smem_limit(decode_mixed_kernel<D, G, VB, 1>, smem_max, done1)
                  : kmode == 2 ? ensure_smem_limit(decode_mixed_kernel<D, G, VB, 2>, smem_max, done2)
                               : ensure_smem_limit(decode_mixed_kernel<D, G, VB, 0>, smem_max, done0);
  if (e != cudaSuccess) return e;
  if (kmode == 1)
    decode_mixed_kernel<D, G, VB, 1><<<ctas, kWarps * 32, smem, st>>>(a, kmap);
  else if (kmode == 2)
    decode_mixed_kernel<D, G, VB, 2><<<ctas, kWarps * 32, smem, st>>>(a, kmap);
  else
    decode_mixed_kernel<D, G, VB, 0><<<ctas, kWarps * 32, smem, st>>>(a, kmap);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return splitk::launch_merge<D, G>(a, st);
}

template <int D, int G>
cudaError_t launch_dg(const DecodeArgs& a, int ctas, cudaStream_t st, bool rows) {
  switch (a.vbits) {
    case 2: return launch_dgv<D, G, 2>(a, ctas, st, rows);
    case 3: return launch_dgv<D, G, 3>(a, ctas, st, rows);
    case 4: return launch_dgv<D, G, 4>(a, ctas, st, rows);
    case 8: return launch_dgv<D, G, 8>(a, ctas, st, rows);
    default: return cudaErrorInvalidValue;
  }
}

template <int D>
cudaError_t launch_append_d(const AppendArgs& a, cudaStream_t st) {
  const int warps = a.T * a.Hkv;
  append_mixed_kernel<D><<<(warps + kAppendThreads / 32 - 1) / (kAppendThreads / 32), kAppendThreads, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_mixed_score(const ScoreArgs& a, int D, cudaStream_t st) {
  note_launches(1);
  if (D == 128) mixed_score_kernel<128><<<a.Hkv, 64, 0, st>>>(a);
  else mixed_score_kernel<64><<<a.Hkv, 32, 0, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_append_mixed(const AppendArgs& a, int D, cudaStream_t st) {
  if (a.T <= 0) return cudaSuccess;
  note_launches(1);
  return D == 128 ? launch_append_d<128>(a, st) : launch_append_d<64>(a, st);
}

int mixed_decode_warps_per_cta() { return kWarps; }

// Two CTAs per SM where their shared memory fits (rows of up to 12 bytes per dimension pair at
// D = 128, e.g. K3V3 or K4V4), else one.
int mixed_decode_ctas_per_sm(int D, int G, int VB, int KB) {
  const int KR = KB * D / 8, VR = VB * D / 8;
  size_t bytes = 0;
  if (D == 128)
    bytes = G == 4 ? mixed_smem_bytes<128, 4>(KR, VR) : G == 2 ? mixed_smem_bytes<128, 2>(KR, VR)
                                                       : mixed_smem_bytes<128, 1>(KR, VR);
  else
    bytes = G == 4 ? mixed_smem_bytes<64, 4>(KR, VR) : G == 2 ? mixed_smem_bytes<64, 2>(KR, VR)
                                                     : mixed_smem_bytes<64, 1>(KR, VR);
  return 2 * (bytes + 1024) <= 227u * 1024u ? 2 : 1;
}

cudaError_t launch_decode_mixed(DecodeArgs a, int D, int G, int ctas, cudaStream_t st, bool row_copies) {
  a.W = ctas * kWarps;
  note_launches(2);
  if (D == 128) {
    if (G == 4) return launch_dg<128, 4>(a, ctas, st, row_copies);
    if (G == 2) return launch_dg<128, 2>(a, ctas, st, row_copies);
    return launch_dg<128, 1>(a, ctas, st, row_copies);
  }
  if (G == 4) return launch_dg<64, 4>(a, ctas, st, row_copies);
  if (G == 2) return launch_dg<64, 2>(a, ctas, st, row_copies);
  return launch_dg<64, 1>(a, ctas, st, row_copies);
}

}  // namespace kv4
