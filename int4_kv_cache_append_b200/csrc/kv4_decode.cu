// kv4_decode.cu -- decode-step attention over the paged INT4 cache and the INT8 side cache.
//
// Method: KV4-RL (ai.info summary), "Methodology in Plain English" paragraph 2: the packed INT4
// codes are consumed directly (no reconstruction in HBM), scale and offset are applied after
// the dot-product reduction (q . k^ = s (q . c) + z sum(q); sum_t p_t v^_t = sum_t (p_t s_t) c_t +
// sum_t p_t z_t), and the query is rotated to the keys' Hadamard basis; paragraph 3 and "Key
// Contributions" item 4: sink and recent positions come from an INT8 side cache, attended as
// disjoint regions whose softmax statistics (running max, sum) are merged.
//
// Work decomposition (flattened split-K): every (sequence b, KV head g) has an INT8 segment of
// ceil((s+w)/16) tiles (with a side cache over 16 tiles, only the tiles in use) and an INT4
// segment of the 16-position tiles covering [s, max(s, L-w)).
// An INT4 tile costs 1 unit (16*(D+8) bytes), an INT8 tile 2 units (about twice the bytes).  All
// tiles of all segments form one sequence of units; warp w of the launch takes the tiles whose
// first unit lies in [w*Q, (w+1)*Q), Q = ceil(total / warps), so every warp streams about the
// same number of bytes whatever the length mix.  A warp writes one partial (o, m, l) for every
// segment it touches, at index w + segment_id (unique: each step along the sequence advances the
// warp, the segment, or both); a second kernel (merge_int4_kernel) merges the partials of each
// (b, g) with the LSE rule.  A (b, g) whose positions all fell to one warp segment is written
// directly.  One CTA of 16 warps per SM.
//
// Per warp: kStages shared-memory stages of two tile blocks each, fed by 1-D bulk copies
// (cp.async.bulk, issued by lane 0 kStages-1 slots ahead, completion on one mbarrier per stage).
// A slot is two INT4 tiles (32 positions) or one INT8 tile (its K half and V half).  Slot
// descriptors (sources, 32-row validity mask, segment index, last-slot flag) are computed 16 slots
// at a time, one slot per lane, into a small ring, so the per-slot bookkeeping is a few
// instructions.  QK^T runs on 8-bit integer MMAs (m16n8k32): the INT4 key codes, unpacked to
// bytes by masks (pair-rows: rows r and r + 8 share a byte), are the A operand; the rotated
// query, rounded to a 22-bit integer and split into three signed base-256 digits, is the B
// operand (G heads x 3 digits in two n-blocks), so q . c is exact in int32.  PV runs on m16n8k16 fp16 MMAs: 16 dims x 16 positions with the centred V codes as the
// A operand and the hi/lo fp16 halves of p * scale of the G heads as the 8 columns of B.  Softmax,
// scale/offset and rescaling run in fp32 registers.
#include <cuda_bf16.h>
#include <math.h>

#include <type_traits>

#include "kv4_device.cuh"
#include "kv4_internal.h"
#include "kv4_layout.cuh"

namespace kv4 {
namespace {

constexpr unsigned FULL = 0xffffffffu;
// One CTA of 16 warps per SM: the SM's warp schedulers favour the older of two co-resident CTAs,
// so two 8-warp CTAs per SM finish unevenly; warps of one CTA progress at the same rate.
constexpr int kWarps = 16;
constexpr int kCtasPerSm = 1;
constexpr int kStages = 2;
constexpr int kChunk = 16;  // slots per descriptor fill (a fill of 32 measured slower on short batches)
constexpr int kRing = 32;   // descriptor ring (two chunks)
constexpr int kLensRegs = 8;  // sequence lengths held in registers by the schedule (B <= 256)
constexpr float kNegInf = -__builtin_huge_valf();

// ------------------------------------------------------------------ schedule
//
// Unit positions are 32-bit: the host refuses launches whose worst-case unit count
// B * Hkv * (2 * nt8 + stride * P / 16) reaches 2^31.

typedef unsigned int u32;

struct SegInfo {
  int n8;     // INT8 tiles (2 units each)
  int n4;     // INT4 tiles (1 unit each)
  int t4a;    // first INT4 tile (absolute 16-position tile index)
  int m_end;  // INT4 region end position
  int L;
};

__device__ __forceinline__ int clamp_len(int L, int cap) { return L < 0 ? 0 : (L > cap ? cap : L); }

// Side tiles visited: those up to the highest side row that holds a position.  Position j < s
// is row j; position j >= s is row s + (j mod w), so until the recent ring wraps
// (L + (s mod w) <= s + w) the rows in use end at L + (s mod w) (at L when L <= s): short
// sequences, and the all-INT8 configuration (w >= every length), read only the tiles they fill.
// smw = s mod w, precomputed on the host (0 when w = 0, which always gives nt8 for L > s).
__device__ __forceinline__ int side_tiles_used(int L, int s, int w, int nt8, int smw) {
  const int top = L <= s ? L : L + smw;
  return L <= 0 ? 0 : (top <= s + w ? (top + 15) >> 4 : nt8);
}

// T8: side caches larger than kTightSideTiles tiles (long recent windows, the all-INT8
// configuration) visit only the side tiles in use; smaller ones visit all of theirs (a few tiles,
// masked), which keeps this bound out of the common kernels' code.
constexpr int kTightSideTiles = 16;
template <bool T8>
__device__ __forceinline__ SegInfo seg_info(int L, int s, int w, int nt8, int smw) {
  SegInfo r;
  r.L = L;
  r.n8 = T8 ? side_tiles_used(L, s, w, nt8, smw) : (L > 0 ? nt8 : 0);
  r.m_end = max(s, L - w);
  r.t4a = s >> 4;
  r.n4 = (r.m_end > s) ? ((r.m_end - 1) >> 4) - r.t4a + 1 : 0;
  return r;
}

// Cost units of an INT8 side tile: 2 with INT4 values (its bytes are about twice an INT4 tile's),
// 1 with bf16 values (a side tile and a page tile then move about the same bytes).
template <bool VB>
constexpr u32 kU8 = VB ? 1u : 2u;

template <bool VB>
__device__ __forceinline__ u32 head_cost(const SegInfo& si) { return kU8<VB> * si.n8 + si.n4; }

template <bool T8, bool VB>
__device__ __forceinline__ u32 seq_cost(const DecodeArgs& a, int cap, int b) {
  return static_cast<u32>(a.Hkv) * head_cost<VB>(seg_info<T8>(clamp_len(a.lens[b], cap), a.s, a.w, a.nt8, a.smw));
}

__device__ __forceinline__ u32 warp_incl_scan(u32 v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const u32 t = __shfl_up_sync(FULL, v, o);
    if (lane >= o) v += t;
  }
  return v;
}

template <bool T8, bool VB>
__device__ u32 total_cost(const DecodeArgs& a, int cap, int lane) {
  u32 run = 0;
  for (int base = 0; base < a.B; base += 32) {
    const int b = base + lane;
    const u32 c = b < a.B ? seq_cost<T8, VB>(a, cap, b) : 0u;
    run += __shfl_sync(FULL, warp_incl_scan(c, lane), 31);
  }
  return run;
}

// Sequence containing unit c (c < total); *bstart = first unit of that sequence.
template <bool T8, bool VB>
__device__ int find_seq(const DecodeArgs& a, int cap, int lane, u32 c, u32* bstart) {
  u32 run = 0;
  for (int base = 0; base < a.B; base += 32) {
    const int b = base + lane;
    const u32 cb = b < a.B ? seq_cost<T8, VB>(a, cap, b) : 0u;
    const u32 incl = warp_incl_scan(cb, lane);
    const u32 tot = __shfl_sync(FULL, incl, 31);
    if (c < run + tot) {
      const unsigned m = __ballot_sync(FULL, c < run + incl);
      const int l = __ffs(m) - 1;
      *bstart = run + __shfl_sync(FULL, incl - cb, l);
      return base + l;
    }
    run += tot;
  }
  *bstart = run;
  return a.B;
}

// Division by a per-launch constant d >= 2 for n < 2^31: q = umulhi(n, ceil(2^32 / d)) is
// floor(n / d) or one more; one multiply-compare fixes it.  ceil(2^32 / d) = floor((2^32 - 1) / d)
// + 1 for every d >= 2, a 32-bit division.
struct FastDiv {
  u32 d, m;
  __device__ explicit FastDiv(u32 dd) : d(dd), m(0xFFFFFFFFu / dd + 1u) {}
  __device__ __forceinline__ u32 div(u32 n) const {
    u32 q = __umulhi(n, m);
    if (q * d > n) --q;
    return q;
  }
};

// Position in the tile sequence (warp-uniform): tile i of segment seg of (b, g).
struct Cursor {
  int b, g, seg;  // seg 0 = INT8 region, 1 = INT4 region
  int i;          // tile index within the segment
  int n;          // tiles in the segment
  u32 cost;       // first unit of tile i
  u32 cs8;        // first unit of the INT8 segment of (b, g)
  SegInfo si;
  bool valid;
};

// Move forward to the first non-empty segment at or after the current one.
template <bool T8, bool VB>
__device__ void settle(const DecodeArgs& a, int cap, Cursor& c) {
  while (true) {
    if (c.b >= a.B) {
      c.valid = false;
      return;
    }
    c.n = c.seg == 0 ? c.si.n8 : c.si.n4;
    if (c.i < c.n) return;
    c.i = 0;
    if (c.seg == 0) {
      c.seg = 1;
    } else {
      c.seg = 0;
      c.cs8 += head_cost<VB>(c.si);
      if (++c.g == a.Hkv) {
        c.g = 0;
        if (++c.b < a.B) c.si = seg_info<T8>(clamp_len(a.lens[c.b], cap), a.s, a.w, a.nt8, a.smw);
      }
    }
  }
}

// Unit position of the cursor's tile (after settle moved it to another segment).
template <bool VB>
__device__ __forceinline__ void recost(Cursor& c) {
  c.cost = c.seg == 0 ? c.cs8 + kU8<VB> * c.i : c.cs8 + kU8<VB> * c.si.n8 + c.i;
}

// First tile whose first unit is >= c0, in sequence b (first unit bstart, raw length Lraw).
template <bool T8, bool VB>
__device__ Cursor cursor_at(const DecodeArgs& a, int cap, int b, u32 bstart, u32 c0, int Lraw) {
  Cursor c;
  c.b = b;
  c.valid = b < a.B;
  if (!c.valid) return c;
  c.si = seg_info<T8>(clamp_len(Lraw, cap), a.s, a.w, a.nt8, a.smw);
  const u32 ch = head_cost<VB>(c.si);
  const u32 off = c0 - bstart;
  c.g = static_cast<int>(off / ch);
  c.cs8 = bstart + static_cast<u32>(c.g) * ch;
  const u32 r = off - static_cast<u32>(c.g) * ch;
  if (r < kU8<VB> * c.si.n8) {
    c.seg = 0;
    c.i = static_cast<int>(VB ? r : (r + 1) >> 1);
  } else {
    c.seg = 1;
    c.i = static_cast<int>(r - kU8<VB> * c.si.n8);
  }
  settle<T8, VB>(a, cap, c);
  if (c.valid) recost<VB>(c);
  return c;
}

// Page-table column and tile-in-page of absolute tile ti (16 positions each).
__device__ __forceinline__ void tile_page(const DecodeArgs& a, int ti, int* lp, int* tin) {
  if (a.tp_shift >= 0) {
    *lp = ti >> a.tp_shift;
    *tin = ti & ((1 << a.tp_shift) - 1);
  } else {
    *lp = (ti * 16) / a.P;
    *tin = ti - *lp * (a.P >> 4);
  }
}

// ------------------------------------------------------------------ per-warp shared memory

// Stage of the shared-memory ring: two INT4 page tiles or one INT8 side tile; with bf16 values
// one page tile or one side tile (the larger).
template <int D, bool VB>
constexpr int kStageBytes = VB ? Geo<D>::T8V : 2 * Geo<D>::T4B;

template <int D, bool VB>
struct Smem {
  uint8_t ring[kWarps][kStages][kStageBytes<D, VB>];
  unsigned long long src[kWarps][kRing][2];      // bulk-copy sources of each slot (0 = none)
  unsigned int mask[kWarps][kRing];              // valid rows: tile A bits 0-15, tile B 16-31
  unsigned int meta[kWarps][kRing];              // kind | flags | segment index << 8
  unsigned long long seg[kWarps][kRing];         // segment table: cs8 | seg<<32 | g<<33 | b<<41
  Cursor cur[kWarps];                                // descriptor cursor between fills
  unsigned segno[kWarps];                            // segments entered so far
  uint64_t bar[kWarps][kStages];
  uint64_t stall[kWarps];  // never arrived on: the wait-limit test (kv4_debug_force_wait_timeout)
};

// slot meta word
constexpr unsigned kKindInt4 = 0u, kKindInt8 = 1u, kKindNone = 2u;
constexpr unsigned kMetaLast = 4u;  // last slot of its segment in this warp's stream
constexpr unsigned kMetaTwo = 8u;   // INT4 slot with a second tile
constexpr unsigned kMetaBad = 16u;  // a page id outside the pool (tile skipped)
__device__ __forceinline__ unsigned meta_kind(unsigned m) { return m & 3u; }
__device__ __forceinline__ unsigned meta_seg(unsigned m) { return (m >> 8) & (kRing - 1); }

__device__ __forceinline__ unsigned long long pack_seg(int b, int g, int seg, u32 cs8) {
  return static_cast<unsigned long long>(cs8) | (static_cast<unsigned long long>(seg) << 32) |
         (static_cast<unsigned long long>(g) << 33) | (static_cast<unsigned long long>(b) << 41);
}
__device__ __forceinline__ u32 seg_cs8(unsigned long long e) { return static_cast<u32>(e); }
__device__ __forceinline__ int seg_kind(unsigned long long e) { return static_cast<int>((e >> 32) & 1ull); }
__device__ __forceinline__ int seg_g(unsigned long long e) { return static_cast<int>((e >> 33) & 255ull); }
__device__ __forceinline__ int seg_b(unsigned long long e) { return static_cast<int>(e >> 41); }

// Bits r (0..15) of the 16 rows starting at t0 whose index lies in [lo, hi).
__device__ __forceinline__ unsigned range_bits(int lo, int hi, int t0) {
  const int l = min(max(lo - t0, 0), 16), h = min(max(hi - t0, 0), 16);
  return h > l ? (((1u << h) - 1u) & ~((1u << l) - 1u)) : 0u;
}

// Valid side rows of INT8 tile i for a sequence of length L: sink rows R < min(s, L); ring row
// s + idx holds the recent position j in [max(s, L - w), L) with j mod w = idx, i.e. the cyclic
// interval of idx starting at s mod w of length min(L - s, w); rows past s + w are padding.
__device__ __forceinline__ unsigned side_tile_mask(int i, int L, int s, int w) {
  const int t0 = 16 * i;
  unsigned m = range_bits(0, min(s, L), t0);
  if (L > s && w > 0) {
    const int n = min(L - s, w);
    if (n == w) {
      m |= range_bits(s, s + w, t0);
    } else {
      const int a0 = s % w;
      m |= range_bits(s + a0, s + min(w, a0 + n), t0);
      if (a0 + n > w) m |= range_bits(s, s + (a0 + n - w), t0);
    }
  }
  return m;
}

// Descriptors of the kChunk slots that follow cursor `c` (lane j < kChunk takes slot base + j),
// written to ring position (base + j) % kRing, plus one segment-table entry per segment entered.
// `c` is advanced past them; slots past the warp's stream get kind None.  `segno` counts the
// segments this warp has entered.
template <int D, bool T8, bool VB>
__device__ void fill_descriptors(const DecodeArgs& a, int cap, u32 c1, Cursor& c, int lane,
                                 Smem<D, VB>& sm, int warp, int base, unsigned& segno) {
  using Gm = Geo<D>;
  constexpr int TPS = VB ? 1 : 2;                         // page tiles per slot
  constexpr int T4 = VB ? Gm::T4V : Gm::T4B;              // page tile bytes
  constexpr int TS = VB ? Gm::T8V : Gm::T8B;              // side tile bytes
  unsigned long long s0 = 0ull, s1 = 0ull;
  unsigned msk = 0u, meta = kKindNone;
  int done = 0;
  while (done < kChunk && c.valid && c.cost < c1) {
    const unsigned sidx = segno & (kRing - 1);
    if (lane == 0) sm.seg[warp][sidx] = pack_seg(c.b, c.g, c.seg, c.cs8);
    int avail_tiles, avail_slots;
    if (c.seg == 1) {
      avail_tiles = static_cast<int>(min(static_cast<u32>(c.n - c.i), c1 - c.cost));
      avail_slots = VB ? avail_tiles : (avail_tiles + 1) >> 1;
    } else {
      avail_tiles = static_cast<int>(min(static_cast<u32>(c.n - c.i), VB ? c1 - c.cost : (c1 - c.cost + 1) >> 1));
      avail_slots = avail_tiles;
    }
    const int take = min(kChunk - done, avail_slots);
    const int u = lane - done;
    if (u >= 0 && u < take) {
      meta = (sidx << 8) | ((take == avail_slots && u == take - 1) ? kMetaLast : 0u);
      if (c.seg == 1) {
        meta |= kKindInt4;
        const int t0 = c.i + TPS * u;
        const int nt = min(TPS, avail_tiles - TPS * u);
        if (nt == 2) meta |= kMetaTwo;
#pragma unroll
        for (int j = 0; j < TPS; ++j) {
          if (j < nt) {
            const int ti = c.si.t4a + t0 + j;
            int lp, tin;
            tile_page(a, ti, &lp, &tin);
            const int page = a.page_table[static_cast<size_t>(c.b) * a.stride + lp];
            unsigned long long addr = 0ull;
            if (page >= 0 && page < a.max_pages) {
              addr = reinterpret_cast<unsigned long long>(a.pool + static_cast<size_t>(page) * a.page_bytes +
                                                          static_cast<size_t>(c.g) * (a.P / 16) * T4 +
                                                          static_cast<size_t>(tin) * T4);
              msk |= range_bits(a.s, c.si.m_end, 16 * ti) << (16 * j);
            } else {
              meta |= kMetaBad;
            }
            if (j == 0) s0 = addr; else s1 = addr;
          }
        }
      } else {
        meta |= kKindInt8;
        const int ti = c.i + u;
        s0 = reinterpret_cast<unsigned long long>(a.side + static_cast<size_t>(c.b) * a.side_slot_bytes +
                                                  static_cast<size_t>(c.g) * a.nt8 * TS +
                                                  static_cast<size_t>(ti) * TS);
        s1 = VB ? 0ull : s0 + Gm::H8B;  // bf16 values: the side tile is one copy
        msk = side_tile_mask(ti, c.si.L, a.s, a.w);
      }
    }
    // advance the cursor past the taken slots; at the end of the segment move to the next one.
    // If the stream limit c1 cut the segment, the next tile starts at or past c1.
    if (c.seg == 1) {
      const int tiles = min(TPS * take, avail_tiles);
      c.i += tiles;
      c.cost += static_cast<u32>(tiles);
    } else {
      c.i += take;
      c.cost += kU8<VB> * take;
    }
    done += take;
    if (c.i >= c.n) {
      settle<T8, VB>(a, cap, c);
      ++segno;
      if (c.valid) recost<VB>(c);
    }
  }
  if (lane < kChunk) {
    const int p = (base + lane) % kRing;
    sm.src[warp][p][0] = s0;
    sm.src[warp][p][1] = s1;
    sm.mask[warp][p] = msk;
    sm.meta[warp][p] = meta;
  }
}

// ------------------------------------------------------------------ conversions

// V codes for the PV A operand: nibble k of each 16-bit half of word w (k = 0, 1 from w, k = 2, 3
// from w8 = w >> 8) becomes the exact fp16 (c - 8) (even k) or 16 (c - 8) (odd k); the factor 16
// of odd k is removed from the corresponding output rows when the partial is written.  V stays in
// normal fp16: the (p * scale) operand is small, and subnormal codes against it lose accuracy in
// the tensor-core accumulation over long sequences.
// Written as one lop3 (mask and magic exponent) and one packed fp16 subtraction: the same steps
// through the half2 intrinsics measured about 30 more integer-pipe instructions per tile.
template <int K>
__device__ __forceinline__ uint32_t vcode(uint32_t w, uint32_t w8) {
  const uint32_t src = K < 2 ? w : w8;
  uint32_t h, r;
  if constexpr ((K & 1) != 0) {
    // (src & 0x00F000F0) | 0x64006400 = 1024 + 16 c; minus 1152 = 1024 + 16 * 8
    asm("lop3.b32 %0, %1, 0x00F000F0, 0x64006400, 0xea;" : "=r"(h) : "r"(src));
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(h), "r"(0x64806480u));
  } else {
    // (src & 0x000F000F) | 0x64006400 = 1024 + c; minus 1032 = 1024 + 8
    asm("lop3.b32 %0, %1, 0x000F000F, 0x64006400, 0xea;" : "=r"(h) : "r"(src));
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(h), "r"(0x64086408u));
  }
  return r;
}

// This lane's part of two fp32 values as an fp16 pair: the value truncated to 11 significant bits
// (hi lanes) or the exact remainder rounded to fp16 (lo lanes); hi + lo carries ~22 bits.
__device__ __forceinline__ uint32_t split_pair(float x0, float x1, bool lo) {
  const float t0 = __uint_as_float(__float_as_uint(x0) & 0xFFFFE000u);
  const float t1 = __uint_as_float(__float_as_uint(x1) & 0xFFFFE000u);
  const float y0 = lo ? x0 - t0 : t0;
  const float y1 = lo ? x1 - t1 : t1;
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(y1), "f"(y0));
  return r;
}

// The bf16 counterpart of split_pair (bf16 values): the value truncated to 8 significant bits (hi
// lanes) or the remainder rounded to bf16 (lo lanes); hi + lo carries ~16 bits.
__device__ __forceinline__ uint32_t split_pair_bf16(float x0, float x1, bool lo) {
  const float t0 = __uint_as_float(__float_as_uint(x0) & 0xFFFF0000u);
  const float t1 = __uint_as_float(__float_as_uint(x1) & 0xFFFF0000u);
  const float y0 = lo ? x0 - t0 : t0;
  const float y1 = lo ? x1 - t1 : t1;
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(y1), "f"(y0));
  return r;
}

__device__ __forceinline__ float exp2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <int QT>
__device__ __forceinline__ float load_q(const void* q, size_t i) {
  if constexpr (QT == KV4_F32) return reinterpret_cast<const float*>(q)[i];
  else if constexpr (QT == KV4_BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(q)[i]);
  else return __half2float(reinterpret_cast<const __half*>(q)[i]);
}

__device__ __forceinline__ float half_lo(uint32_t w) { return __half2float(__ushort_as_half(static_cast<unsigned short>(w & 0xffffu))); }
__device__ __forceinline__ float half_hi(uint32_t w) { return __half2float(__ushort_as_half(static_cast<unsigned short>(w >> 16))); }

template <int WPC>
__device__ __forceinline__ void lds_words(const uint8_t* p, uint32_t (&w)[WPC]) {
  if constexpr (WPC == 4) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    w[0] = u.x;
    w[1] = u.y;
    w[2] = u.z;
    w[3] = u.w;
  } else {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    w[0] = u.x;
    w[1] = u.y;
  }
}

// ------------------------------------------------------------------ LSE merge of split partials

// Where the rows of the partials of one (b, g) live: partial j (INT8-region owners first, then
// INT4) has index w8a + j + sid8 (j < n8p) or w4a + (j - n8p) + sid8 + 1, and its G rows of
// (o[D], m, l) start at index * G * kPartRow.
struct PartRows {
  int n8p;
  u32 w8a, w4a, sid8;
  __device__ __forceinline__ unsigned long long row(int j, int G, int stride) const {
    const u32 idx = j < n8p ? (w8a + static_cast<u32>(j) + sid8) : (w4a + static_cast<u32>(j - n8p) + sid8 + 1u);
    return static_cast<unsigned long long>(idx) * G * stride;
  }
};

// ------------------------------------------------------------------ the decode kernel

// VB: values stored as bf16 (KV4_VALUES_BF16): one page tile per slot, PV on bf16 MMAs with the
// probabilities as bf16 hi/lo halves, no value scale or offset.
template <int D, int G, int QT, bool T8, bool VB>
__global__ void __launch_bounds__(kWarps * 32, kCtasPerSm) decode_int4_kernel(const DecodeArgs a) {
  using Gm = Geo<D>;
  constexpr int NKB = Gm::NKB;
  constexpr int WPC = Gm::WPC;
  constexpr int NK32 = D / 32;  // 32-dim blocks of the QK^T integer MMAs
  constexpr int T4B = Gm::T4B;
  constexpr int KPO = VB ? 8 * D : 16 * D;  // K {scale, zero} in a page tile
  extern __shared__ __align__(128) uint8_t smem_raw[];
  Smem<D, VB>& sm = *reinterpret_cast<Smem<D, VB>*>(smem_raw);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, tig = lane & 3;
  const int wid = blockIdx.x * kWarps + warp;
  const int cap = a.stride * a.P;
  // No early griddepcontrol.launch_dependents: the merge kernel launches when this grid completes.
  // Launched early, its waiting CTAs sat beside this kernel's warps and slowed them (1-2 %).

  // Launched as a programmatic dependent of the preceding kernel.  By default nothing is read
  // before that kernel completes; with a.early the schedule and the first descriptors (which read
  // only lens and page_table) are built first, and the wait comes before anything else.
  if (!a.early) pdl_wait();
  uint64_t* bars = sm.bar[warp];
  if (lane == 0) {
    for (int i = 0; i < kStages; ++i) mbar_init(&bars[i], 1);
    mbar_init(&sm.stall[warp], 1);
    fence_mbar_init();
  }

  // Lengths: read once (one load per lane and 32 sequences, all in flight together) and kept in
  // registers for the schedule when B <= 32 * kLensRegs; larger batches re-read them.
  const bool cached = a.B <= 32 * kLensRegs;
  int lr[kLensRegs];
#pragma unroll
  for (int r = 0; r < kLensRegs; ++r) {
    const int b = 32 * r + lane;
    lr[r] = (cached && b < a.B) ? a.lens[b] : 0;
  }
  auto cached_len = [&](int b) {  // raw length of sequence b (warp-uniform b < B <= 32 kLensRegs)
    int v = lr[0];
#pragma unroll
    for (int r = 1; r < kLensRegs; ++r)
      if ((b >> 5) == r) v = lr[r];
    return __shfl_sync(FULL, v, b & 31);
  };
  u32 total = 0;
  if (cached) {
#pragma unroll
    for (int r = 0; r < kLensRegs; ++r)
      if (32 * r < a.B) {
        const u32 c = 32 * r + lane < a.B ? static_cast<u32>(a.Hkv) * head_cost<VB>(seg_info<T8>(clamp_len(lr[r], cap), a.s, a.w, a.nt8, a.smw)) : 0u;
        total += __shfl_sync(FULL, warp_incl_scan(c, lane), 31);
      }
  } else {
    total = total_cost<T8, VB>(a, cap, lane);
  }
  const u32 Q = max(2u, (total + a.W - 1) / static_cast<u32>(a.W));
  const FastDiv divQ(Q);
  const unsigned long long c0l = static_cast<unsigned long long>(wid) * Q;
  const bool any = c0l < total;
  const u32 c0 = static_cast<u32>(c0l);
  const u32 c1 = c0 + Q;
  u32 bstart = 0;
  int b0 = a.B;
  if (cached) {
    u32 run = 0;
#pragma unroll
    for (int r = 0; r < kLensRegs; ++r)
      if (32 * r < a.B && b0 == a.B) {
        const u32 cb = 32 * r + lane < a.B ? static_cast<u32>(a.Hkv) * head_cost<VB>(seg_info<T8>(clamp_len(lr[r], cap), a.s, a.w, a.nt8, a.smw)) : 0u;
        const u32 incl = warp_incl_scan(cb, lane);
        const u32 tot = __shfl_sync(FULL, incl, 31);
        if (c0 < run + tot) {
          const int l = __ffs(__ballot_sync(FULL, c0 < run + incl)) - 1;
          bstart = run + __shfl_sync(FULL, incl - cb, l);
          b0 = 32 * r + l;
        }
        run += tot;
      }
  } else {
    b0 = find_seq<T8, VB>(a, cap, lane, c0, &bstart);
  }
  Cursor dcur = cursor_at<T8, VB>(a, cap, b0, bstart, c0, (any && b0 < a.B) ? (cached ? cached_len(b0) : a.lens[b0]) : 0);
  const bool active = any && dcur.valid && dcur.cost < c1;

  // Query of the first (b, g): loaded during the first descriptor fill, or after the wait on the
  // preceding kernel when the schedule is built early.
  float qx[G][4];
  auto load_q_regs = [&](int b, int g) {
    const bool act = lane < D / 4;
#pragma unroll
    for (int i = 0; i < G; ++i) {
      const size_t q0 = (static_cast<size_t>(b) * a.Hq + static_cast<size_t>(g) * G + i) * D + 4 * lane;
#pragma unroll
      for (int e = 0; e < 4; ++e) qx[i][e] = act ? load_q<QT>(a.q, q0 + e) : 0.f;
    }
  };
  const int qb0 = dcur.b, qg0 = dcur.g;  // first (b, g); the fill below moves dcur on
  if (active && !a.early) load_q_regs(qb0, qg0);  // in flight during the descriptor fill

  unsigned segno = 0;
  if (active) fill_descriptors<D, T8, VB>(a, cap, c1, dcur, lane, sm, warp, 0, segno);
  // the cursor waits in shared memory between fills (its registers are free in the main loop)
  if (lane == 0) {
    sm.cur[warp] = dcur;
    sm.segno[warp] = segno;
  }
  __syncwarp();
  if (a.early) pdl_wait();

  // Sequences with no positions get out = 0, lse = -inf here (nothing else touches them).
  for (int b = wid; b < a.B; b += a.W) {
    const int Lraw = cached ? cached_len(b) : a.lens[b];
    if (lane == 0 && Lraw > cap) atomicOr(a.err, KV4_DEVERR_LENGTH);
    if (clamp_len(Lraw, cap) == 0) {
      for (int e = lane; e < a.Hq * D; e += 32) a.out[static_cast<size_t>(b) * a.Hq * D + e] = 0.f;
      if (a.lse)
        for (int e = lane; e < a.Hq; e += 32) a.lse[static_cast<size_t>(b) * a.Hq + e] = kNegInf;
      for (int g = lane; g < a.Hkv; g += 32) *reinterpret_cast<uint4*>(a.meta + 4 * (b * a.Hkv + g)) = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  __syncwarp();

  if (!active) return;
  if (a.early) load_q_regs(qb0, qg0);

  // Issue the bulk copies of slot k into stage k % kStages (lane 0).  Returns false past the end.
  auto issue = [&](int k) {
    const int p = k % kRing;
    const unsigned meta = sm.meta[warp][p];
    if (meta_kind(meta) == kKindNone) return false;
    const int st = k % kStages;
    const unsigned long long s0 = sm.src[warp][p][0], s1 = sm.src[warp][p][1];
    const uint32_t nb = meta_kind(meta) == kKindInt8 ? (VB ? Gm::T8V : Gm::H8B) : (VB ? Gm::T4V : T4B);
    const uint32_t bytes = (s0 ? nb : 0u) + (s1 ? nb : 0u);
    if (meta & kMetaBad) atomicOr(a.err, KV4_DEVERR_PAGE_RANGE);
    mbar_arrive_expect_tx(&bars[st], bytes);
    // the cache is read once per decode: evict it first from L2, so that lens, the page table,
    // the queries and the split partials stay there
    const uint64_t pol = l2_policy_evict_first();
    if (s0) bulk_g2s_hint(sm.ring[warp][st], reinterpret_cast<const void*>(s0), nb, &bars[st], pol);
    if (s1) bulk_g2s_hint(sm.ring[warp][st] + T4B, reinterpret_cast<const void*>(s1), nb, &bars[st], pol);
    return true;
  };

  int issued = 0;
  if (lane == 0)
    for (int k = 0; k < kStages - 1; ++k)
      if (issue(k)) ++issued;
  issued = __shfl_sync(FULL, issued, 0);

  // ---- per-(b, g) query state
  // Query of head tig as the integer q_int = rint(q * 2^e) with |q_int| < 2^22, split into three
  // signed base-256 digits; qd[j] holds the s8 B fragments of 32-dim block j: n-block A (columns
  // 2h, 2h+1 = digits 2, 1 of head h), then n-block B (column 2h = digit 0 of head h).
  uint32_t qd[NK32][4];
  float sumq = 0.f, qinv = 1.f;  // sum of q_int over the dims of head tig; 2^-e

  // Rotate the G query heads held in qx (H/h), scale to log2 softmax units, normalise each head
  // by a power of two so that its fp16 hi/lo halves stay in the normal range, and build this
  // lane's MMA B fragments through `scratch` (a free stage buffer).
  auto build_query = [&](uint8_t* scratch) {
    const bool act = lane < D / 4;
    const int h = a.h;
    {
      // the keys' randomised signs (lane holds dims 4 lane .. 4 lane + 3)
      const uint32_t sb = act ? (a.signs[lane >> 3] >> (4 * (lane & 7))) & 15u : 0u;
#pragma unroll
      for (int i = 0; i < G; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) qx[i][e] = __uint_as_float(__float_as_uint(qx[i][e]) ^ (((sb >> e) & 1u) << 31));
    }
    // Butterfly strides 1 and 2 within the lane, then 4 .. h/2 across lanes (lane xor stride/4),
    // every stage over all G heads so that their shuffles overlap.
#pragma unroll
    for (int i = 0; i < G; ++i) {
      float* x = qx[i];
      if (h >= 2) {
        float u = x[0], v = x[1];
        x[0] = u + v;
        x[1] = u - v;
        u = x[2];
        v = x[3];
        x[2] = u + v;
        x[3] = u - v;
      }
      if (h >= 4) {
        float u = x[0], v = x[2];
        x[0] = u + v;
        x[2] = u - v;
        u = x[1];
        v = x[3];
        x[1] = u + v;
        x[3] = u - v;
      }
    }
#pragma unroll
    for (int st = 4; st < D; st <<= 1) {
      if (st < h) {
        const int m = st >> 2;
        const float sgn = (lane & m) ? -1.f : 1.f;  // upper half of the pair: o - x, lower: x + o
#pragma unroll
        for (int i = 0; i < G; ++i)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float o = __shfl_xor_sync(FULL, qx[i][e], m);
            qx[i][e] = fmaf(qx[i][e], sgn, o);  // exact: one rounding of o -+ x
          }
      }
    }
    const float sc = a.qscale / static_cast<float>(h);
    float amax[G];
#pragma unroll
    for (int i = 0; i < G; ++i) {
      amax[i] = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        qx[i][e] *= sc;
        amax[i] = fmaxf(amax[i], fabsf(qx[i][e]));
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1)
#pragma unroll
      for (int i = 0; i < G; ++i) amax[i] = fmaxf(amax[i], __shfl_xor_sync(FULL, amax[i], o));
    int qsum[G];
#pragma unroll
    for (int i = 0; i < G; ++i) {
      // 2^(21 - floor(log2 amax)) puts max|q| in [2^21, 2^22).
      int ex = amax[i] > 0.f ? ((__float_as_int(amax[i]) >> 23) & 0xff) - 127 : 0;
      ex = max(min(ex, 100), -100);
      const float up = __int_as_float((127 + 21 - ex) << 23);
      const float down = __int_as_float((127 - 21 + ex) << 23);
      if (tig == i) qinv = down;
      // digits of the lane's dims 4 lane + e: q = d2 2^16 + d1 2^8 + d0, each in [-128, 127]; in
      // the scratch each 8-dim group keeps its even dims in bytes 0-3 and odd dims in 4-7, the
      // order in which the K code bytes of a group enter the MMA.
      unsigned dg[3][2] = {{0u, 0u}, {0u, 0u}, {0u, 0u}};  // [digit][dims {0,2} | {1,3}] packed
      qsum[i] = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int qv = act ? __float2int_rn(qx[i][e] * up) : 0;
        qsum[i] += qv;
        const int d0 = ((qv + 128) & 255) - 128;
        const int q1 = (qv - d0) >> 8;
        const int d1 = ((q1 + 128) & 255) - 128;
        const int d2 = (q1 - d1) >> 8;
        const int sh = 8 * (e >> 1);
        dg[0][e & 1] |= static_cast<unsigned>(d0 & 255) << sh;
        dg[1][e & 1] |= static_cast<unsigned>(d1 & 255) << sh;
        dg[2][e & 1] |= static_cast<unsigned>(d2 & 255) << sh;
      }
      if (act) {
        // lane holds dims 0-3 (even lane) or 4-7 (odd lane) of group lane / 2: even dims go to
        // bytes (0, 1) or (2, 3) of the group, odd dims to bytes (4, 5) or (6, 7).
        const int gb = 8 * (lane >> 1) + 2 * (lane & 1);
#pragma unroll
        for (int dgt = 0; dgt < 3; ++dgt) {
          uint8_t* row = scratch + (i * 3 + dgt) * D + gb;
          *reinterpret_cast<unsigned short*>(row) = static_cast<unsigned short>(dg[dgt][0]);
          *reinterpret_cast<unsigned short*>(row + 4) = static_cast<unsigned short>(dg[dgt][1]);
        }
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1)
#pragma unroll
      for (int i = 0; i < G; ++i) qsum[i] += __shfl_xor_sync(FULL, qsum[i], o);
#pragma unroll
    for (int i = 0; i < G; ++i)
      if (tig == i) sumq = static_cast<float>(qsum[i]);
    __syncwarp();
    // B fragments: lane (gq, tig) supplies column gq, bytes of its dims 32 tig + 8 j + (0, 2, 4, 6)
    // (b0) and (1, 3, 5, 7) (b1).
    const int hA = gq >> 1, digA = (gq & 1) ? 1 : 2;
    const int hB = gq >> 1;
    const bool useB = (gq & 1) == 0;
#pragma unroll
    for (int j = 0; j < NK32; ++j) {
      const int grp = WPC * tig + j;
      if (hA < G) {
        const uint2 v = *reinterpret_cast<const uint2*>(scratch + (hA * 3 + digA) * D + 8 * grp);
        qd[j][0] = v.x;
        qd[j][1] = v.y;
      } else {
        qd[j][0] = qd[j][1] = 0u;
      }
      if (useB && hB < G) {
        const uint2 v = *reinterpret_cast<const uint2*>(scratch + (hB * 3 + 0) * D + 8 * grp);
        qd[j][2] = v.x;
        qd[j][3] = v.y;
      } else {
        qd[j][2] = qd[j][3] = 0u;
      }
    }
    // the scratch is a ring stage that a bulk copy (async proxy) refills later: order this lane's
    // generic accesses to it before that copy
    fence_proxy_async_smem();
    __syncwarp();
  };

  // ---- per-segment softmax state (head tig; lane-partial l and beta)
  float oacc[NKB][4];
  float m_run, l_part, beta_part;
  auto reset = [&]() {
#pragma unroll
    for (int mb = 0; mb < NKB; ++mb) oacc[mb][0] = oacc[mb][1] = oacc[mb][2] = oacc[mb][3] = 0.f;
    m_run = kNegInf;
    l_part = 0.f;
    beta_part = 0.f;
  };

  // Which warps hold the partials of (b, g) (segment-table entry se of either segment): the
  // first INT8 / INT4 warps and their counts.  When one warp holds the whole INT8 segment and
  // the start of the INT4 segment, it runs one softmax across both regions (continuation) and
  // writes no INT8 partial: the INT8 count is then 0.  Every warp computes the same record.
  auto pair_split = [&](unsigned long long se, u32& w8a, u32& w4a, u32& n8p, u32& n4p) {
    const int cb = seg_b(se);
    const u32 cs8 = seg_cs8(se);
    const SegInfo si = seg_info<T8>(clamp_len(a.lens[cb], cap), a.s, a.w, a.nt8, a.smw);
    const u32 cs4 = cs8 + kU8<VB> * si.n8;
    w8a = divQ.div(cs8);
    w4a = divQ.div(cs4);
    n8p = si.n8 ? divQ.div(cs4 - kU8<VB>) - w8a + 1 : 0u;
    n4p = si.n4 ? divQ.div(cs4 + si.n4 - 1) - w4a + 1 : 0u;
    if (n8p == 1u && n4p >= 1u && w8a == w4a) n8p = 0u;
  };

  // Write the partial of the segment `se` (a segment-table entry).  The partials of (b, g) are
  // merged by merge_int4_kernel; when this is the only partial of (b, g) it is the output.
  auto flush = [&](unsigned long long se) {
    const int cb = seg_b(se), cg = seg_g(se), cseg = seg_kind(se);
    float l = l_part, beta = beta_part;
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      l += __shfl_xor_sync(FULL, l, o);
      beta += __shfl_xor_sync(FULL, beta, o);
    }
    u32 w8a, w4a, n8p, n4p;
    pair_split(se, w8a, w4a, n8p, n4p);
    const bool only = n8p + n4p == 1u && !a.rotate_v;  // rotated values: the merge rotates back
    const u32 sid = 2u * static_cast<u32>(cb * a.Hkv + cg) + static_cast<u32>(cseg);
    // where the merge finds the partials of (b, g); every writer of (b, g) stores the same record
    if (lane == 0) *reinterpret_cast<uint4*>(a.meta + 4 * (cb * a.Hkv + cg)) = make_uint4(w8a, w4a, n8p, n4p);
    if (tig < G) {
      // INT4: even output rows carry (c - 8), odd rows 16 (c - 8); INT8 rows carry c; bf16 values
      // carry the values.
      const float f1 = (cseg == 1 && !VB) ? 0.0625f : 1.f;
      const float sc = only ? (l > 0.f ? 1.f / l : 0.f) : 1.f;
      float* p = only ? a.out + (static_cast<size_t>(cb) * a.Hq + cg * G + tig) * D
                      : a.part + (static_cast<size_t>(wid + sid) * G + tig) * kPartRow<D>;
#pragma unroll
      for (int mb = 0; mb < NKB; ++mb) {
        const int d = Gm::DG * gq + 2 * mb;
        *reinterpret_cast<float2*>(p + d) = make_float2(((oacc[mb][0] + oacc[mb][1]) + beta) * sc,
                                                         (f1 * (oacc[mb][2] + oacc[mb][3]) + beta) * sc);
      }
      if (gq == 0) {
        if (!only)
          *reinterpret_cast<float2*>(p + D) = make_float2(m_run * qinv, l);
        else if (a.lse)
          a.lse[static_cast<size_t>(cb) * a.Hq + cg * G + tig] = l > 0.f ? (m_run * qinv + log2f(l)) * 0.69314718055994531f : kNegInf;
      }
    }
  };



  // Running-max update for this lane's logits of head tig.  Logits and the running max m_run are
  // kept unscaled (log2 units times 2^e, e the query's power-of-two normalisation); the returned
  // offset -m_run 2^-e makes exp2(fmaf(logit, qinv, offset)) the probability.
  auto softmax_update = [&](float tm) {
    tm = fmaxf(tm, __shfl_xor_sync(FULL, tm, 4));
    tm = fmaxf(tm, __shfl_xor_sync(FULL, tm, 8));
    tm = fmaxf(tm, __shfl_xor_sync(FULL, tm, 16));
    const float mn = fmaxf(m_run, tm);
    const bool grow = mn > m_run;
    if (__any_sync(FULL, grow)) {
      const float alpha = grow ? (m_run == kNegInf ? 0.f : exp2_fast((m_run - mn) * qinv)) : 1.f;
#pragma unroll
      for (int mb = 0; mb < NKB; ++mb) {
        oacc[mb][0] *= alpha;
        oacc[mb][1] *= alpha;
        oacc[mb][2] *= alpha;
        oacc[mb][3] *= alpha;
      }
      l_part *= alpha;
      beta_part *= alpha;
      m_run = mn;
    }
    return m_run == kNegInf ? 0.f : -m_run * qinv;
  };
  auto prob = [&](float lg, float off) { return exp2_fast(fmaf(lg, qinv, off)); };

  // PV B operand: hi/lo halves of pv for head gq>>1 of this lane's column, positions 2tig, 2tig+1
  // (b0) and 2tig+8, 2tig+9 (b1), gathered from the lanes that computed them.
  auto pv_fragments = [&](float pv0, float pv1, uint32_t& b0, uint32_t& b1) {
    const int hh = gq >> 1;
    const bool lo = gq & 1;
    const int src0 = 8 * tig + hh, src1 = src0 + 4;
    const float x0 = __shfl_sync(FULL, pv0, src0), x1 = __shfl_sync(FULL, pv0, src1);
    const float x2 = __shfl_sync(FULL, pv1, src0), x3 = __shfl_sync(FULL, pv1, src1);
    if (hh < G) {
      b0 = VB ? split_pair_bf16(x0, x1, lo) : split_pair(x0, x1, lo);
      b1 = VB ? split_pair_bf16(x2, x3, lo) : split_pair(x2, x3, lo);
    } else {
      b0 = b1 = 0u;
    }
  };

  // PV of one 16-row block of bf16 values (bf16 values) with probabilities p0, p1 (rows gq, gq + 8
  // of head tig).  Rows whose bit in `rows` is clear are zeroed in the A operand: their bytes may
  // be stale (a zero weight does not cancel a NaN pattern).
  auto pv_bf16 = [&](const uint8_t* vb, bool v0, bool v1, float p0, float p1, unsigned rows) {
    const float w0 = v0 ? p0 : 0.f, w1 = v1 ? p1 : 0.f;
    l_part += w0 + w1;
    uint32_t b0, b1;
    pv_fragments(w0, w1, b0, b1);
    constexpr int UPC = D / 32;
    uint32_t vw0[D / 8], vw1[D / 8];
#pragma unroll
    for (int u = 0; u < UPC; ++u) {
      const int uu = u ^ bf16_swz(D, tig, gq);
      const uint4 y0 = *reinterpret_cast<const uint4*>(vb + ((0 * 8 + gq) * 4 + tig) * (D / 2) + 16 * uu);
      const uint4 y1 = *reinterpret_cast<const uint4*>(vb + ((1 * 8 + gq) * 4 + tig) * (D / 2) + 16 * uu);
      vw0[4 * u] = y0.x; vw0[4 * u + 1] = y0.y; vw0[4 * u + 2] = y0.z; vw0[4 * u + 3] = y0.w;
      vw1[4 * u] = y1.x; vw1[4 * u + 1] = y1.y; vw1[4 * u + 2] = y1.z; vw1[4 * u + 3] = y1.w;
    }
    if (rows != 0xFFFFu) {
      const int t0 = 2 * tig;
      const uint32_t m0 = (((rows >> t0) & 1u) ? 0x0000ffffu : 0u) | (((rows >> (t0 + 1)) & 1u) ? 0xffff0000u : 0u);
      const uint32_t m1 = (((rows >> (t0 + 8)) & 1u) ? 0x0000ffffu : 0u) | (((rows >> (t0 + 9)) & 1u) ? 0xffff0000u : 0u);
#pragma unroll
      for (int x = 0; x < D / 8; ++x) {
        vw0[x] &= m0;
        vw1[x] &= m1;
      }
    }
#pragma unroll
    for (int mb = 0; mb < NKB; ++mb) mma_bf16(oacc[mb], vw0[2 * mb], vw0[2 * mb + 1], vw1[2 * mb], vw1[2 * mb + 1], b0, b1);
  };

  // QK^T of one INT4 tile block: logits (log2 units) of rows gq and gq + 8 for head tig.
  auto qk_int4 = [&](const uint8_t* tb, bool v0, bool v1, float& lg0, float& lg1) {
    // pair-row gq holds rows gq (low nibbles) and gq + 8 (high nibbles); this lane's 8-dim
    // groups 4 tig .. 4 tig + 3 are 8 W bytes at 8 W tig (16-byte halves swapped for odd gq
    // when D = 128): per group, word 0 = its even dims, word 1 = its odd dims
    uint32_t kw[2 * WPC];
    if constexpr (D == 128) {
      const int sw = gq & 1;
      lds_words<4>(tb + gq * D + 16 * ((2 * tig) ^ sw), *reinterpret_cast<uint32_t(*)[4]>(&kw[0]));
      lds_words<4>(tb + gq * D + 16 * ((2 * tig + 1) ^ sw), *reinterpret_cast<uint32_t(*)[4]>(&kw[4]));
    } else {
      lds_words<4>(tb + gq * D + 16 * tig, *reinterpret_cast<uint32_t(*)[4]>(&kw[0]));
    }
    int SA[4] = {0, 0, 0, 0}, SB[4] = {0, 0, 0, 0};
#pragma unroll
    for (int j = 0; j < NK32; ++j) {
      // A fragment: row gq = low nibbles, row gq + 8 = high nibbles kept in place (16 c, the
      // factor is removed from that row's logit below); k 0-15 even dims, k 16-31 odd dims
      const uint32_t e = kw[2 * j], o = kw[2 * j + 1];
      const uint32_t a0 = e & 0x0F0F0F0Fu, a1 = e & 0xF0F0F0F0u;
      const uint32_t a2 = o & 0x0F0F0F0Fu, a3 = o & 0xF0F0F0F0u;
      mma_u8s8(SA, a0, a1, a2, a3, qd[j][0], qd[j][1]);
      mma_u8s8(SB, a0, a1, a2, a3, qd[j][2], qd[j][3]);
    }
    const uint32_t kp0 = *reinterpret_cast<const uint32_t*>(tb + KPO + 4 * gq);
    const uint32_t kp1 = *reinterpret_cast<const uint32_t*>(tb + KPO + 4 * (gq + 8));
    const float ks0 = half_lo(kp0), kz0 = half_hi(kp0), ks1 = half_lo(kp1) * 0.0625f, kz1 = half_hi(kp1);
    // logit 2^e = s q_int.c + z sum(q_int), q_int.c = 2^16 S2 + (2^8 S1 + S0); the bracket is
    // below 2^30 in magnitude and exact in int32 (row gq + 8: 16 q_int.c, hence s / 16)
    const float R0 = fmaf(65536.f, static_cast<float>(SA[0]), static_cast<float>(SA[1] * 256 + SB[0]));
    const float R1 = fmaf(65536.f, static_cast<float>(SA[2]), static_cast<float>(SA[3] * 256 + SB[2]));
    lg0 = v0 ? fmaf(ks0, R0, kz0 * sumq) : kNegInf;
    lg1 = v1 ? fmaf(ks1, R1, kz1 * sumq) : kNegInf;
  };

  // PV of one INT4 tile block with probabilities p0, p1 (rows gq, gq + 8 of head tig).
  auto pv_int4 = [&](const uint8_t* tb, bool v0, bool v1, float p0, float p1) {
    const uint32_t vp0 = *reinterpret_cast<const uint32_t*>(tb + 16 * D + 64 + 4 * gq);
    const uint32_t vp1 = *reinterpret_cast<const uint32_t*>(tb + 16 * D + 64 + 4 * (gq + 8));
    const float vs0 = half_lo(vp0), vz0 = half_hi(vp0), vs1 = half_lo(vp1), vz1 = half_hi(vp1);
    l_part += (v0 ? p0 : 0.f) + (v1 ? p1 : 0.f);
    // v^ = z + s c = (z + 8 s) + s (c - 8): the MMA sees the centred codes, the per-position
    // constant goes to the scalar sum.
    beta_part += (v0 ? p0 * (vz0 + 8.f * vs0) : 0.f) + (v1 ? p1 * (vz1 + 8.f * vs1) : 0.f);
    uint32_t b0, b1;
    pv_fragments(v0 ? p0 * vs0 : 0.f, v1 ? p1 * vs1 : 0.f, b0, b1);
    uint32_t vw0[WPC], vw1[WPC];
    const uint8_t* vb = tb + 8 * D;
    lds_words<WPC>(vb + ((0 * 8 + gq) * 4 + tig) * Gm::CH, vw0);
    lds_words<WPC>(vb + ((1 * 8 + gq) * 4 + tig) * Gm::CH, vw1);
#pragma unroll
    for (int j = 0; j < WPC; ++j) {
      const uint32_t a8 = vw0[j] >> 8, c8 = vw1[j] >> 8;
      // m-blocks 2j (nibbles 0, 1) and 2j + 1 (nibbles 2, 3)
      mma_f16(oacc[2 * j], vcode<0>(vw0[j], a8), vcode<1>(vw0[j], a8), vcode<0>(vw1[j], c8), vcode<1>(vw1[j], c8),
              b0, b1);
      mma_f16(oacc[2 * j + 1], vcode<2>(vw0[j], a8), vcode<3>(vw0[j], a8), vcode<2>(vw1[j], c8),
              vcode<3>(vw1[j], c8), b0, b1);
    }
  };

  // ---- main loop over this warp's slots
  reset();
  build_query(sm.ring[warp][kStages - 1]);  // stage kStages-1 is not in flight
  int cur_bg;  // (b, g) whose query fragments are loaded
  {
    const unsigned long long se = sm.seg[warp][meta_seg(sm.meta[warp][0])];
    cur_bg = seg_b(se) * a.Hkv + seg_g(se);
  }
  // The wait-limit test: a wait on a barrier that nothing arrives on runs out, and the warp takes
  // the failure path below with its first copies in flight.
  bool failed = a.stall_test && !mbar_wait_bounded(&sm.stall[warp], 0u, a.err, a.wait_ns);
  int k = 0;
  while (!failed) {
    // the next slot's copies first: its descriptor is in the chunk being consumed, and the fill
    // below (page-table loads) then overlaps copies in flight
    if (lane == 0 && issue(k + kStages - 1)) ++issued;
    if ((k % kChunk) == 0) {
      // descriptors of slots [k + kChunk, k + 2 kChunk) while this chunk is consumed
      Cursor fc = sm.cur[warp];
      unsigned fs = sm.segno[warp];
      __syncwarp();
      fill_descriptors<D, T8, VB>(a, cap, c1, fc, lane, sm, warp, k + kChunk, fs);
      if (lane == 0) {
        sm.cur[warp] = fc;
        sm.segno[warp] = fs;
      }
      __syncwarp();
    }
    const int st = k % kStages;
    const bool ok = mbar_wait_bounded(&bars[st], static_cast<uint32_t>((k / kStages) & 1), a.err, a.wait_ns);
    if (__any_sync(FULL, !ok)) {
      failed = true;
      break;
    }
    const uint8_t* buf = sm.ring[warp][st];
    const int p = k % kRing;
    const unsigned meta = sm.meta[warp][p];
    const unsigned msk = sm.mask[warp][p];
    if (VB && meta_kind(meta) == kKindInt4) {
      // ----------------------------------------------------------- one page tile, bf16 values
      float l0, l1;
      if (msk == 0xFFFFu) {
        qk_int4(buf, true, true, l0, l1);
        const float off = softmax_update(fmaxf(l0, l1));
        pv_bf16(buf + Gm::VBO, true, true, prob(l0, off), prob(l1, off), 0xFFFFu);
      } else {
        const bool v0 = tig < G && ((msk >> gq) & 1u), v1 = tig < G && ((msk >> (gq + 8)) & 1u);
        qk_int4(buf, v0, v1, l0, l1);
        const float off = softmax_update(fmaxf(l0, l1));
        pv_bf16(buf + Gm::VBO, v0, v1, prob(l0, off), prob(l1, off), msk);
      }
    } else if (meta_kind(meta) == kKindInt4) {
      // ----------------------------------------------------------- two INT4 tiles
      float lA0, lA1, lB0 = kNegInf, lB1 = kNegInf;
      if (msk == 0xFFFFFFFFu) {
        // both tiles present with all 32 rows valid (the common case): no row masking.  Lanes of
        // absent heads (tig >= G) compute finite values that nothing reads.
        qk_int4(buf, true, true, lA0, lA1);
        qk_int4(buf + T4B, true, true, lB0, lB1);
        const float off = softmax_update(fmaxf(fmaxf(lA0, lA1), fmaxf(lB0, lB1)));
        pv_int4(buf, true, true, prob(lA0, off), prob(lA1, off));
        pv_int4(buf + T4B, true, true, prob(lB0, off), prob(lB1, off));
      } else {
        const bool two = (meta & kMetaTwo) != 0;
        const bool vA0 = tig < G && ((msk >> gq) & 1u), vA1 = tig < G && ((msk >> (gq + 8)) & 1u);
        const bool vB0 = tig < G && ((msk >> (gq + 16)) & 1u), vB1 = tig < G && ((msk >> (gq + 24)) & 1u);
        qk_int4(buf, vA0, vA1, lA0, lA1);
        if (two) qk_int4(buf + T4B, vB0, vB1, lB0, lB1);
        const float off = softmax_update(fmaxf(fmaxf(lA0, lA1), fmaxf(lB0, lB1)));
        pv_int4(buf, vA0, vA1, prob(lA0, off), prob(lA1, off));
        if (two) pv_int4(buf + T4B, vB0, vB1, prob(lB0, off), prob(lB1, off));
      }
    } else {
      // ----------------------------------------------------------- one INT8 tile (K half, V half)
      const bool v0 = tig < G && ((msk >> gq) & 1u), v1 = tig < G && ((msk >> (gq + 8)) & 1u);
      constexpr int NW8 = 2 * WPC;  // int8 words per row chunk
      uint32_t kw0[NW8], kw1[NW8];
#pragma unroll
      for (int u = 0; u < NW8 / 4; ++u) {
        const int lu = (NW8 / 4) * tig + u;  // logical 16-byte unit of the row
        const uint4 x0 = *reinterpret_cast<const uint4*>(buf + gq * D + 16 * (lu ^ (gq & 1)));
        const uint4 x1 = *reinterpret_cast<const uint4*>(buf + (gq + 8) * D + 16 * (lu ^ ((gq + 8) & 1)));
        kw0[4 * u] = x0.x; kw0[4 * u + 1] = x0.y; kw0[4 * u + 2] = x0.z; kw0[4 * u + 3] = x0.w;
        kw1[4 * u] = x1.x; kw1[4 * u + 1] = x1.y; kw1[4 * u + 2] = x1.z; kw1[4 * u + 3] = x1.w;
      }
      int SA[4] = {0, 0, 0, 0}, SB[4] = {0, 0, 0, 0};
#pragma unroll
      for (int j = 0; j < NK32; ++j) {
        // words 2j, 2j + 1 of a row: dims 8W + 0..3 and 8W + 4..7; even dims, then odd dims
        const uint32_t a0 = prmt(kw0[2 * j], kw0[2 * j + 1], 0x6420u), a2 = prmt(kw0[2 * j], kw0[2 * j + 1], 0x7531u);
        const uint32_t a1 = prmt(kw1[2 * j], kw1[2 * j + 1], 0x6420u), a3 = prmt(kw1[2 * j], kw1[2 * j + 1], 0x7531u);
        mma_s8s8(SA, a0, a1, a2, a3, qd[j][0], qd[j][1]);
        mma_s8s8(SB, a0, a1, a2, a3, qd[j][2], qd[j][3]);
      }
      const float ks0 = __half2float(*reinterpret_cast<const __half*>(buf + 16 * D + 2 * gq));
      const float ks1 = __half2float(*reinterpret_cast<const __half*>(buf + 16 * D + 2 * (gq + 8)));
      // |2^8 S1 + S0| < 2^31 for 8-bit codes
      const float R0 = fmaf(65536.f, static_cast<float>(SA[0]), static_cast<float>(SA[1] * 256 + SB[0]));
      const float R1 = fmaf(65536.f, static_cast<float>(SA[2]), static_cast<float>(SA[3] * 256 + SB[2]));
      const float lg0 = v0 ? ks0 * R0 : kNegInf;
      const float lg1 = v1 ? ks1 * R1 : kNegInf;
      const float off = softmax_update(fmaxf(lg0, lg1));
      const float p0 = prob(lg0, off), p1 = prob(lg1, off);
      if constexpr (VB) {
        pv_bf16(buf + Gm::VB8O, v0, v1, p0, p1, msk);
      } else {
        l_part += (v0 ? p0 : 0.f) + (v1 ? p1 : 0.f);
        const uint8_t* vb = buf + T4B;  // V half
        const float vs0 = __half2float(*reinterpret_cast<const __half*>(vb + 16 * D + 2 * gq));
        const float vs1 = __half2float(*reinterpret_cast<const __half*>(vb + 16 * D + 2 * (gq + 8)));
        uint32_t b0, b1;
        pv_fragments(v0 ? p0 * vs0 : 0.f, v1 ? p1 * vs1 : 0.f, b0, b1);
        constexpr int NW = Gm::CH8 / 4;  // words per pair chunk (8 or 4)
        uint32_t vw0[NW], vw1[NW];
#pragma unroll
        for (int hv = 0; hv < NW / 4; ++hv) {
          const int phys = (Gm::CH8 >= 32) ? (hv ^ (gq & 1)) : hv;
          const uint4 x0 = *reinterpret_cast<const uint4*>(vb + ((0 * 8 + gq) * 4 + tig) * Gm::CH8 + 16 * phys);
          const uint4 x1 = *reinterpret_cast<const uint4*>(vb + ((1 * 8 + gq) * 4 + tig) * Gm::CH8 + 16 * phys);
          vw0[4 * hv] = x0.x; vw0[4 * hv + 1] = x0.y; vw0[4 * hv + 2] = x0.z; vw0[4 * hv + 3] = x0.w;
          vw1[4 * hv] = x1.x; vw1[4 * hv + 1] = x1.y; vw1[4 * hv + 2] = x1.z; vw1[4 * hv + 3] = x1.w;
        }
#pragma unroll
        for (int mb = 0; mb < NKB; ++mb) {
          const uint32_t w0 = vw0[mb] ^ 0x80808080u, w1 = vw1[mb] ^ 0x80808080u;
          mma_f16(oacc[mb], i8x2_to_h2<0x4140>(w0), i8x2_to_h2<0x4342>(w0), i8x2_to_h2<0x4140>(w1),
                  i8x2_to_h2<0x4342>(w1), b0, b1);
        }
      }
    }
    __syncwarp();

    if (meta & kMetaLast) {
      const unsigned long long se = sm.seg[warp][meta_seg(meta)];
      bool cont = false;  // region continuation into the INT4 segment of the same (b, g)
      if (seg_kind(se) == 0) {
        u32 w8a, w4a, n8p, n4p;
        pair_split(se, w8a, w4a, n8p, n4p);
        cont = n8p == 0u && n4p >= 1u && w4a == static_cast<u32>(wid);
      }
      if (cont) {
        // INT4 slots accumulate their odd output rows 16x (removed when the partial is written):
        // bring the INT8 region's rows to that convention
        if constexpr (!VB) {
#pragma unroll
          for (int mb = 0; mb < NKB; ++mb) {
            oacc[mb][2] *= 16.f;
            oacc[mb][3] *= 16.f;
          }
        }
      } else {
        flush(se);
        reset();
      }
      const unsigned nmeta = sm.meta[warp][(k + 1) % kRing];
      if (meta_kind(nmeta) == kKindNone) break;  // end of this warp's stream
      const unsigned long long ns = sm.seg[warp][meta_seg(nmeta)];
      const int nbg = seg_b(ns) * a.Hkv + seg_g(ns);
      if (nbg != cur_bg) {
        cur_bg = nbg;
        load_q_regs(seg_b(ns), seg_g(ns));
        build_query(sm.ring[warp][st]);  // this slot's stage is free now
      }
    }
    ++k;
  }
  if (failed) {
    // A copy did not arrive in time: wait (bounded) for every copy this warp still has in
    // flight so none lands in shared memory after the CTA exits, then leave.
    issued = __shfl_sync(FULL, issued, 0);
    for (int j = k; j < issued; ++j)
      mbar_wait_bounded(&bars[j % kStages], static_cast<uint32_t>((j / kStages) & 1), a.err, a.wait_ns);
  }
}

// ------------------------------------------------------------------ LSE merge kernel

// Merge of the partials of (sequence b, query head j): MW warps per (b, j), MW chosen on the host
// so that a warp has at most kMergeBatch partials (MW = 1: four (b, j) per CTA of 4 warps; else one
// (b, j) per CTA of MW warps).  The decode kernel left, per (b, g), where the n partials are
// (meta); warp w of the MW merges head j % G of partials [w n / MW, (w+1) n / MW) in one pass of
// batches of kMergeBatch rows, each batch one round trip.  With MW > 1, warp 0 combines the
// warps' (M, L, o) through shared memory.  (b, g) with at most one partial, and sequences of
// length 0 (record of zeros), were written by the decode kernel.  Launched as a programmatic
// dependent of the decode kernel: griddepcontrol.wait orders every read of its results after its
// completion.
constexpr int kMergeThreads = 128;
constexpr int kMergeBatch = 16;

template <int D, int G, int MW>
__global__ void __launch_bounds__(MW == 1 ? kMergeThreads : 32 * MW) merge_int4_kernel(const DecodeArgs a) {
  constexpr int PER = D / 32;
  constexpr int kInFlight = kMergeBatch;
  constexpr int RS = kPartRow<D>;
  using VecT = typename std::conditional<PER == 4, float4, float2>::type;
  __shared__ float smo[MW][D];
  __shared__ float smM[MW], smL[MW];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int sub = MW == 1 ? 0 : warp;                       // warp within the item
  const int item = MW == 1 ? blockIdx.x * (kMergeThreads / 32) + warp : blockIdx.x;
  if (item >= a.B * a.Hq) return;
  const int b = item / a.Hq, j = item - b * a.Hq;
  const int g = j / G, hd = j - g * G;
  pdl_wait();
  const uint4 mt = *reinterpret_cast<const uint4*>(a.meta + 4 * (b * a.Hkv + g));
  {
    // A record whose partial rows fall outside the workspace can only be left over from a decode
    // that stopped early (a wait that ran out): report it and write no output from it.
    const unsigned long long rows = static_cast<unsigned long long>(a.W) + 2ull * a.B * a.Hkv;
    const unsigned long long sid8 = 2ull * (b * a.Hkv + g);
    const bool bad8 = mt.z && static_cast<unsigned long long>(mt.x) + mt.z + sid8 > rows;
    const bool bad4 = mt.w && static_cast<unsigned long long>(mt.y) + mt.w + sid8 + 1ull > rows;
    if (bad8 || bad4 || mt.z > rows || mt.w > rows) {
      if (lane == 0 && sub == 0) atomicOr(a.err, KV4_DEVERR_RECORD);
      return;
    }
  }
  const int n8p = static_cast<int>(mt.z), n = static_cast<int>(mt.z + mt.w);
  if (n == 0 || (n == 1 && !a.rotate_v)) return;  // uniform over the item's warps
  const PartRows pr{n8p, mt.x, mt.y, 2u * static_cast<u32>(b * a.Hkv + g)};
  const int t0 = sub * n / MW, t1 = (sub + 1) * n / MW;
  float M = kNegInf, L = 0.f, o[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) o[e] = 0.f;
  // One pass, kInFlight partials at a time: every lane loads its slice of each row together with
  // the row's (m, l) (the same address in every lane), so a batch costs one memory round trip; the
  // running maximum is raised partial by partial (warp-uniform).
  for (int base = t0; base < t1; base += kInFlight) {
    VecT v[kInFlight];
    float2 ml[kInFlight];
#pragma unroll
    for (int u = 0; u < kInFlight; ++u) {
      const int t = base + u < t1 ? base + u : t0;  // past the end: reload the first row, unused
      const unsigned long long row = pr.row(t, G, RS) + hd * RS;
      v[u] = __ldcg(reinterpret_cast<const VecT*>(a.part + row + lane * PER));
      ml[u] = __ldcg(reinterpret_cast<const float2*>(a.part + row + D));
    }
#pragma unroll
    for (int u = 0; u < kInFlight; ++u) {
      if (base + u >= t1 || !(ml[u].y > 0.f)) continue;
      if (ml[u].x > M) {
        const float sc = M == kNegInf ? 0.f : exp2f(M - ml[u].x);
        L *= sc;
#pragma unroll
        for (int e = 0; e < PER; ++e) o[e] *= sc;
        M = ml[u].x;
      }
      const float w = exp2f(ml[u].x - M);
      L = fmaf(w, ml[u].y, L);
      const float* vv = reinterpret_cast<const float*>(&v[u]);
#pragma unroll
      for (int e = 0; e < PER; ++e) o[e] = fmaf(w, vv[e], o[e]);
    }
  }
  if constexpr (MW > 1) {
#pragma unroll
    for (int e = 0; e < PER; ++e) smo[sub][lane * PER + e] = o[e];
    if (lane == 0) {
      smM[sub] = M;
      smL[sub] = L;
    }
    __syncthreads();
    if (sub != 0) return;
    M = kNegInf;
#pragma unroll
    for (int w = 0; w < MW; ++w)
      if (smL[w] > 0.f) M = fmaxf(M, smM[w]);
    L = 0.f;
#pragma unroll
    for (int e = 0; e < PER; ++e) o[e] = 0.f;
#pragma unroll
    for (int w = 0; w < MW; ++w) {
      const float f = smL[w] > 0.f ? exp2f(smM[w] - M) : 0.f;
      L += f * smL[w];
#pragma unroll
      for (int e = 0; e < PER; ++e) o[e] = fmaf(f, smo[w][lane * PER + e], o[e]);
    }
  }
  float* out = a.out + (static_cast<size_t>(b) * a.Hq + j) * D + lane * PER;
  const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
  for (int e = 0; e < PER; ++e) o[e] *= inv;
  if (a.rotate_v) {
    // values were stored as H diag(s) v: o = diag(s) H o_rot / h (lane holds dims PER lane + e)
    const int h = a.h;
#pragma unroll
    for (int st = 1; st < PER; st <<= 1)
      if (st < h)
#pragma unroll
        for (int e = 0; e < PER; ++e)
          if ((e & st) == 0) {
            const float x0 = o[e], x1 = o[e + st];
            o[e] = x0 + x1;
            o[e + st] = x0 - x1;
          }
#pragma unroll
    for (int st = PER; st < D; st <<= 1)
      if (st < h) {
        const int m = st / PER;
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int e = 0; e < PER; ++e) {
          const float x = __shfl_xor_sync(FULL, o[e], m);
          o[e] = upper ? x - o[e] : o[e] + x;
        }
      }
    const float ih = 1.f / static_cast<float>(h);
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      const int d = lane * PER + e;
      o[e] = __uint_as_float(__float_as_uint(o[e] * ih) ^ (((a.signs[d >> 5] >> (d & 31)) & 1u) << 31));
    }
  }
  if constexpr (PER == 4)
    *reinterpret_cast<float4*>(out) = make_float4(o[0], o[1], o[2], o[3]);
  else
    *reinterpret_cast<float2*>(out) = make_float2(o[0], o[1]);
  if (a.lse && lane == 0) a.lse[static_cast<size_t>(b) * a.Hq + j] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : kNegInf;
}

// Launch of the merge kernel as a programmatic dependent of the preceding decode kernel.
template <int D, int G>
cudaError_t launch_merge(const DecodeArgs& a, cudaStream_t st) {
  const int items = a.B * a.Hq;
  // partials of an average (b, g): its share of the split warps, plus the two segment ends
  const long long per = static_cast<long long>(a.W) / (static_cast<long long>(a.B) * a.Hkv) + 2;
  const int mw = per <= kMergeBatch ? 1 : per <= 4 * kMergeBatch ? 4 : per <= 8 * kMergeBatch ? 8 : 16;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(mw > 1 ? items : (items + kMergeThreads / 32 - 1) / (kMergeThreads / 32)));
  cfg.blockDim = dim3(mw > 1 ? 32 * mw : kMergeThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  switch (mw) {
    case 1: return cudaLaunchKernelEx(&cfg, merge_int4_kernel<D, G, 1>, a);
    case 4: return cudaLaunchKernelEx(&cfg, merge_int4_kernel<D, G, 4>, a);
    case 8: return cudaLaunchKernelEx(&cfg, merge_int4_kernel<D, G, 8>, a);
    default: return cudaLaunchKernelEx(&cfg, merge_int4_kernel<D, G, 16>, a);
  }
}

// One instantiation of the split-K kernel, launched as a programmatic dependent (its dynamic
// shared-memory limit raised once per device).
template <int D, int G, int QT, bool T8, bool VB>
cudaError_t launch_variant(const cudaLaunchConfig_t& cfg0, const DecodeArgs& a, std::atomic<uint64_t>& done) {
  const int smem = static_cast<int>(sizeof(Smem<D, VB>));
  cudaError_t e = ensure_smem_limit(decode_int4_kernel<D, G, QT, T8, VB>, smem, done);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = cfg0;
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  return cudaLaunchKernelEx(&cfg, decode_int4_kernel<D, G, QT, T8, VB>, a);
}

template <int D, int G, int QT>
cudaError_t launch_qt(const cudaLaunchConfig_t& cfg, const DecodeArgs& a, std::atomic<uint64_t>* done) {
  // bf16 values: every side tile is visited (masked), so one kernel serves every side-cache size
  if (a.vbf) return launch_variant<D, G, QT, false, true>(cfg, a, done[2]);
  if (a.nt8 > kTightSideTiles) return launch_variant<D, G, QT, true, false>(cfg, a, done[1]);
  return launch_variant<D, G, QT, false, false>(cfg, a, done[0]);
}

template <int D, int G>
cudaError_t launch_dg(const DecodeArgs& a, int ctas, cudaStream_t st) {
  static std::atomic<uint64_t> done[3][3];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(ctas));
  cfg.blockDim = dim3(kWarps * 32);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e;
  if (a.q_dtype == KV4_F32) e = launch_qt<D, G, KV4_F32>(cfg, a, done[0]);
  else if (a.q_dtype == KV4_BF16) e = launch_qt<D, G, KV4_BF16>(cfg, a, done[1]);
  else e = launch_qt<D, G, KV4_F16>(cfg, a, done[2]);
  if (e != cudaSuccess) return e;
  return launch_merge<D, G>(a, st);
}

}  // namespace

int decode_warps_per_cta() { return kWarps; }
int decode_ctas_per_sm() { return kCtasPerSm; }

size_t decode_smem_bytes(int D, int G) {
  (void)G;
  return D == 128 ? sizeof(Smem<128, true>) : sizeof(Smem<64, true>);
}

cudaError_t launch_decode_int4(DecodeArgs a, int D, int G, int ctas, cudaStream_t st) {
  a.W = ctas * kWarps;
  note_launches(2);
  if (D == 128) {
    if (G == 4) return launch_dg<128, 4>(a, ctas, st);
    if (G == 2) return launch_dg<128, 2>(a, ctas, st);
    return launch_dg<128, 1>(a, ctas, st);
  }
  if (G == 4) return launch_dg<64, 4>(a, ctas, st);
  if (G == 2) return launch_dg<64, 2>(a, ctas, st);
  return launch_dg<64, 1>(a, ctas, st);
}

}  // namespace kv4
