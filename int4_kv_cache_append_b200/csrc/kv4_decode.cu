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
// ceil((s+w)/16) tiles and an INT4 segment of the 16-position tiles covering [s, max(s, L-w)).
// A tile is one or two "slots" of at most 16*(D+8) bytes: an INT4 tile is one slot, an INT8 tile
// two (its K half and its V half).  All slots of all segments form one sequence; warp w of the
// launch takes the tiles whose first slot lies in [w*Q, (w+1)*Q), Q = ceil(total / warps), so
// every warp streams the same number of bytes regardless of the length mix.  A warp writes one
// partial (o, m, l) for every segment it touches, at index w + segment_id (unique because each
// step along the sequence advances the warp, the segment, or both), and a second kernel merges
// the partials of each (b, q head) with the LSE rule.
//
// Per warp: a ring of kStages shared-memory stages fed by 1-D bulk copies (cp.async.bulk, one
// per slot, issued by lane 0 kStages-1 slots ahead, completion on an mbarrier per stage).  The
// G query heads of the KV group and hi/lo fp16 halves of each query form the 8 columns of an
// m16n8k16 MMA: QK^T takes 16 positions x 16 dims per MMA with the codes as the A operand
// converted in registers; PV takes 16 dims x 16 positions with the (p * scale) hi/lo halves as
// the B operand.  Everything else (softmax, scale/offset, rescaling) runs in fp32 registers.
#include <cuda_bf16.h>
#include <math.h>

#include "kv4_device.cuh"
#include "kv4_internal.h"
#include "kv4_layout.cuh"

namespace kv4 {
namespace {

constexpr unsigned FULL = 0xffffffffu;
constexpr int kWarps = 8;
constexpr int kStages = 4;
constexpr float kNegInf = -__builtin_huge_valf();

// ------------------------------------------------------------------ schedule (shared with merge)

struct SegInfo {
  int n8;     // INT8 tiles (each 2 slots)
  int n4;     // INT4 tiles (each 1 slot)
  int t4a;    // first INT4 tile (absolute 16-position tile index)
  int m_end;  // INT4 region end position
  int L;
};

__device__ __forceinline__ int clamp_len(int L, int cap) { return L < 0 ? 0 : (L > cap ? cap : L); }

__device__ __forceinline__ SegInfo seg_info(int L, int s, int w, int nt8) {
  SegInfo r;
  r.L = L;
  r.n8 = L > 0 ? nt8 : 0;
  r.m_end = max(s, L - w);
  r.t4a = s >> 4;
  r.n4 = (r.m_end > s) ? ((r.m_end - 1) >> 4) - r.t4a + 1 : 0;
  return r;
}

__device__ __forceinline__ long long head_cost(const SegInfo& si) { return 2LL * si.n8 + si.n4; }

__device__ __forceinline__ long long warp_incl_scan(long long v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long t = __shfl_up_sync(FULL, v, o);
    if (lane >= o) v += t;
  }
  return v;
}

// Total slot count over all sequences (every lane gets the same value).
__device__ long long total_cost(const DecodeArgs& a, int cap, int lane) {
  long long run = 0;
  for (int base = 0; base < a.B; base += 32) {
    const int b = base + lane;
    long long c = 0;
    if (b < a.B) c = a.Hkv * head_cost(seg_info(clamp_len(a.lens[b], cap), a.s, a.w, a.nt8));
    run += __shfl_sync(FULL, warp_incl_scan(c, lane), 31);
  }
  return run;
}

// Sequence containing slot position c (c < total); *bstart = first slot of that sequence.
__device__ int find_seq(const DecodeArgs& a, int cap, int lane, long long c, long long* bstart) {
  long long run = 0;
  for (int base = 0; base < a.B; base += 32) {
    const int b = base + lane;
    long long cb = 0;
    if (b < a.B) cb = a.Hkv * head_cost(seg_info(clamp_len(a.lens[b], cap), a.s, a.w, a.nt8));
    const long long incl = warp_incl_scan(cb, lane);
    const long long tot = __shfl_sync(FULL, incl, 31);
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

__device__ __forceinline__ long long quota(long long total, int W) {
  long long q = (total + W - 1) / W;
  return q < 2 ? 2 : q;
}

// ------------------------------------------------------------------ slot cursor

struct Cursor {
  int b, g, seg;        // seg 0 = INT8 region, 1 = INT4 region
  int i;                // tile index within the segment
  int half;             // INT8 tiles: 0 = K half, 1 = V half
  int n;                // tiles in the segment
  long long cost;       // slot position
  SegInfo si;
  bool valid;
};

__device__ __forceinline__ long long tile_start(const Cursor& c) { return c.seg == 0 ? c.cost - c.half : c.cost; }

// Move to the next non-empty segment starting at (b, g, seg) (inclusive).
__device__ void settle(const DecodeArgs& a, int cap, Cursor& c) {
  while (true) {
    if (c.b >= a.B) {
      c.valid = false;
      return;
    }
    c.n = c.seg == 0 ? c.si.n8 : c.si.n4;
    if (c.i < c.n) return;
    c.i = 0;
    c.half = 0;
    if (c.seg == 0) {
      c.seg = 1;
    } else {
      c.seg = 0;
      if (++c.g == a.Hkv) {
        c.g = 0;
        if (++c.b < a.B) c.si = seg_info(clamp_len(a.lens[c.b], cap), a.s, a.w, a.nt8);
      }
    }
  }
}

__device__ __forceinline__ void advance(const DecodeArgs& a, int cap, Cursor& c) {
  c.cost += 1;
  if (c.seg == 0 && c.half == 0) {
    c.half = 1;
    return;
  }
  c.half = 0;
  c.i += 1;
  settle(a, cap, c);
}

// First slot of the first tile whose start is >= c0.
__device__ Cursor cursor_at(const DecodeArgs& a, int cap, int lane, long long c0) {
  Cursor c;
  long long bstart;
  c.b = find_seq(a, cap, lane, c0, &bstart);
  c.valid = c.b < a.B;
  if (!c.valid) return c;
  c.si = seg_info(clamp_len(a.lens[c.b], cap), a.s, a.w, a.nt8);
  const long long ch = head_cost(c.si);
  const long long off = c0 - bstart;
  c.g = static_cast<int>(off / ch);
  const long long r = off - c.g * ch;
  c.half = 0;
  if (r < 2LL * c.si.n8) {
    c.seg = 0;
    c.i = static_cast<int>((r + 1) >> 1);
    c.cost = c0 + (r & 1);
  } else {
    c.seg = 1;
    c.i = static_cast<int>(r - 2LL * c.si.n8);
    c.cost = c0;
  }
  settle(a, cap, c);
  return c;
}

// ------------------------------------------------------------------ the partial kernel

template <int D, int G>
struct Smem {
  uint8_t ring[kWarps][kStages][Geo<D>::T4B];
  float qbuf[kWarps][G][D];
  uint64_t bar[kWarps][kStages];
};

__device__ __forceinline__ uint32_t nib2h_rt(uint32_t w, int k) {
  if (k == 0) return nib2h<0>(w);
  if (k == 1) return nib2h<1>(w);
  if (k == 2) return nib2h<2>(w);
  return nib2h<3>(w);
}

// (1 + c/16) - 1.5 = (c - 8)/16, exact in fp16: centred V codes keep the PV accumulators near
// the size of the result instead of carrying the affine offset through every tile.
__device__ __forceinline__ uint32_t centred(uint32_t x) {
  __half2 v = *reinterpret_cast<const __half2*>(&x);
  v = __hsub2(v, __halves2half2(__ushort_as_half(0x3E00), __ushort_as_half(0x3E00)));  // 1.5
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ __half split_part(float x, bool lo) {
  const __half hi = __float2half_rn(x);
  return lo ? __float2half_rn(x - __half2float(hi)) : hi;
}

__device__ __forceinline__ float exp2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Valid side rows for a sequence of length L: sink rows R < min(s, L); ring row s + i holds
// the recent position j in [max(s, L-w), L) with j mod w = i.
__device__ __forceinline__ bool side_row_valid(int R, int L, int s, int w) {
  if (R < s) return R < L;
  if (R >= s + w || L <= s) return false;
  const int n = L - s;
  if (n >= w) return true;
  const int i = R - s;
  int d = (i - s) % w;
  if (d < 0) d += w;
  return d < n;
}

template <int D, int G, int QT>
__device__ __forceinline__ float load_q(const void* q, size_t i) {
  if constexpr (QT == KV4_F32) return reinterpret_cast<const float*>(q)[i];
  else if constexpr (QT == KV4_BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(q)[i]);
  else return __half2float(reinterpret_cast<const __half*>(q)[i]);
}

template <int D, int G, int QT>
__global__ void __launch_bounds__(kWarps * 32, 2) decode_int4_kernel(const DecodeArgs a) {
  using Gm = Geo<D>;
  constexpr int NKB = Gm::NKB;
  constexpr int WPC = Gm::WPC;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  Smem<D, G>& sm = *reinterpret_cast<Smem<D, G>*>(smem_raw);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, tig = lane & 3;
  const int wid = blockIdx.x * kWarps + warp;
  const int cap = a.stride * a.P;

  uint64_t* bars = sm.bar[warp];
  if (lane == 0) {
    for (int i = 0; i < kStages; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
  }
  __syncwarp();

  const long long total = total_cost(a, cap, lane);
  const long long Q = quota(total, a.W);
  const long long c0 = static_cast<long long>(wid) * Q;
  if (c0 >= total) return;
  const long long c1 = c0 + Q;

  Cursor cons = cursor_at(a, cap, lane, c0);
  if (!cons.valid || tile_start(cons) >= c1) return;
  Cursor prod = cons;  // lane 0 uses it

  // Issue the bulk copy of one slot into stage `st`.
  auto issue = [&](const Cursor& c, int st) {
    const void* src = nullptr;
    uint32_t bytes;
    if (c.seg == 1) {
      const int ti = c.si.t4a + c.i;
      const int lp = (ti * 16) / a.P;
      const int page = a.page_table[static_cast<size_t>(c.b) * a.stride + lp];
      bytes = Gm::T4B;
      if (page >= 0 && page < a.max_pages)
        src = a.pool + static_cast<size_t>(page) * a.page_bytes + static_cast<size_t>(c.g) * a.P * (D + 8) +
              static_cast<size_t>((ti * 16 - lp * a.P) >> 4) * Gm::T4B;
    } else {
      bytes = Gm::H8B;
      src = a.side + static_cast<size_t>(c.b) * a.side_slot_bytes + static_cast<size_t>(c.g) * a.nt8 * Gm::T8B +
            static_cast<size_t>(c.i) * Gm::T8B + static_cast<size_t>(c.half) * Gm::H8B;
    }
    if (src) {
      mbar_arrive_expect_tx(&bars[st], bytes);
      bulk_g2s(sm.ring[warp][st], src, bytes, &bars[st]);
    } else {
      atomicOr(a.err, KV4_DEVERR_PAGE_RANGE);
      mbar_arrive_expect_tx(&bars[st], 0);
    }
  };

  // ---- per-(b, g) query state
  uint32_t qf[NKB][2];
  float sumq = 0.f, qinv = 1.f;
  float* qb = &sm.qbuf[warp][0][0];

  auto load_query = [&](int b, int g) {
    // Rotate each query head of the group (H/h), scale to log2 softmax units, normalise by a
    // power of two so that the fp16 hi/lo halves stay in the normal range.
    const bool act = lane < D / 4;
#pragma unroll
    for (int i = 0; i < G; ++i) {
      const size_t q0 = (static_cast<size_t>(b) * a.Hq + static_cast<size_t>(g) * G + i) * D + 4 * lane;
      float x[4] = {0.f, 0.f, 0.f, 0.f};
      if (act)
#pragma unroll
        for (int e = 0; e < 4; ++e) x[e] = load_q<D, G, QT>(a.q, q0 + e);
      const int h = a.h;
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
      for (int st = 4; st < h; st <<= 1) {
        const int m = st >> 2;
        const bool upper = (lane & m) != 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float o = __shfl_xor_sync(FULL, x[e], m);
          x[e] = upper ? o - x[e] : x[e] + o;
        }
      }
      const float sc = a.qscale / static_cast<float>(h);
      float amax = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        x[e] *= sc;
        amax = fmaxf(amax, fabsf(x[e]));
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(FULL, amax, o));
      // 2^(14 - floor(log2 amax)) puts max|q| in [2^14, 2^15).
      int ex = amax > 0.f ? ((__float_as_int(amax) >> 23) & 0xff) - 127 : 0;
      ex = max(min(ex, 100), -100);
      const float up = __int_as_float((127 + 14 - ex) << 23);
      const float down = __int_as_float((127 - 14 + ex) << 23);
      float ps = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        x[e] *= up;
        const __half hi = __float2half_rn(x[e]);
        const __half lo = __float2half_rn(x[e] - __half2float(hi));
        ps += __half2float(hi) + __half2float(lo);
      }
      if (act) *reinterpret_cast<float4*>(qb + i * D + 4 * lane) = make_float4(x[0], x[1], x[2], x[3]);
#pragma unroll
      for (int o = 16; o; o >>= 1) ps += __shfl_xor_sync(FULL, ps, o);
      if (tig == i) {
        sumq = ps;
        qinv = down;
      }
    }
    __syncwarp();
    const int hh = gq >> 1;
    const bool lo = gq & 1;
#pragma unroll
    for (int kb = 0; kb < NKB; ++kb) {
      const int W = WPC * tig + (kb >> 1), k0 = 2 * (kb & 1);
      if (hh < G) {
        const float* qh = qb + hh * D;
        qf[kb][0] = pack_h2(split_part(qh[8 * W + k0], lo), split_part(qh[8 * W + k0 + 4], lo));
        qf[kb][1] = pack_h2(split_part(qh[8 * W + k0 + 1], lo), split_part(qh[8 * W + k0 + 5], lo));
      } else {
        qf[kb][0] = 0u;
        qf[kb][1] = 0u;
      }
    }
    __syncwarp();
  };

  // ---- per-segment softmax state (head tig; lane-partial l and beta)
  float oacc[NKB][4];
  float m_run, l_part, beta_part;
  float p_keep0 = 0.f, p_keep1 = 0.f;  // INT8: probabilities carried from the K half to the V half
  bool v_keep0 = false, v_keep1 = false;
  auto reset = [&]() {
#pragma unroll
    for (int mb = 0; mb < NKB; ++mb) oacc[mb][0] = oacc[mb][1] = oacc[mb][2] = oacc[mb][3] = 0.f;
    m_run = kNegInf;
    l_part = 0.f;
    beta_part = 0.f;
  };

  auto flush = [&](const Cursor& c) {
    float l = l_part, beta = beta_part;
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      l += __shfl_xor_sync(FULL, l, o);
      beta += __shfl_xor_sync(FULL, beta, o);
    }
    if (tig < G) {
      const float fV = c.seg == 1 ? 16.f : 1.f;
      const long long sid = 2LL * (static_cast<long long>(c.b) * a.Hkv + c.g) + c.seg;
      float* p = a.part + (static_cast<size_t>(wid + sid) * G + tig) * (D + 2);
#pragma unroll
      for (int mb = 0; mb < NKB; ++mb) {
        const int d = Gm::DG * gq + 2 * mb;
        *reinterpret_cast<float2*>(p + d) =
            make_float2(fV * (oacc[mb][0] + oacc[mb][1]) + beta, fV * (oacc[mb][2] + oacc[mb][3]) + beta);
      }
      if (gq == 0) *reinterpret_cast<float2*>(p + D) = make_float2(m_run, l);
    }
  };

  // Softmax update for this lane's two positions (gq and gq + 8) of head tig.
  auto softmax_step = [&](float lg0, float lg1, float& p0, float& p1) {
    float tm = fmaxf(lg0, lg1);
    tm = fmaxf(tm, __shfl_xor_sync(FULL, tm, 4));
    tm = fmaxf(tm, __shfl_xor_sync(FULL, tm, 8));
    tm = fmaxf(tm, __shfl_xor_sync(FULL, tm, 16));
    const float mn = fmaxf(m_run, tm);
    const bool grow = mn > m_run;
    if (__any_sync(FULL, grow)) {
      const float alpha = grow ? (m_run == kNegInf ? 0.f : exp2_fast(m_run - mn)) : 1.f;
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
    const float mu = m_run == kNegInf ? 0.f : m_run;
    p0 = exp2_fast(lg0 - mu);
    p1 = exp2_fast(lg1 - mu);
  };

  // PV for one 16-position tile: B = hi/lo halves of pv (head gq>>1 of this lane's column).
  auto pv_fragments = [&](float pv0, float pv1, uint32_t& b0, uint32_t& b1) {
    const int hh = gq >> 1;
    const bool lo = gq & 1;
    const int src0 = 8 * tig + (hh < 4 ? hh : 0), src1 = src0 + 4;
    const float x0 = __shfl_sync(FULL, pv0, src0), x1 = __shfl_sync(FULL, pv0, src1);
    const float x2 = __shfl_sync(FULL, pv1, src0), x3 = __shfl_sync(FULL, pv1, src1);
    if (hh < G) {
      b0 = pack_h2(split_part(x0, lo), split_part(x1, lo));
      b1 = pack_h2(split_part(x2, lo), split_part(x3, lo));
    } else {
      b0 = b1 = 0u;
    }
  };

  // ---- pipeline
  int issued = 0;
  long long processed = 0;
  if (lane == 0) {
    for (int k = 0; k < kStages - 1; ++k) {
      if (!prod.valid || tile_start(prod) >= c1) break;
      issue(prod, k % kStages);
      advance(a, cap, prod);
      ++issued;
    }
  }
  issued = __shfl_sync(FULL, issued, 0);

  reset();
  load_query(cons.b, cons.g);
  bool failed = false;
  int k = 0;
  while (true) {
    if (lane == 0) {
      if (prod.valid && tile_start(prod) < c1) {
        fence_proxy_async_smem();
        issue(prod, (k + kStages - 1) % kStages);
        advance(a, cap, prod);
        ++issued;
      }
    }
    const int st = k % kStages;
    const bool ok = mbar_wait_bounded(&bars[st], (k / kStages) & 1, a.err);
    if (__any_sync(FULL, !ok)) {
      failed = true;
      break;
    }
    const uint8_t* buf = sm.ring[warp][st];
    if (cons.seg == 1) {
      // ----------------------------------------------------------- INT4 tile
      const int ti = cons.si.t4a + cons.i;
      const int lp = (ti * 16) / a.P;
      const int page = a.page_table[static_cast<size_t>(cons.b) * a.stride + lp];
      const bool page_ok = page >= 0 && page < a.max_pages;
      const int pos0 = ti * 16 + gq, pos1 = pos0 + 8;
      const bool v0 = page_ok && tig < G && pos0 >= a.s && pos0 < cons.si.m_end;
      const bool v1 = page_ok && tig < G && pos1 >= a.s && pos1 < cons.si.m_end;
      uint32_t kw0[WPC], kw1[WPC];
      {
        const uint8_t* k0p = buf + gq * (D / 2) + tig * Gm::CH;
        const uint8_t* k1p = k0p + 8 * (D / 2);
        if constexpr (WPC == 4) {
          const uint4 u0 = *reinterpret_cast<const uint4*>(k0p), u1 = *reinterpret_cast<const uint4*>(k1p);
          kw0[0] = u0.x; kw0[1] = u0.y; kw0[2] = u0.z; kw0[3] = u0.w;
          kw1[0] = u1.x; kw1[1] = u1.y; kw1[2] = u1.z; kw1[3] = u1.w;
        } else {
          const uint2 u0 = *reinterpret_cast<const uint2*>(k0p), u1 = *reinterpret_cast<const uint2*>(k1p);
          kw0[0] = u0.x; kw0[1] = u0.y;
          kw1[0] = u1.x; kw1[1] = u1.y;
        }
      }
      float S[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int kb = 0; kb < NKB; ++kb) {
        const int j = kb >> 1, k0 = 2 * (kb & 1);
        mma_f16(S, nib2h_rt(kw0[j], k0), nib2h_rt(kw1[j], k0), nib2h_rt(kw0[j], k0 + 1), nib2h_rt(kw1[j], k0 + 1),
                qf[kb][0], qf[kb][1]);
      }
      const uint32_t kp0 = *reinterpret_cast<const uint32_t*>(buf + 16 * D + 4 * gq);
      const uint32_t kp1 = *reinterpret_cast<const uint32_t*>(buf + 16 * D + 4 * (gq + 8));
      const uint32_t vp0 = *reinterpret_cast<const uint32_t*>(buf + 16 * D + 64 + 4 * gq);
      const uint32_t vp1 = *reinterpret_cast<const uint32_t*>(buf + 16 * D + 64 + 4 * (gq + 8));
      const float ks0 = __half2float(__ushort_as_half(kp0 & 0xffff)), kz0 = __half2float(__ushort_as_half(kp0 >> 16));
      const float ks1 = __half2float(__ushort_as_half(kp1 & 0xffff)), kz1 = __half2float(__ushort_as_half(kp1 >> 16));
      // logit (log2 units) = (16 s R + (z - 16 s) sum(q)) / 2^e
      const float lg0 = v0 ? (16.f * ks0 * (S[0] + S[1]) + (kz0 - 16.f * ks0) * sumq) * qinv : kNegInf;
      const float lg1 = v1 ? (16.f * ks1 * (S[2] + S[3]) + (kz1 - 16.f * ks1) * sumq) * qinv : kNegInf;
      float p0, p1;
      softmax_step(lg0, lg1, p0, p1);
      const float vs0 = __half2float(__ushort_as_half(vp0 & 0xffff)), vz0 = __half2float(__ushort_as_half(vp0 >> 16));
      const float vs1 = __half2float(__ushort_as_half(vp1 & 0xffff)), vz1 = __half2float(__ushort_as_half(vp1 >> 16));
      const float pv0 = v0 ? p0 * vs0 : 0.f, pv1 = v1 ? p1 * vs1 : 0.f;
      l_part += (v0 ? p0 : 0.f) + (v1 ? p1 : 0.f);
      // v^ = z + s c = (z + 8 s) + 16 s (c - 8)/16: the MMA sees the centred codes, the
      // per-token constant goes to the scalar sum.
      beta_part += (v0 ? p0 * (vz0 + 8.f * vs0) : 0.f) + (v1 ? p1 * (vz1 + 8.f * vs1) : 0.f);
      uint32_t b0, b1;
      pv_fragments(pv0, pv1, b0, b1);
      uint32_t vw0[WPC], vw1[WPC];
      {
        const uint8_t* vb = buf + 8 * D;
        const uint8_t* v0p = vb + ((0 * 8 + gq) * 4 + tig) * Gm::CH;
        const uint8_t* v1p = vb + ((1 * 8 + gq) * 4 + tig) * Gm::CH;
        if constexpr (WPC == 4) {
          const uint4 u0 = *reinterpret_cast<const uint4*>(v0p), u1 = *reinterpret_cast<const uint4*>(v1p);
          vw0[0] = u0.x; vw0[1] = u0.y; vw0[2] = u0.z; vw0[3] = u0.w;
          vw1[0] = u1.x; vw1[1] = u1.y; vw1[2] = u1.z; vw1[3] = u1.w;
        } else {
          const uint2 u0 = *reinterpret_cast<const uint2*>(v0p), u1 = *reinterpret_cast<const uint2*>(v1p);
          vw0[0] = u0.x; vw0[1] = u0.y;
          vw1[0] = u1.x; vw1[1] = u1.y;
        }
      }
#pragma unroll
      for (int mb = 0; mb < NKB; ++mb) {
        const int j = mb >> 1, k0 = 2 * (mb & 1);
        mma_f16(oacc[mb], centred(nib2h_rt(vw0[j], k0)), centred(nib2h_rt(vw0[j], k0 + 1)),
                centred(nib2h_rt(vw1[j], k0)), centred(nib2h_rt(vw1[j], k0 + 1)), b0, b1);
      }
    } else if (cons.half == 0) {
      // ----------------------------------------------------------- INT8 tile, K half
      const int R0 = cons.i * 16 + gq, R1 = R0 + 8;
      const bool v0 = tig < G && side_row_valid(R0, cons.si.L, a.s, a.w);
      const bool v1 = tig < G && side_row_valid(R1, cons.si.L, a.s, a.w);
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
      float S[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int kb = 0; kb < NKB; ++kb) {
        const int j = kb >> 1;
        const uint32_t A0 = kw0[2 * j] ^ 0x80808080u, B0 = kw0[2 * j + 1] ^ 0x80808080u;
        const uint32_t A1 = kw1[2 * j] ^ 0x80808080u, B1 = kw1[2 * j + 1] ^ 0x80808080u;
        const uint32_t sel = (kb & 1) ? 0x7362u : 0x5140u;
        const uint32_t t0 = prmt(A0, B0, sel), t1 = prmt(A1, B1, sel);
        mma_f16(S, i8x2_to_h2<0x4140>(t0), i8x2_to_h2<0x4140>(t1), i8x2_to_h2<0x4342>(t0), i8x2_to_h2<0x4342>(t1),
                qf[kb][0], qf[kb][1]);
      }
      const float ks0 = __half2float(*reinterpret_cast<const __half*>(buf + 16 * D + 2 * gq));
      const float ks1 = __half2float(*reinterpret_cast<const __half*>(buf + 16 * D + 2 * (gq + 8)));
      const float lg0 = v0 ? ks0 * (S[0] + S[1]) * qinv : kNegInf;
      const float lg1 = v1 ? ks1 * (S[2] + S[3]) * qinv : kNegInf;
      softmax_step(lg0, lg1, p_keep0, p_keep1);
      v_keep0 = v0;
      v_keep1 = v1;
      l_part += (v0 ? p_keep0 : 0.f) + (v1 ? p_keep1 : 0.f);
    } else {
      // ----------------------------------------------------------- INT8 tile, V half
      const float vs0 = __half2float(*reinterpret_cast<const __half*>(buf + 16 * D + 2 * gq));
      const float vs1 = __half2float(*reinterpret_cast<const __half*>(buf + 16 * D + 2 * (gq + 8)));
      const float pv0 = v_keep0 ? p_keep0 * vs0 : 0.f, pv1 = v_keep1 ? p_keep1 * vs1 : 0.f;
      uint32_t b0, b1;
      pv_fragments(pv0, pv1, b0, b1);
      constexpr int NW = Gm::CH8 / 4;  // words per pair chunk (8 or 4)
      uint32_t vw0[NW], vw1[NW];
#pragma unroll
      for (int hv = 0; hv < NW / 4; ++hv) {
        const int phys = (Gm::CH8 >= 32) ? (hv ^ (gq & 1)) : hv;
        const uint4 x0 = *reinterpret_cast<const uint4*>(buf + ((0 * 8 + gq) * 4 + tig) * Gm::CH8 + 16 * phys);
        const uint4 x1 = *reinterpret_cast<const uint4*>(buf + ((1 * 8 + gq) * 4 + tig) * Gm::CH8 + 16 * phys);
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
    __syncwarp();
    ++processed;

    Cursor nxt = cons;
    advance(a, cap, nxt);
    const bool more = nxt.valid && tile_start(nxt) < c1;
    const bool seg_change = !more || nxt.b != cons.b || nxt.g != cons.g || nxt.seg != cons.seg;
    if (seg_change) {
      flush(cons);
      reset();
      if (more && (nxt.b != cons.b || nxt.g != cons.g)) load_query(nxt.b, nxt.g);
    }
    if (!more) break;
    cons = nxt;
    ++k;
  }
  if (failed) {
    // A copy did not arrive in time: wait (bounded) for every copy this warp still has in
    // flight so none lands in shared memory after the CTA exits, then leave.
    issued = __shfl_sync(FULL, issued, 0);
    for (long long j = processed; j < issued; ++j) {
      const int st = static_cast<int>(j % kStages);
      mbar_wait_bounded(&bars[st], static_cast<uint32_t>((j / kStages) & 1), a.err);
    }
  }
}

// ------------------------------------------------------------------ merge kernel

// One warp per (b, q head): LSE merge of the partials of the INT8 and INT4 segments.
template <int D, int G>
__global__ void __launch_bounds__(256) merge_kernel(const DecodeArgs a) {
  const int lane = threadIdx.x & 31;
  const int item = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  if (item >= a.B * a.Hq) return;
  const int b = item / a.Hq, j = item - b * a.Hq;
  const int g = j / G, hi = j - g * G;
  const int cap = a.stride * a.P;
  const long long total = total_cost(a, cap, lane);
  const long long Q = quota(total, a.W);
  long long bstart = 0;
  // prefix of sequence b
  {
    long long run = 0;
    for (int base = 0; base < b; base += 32) {
      const int bb = base + lane;
      long long c = 0;
      if (bb < b) c = a.Hkv * head_cost(seg_info(clamp_len(a.lens[bb], cap), a.s, a.w, a.nt8));
      run += __shfl_sync(FULL, warp_incl_scan(c, lane), 31);
    }
    bstart = run;
  }
  const int Lraw = a.lens[b];
  const SegInfo si = seg_info(clamp_len(Lraw, cap), a.s, a.w, a.nt8);
  if (lane == 0 && Lraw > cap) atomicOr(a.err, KV4_DEVERR_LENGTH);
  const long long hstart = bstart + g * head_cost(si);

  constexpr int PER = D / 32;
  float o[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) o[e] = 0.f;
  float m = kNegInf, l = 0.f;
  for (int seg = 0; seg < 2; ++seg) {
    const long long cs = hstart + (seg == 0 ? 0 : 2LL * si.n8);
    const long long ce = cs + (seg == 0 ? 2LL * si.n8 : si.n4);
    if (ce <= cs) continue;
    const long long tc = seg == 0 ? 2 : 1;
    const long long wf = cs / Q, wl = (ce - tc) / Q;
    const long long sid = 2LL * (static_cast<long long>(b) * a.Hkv + g) + seg;
    for (long long w = wf; w <= wl; ++w) {
      const float* p = a.part + (static_cast<size_t>(w + sid) * G + hi) * (D + 2);
      const float pm = p[D], pl = p[D + 1];
      if (!(pl > 0.f)) continue;
      const float mn = fmaxf(m, pm);
      const float fo = m == kNegInf ? 0.f : exp2f(m - mn), fp = exp2f(pm - mn);
      l = l * fo + pl * fp;
#pragma unroll
      for (int e = 0; e < PER; ++e) o[e] = o[e] * fo + p[lane * PER + e] * fp;
      m = mn;
    }
  }
  float* out = a.out + (static_cast<size_t>(b) * a.Hq + j) * D + lane * PER;
  const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
  for (int e = 0; e < PER; ++e) out[e] = o[e] * inv;
  if (a.lse && lane == 0) a.lse[static_cast<size_t>(b) * a.Hq + j] = l > 0.f ? (m + log2f(l)) * 0.69314718055994531f : kNegInf;
}

template <int D, int G>
cudaError_t launch_dg(const DecodeArgs& a, int ctas, cudaStream_t st) {
  const int smem = static_cast<int>(sizeof(Smem<D, G>));
  static std::atomic<uint64_t> done[3];
  cudaError_t e;
  if (a.q_dtype == KV4_F32) {
    if ((e = ensure_smem_limit(decode_int4_kernel<D, G, KV4_F32>, smem, done[0])) != cudaSuccess) return e;
    decode_int4_kernel<D, G, KV4_F32><<<ctas, kWarps * 32, smem, st>>>(a);
  } else if (a.q_dtype == KV4_BF16) {
    if ((e = ensure_smem_limit(decode_int4_kernel<D, G, KV4_BF16>, smem, done[1])) != cudaSuccess) return e;
    decode_int4_kernel<D, G, KV4_BF16><<<ctas, kWarps * 32, smem, st>>>(a);
  } else {
    if ((e = ensure_smem_limit(decode_int4_kernel<D, G, KV4_F16>, smem, done[2])) != cudaSuccess) return e;
    decode_int4_kernel<D, G, KV4_F16><<<ctas, kWarps * 32, smem, st>>>(a);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int items = a.B * a.Hq;
  merge_kernel<D, G><<<(items + 7) / 8, 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

int decode_warps_per_cta() { return kWarps; }

size_t decode_smem_bytes(int D, int G) {
  if (D == 128) return G == 4 ? sizeof(Smem<128, 4>) : G == 2 ? sizeof(Smem<128, 2>) : sizeof(Smem<128, 1>);
  return G == 4 ? sizeof(Smem<64, 4>) : G == 2 ? sizeof(Smem<64, 2>) : sizeof(Smem<64, 1>);
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
