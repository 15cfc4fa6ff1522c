// kv4_bf16.cu -- BF16-KV paged decode attention: the baseline the INT4 cache is measured
// against (KV4-RL, "Main Findings": speedups are quoted relative to BF16 KV).
//
// Flattened split-K over 16-position tiles (kv4_splitk.cuh), one bulk copy per tile into a
// per-warp shared-memory ring, m16n8k16 MMA with the GQA group's query heads as the N columns,
// LSE merge; K and V are bf16 in the pages, so the MMA operands are read as-is.
// Queries enter as bf16 hi/lo halves (exact for bf16 queries); P enters as bf16 hi/lo halves.
#include <cuda_bf16.h>
#include <math.h>

#include "kv4_device.cuh"
#include "kv4_internal.h"
#include "kv4_layout.cuh"
#include "kv4_splitk.cuh"

namespace kv4 {
namespace {

constexpr unsigned FULL = 0xffffffffu;
constexpr int kWarps = 8;
constexpr int kStages = 3;
constexpr float kNegInf = -__builtin_huge_valf();

using splitk::clamp_len;
using splitk::Cur;
using splitk::prefix_cost;
using splitk::quota;
using splitk::settle;

template <int D, int G>
struct SmemBF {
  uint8_t ring[kWarps][kStages][Geo<D>::TBF];
  float qbuf[kWarps][G][D];
  uint64_t bar[kWarps][kStages];
};

__device__ __forceinline__ float exp2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ __nv_bfloat16 split_bf(float x, bool lo) {
  const __nv_bfloat16 hi = __float2bfloat16_rn(x);
  return lo ? __float2bfloat16_rn(x - __bfloat162float(hi)) : hi;
}

template <int D, int G, int QT>
__global__ void __launch_bounds__(kWarps * 32, 1) decode_bf16_kernel(const DecodeArgs a) {
  using Gm = Geo<D>;
  constexpr int NKB = Gm::NKB;
  constexpr int EPT = Gm::EPT;     // elements per thread chunk (32 or 16)
  constexpr int UPC = D / 32;      // 16-byte units per chunk (4 or 2)
  extern __shared__ __align__(128) uint8_t smem_raw[];
  SmemBF<D, G>& sm = *reinterpret_cast<SmemBF<D, G>*>(smem_raw);
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

  const long long total = prefix_cost(a, cap, lane, a.B);
  const long long Q = quota(total, a.W);
  const long long c0 = static_cast<long long>(wid) * Q;
  if (c0 >= total) return;
  const long long c1 = c0 + Q < total ? c0 + Q : total;

  Cur cons = splitk::cursor_at(a, cap, lane, c0);
  Cur prod = cons;
  const long long nslots = c1 - c0;

  auto issue = [&](const Cur& c, int st) {
    const int lp = (c.i * 16) / a.P;
    const int page = a.page_table[static_cast<size_t>(c.b) * a.stride + lp];
    if (page >= 0 && page < a.max_pages) {
      const uint8_t* src = a.pool + static_cast<size_t>(page) * a.page_bytes + static_cast<size_t>(c.g) * a.P * 4 * D +
                           static_cast<size_t>((c.i * 16 - lp * a.P) >> 4) * Gm::TBF;
      mbar_arrive_expect_tx(&bars[st], Gm::TBF);
      bulk_g2s_hint(sm.ring[warp][st], src, Gm::TBF, &bars[st], l2_policy_evict_first());
    } else {
      atomicOr(a.err, KV4_DEVERR_PAGE_RANGE);
      mbar_arrive_expect_tx(&bars[st], 0);
    }
  };

  uint32_t qf[NKB][2];
  float* qb = &sm.qbuf[warp][0][0];
  auto load_query = [&](int b, int g) {
    for (int idx = lane; idx < G * D; idx += 32) {
      const size_t qi = (static_cast<size_t>(b) * a.Hq + static_cast<size_t>(g) * G) * D + idx;
      float x;
      if constexpr (QT == KV4_F32) x = reinterpret_cast<const float*>(a.q)[qi];
      else if constexpr (QT == KV4_BF16) x = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(a.q)[qi]);
      else x = __half2float(reinterpret_cast<const __half*>(a.q)[qi]);
      qb[idx] = x;
    }
    __syncwarp();
    const int hh = gq >> 1;
    const bool lo = gq & 1;
#pragma unroll
    for (int kb = 0; kb < NKB; ++kb) {
      const int e0 = EPT * tig + 4 * kb;
      if (hh < G) {
        const float* qh = qb + hh * D;
        qf[kb][0] = pack_bf2(split_bf(qh[e0], lo), split_bf(qh[e0 + 1], lo));
        qf[kb][1] = pack_bf2(split_bf(qh[e0 + 2], lo), split_bf(qh[e0 + 3], lo));
      } else {
        qf[kb][0] = qf[kb][1] = 0u;
      }
    }
    __syncwarp();
  };

  float oacc[NKB][4];
  float m_run, l_part;
  auto reset = [&]() {
#pragma unroll
    for (int mb = 0; mb < NKB; ++mb) oacc[mb][0] = oacc[mb][1] = oacc[mb][2] = oacc[mb][3] = 0.f;
    m_run = kNegInf;
    l_part = 0.f;
  };
  auto flush = [&](const Cur& c) {
    float l = l_part;
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) l += __shfl_xor_sync(FULL, l, o);
    if (tig < G) {
      const long long sid = static_cast<long long>(c.b) * a.Hkv + c.g;
      float* p = a.part + (static_cast<size_t>(wid + sid) * G + tig) * kPartRow<D>;
#pragma unroll
      for (int mb = 0; mb < NKB; ++mb) {
        const int d = Gm::DG * gq + 2 * mb;
        *reinterpret_cast<float2*>(p + d) = make_float2(oacc[mb][0] + oacc[mb][1], oacc[mb][2] + oacc[mb][3]);
      }
      if (gq == 0) *reinterpret_cast<float2*>(p + D) = make_float2(m_run, l);
    }
  };

  int issued = 0;
  if (lane == 0) {
    for (int k = 0; k < kStages - 1 && k < nslots; ++k) {
      issue(prod, k);
      ++prod.i;
      settle(a, cap, prod);
      ++issued;
    }
  }
  reset();
  load_query(cons.b, cons.g);
  bool failed = false;
  long long k = 0;
  for (; k < nslots; ++k) {
    if (lane == 0 && issued < nslots) {
      fence_proxy_async_smem();
      issue(prod, static_cast<int>((k + kStages - 1) % kStages));
      ++prod.i;
      settle(a, cap, prod);
      ++issued;
    }
    const int st = static_cast<int>(k % kStages);
    const bool ok = mbar_wait_bounded(&bars[st], static_cast<uint32_t>((k / kStages) & 1), a.err);
    if (__any_sync(FULL, !ok)) {
      failed = true;
      break;
    }
    const uint8_t* buf = sm.ring[warp][st];
    const int lp = (cons.i * 16) / a.P;
    const int page = a.page_table[static_cast<size_t>(cons.b) * a.stride + lp];
    const bool page_ok = page >= 0 && page < a.max_pages;
    const int L = clamp_len(a.lens[cons.b], cap);
    const int pos0 = cons.i * 16 + gq, pos1 = pos0 + 8;
    const bool v0 = page_ok && tig < G && pos0 < L, v1 = page_ok && tig < G && pos1 < L;

    // QK: A = K rows gq and gq + 8, thread chunk tig (units swizzled).
    float S[4] = {0.f, 0.f, 0.f, 0.f};
    uint32_t kw0[EPT / 2], kw1[EPT / 2];
#pragma unroll
    for (int u = 0; u < UPC; ++u) {
      const uint4 x0 = *reinterpret_cast<const uint4*>(buf + gq * 2 * D + tig * (D / 2) + 16 * (u ^ bf16_swz(D, tig, gq)));
      const uint4 x1 =
          *reinterpret_cast<const uint4*>(buf + (gq + 8) * 2 * D + tig * (D / 2) + 16 * (u ^ bf16_swz(D, tig, gq + 8)));
      kw0[4 * u] = x0.x; kw0[4 * u + 1] = x0.y; kw0[4 * u + 2] = x0.z; kw0[4 * u + 3] = x0.w;
      kw1[4 * u] = x1.x; kw1[4 * u + 1] = x1.y; kw1[4 * u + 2] = x1.z; kw1[4 * u + 3] = x1.w;
    }
#pragma unroll
    for (int kb = 0; kb < NKB; ++kb) mma_bf16(S, kw0[2 * kb], kw1[2 * kb], kw0[2 * kb + 1], kw1[2 * kb + 1], qf[kb][0], qf[kb][1]);
    const float lg0 = v0 ? (S[0] + S[1]) * a.qscale : kNegInf;
    const float lg1 = v1 ? (S[2] + S[3]) * a.qscale : kNegInf;

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
      m_run = mn;
    }
    const float mu = m_run == kNegInf ? 0.f : m_run;
    const float p0 = v0 ? exp2_fast(lg0 - mu) : 0.f, p1 = v1 ? exp2_fast(lg1 - mu) : 0.f;
    l_part += p0 + p1;

    const int hh = gq >> 1;
    const bool lo = gq & 1;
    const int src0 = 8 * tig + hh, src1 = src0 + 4;
    const float x0 = __shfl_sync(FULL, p0, src0), x1 = __shfl_sync(FULL, p0, src1);
    const float x2 = __shfl_sync(FULL, p1, src0), x3 = __shfl_sync(FULL, p1, src1);
    uint32_t b0 = 0u, b1 = 0u;
    if (hh < G) {
      b0 = pack_bf2(split_bf(x0, lo), split_bf(x1, lo));
      b1 = pack_bf2(split_bf(x2, lo), split_bf(x3, lo));
    }
    // PV: A = V^T from the pair chunks of pairs tig and tig + 4, group gq.
    const uint8_t* vb = buf + 32 * D;
    uint32_t vw0[D / 8], vw1[D / 8];
#pragma unroll
    for (int u = 0; u < UPC; ++u) {
      const uint4 y0 = *reinterpret_cast<const uint4*>(vb + ((0 * 8 + gq) * 4 + tig) * (D / 2) + 16 * (u ^ bf16_swz(D, tig, gq)));
      const uint4 y1 = *reinterpret_cast<const uint4*>(vb + ((1 * 8 + gq) * 4 + tig) * (D / 2) + 16 * (u ^ bf16_swz(D, tig, gq)));
      vw0[4 * u] = y0.x; vw0[4 * u + 1] = y0.y; vw0[4 * u + 2] = y0.z; vw0[4 * u + 3] = y0.w;
      vw1[4 * u] = y1.x; vw1[4 * u + 1] = y1.y; vw1[4 * u + 2] = y1.z; vw1[4 * u + 3] = y1.w;
    }
    if (cons.i * 16 + 16 > L) {
      // Partial last tile: slots past L were never written and may hold NaN patterns, which a
      // zero weight does not cancel (0 * NaN); clear those positions in the A operand.
      const int t0 = cons.i * 16 + 2 * tig;
      const uint32_t m0 = (t0 < L ? 0x0000ffffu : 0u) | (t0 + 1 < L ? 0xffff0000u : 0u);
      const uint32_t m1 = (t0 + 8 < L ? 0x0000ffffu : 0u) | (t0 + 9 < L ? 0xffff0000u : 0u);
#pragma unroll
      for (int x = 0; x < D / 8; ++x) {
        vw0[x] &= m0;
        vw1[x] &= m1;
      }
    }
#pragma unroll
    for (int mb = 0; mb < NKB; ++mb) mma_bf16(oacc[mb], vw0[2 * mb], vw0[2 * mb + 1], vw1[2 * mb], vw1[2 * mb + 1], b0, b1);
    __syncwarp();

    Cur nxt = cons;
    ++nxt.i;
    settle(a, cap, nxt);
    const bool more = k + 1 < nslots;
    if (!more || nxt.b != cons.b || nxt.g != cons.g) {
      flush(cons);
      reset();
      if (more) load_query(nxt.b, nxt.g);
    }
    cons = nxt;
  }
  if (failed) {
    issued = __shfl_sync(FULL, issued, 0);
    for (long long j = k; j < issued; ++j)
      mbar_wait_bounded(&bars[j % kStages], static_cast<uint32_t>((j / kStages) & 1), a.err);
  }
}

template <int D, int G>
cudaError_t launch_dg(const DecodeArgs& a, int ctas, cudaStream_t st) {
  const int smem = static_cast<int>(sizeof(SmemBF<D, G>));
  static std::atomic<uint64_t> done[3];
  cudaError_t e;
  if (a.q_dtype == KV4_F32) {
    if ((e = ensure_smem_limit(decode_bf16_kernel<D, G, KV4_F32>, smem, done[0])) != cudaSuccess) return e;
    decode_bf16_kernel<D, G, KV4_F32><<<ctas, kWarps * 32, smem, st>>>(a);
  } else if (a.q_dtype == KV4_BF16) {
    if ((e = ensure_smem_limit(decode_bf16_kernel<D, G, KV4_BF16>, smem, done[1])) != cudaSuccess) return e;
    decode_bf16_kernel<D, G, KV4_BF16><<<ctas, kWarps * 32, smem, st>>>(a);
  } else {
    if ((e = ensure_smem_limit(decode_bf16_kernel<D, G, KV4_F16>, smem, done[2])) != cudaSuccess) return e;
    decode_bf16_kernel<D, G, KV4_F16><<<ctas, kWarps * 32, smem, st>>>(a);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return splitk::launch_merge<D, G>(a, st);
}

}  // namespace

int bf16_decode_warps_per_cta() { return kWarps; }

size_t bf16_decode_smem_bytes(int D, int G) {
  if (D == 128) return G == 4 ? sizeof(SmemBF<128, 4>) : G == 2 ? sizeof(SmemBF<128, 2>) : sizeof(SmemBF<128, 1>);
  return G == 4 ? sizeof(SmemBF<64, 4>) : G == 2 ? sizeof(SmemBF<64, 2>) : sizeof(SmemBF<64, 1>);
}

cudaError_t launch_decode_bf16(DecodeArgs a, int D, int G, int ctas, cudaStream_t st) {
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
