// kv4_splitk.cuh -- the flattened split-K schedule shared by the single-region decode kernels (the
// BF16 baseline and the mixed bit-width key cache): every (sequence, KV head) is cut into
// 16-position tiles, the tiles of all pairs are laid end to end in (sequence, head, tile) order,
// and warp w of W takes the w-th run of ceil(total / W) of them.  A warp writes one partial row
// group (o[D], m, l) per (sequence, head) segment it touches, at index w + b * Hkv + g (unique:
// consecutive warps overlap in at most one segment); the merge kernel finds the warps that
// covered a pair from the same arithmetic and combines their partials by log-sum-exp.
#pragma once

#include <cuda_runtime.h>
#include <math.h>

#include "kv4_internal.h"
#include "kv4_layout.cuh"

namespace kv4 {
namespace splitk {

constexpr unsigned kFull = 0xffffffffu;
constexpr float kNegInfF = -__builtin_huge_valf();

__device__ __forceinline__ int clamp_len(int L, int cap) { return L < 0 ? 0 : (L > cap ? cap : L); }
__device__ __forceinline__ long long seq_cost(const DecodeArgs& a, int L) {
  return static_cast<long long>(a.Hkv) * ((L + 15) >> 4);
}

__device__ __forceinline__ long long warp_incl_scan(long long v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long t = __shfl_up_sync(kFull, v, o);
    if (lane >= o) v += t;
  }
  return v;
}

// tiles of sequences [0, upto)
__device__ __forceinline__ long long prefix_cost(const DecodeArgs& a, int cap, int lane, int upto) {
  long long run = 0;
  for (int base = 0; base < upto; base += 32) {
    const int b = base + lane;
    const long long c = b < upto ? seq_cost(a, clamp_len(a.lens[b], cap)) : 0;
    run += __shfl_sync(kFull, warp_incl_scan(c, lane), 31);
  }
  return run;
}

// the sequence holding flattened tile c, and the index of its first tile
__device__ __forceinline__ int find_seq(const DecodeArgs& a, int cap, int lane, long long c, long long* bstart) {
  long long run = 0;
  for (int base = 0; base < a.B; base += 32) {
    const int b = base + lane;
    const long long cb = b < a.B ? seq_cost(a, clamp_len(a.lens[b], cap)) : 0;
    const long long incl = warp_incl_scan(cb, lane);
    const long long tot = __shfl_sync(kFull, incl, 31);
    if (c < run + tot) {
      const unsigned m = __ballot_sync(kFull, c < run + incl);
      const int l = __ffs(m) - 1;
      *bstart = run + __shfl_sync(kFull, incl - cb, l);
      return base + l;
    }
    run += tot;
  }
  *bstart = run;
  return a.B;
}

__device__ __forceinline__ long long quota(long long total, int W) {
  const long long q = (total + W - 1) / W;
  return q < 1 ? 1 : q;
}

// position in the flattened order: sequence b, KV head g, tile i of n
struct Cur {
  int b, g, i, n;
  bool valid;
};

__device__ __forceinline__ void settle(const DecodeArgs& a, int cap, Cur& c) {
  while (c.b < a.B && c.i >= c.n) {
    c.i = 0;
    if (++c.g == a.Hkv) {
      c.g = 0;
      if (++c.b < a.B) c.n = (clamp_len(a.lens[c.b], cap) + 15) >> 4;
    }
  }
  c.valid = c.b < a.B;
}

// The cursor of flattened tile c0.
__device__ __forceinline__ Cur cursor_at(const DecodeArgs& a, int cap, int lane, long long c0) {
  Cur c;
  long long bstart;
  c.b = find_seq(a, cap, lane, c0, &bstart);
  const int L = clamp_len(a.lens[c.b], cap);
  c.n = (L + 15) >> 4;
  const long long off = c0 - bstart;
  c.g = static_cast<int>(off / c.n);
  c.i = static_cast<int>(off - static_cast<long long>(c.g) * c.n);
  c.valid = true;
  return c;
}

// Combine the partials of the warps that covered a (sequence, query head) pair.  MW = 1: one warp
// per pair, 8 pairs per CTA.  MW = 8, for batches with few pairs (and long runs of partials each):
// one pair per CTA, its partials split in 8 consecutive runs folded by the 8 warps, whose states
// warp 0 then combines.  At most 64 registers (4 CTAs per SM): the batched loads of long runs would
// otherwise halve the occupancy that short runs need.
template <int D, int G, int MW>
__global__ void __launch_bounds__(256, 4) merge_kernel(const DecodeArgs a) {
  static_assert(MW == 1 || MW == 8, "one warp per pair, or a CTA of 8 warps per pair");
  // The tile offsets of the warps' sequences and the total, from one pass of the CTA over the
  // sequences' lengths (256 at a time, block-wide scan) instead of two scans per warp.
  __shared__ long long incl_s[256];
  __shared__ long long wsum_s[8];
  __shared__ long long carry_s;
  __shared__ float smo[MW][D];
  __shared__ float smM[MW], smL[MW];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int item = MW == 1 ? static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5) : static_cast<int>(blockIdx.x);
  const int sub = MW == 1 ? 0 : warp;  // this warp's run of the pair's partials
  const bool valid = item < a.B * a.Hq;
  const int b = valid ? item / a.Hq : 0, j = valid ? item - b * a.Hq : 0;
  const int cap = a.stride * a.P;
  long long bstart = 0;
  if (threadIdx.x == 0) carry_s = 0;
  __syncthreads();
  for (int base = 0; base < a.B; base += 256) {
    const int bt = base + static_cast<int>(threadIdx.x);
    const long long c = bt < a.B ? seq_cost(a, clamp_len(a.lens[bt], cap)) : 0;
    const long long wi = warp_incl_scan(c, lane);
    if (lane == 31) wsum_s[warp] = wi;
    __syncthreads();
    long long off = carry_s;
    for (int w = 0; w < warp; ++w) off += wsum_s[w];
    incl_s[threadIdx.x] = off + wi;
    __syncthreads();
    if (valid && b >= base && b < base + 256)  // exclusive prefix of sequence b (b < B when valid)
      bstart = incl_s[b - base] - seq_cost(a, clamp_len(a.lens[b], cap));
    if (threadIdx.x == 255) carry_s = incl_s[255];
    __syncthreads();
  }
  const long long total = carry_s;
  if (!valid) return;  // uniform over the CTA when MW = 8
  const int g = j / G, hi = j - g * G;
  const long long Q = quota(total, a.W);
  const int L = clamp_len(a.lens[b], cap);
  const long long n = (L + 15) >> 4;
  constexpr int PER = D / 32;
  float o[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) o[e] = 0.f;
  float m = kNegInfF, l = 0.f;
  if (n > 0) {
    const long long cs = bstart + g * n, ce = cs + n;
    const long long sid = static_cast<long long>(b) * a.Hkv + g;
    const long long f0 = cs / Q, f1 = (ce - 1) / Q;  // the warps that covered the pair
    const long long cnt = f1 - f0 + 1;
    const long long w0 = f0 + sub * cnt / MW, w1 = f0 + (sub + 1) * cnt / MW - 1;  // this warp's run
    auto fold = [&](float pm, float pl, const float (&pr)[PER]) {
      if (!(pl > 0.f)) return;
      const float mn = fmaxf(m, pm);
      const float fo = m == kNegInfF ? 0.f : exp2f(m - mn), fp = exp2f(pm - mn);
      l = l * fo + pl * fp;
#pragma unroll
      for (int e = 0; e < PER; ++e) o[e] = o[e] * fo + pr[e] * fp;
      m = mn;
    };
    auto row = [&](long long w) { return a.part + (static_cast<size_t>(w + sid) * G + hi) * kPartRow<D>; };
    // Long runs of partials kBatch at a time: their loads are issued together (one memory round
    // trip per batch), then folded in warp order; the rest one by one.
    constexpr int kBatch = 8;
    long long w = w0;
    for (; w + kBatch - 1 <= w1; w += kBatch) {
      float2 ml[kBatch];
      float pv[kBatch][PER];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const float* p = row(w + u);
        ml[u] = *reinterpret_cast<const float2*>(p + D);
#pragma unroll
        for (int e = 0; e < PER; ++e) pv[u][e] = p[lane * PER + e];
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) fold(ml[u].x, ml[u].y, pv[u]);
    }
    for (; w <= w1; ++w) {
      const float* p = row(w);
      const float pm = p[D], pl = p[D + 1];
      if (!(pl > 0.f)) continue;
      float pr[PER];
#pragma unroll
      for (int e = 0; e < PER; ++e) pr[e] = p[lane * PER + e];
      fold(pm, pl, pr);
    }
  }
  if constexpr (MW > 1) {
    // warp 0 combines the 8 runs' (m, l, o), in run order
#pragma unroll
    for (int e = 0; e < PER; ++e) smo[sub][lane * PER + e] = o[e];
    if (lane == 0) {
      smM[sub] = m;
      smL[sub] = l;
    }
    __syncthreads();
    if (sub != 0) return;
    m = kNegInfF;
#pragma unroll
    for (int w = 0; w < MW; ++w)
      if (smL[w] > 0.f) m = fmaxf(m, smM[w]);
    l = 0.f;
#pragma unroll
    for (int e = 0; e < PER; ++e) o[e] = 0.f;
#pragma unroll
    for (int w = 0; w < MW; ++w) {
      const float f = smL[w] > 0.f ? exp2f(smM[w] - m) : 0.f;
      l += f * smL[w];
#pragma unroll
      for (int e = 0; e < PER; ++e) o[e] = fmaf(f, smo[w][lane * PER + e], o[e]);
    }
  }
  float* out = a.out + (static_cast<size_t>(b) * a.Hq + j) * D + lane * PER;
  const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
  for (int e = 0; e < PER; ++e) out[e] = o[e] * inv;
  if (a.lse && lane == 0) a.lse[static_cast<size_t>(b) * a.Hq + j] = l > 0.f ? (m + log2f(l)) * 0.69314718055994531f : kNegInfF;
}

// Pairs below which the merge gives each pair a CTA of 8 warps: fewer pairs than about one wave
// of warps on 148 SMs leave most of the GPU idle with one warp per pair.
constexpr int kWideMergePairs = 1024;

template <int D, int G>
cudaError_t launch_merge(const DecodeArgs& a, cudaStream_t st) {
  const int items = a.B * a.Hq;
  if (items < kWideMergePairs)
    merge_kernel<D, G, 8><<<items, 256, 0, st>>>(a);
  else
    merge_kernel<D, G, 1><<<(items + 7) / 8, 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace splitk
}  // namespace kv4
