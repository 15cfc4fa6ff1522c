// kv4_append.cu -- fused append: block-Hadamard rotation of K, per-token affine INT4
// quantisation of rotated K and of V, nibble packing into the page slot, INT8 routing of
// sink / recent positions into the side cache.  Plus the BF16 pool append of the baseline.
//
// Method: KV4-RL (ai.info summary), "Methodology in Plain English" paragraph 2 (one affine INT4
// group per token-head vector, FP16 scale and offset, keys Hadamard-rotated before
// quantisation) and paragraph 3 (INT8 side cache for the first s and last w positions);
// SAW-INT4 (gist.science summary), section 2 (block-diagonal rotation in blocks of h, fused with
// quantisation in one kernel).
//
// One warp per (token, KV head); lane l holds elements 4l..4l+3 (D = 128 uses all 32 lanes,
// D = 64 the first 16).  Bit-exact rules: the butterfly runs strides 1, 2, ..., h/2 in that
// order with plain fp32 add/sub (a + b, a - b); the quantiser uses IEEE fp32 sub/div, rint
// (ties to even) and directed fp16 conversions; min and max are taken as values (+0 for zero).
#include <cuda_bf16.h>

#include "kv4_device.cuh"
#include "kv4_internal.h"
#include "kv4_layout.cuh"

namespace kv4 {
namespace {

constexpr unsigned FULL = 0xffffffffu;
constexpr int kAppendThreads = 256;

template <typename T>
__device__ __forceinline__ void load4(const void* base, size_t i, float (&x)[4]);

template <>
__device__ __forceinline__ void load4<float>(const void* base, size_t i, float (&x)[4]) {
  const float4 v = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + i);
  x[0] = v.x;
  x[1] = v.y;
  x[2] = v.z;
  x[3] = v.w;
}

template <>
__device__ __forceinline__ void load4<__nv_bfloat16>(const void* base, size_t i, float (&x)[4]) {
  const uint2 v = *reinterpret_cast<const uint2*>(reinterpret_cast<const __nv_bfloat16*>(base) + i);
  x[0] = __uint_as_float(v.x << 16);
  x[1] = __uint_as_float(v.x & 0xffff0000u);
  x[2] = __uint_as_float(v.y << 16);
  x[3] = __uint_as_float(v.y & 0xffff0000u);
}

// Sylvester block Hadamard on blocks of h over the warp's D elements (lane holds 4).
__device__ __forceinline__ void hadamard4(float (&x)[4], int lane, int h) {
  if (h >= 2) {
    float a = x[0], b = x[1];
    x[0] = __fadd_rn(a, b);
    x[1] = __fsub_rn(a, b);
    a = x[2];
    b = x[3];
    x[2] = __fadd_rn(a, b);
    x[3] = __fsub_rn(a, b);
  }
  if (h >= 4) {
    float a = x[0], b = x[2];
    x[0] = __fadd_rn(a, b);
    x[2] = __fsub_rn(a, b);
    a = x[1];
    b = x[3];
    x[1] = __fadd_rn(a, b);
    x[3] = __fsub_rn(a, b);
  }
  for (int st = 4; st < h; st <<= 1) {
    const int m = st >> 2;
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float o = __shfl_xor_sync(FULL, x[i], m);
      x[i] = upper ? __fsub_rn(o, x[i]) : __fadd_rn(x[i], o);
    }
  }
}

__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fminf(v, __shfl_xor_sync(FULL, v, o));
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(FULL, v, o));
  return v;
}

// INT4 codes of the lane's 4 elements packed as elements 0..3 in bits 0..15 (4 bits each);
// *sz receives (fp16 scale bits) | (fp16 zero bits << 16).  A vector whose zero or scale is not a
// finite fp16 (values beyond the fp16 range) keeps those parameters, gets all-zero codes and sets
// *bad (warp-uniform: the parameters come from warp reductions).
__device__ __forceinline__ uint32_t quant_int4(const float (&x)[4], bool act, uint32_t* sz, bool* bad) {
  float mn = act ? fminf(fminf(x[0], x[1]), fminf(x[2], x[3])) : __int_as_float(0x7f800000);
  float mx = act ? fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3])) : __int_as_float(0xff800000);
  mn = __fadd_rn(warp_min(mn), 0.0f);
  mx = __fadd_rn(warp_max(mx), 0.0f);
  const __half zh = __float2half_rd(mn);
  const float zf = __half2float(zh);
  const float r = __fsub_rn(mx, zf);
  const __half sh = __float2half_ru(__fdiv_rn(r, 15.0f));
  const float sf = __half2float(sh);
  *bad = !(isfinite(zf) && isfinite(sf));
  uint32_t packed = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int c = 0;
    if (sf != 0.0f && !*bad) {
      c = static_cast<int>(rintf(__fdiv_rn(__fsub_rn(x[i], zf), sf)));
      c = min(max(c, 0), 15);
    }
    packed |= static_cast<uint32_t>(c) << (4 * i);
  }
  *sz = static_cast<uint32_t>(__half_as_ushort(sh)) | (static_cast<uint32_t>(__half_as_ushort(zh)) << 16);
  return packed;
}

// Symmetric INT8 codes of the lane's 4 elements (bytes 0..3), fp16 scale bits in *sc; a scale
// that is not a finite fp16 gives all-zero codes and sets *bad, as for INT4.
__device__ __forceinline__ uint32_t quant_int8(const float (&x)[4], bool act, uint16_t* sc, bool* bad) {
  float a = act ? fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3]))) : 0.0f;
  a = warp_max(a);
  const __half sh = __float2half_ru(__fdiv_rn(a, 127.0f));
  const float sf = __half2float(sh);
  *bad = !isfinite(sf);
  uint32_t packed = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int c = 0;
    if (sf != 0.0f && !*bad) {
      c = static_cast<int>(rintf(__fdiv_rn(x[i], sf)));
      c = min(max(c, -127), 127);
    }
    packed |= (static_cast<uint32_t>(c) & 0xffu) << (8 * i);
  }
  *sc = __half_as_ushort(sh);
  return packed;
}

// Offset of value element e of row r in a 16-row bf16 V block (the BF16 pool's V order).
template <int D>
__device__ __forceinline__ int vbf_offset(int r, int e) {
  using Gm = Geo<D>;
  const int p = r >> 1, half = p >> 2, pl = p & 3;
  const int gq = e / Gm::DG, m = e % Gm::DG, uu = m >> 2;
  return ((half * 8 + gq) * 4 + pl) * (D / 2) + ((uu ^ bf16_swz(D, pl, gq)) << 4) + (m & 3) * 4 + (r & 1) * 2;
}

// VB: values kept as bf16 (KV4_VALUES_BF16) instead of INT4 / INT8.
template <int D, typename KT, typename VT, bool VB>
__global__ void __launch_bounds__(kAppendThreads) append_int4_kernel(AppendArgs a) {
  using Gm = Geo<D>;
  constexpr int PB = VB ? D / 2 + 4 + 2 * D : D + 8;  // bytes of one position of one head in a page
  constexpr int KPO = VB ? 8 * D : 16 * D;             // K parameters in a page tile
  constexpr int T8 = VB ? Gm::T8V : Gm::T8B;           // side tile
  pdl_launch_dependents();  // the decode kernel that follows may start its launch now
  const int gw = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (gw >= a.T * a.Hkv) return;
  const int t = gw / a.Hkv, g = gw - t * a.Hkv;
  // Three dependent round trips at most: {token's slot and position, its K and V} -> {page-table
  // entry, length after the call} -> stores.  K and V are read before the checks (every t < T is
  // a valid input row).
  const bool act = lane < D / 4;
  float k[4] = {0.f, 0.f, 0.f, 0.f}, v[4] = {0.f, 0.f, 0.f, 0.f};
  const size_t in0 = (static_cast<size_t>(t) * a.Hkv + g) * D + 4 * lane;
  if (act) {
    load4<KT>(a.K, in0, k);
    load4<VT>(a.V, in0, v);
  }
  const int b = a.seq_slot[t], pos = a.pos[t];
  if (b < 0 || b >= a.max_seqs || pos < 0 || pos / a.P >= a.stride) {
    if (lane == 0) atomicOr(a.err, KV4_DEVERR_LENGTH);
    return;
  }
  const int page = a.page_table[static_cast<size_t>(b) * a.stride + pos / a.P];
  const int len_after = a.w > 0 && pos >= a.s ? a.lens_after[b] : 0;
  if (page < 0 || page >= a.max_pages) {
    if (lane == 0) atomicOr(a.err, KV4_DEVERR_PAGE_RANGE);
    return;
  }
  {
    // randomised-sign rotation: dims of set bits are negated first (exact: the sign bit flips)
    const uint32_t sb = (a.signs[lane >> 3] >> (4 * (lane & 7))) & 15u;
#pragma unroll
    for (int e = 0; e < 4; ++e) k[e] = __uint_as_float(__float_as_uint(k[e]) ^ (((sb >> e) & 1u) << 31));
  }
  hadamard4(k, lane, a.h);
  if (a.rotate_v) {  // value rotation: the same H diag(s) as the keys
    const uint32_t sb = (a.signs[lane >> 3] >> (4 * (lane & 7))) & 15u;
#pragma unroll
    for (int e = 0; e < 4; ++e) v[e] = __uint_as_float(__float_as_uint(v[e]) ^ (((sb >> e) & 1u) << 31));
    hadamard4(v, lane, a.h);
  }

  const int pp = pos % a.P, r = pp & 15;
  uint8_t* tile = a.pool + static_cast<size_t>(page) * a.page_bytes + static_cast<size_t>(g) * a.P * PB +
                  static_cast<size_t>(pp >> 4) * (16 * PB);
  uint32_t ksz, vsz = 0;
  bool kbad, vbad = false;
  const uint32_t kc = quant_int4(k, act, &ksz, &kbad);
  uint32_t vc = 0;
  if constexpr (!VB) vc = quant_int4(v, act, &vsz, &vbad);
  if (lane == 0 && (kbad || vbad)) atomicOr(a.err, KV4_DEVERR_RANGE);
  if (act) {
    // K: row r shares pair-row r % 8 with row r ^ 8 (low nibbles rows 0-7, high nibbles rows
    // 8-15), so its nibbles are merged in with atomics (another token of the tile may be written
    // by another warp of this launch).  Elements 4l, 4l+2 go to bytes 2(l&1), 2(l&1)+1 of word 0
    // of 8-byte group l/2, elements 4l+1, 4l+3 to the same bytes of word 1.
    const int pr = r & 7, hi4 = 4 * (r >> 3);
    const int gb = 8 * (lane >> 1);                                    // group byte in the pair-row
    const int unit = (gb >> 4) ^ (D >= 128 ? (pr & 1) : 0);
    uint32_t* w0 = reinterpret_cast<uint32_t*>(tile + pr * D + 16 * unit + (gb & 15));
    const int sh = 16 * (lane & 1) + hi4;                              // bit of byte 2(l&1)
    const uint32_t e0 = kc & 15u, e1 = (kc >> 4) & 15u, e2 = (kc >> 8) & 15u, e3 = (kc >> 12) & 15u;
    const uint32_t clear = ~((0xFu << sh) | (0xFu << (sh + 8)));
    atomicAnd(w0, clear);
    atomicOr(w0, (e0 << sh) | (e2 << (sh + 8)));
    atomicAnd(w0 + 1, clear);
    atomicOr(w0 + 1, (e1 << sh) | (e3 << (sh + 8)));
    if constexpr (VB) {
      // V as bf16 (nearest even), elements 4l..4l+3
#pragma unroll
      for (int i = 0; i < 4; ++i)
        *reinterpret_cast<__nv_bfloat16*>(tile + Gm::VBO + vbf_offset<D>(r, 4 * lane + i)) = __float2bfloat16_rn(v[i]);
    } else {
      // V: 16-bit chunk of quad Q = l.
      const int Q = lane, p = r >> 1, half = p >> 2, pl = p & 3;
      const int off = ((half * 8 + Q / Gm::WPC) * 4 + pl) * Gm::CH + 4 * (Q % Gm::WPC) + 2 * (r & 1);
      *reinterpret_cast<uint16_t*>(tile + 8 * D + off) = static_cast<uint16_t>(vc);
    }
  }
  if (lane == 0) {
    *reinterpret_cast<uint32_t*>(tile + KPO + 4 * r) = ksz;
    if constexpr (!VB) *reinterpret_cast<uint32_t*>(tile + 16 * D + 64 + 4 * r) = vsz;
  }

  // INT8 side cache: sinks and the recent window (warp-uniform decision).
  int row = -1;
  if (pos < a.s)
    row = pos;
  else if (a.w > 0 && pos >= len_after - a.w)
    row = a.s + pos % a.w;
  if (row < 0) return;
  uint8_t* t8 = a.side + static_cast<size_t>(b) * a.side_slot_bytes +
                static_cast<size_t>(g) * a.nt8 * T8 + static_cast<size_t>(row >> 4) * T8;
  const int r8 = row & 15;
  uint16_t ks, vs = 0;
  bool kbad8, vbad8 = false;
  const uint32_t k8 = quant_int8(k, act, &ks, &kbad8);
  uint32_t v8 = 0;
  if constexpr (!VB) v8 = quant_int8(v, act, &vs, &vbad8);
  if (lane == 0 && (kbad8 || vbad8)) atomicOr(a.err, KV4_DEVERR_RANGE);
  if constexpr (VB) {
    if (act) {
      const int e = 4 * lane;
      *reinterpret_cast<uint32_t*>(t8 + r8 * D + 16 * ((e >> 4) ^ (r8 & 1)) + (e & 15)) = k8;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        *reinterpret_cast<__nv_bfloat16*>(t8 + Gm::VB8O + vbf_offset<D>(r8, e + i)) = __float2bfloat16_rn(v[i]);
    }
    if (lane == 0) *reinterpret_cast<uint16_t*>(t8 + 16 * D + 2 * r8) = ks;
    return;
  }
  if (act) {
    const int e = 4 * lane;
    *reinterpret_cast<uint32_t*>(t8 + r8 * D + 16 * ((e >> 4) ^ (r8 & 1)) + (e & 15)) = k8;
    const int p = r8 >> 1, half = p >> 2, pl = p & 3;
    uint8_t* vbase = t8 + Gm::H8B;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int ei = e + i, gq = ei / Gm::DG, dd = ei % Gm::DG;
      int bb = (dd >> 1) * 4 + (dd & 1) * 2 + (r8 & 1);
      if (Gm::CH8 >= 32) bb ^= 16 * (gq & 1);
      vbase[((half * 8 + gq) * 4 + pl) * Gm::CH8 + bb] = static_cast<uint8_t>(v8 >> (8 * i));
    }
  }
  if (lane == 0) {
    *reinterpret_cast<uint16_t*>(t8 + 16 * D + 2 * r8) = ks;
    *reinterpret_cast<uint16_t*>(t8 + Gm::H8B + 16 * D + 2 * r8) = vs;
  }
}

// BF16 baseline pool append: K and V stored as bf16 (no rotation, no quantisation).
template <int D, typename KT, typename VT>
__global__ void __launch_bounds__(kAppendThreads) append_bf16_kernel(AppendArgs a) {
  using Gm = Geo<D>;
  const int gw = static_cast<int>((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
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
  if (lane >= D / 4) return;
  float k[4], v[4];
  const size_t in0 = (static_cast<size_t>(t) * a.Hkv + g) * D + 4 * lane;
  load4<KT>(a.K, in0, k);
  load4<VT>(a.V, in0, v);
  const int pp = pos % a.P, r = pp & 15;
  uint8_t* tile = a.pool + static_cast<size_t>(page) * a.page_bytes + static_cast<size_t>(g) * a.P * 4 * D +
                  static_cast<size_t>(pp >> 4) * Gm::TBF;
  // K row r: element e in thread chunk c = e / EPT, unit u = (e % EPT) / 8 stored at u ^ sw.
  const int e = 4 * lane, c = e / Gm::EPT, u = (e % Gm::EPT) >> 3;
  const int kofs = r * 2 * D + c * 2 * Gm::EPT + ((u ^ bf16_swz(D, c, r)) << 4) + (e & 7) * 2;
  uint2 kw;
  kw.x = pack_bf2(__float2bfloat16_rn(k[0]), __float2bfloat16_rn(k[1]));
  kw.y = pack_bf2(__float2bfloat16_rn(k[2]), __float2bfloat16_rn(k[3]));
  *reinterpret_cast<uint2*>(tile + kofs) = kw;
  // V: pair p = r >> 1, group gq = e / DG, word m = e % DG of the chunk.
  const int p = r >> 1, half = p >> 2, pl = p & 3;
  uint8_t* vb = tile + 32 * D;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int ei = e + i, gq = ei / Gm::DG, m = ei % Gm::DG, uu = m >> 2;
    const int ofs = ((half * 8 + gq) * 4 + pl) * (D / 2) + ((uu ^ bf16_swz(D, pl, gq)) << 4) + (m & 3) * 4 + (r & 1) * 2;
    *reinterpret_cast<__nv_bfloat16*>(vb + ofs) = __float2bfloat16_rn(v[i]);
  }
}

#define KV4_APPEND_LAUNCH(KERN, KT, VT) KERN<D, KT, VT><<<grid, block, 0, st>>>(a)
#define KV4_APPEND_LAUNCH4(KT, VT)                                   \
  do {                                                               \
    if (a.vbf) append_int4_kernel<D, KT, VT, true><<<grid, block, 0, st>>>(a); \
    else append_int4_kernel<D, KT, VT, false><<<grid, block, 0, st>>>(a);      \
  } while (0)

template <int D, bool BF16_POOL>
cudaError_t dispatch_types(const AppendArgs& a, cudaStream_t st) {
  // 8-warp blocks: a block of this kernel keeps the following decode kernel's block (which needs a
  // whole SM) off its SM until it exits, but spreading the append over more SMs ends it sooner,
  // and that measured better for the whole step than fewer 32-warp blocks (0.0606 vs 0.0633 ms).
  const int warps = a.T * a.Hkv;
  const dim3 grid((warps + kAppendThreads / 32 - 1) / (kAppendThreads / 32)), block(kAppendThreads);
  const bool kf = a.k_dtype == KV4_F32, vf = a.v_dtype == KV4_F32;
  if (BF16_POOL) {
    if (kf && vf) KV4_APPEND_LAUNCH(append_bf16_kernel, float, float);
    else if (kf) KV4_APPEND_LAUNCH(append_bf16_kernel, float, __nv_bfloat16);
    else if (vf) KV4_APPEND_LAUNCH(append_bf16_kernel, __nv_bfloat16, float);
    else KV4_APPEND_LAUNCH(append_bf16_kernel, __nv_bfloat16, __nv_bfloat16);
  } else {
    if (kf && vf) KV4_APPEND_LAUNCH4(float, float);
    else if (kf) KV4_APPEND_LAUNCH4(float, __nv_bfloat16);
    else if (vf) KV4_APPEND_LAUNCH4(__nv_bfloat16, float);
    else KV4_APPEND_LAUNCH4(__nv_bfloat16, __nv_bfloat16);
  }
  return cudaGetLastError();
}

#undef KV4_APPEND_LAUNCH
#undef KV4_APPEND_LAUNCH4

}  // namespace

cudaError_t launch_append_int4(const AppendArgs& a, int D, cudaStream_t st) {
  if (a.T <= 0) return cudaSuccess;
  note_launches(1);
  return D == 128 ? dispatch_types<128, false>(a, st) : dispatch_types<64, false>(a, st);
}

cudaError_t launch_append_bf16(const AppendArgs& a, int D, cudaStream_t st) {
  if (a.T <= 0) return cudaSuccess;
  note_launches(1);
  return D == 128 ? dispatch_types<128, true>(a, st) : dispatch_types<64, true>(a, st);
}

}  // namespace kv4
