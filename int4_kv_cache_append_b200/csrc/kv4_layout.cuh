// kv4_layout.cuh -- byte layout of the INT4 page pool, the INT8 side cache and the BF16 pool.
//
// The method pages fix what is stored (one INT4 group per token-head vector with fp16 scale and
// offset; an INT8 side cache for sink and recent positions -- KV4-RL, "Methodology in Plain
// English" paragraphs 2-3) but not where; this layout is this library's own, chosen so that one
// 16-token tile of one KV head is a single contiguous block that one bulk copy brings into
// shared memory, and so that each decode thread's MMA operand bytes are 16-byte contiguous and
// bank-conflict free.
//
// INT4 page pool (one layer): page = Hkv head blocks of P*(D+8) bytes; head block = P/16 tiles
// of T4B = 16*(D+8) bytes; in a tile (row r = position % 16):
//   [0, 8D)            K codes in 8 pair-rows of D bytes: pair-row p = r % 8 holds row p in the
//                      low nibbles and row p + 8 in the high nibbles, one byte per element e:
//                      byte 8*(e/8) + 4*(e%2) + (e%8)/2 (even elements, then odd, per 8-group);
//                      for D = 128 the 16-byte halves of each 32 bytes are swapped in odd
//                      pair-rows.  A decode lane's unpack is then one mask per four codes.
//   [8D, 16D)          V codes: 16-bit chunk (r, quad Q) holds elements 4Q..4Q+3 (4Q+k in bits
//                      4k..4k+3); rows 2p, 2p+1 share a 32-bit word (2p low half); word groups
//                      at byte ((half*8 + Q/WPC)*4 + (p&3))*CH + 4*(Q%WPC), half = p>>2.
//   [16D, 16D+64)      K {fp16 scale, fp16 zero} per row, 4 bytes at 4r.
//   [16D+64, 16D+128)  V {scale, zero}.
// INT8 side cache (one layer): slot = Hkv head blocks of NT8 = ceil((s+w)/16) tiles of
// T8B = 2*H8B bytes, H8B = 16D + 32; side row R in tile R/16, row r = R % 16:
//   [0, 16D)           K int8, row r at r*D, 16-byte unit u at unit u ^ (r & 1).
//   [16D, 16D+32)      K fp16 scale per row at 2r.
//   [H8B, H8B+16D)     V int8: for pair p = r>>1 and group gq = e/(D/8), a CH8 = D/4 byte chunk at
//                      ((half*8 + gq)*4 + (p&3))*CH8 holds words (c[2p][d], c[2p+1][d],
//                      c[2p][d+1], c[2p+1][d+1]) for d = gq*D/8 + 2m; 16-byte halves of the
//                      chunk swapped when CH8 = 32 and gq is odd.
//   [H8B+16D, T8B)     V fp16 scale per row.
// bf16 values (KV4_VALUES_BF16): a page tile is T4V = 16*(D/2 + 4 + 2D) bytes:
//   [0, 8D)            K codes as above;  [8D, 8D+64)  K {scale, zero} per row;
//   [8D+64, 40D+64)    V bf16 in the BF16 pool's V order (below).
// and a side tile T8V = 16*(3D + 2) bytes: [0, 16D+32) K int8 codes and scales as above, then
// [16D+32, 48D+32) V bf16 in the same order.
// BF16 pool (baseline): page = Hkv head blocks of P/16 tiles of 64*D bytes:
//   [0, 32D)   K bf16 row-major; row r, thread chunk c = e/(D/4) of D/2 bytes, 16-byte unit u of
//              the chunk stored at unit u ^ sw(c, r).
//   [32D, 64D) V bf16: pair p, group gq: chunk of D/2 bytes at ((half*8 + gq)*4 + (p&3))*D/2;
//              word m of the chunk = (V[2p][gq*D/8 + m], V[2p+1][...]); 16-byte unit u at
//              u ^ sw(p&3, gq).   sw(a, b) = (a & 2) | (b & 1) when D = 128, (b & 1) when D = 64.
#pragma once

namespace kv4 {

template <int D>
struct Geo {
  static_assert(D == 64 || D == 128, "head_dim 64 or 128");
  static constexpr int WPC = D / 32;          // INT4 words per thread chunk
  static constexpr int CH = 4 * WPC;          // INT4 V chunk bytes
  static constexpr int T4B = 16 * (D + 8);    // INT4 tile block
  static constexpr int H8B = 16 * D + 32;     // INT8 half tile (K or V)
  static constexpr int T8B = 2 * H8B;         // INT8 tile block
  static constexpr int CH8 = D / 4;           // INT8 V chunk bytes
  static constexpr int DG = D / 8;            // dims per thread group
  static constexpr int NKB = D / 16;          // MMA k-blocks (QK) and m-blocks (PV)
  static constexpr int TBF = 64 * D;          // BF16 tile block
  static constexpr int T4V = 40 * D + 64;      // page tile with bf16 values
  static constexpr int T8V = 48 * D + 32;      // side tile with bf16 values
  static constexpr int VBO = 8 * D + 64;       // bf16 values in a page tile
  static constexpr int VB8O = 16 * D + 32;     // bf16 values in a side tile
  static constexpr int EPT = D / 4;           // BF16 elements per thread chunk
};

// Row of one split partial in the decode workspace: o[D] then (m, l), padded to a multiple of
// four floats so that rows start on 16-byte boundaries.
template <int D>
constexpr int kPartRow = D + 4;

__host__ __device__ constexpr int bf16_swz(int D, int a, int b) { return D == 128 ? ((a & 2) | (b & 1)) : (b & 1); }

}  // namespace kv4
