// kv4_internal.h -- host-side launch interfaces between the C ABI layer and the kernels.
#pragma once

#include <cuda_runtime.h>

#include <atomic>
#include <stddef.h>
#include <stdint.h>

#include "../../include/kv4.h"

namespace kv4 {

struct AppendArgs {
  uint8_t* pool;          // layer base of the INT4 page pool (or BF16 pool)
  uint8_t* side;          // layer base of the INT8 side cache (INT4 cache only)
  const void* K;
  const void* V;
  int k_dtype, v_dtype;
  const int32_t* seq_slot;
  const int32_t* pos;
  const int32_t* lens_after;
  const int32_t* page_table;
  int stride;
  int T, Hkv, P, s, w, h, max_seqs, max_pages, nt8;
  size_t page_bytes, side_slot_bytes;
  uint32_t signs[4];      // bit d: key dim d negated before the rotation (randomised-sign Hadamard)
  int rotate_v;           // values stored in the keys' rotated basis too
  int vbf;                // values stored as bf16 (KV4_VALUES_BF16)
  // mixed bit-width keys (KV4_KEYS_MIXED)
  const uint8_t* alloc;   // this layer's block allocation records (per KV head: sigma, widths)
  int kbits, vbits;       // key bits per dimension (average), value bits per dimension
  uint32_t* err;
};

// Mixed bit-width key cache: one layer's block allocation is Hkv records of D/2 fp32 block scales
// followed by D/2 uint8 widths, padded to 16 bytes; the records of all layers follow the pages.
__host__ __device__ inline size_t mixed_alloc_record_bytes(int D) { return (static_cast<size_t>(D) / 2 * 5 + 15) & ~static_cast<size_t>(15); }

struct ScoreArgs {
  const void* K;          // [T][Hkv][D] keys to score
  int k_dtype;
  int T, Hkv, kbits;
  uint8_t* alloc;         // this layer's allocation records (written)
};

struct DecodeArgs {
  const uint8_t* pool;
  const uint8_t* side;
  const void* q;
  int q_dtype;
  const int32_t* page_table;
  int stride;
  const int32_t* lens;
  int B, Hq, Hkv, P, s, w, h, max_pages, nt8;
  int smw;  // s mod w (0 when w = 0): where the recent ring starts being filled
  size_t page_bytes, side_slot_bytes;
  float* part;            // split partials [num_slots][G][D + 4]
  unsigned int* meta;     // per (b, g): first INT8 / INT4 partial warps and their counts
  float* out;
  float* lse;
  float qscale;           // softmax scale in log2 units: log2(e) / sqrt(D)
  int W;                  // warps launched by the partial kernel
  int tp_shift;           // log2(P / 16) when P / 16 is a power of two, else -1
  int early;              // build the schedule before waiting on the preceding kernel
  uint32_t signs[4];      // bit d: query dim d negated before the rotation (as the keys)
  int rotate_v;           // values stored rotated: outputs are rotated back by the merge kernel
  int vbf;                // values stored as bf16 (KV4_VALUES_BF16)
  int stall_test;         // kv4_debug_force_wait_timeout: every warp's first wait runs out
  uint64_t wait_ns;       // bounded-wait limit of the bulk-copy waits
  // mixed bit-width keys (KV4_KEYS_MIXED)
  const uint8_t* alloc;   // this layer's block allocation records
  int kbits, vbits;       // key bits per dimension (average), value bits per dimension
  uint32_t* err;
};

// Launchers return cudaSuccess or the launch error.  `grid_ctas` is filled with the CTA count
// used (decode), so the host can size and check the workspace.
cudaError_t launch_append_int4(const AppendArgs& a, int D, cudaStream_t st);
cudaError_t launch_append_bf16(const AppendArgs& a, int D, cudaStream_t st);

int decode_warps_per_cta();
int decode_ctas_per_sm();
int bf16_decode_warps_per_cta();
size_t decode_smem_bytes(int D, int G);
size_t bf16_decode_smem_bytes(int D, int G);
cudaError_t launch_decode_int4(DecodeArgs a, int D, int G, int ctas, cudaStream_t st);
cudaError_t launch_decode_bf16(DecodeArgs a, int D, int G, int ctas, cudaStream_t st);

// Mixed bit-width key cache (RoPE-block bit allocation): scoring + allocation, append, decode.
cudaError_t launch_mixed_score(const ScoreArgs& a, int D, cudaStream_t st);
cudaError_t launch_append_mixed(const AppendArgs& a, int D, cudaStream_t st);
int mixed_decode_warps_per_cta();
int mixed_decode_ctas_per_sm(int D, int G, int value_bits, int key_bits);
// row_copies: padded key rows by one bulk copy per row instead of the tensor copy (a test hook)
cudaError_t launch_decode_mixed(DecodeArgs a, int D, int G, int ctas, cudaStream_t st, bool row_copies);

// Counts every kernel launch the library issues.
void note_launches(int n);

// Raise a kernel's dynamic shared-memory limit once per device (not on every launch, so that
// launches inside a CUDA-graph capture make no attribute calls).
template <typename Kernel>
cudaError_t ensure_smem_limit(Kernel kernel, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = 1ull << (dev & 63);
  if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

}  // namespace kv4
