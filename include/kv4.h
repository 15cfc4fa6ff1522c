/*
 * kv4.h -- C ABI of libkv4.so: a paged, calibration-free INT4 KV cache with an INT8 sink/recent
 * side cache, and decode-step attention over it, for NVIDIA B200 (sm_100a).
 *
 * The method (page titles and sections it is defined in):
 *   KV4-RL: Unlocking Faster Asynchronous Rollouts for RLVR with INT4 KV Cache Quantization
 *     (ai.info summary), "Methodology in Plain English" paragraphs 2-3 and "Key Contributions"
 *     item 4: every new K/V vector becomes one affine INT4 group per token-head vector with an
 *     FP16 scale and offset, applied after the dot-product reduction; keys are stored in a
 *     Hadamard-rotated basis and queries are rotated to match; the packed codes are read
 *     directly by the attention kernel; an INT8 side cache holds the first s (sink) and the
 *     most recent w positions; the INT4 and INT8 regions are attended as disjoint sets and
 *     combined through regional softmax statistics.
 *   SAW-INT4: System-Aware 4-Bit KV-Cache Quantization (gist.science summary), section 2:
 *     token-wise INT4 in the unchanged paged buffers, block-diagonal Hadamard rotation with
 *     block size h, rotation and quantisation fused in one kernel.
 *
 * Conventions the pages leave open (fixed here, identical in the test oracle):
 *   - Hadamard: Sylvester order, unnormalised, on contiguous blocks of h elements (h a power
 *     of two dividing head_dim; h = 1 means no rotation), optionally after a per-dimension sign
 *     flip (kv4_set_rotation_signs).  Keys are stored rotated; the query is multiplied by the
 *     same rotation over h, so rotated query . rotated key = q . k.  Values are stored as given
 *     unless kv4_set_value_rotation is on (then rotated too, and outputs rotated back).
 *   - INT4: zero = fp16 rounded toward -inf of min(x); scale = fp16 rounded toward +inf of
 *     fl32(max(x) - zero)/15; code = clamp(rint((x - zero)/scale), 0, 15) in IEEE fp32;
 *     x is reconstructed as zero + scale * code.
 *   - INT8 (side cache): symmetric, scale = fp16 rounded toward +inf of max|x|/127,
 *     code = clamp(rint(x/scale), -127, 127).
 *   - Routing: every appended token is written to the INT4 pages; in addition position pos
 *     goes to side row pos when pos < s, and to side row s + (pos mod w) when pos >= s and
 *     pos >= lens_after[seq] - w.  Decode at length L reads sinks [0, min(s, L)) and recent
 *     [max(s, L - w), L) from the side cache and the INT4 region [s, max(s, L - w)) from pages.
 *   - Attention: q head j reads KV head j / (Hq/Hkv); softmax scale 1/sqrt(head_dim);
 *     out is fp32, lse (optional) is m + ln(l) in natural log.
 *
 * Memory: the caller owns every device buffer (page pools, side cache, workspace, inputs,
 * outputs) and the stream.  The library never allocates or frees device memory in these calls;
 * kv4_cache_init allocates only the small host handle.  All launches are asynchronous on the
 * given stream (a cudaStream_t passed as void*; NULL = legacy default stream).
 *
 * Errors: arguments are validated on the host before anything is launched; a failed check
 * returns a status and launches nothing.  A failed launch returns KV4_ERR_CUDA.  Device-side
 * guards (page id outside the pool, a bounded wait that ran out) skip the access and set bits
 * in a per-device error word read by kv4_get_device_error.  No kernel traps or spins forever.
 */
#ifndef KV4_H
#define KV4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KV4_OK = 0,
  KV4_ERR_INVALID_ARG = 1,  /* null pointer, negative size, index out of range          */
  KV4_ERR_UNSUPPORTED = 2,  /* geometry outside the compiled variants (see kv4_config)  */
  KV4_ERR_WORKSPACE = 3,    /* workspace missing or smaller than kv4_*_workspace_bytes  */
  KV4_ERR_CUDA = 4,         /* a CUDA runtime call or kernel launch failed              */
  KV4_ERR_DEVICE = 5,       /* device-side guard fired (kv4_get_device_error has bits)  */
  KV4_ERR_NO_ALLOCATION = 6 /* mixed bit-width keys: the layer has no block allocation yet
                               (kv4_allocate_key_bits or kv4_set_key_allocation)          */
} kv4_status;

typedef enum { KV4_F32 = 0, KV4_BF16 = 1, KV4_F16 = 2 } kv4_dtype;

/* Device error word bits (kv4_get_device_error). */
#define KV4_DEVERR_PAGE_RANGE 0x1u  /* page-table entry outside [0, max_pages)            */
#define KV4_DEVERR_WAIT_LIMIT 0x2u  /* a bounded wait for a bulk copy ran out             */
#define KV4_DEVERR_LENGTH 0x4u      /* a length or position beyond the page-table row     */
#define KV4_DEVERR_RANGE 0x8u       /* an appended vector's fp16 scale or offset overflowed: its
                                       values reach beyond the fp16 range; the vector was stored
                                       with all-zero codes and its non-finite parameters        */
#define KV4_DEVERR_RECORD 0x10u     /* the merge found a split-partial record pointing outside the
                                       workspace (left by a decode that stopped early) and
                                       skipped it                                               */

/* Storage formats (kv4_config.value_format). */
#define KV4_VALUES_INT4 0  /* values as per-token affine INT4 (INT8 in the side cache): KV4       */
#define KV4_VALUES_BF16 1  /* values kept in bf16 in the pages and the side cache, keys as in KV4 */
#define KV4_KEYS_MIXED 2   /* mixed bit-width keys allocated per RoPE block, values at value_bits
                              ("RoPE-Aware Bit Allocation for KV-Cache Quantization", abstract);
                              see kv4_allocate_key_bits                                          */

/*
 * Cache geometry.  Supported: head_dim in {64, 128}; Hq/Hkv in {1, 2, 4}; page_size a
 * multiple of 16; hadamard_block a power of two dividing head_dim; num_sinks >= 0,
 * recent_window >= 0.  One page table (int32 [max_seqs][stride]) is shared by all layers, as in
 * vLLM; page ids index a per-layer pool of max_pages pages.  value_format selects the value
 * storage (KV4-RL, "Main Findings", compares KV4, KV8 and BF16 KV budgets; the K-INT4 / V-BF16
 * variant keeps the INT4 keys and leaves the values unquantised): KV4_VALUES_INT4 (0, the
 * default of a zeroed struct) or KV4_VALUES_BF16 (1).  KV4_KEYS_MIXED (2) selects the mixed
 * bit-width key cache instead: keys take key_bits bits per dimension on average (1..8), split
 * over the RoPE blocks of each KV head by kv4_allocate_key_bits; values take value_bits bits per
 * dimension (2, 3, 4 or 8); it has no side cache and no rotation (num_sinks = recent_window = 0,
 * hadamard_block = 1).  key_bits and value_bits are ignored by the other formats.
 */
typedef struct {
  int num_layers;
  int num_q_heads;      /* Hq                                    */
  int num_kv_heads;     /* Hkv                                   */
  int head_dim;         /* D                                     */
  int page_size;        /* P, positions per page                 */
  int num_sinks;        /* s                                     */
  int recent_window;    /* w                                     */
  int hadamard_block;   /* h                                     */
  int max_seqs;         /* sequence slots of the INT8 side cache */
  int max_pages;        /* pages per layer pool                  */
  int value_format;     /* KV4_VALUES_INT4, KV4_VALUES_BF16 or KV4_KEYS_MIXED */
  int key_bits;         /* KV4_KEYS_MIXED: average key bits per dimension      */
  int value_bits;       /* KV4_KEYS_MIXED: value bits per dimension            */
} kv4_config;

typedef struct kv4_cache kv4_cache;  /* opaque host handle */

/*
 * Byte sizes the caller must allocate (all layers):
 *   page pool:  num_layers * max_pages * Hkv * P * (D + 8)
 *               (per token and KV head: D/2 bytes of K codes + D/2 of V codes + 2x fp16
 *               scale/zero for K and for V; 4 + 32/D bits per element for D = 128 -> 4.25,
 *               the storage KV4-RL, "Methodology in Plain English" paragraph 2, states)
 *   side cache: num_layers * max_seqs * Hkv * ceil((s + w)/16) * 16 * (2D + 4)
 * With KV4_VALUES_BF16 a position takes D/2 + 4 + 2D bytes in a page (K codes and parameters,
 * bf16 V) and 3D + 2 in the side cache (INT8 K and its scale, bf16 V).
 * With KV4_KEYS_MIXED a position takes key_bits*D/8 + value_bits*D/8 + 8 bytes in a page (the
 * packed key and value codes and four fp16: key scale, 0, value zero, value range; a page of one
 * KV head is P/16 slices of 16 positions, each holding its 16 key rows, then 16 value rows, then
 * 16 records; heads in order), the side cache is
 * empty, and the page pool ends with num_layers * Hkv block-allocation records of
 * ceil16(5 D / 2) bytes (D/2 fp32 block scales, then D/2 uint8 block widths).
 * Both must be 16-byte aligned.  Returns KV4_ERR_UNSUPPORTED for geometries outside the list.
 */
kv4_status kv4_query_sizes(const kv4_config* cfg, size_t* page_pool_bytes, size_t* side_cache_bytes);

/* Bind caller-owned device buffers to a host handle (no device work).  *out receives the handle. */
kv4_status kv4_cache_init(const kv4_config* cfg, void* page_pool, void* side_cache, kv4_cache** out);

/* Free the host handle; caller memory is untouched.  NULL is ignored. */
void kv4_cache_destroy(kv4_cache* cache);

/*
 * kv4_append: write T new tokens of one layer.  Fused per (token, KV head): block-Hadamard
 * rotation of K, per-token affine INT4 quantisation of rotated K and of V, nibble packing into
 * the token's page slot (page page_table[seq][pos / P], slot pos % P), and INT8 routing of
 * sink/recent positions into the side cache.  The method of KV4-RL (ai.info summary),
 * "Methodology in Plain English" paragraphs 2-3 (every new K/V vector quantised on the fly to one
 * affine INT4 group with fp16 scale and offset, keys in a Hadamard-rotated basis, an INT8 side
 * cache for the first s and the most recent w positions), and of SAW-INT4 (gist.science
 * summary), section 2 (block-diagonal rotation in blocks of h, fused with quantisation in one
 * kernel).
 *   K, V         device [T][Hkv][D] of k_dtype / v_dtype (KV4_F32 or KV4_BF16), contiguous
 *   seq_slot     device int32 [T]: sequence slot of each token, in [0, max_seqs)
 *   pos          device int32 [T]: position of each token in its sequence
 *   lens_after   device int32 [max_seqs]: sequence length after this call (decides which
 *                positions are "recent"); positions of one sequence must be distinct in a call
 *   page_table   device int32 [max_seqs][stride]
 * Device-side: a page id outside [0, max_pages) or pos / P >= stride sets an error bit and the
 * token is skipped; a vector whose fp16 scale or offset overflows sets KV4_DEVERR_RANGE (stored
 * with zero codes).  With KV4_VALUES_BF16 the values are stored as bf16 (nearest even) instead.
 * With KV4_KEYS_MIXED ("RoPE-Aware Bit Allocation for KV-Cache Quantization", abstract; the
 * layer's allocation from kv4_allocate_key_bits): a key gets one fp16 scale s, rounded up, of
 * max |x_j| / sigma_j over coordinates with bits, and coordinate j of width w the code
 * clamp(floor((x_j / (sigma_j s) + 1) 2^(w-1)), 0, 2^w - 1) (reconstructed as
 * s sigma_j ((2 code + 1) 2^-w - 1); 0 for w = 0); a value gets the per-token affine code of the
 * INT4 cache at value_bits bits (fp16 zero rounded down, fp16 range rounded up, code =
 * rint((x - zero) / (range / (2^b - 1)))); codes packed in coordinate order, least significant
 * bit first; lens_after is not read.
 */
kv4_status kv4_append(kv4_cache* cache, int layer, int T, const void* K, kv4_dtype k_dtype,
                      const void* V, kv4_dtype v_dtype, const int32_t* seq_slot, const int32_t* pos,
                      const int32_t* lens_after, const int32_t* page_table, int stride, void* stream);

/* Workspace bytes kv4_decode_attn needs for a batch of B sequences (upper bound for any lens). */
kv4_status kv4_decode_workspace_bytes(const kv4_cache* cache, int B, size_t* bytes);

/*
 * kv4_decode_attn: one decode step of attention for B sequences (row b of the batch is side-cache
 * slot b) at lengths lens[b] (the just-appended token included).  Rotates each query once
 * (H/h), streams the packed INT4 pages of [s, max(s, L-w)) and the INT8 rows of the sink and
 * recent regions, and merges per-region / per-split softmax statistics.  This is the decode of
 * KV4-RL (ai.info summary), "Methodology in Plain English" paragraphs 2-3 and "Key
 * Contributions" item 4: packed codes read directly, scale and offset applied after the
 * dot-product reduction, queries rotated to the keys' basis, sink and recent regions from the
 * INT8 side cache attended as disjoint regions merged with their softmax statistics.
 *   q            device [B][Hq][D] of q_dtype (KV4_F32, KV4_BF16 or KV4_F16)
 *   page_table   device int32 [>= B][stride];  lens device int32 [B] (0 gives out = 0, lse = -inf)
 *   max_len_hint host upper bound of lens (0 = unknown); only sizes the grid
 *   out          device fp32 [B][Hq][D];  lse device fp32 [B][Hq] or NULL
 *   workspace    device scratch of at least kv4_decode_workspace_bytes(B) bytes, 16-byte aligned;
 *                its contents need no initialisation and are dead after the call.  Calls that
 *                overlap on the GPU must not share a workspace.
 * Two launches on the stream: the split-K pass (one partial (o, m, l) per warp and segment it
 * touches; a warp that holds a whole INT8 region and the start of the INT4 region of a
 * (sequence, KV head) runs one softmax across both; a (sequence, KV head) covered by a single
 * partial is written directly), then the LSE merge of the partials of every other (sequence,
 * KV head).
 * With KV4_KEYS_MIXED the layer's packed pages over [0, L) are attended as one region (no side
 * cache, no rotation) with the keys and values reconstructed as kv4_append describes; two
 * launches as well (split-K pass over 16-position tiles, LSE merge).
 */
kv4_status kv4_decode_attn(kv4_cache* cache, int layer, int B, const void* q, kv4_dtype q_dtype,
                           const int32_t* page_table, int stride, const int32_t* lens, int max_len_hint,
                           float* out, float* lse, void* workspace, size_t ws_bytes, void* stream);

/*
 * kv4_set_rotation_signs: randomised-sign Hadamard rotation for this cache (a precision variant of
 * SAW-INT4's block-diagonal rotation, gist.science summary section 2; default: none).  Bit d of sign_bits (host array of ceil(head_dim / 32) words, bit d % 32 of word
 * d / 32) negates key dimension d before the block Hadamard at append, and query dimension d
 * before the query rotation at decode, so the rotation is H diag(s) with s in {+1, -1}; the
 * attention is unchanged in exact arithmetic.  NULL clears it.  The signs are part of the stored
 * format: set them before the first append to the cache and keep them.  Returns
 * KV4_ERR_INVALID_ARG for a NULL or BF16 cache.
 */
kv4_status kv4_set_rotation_signs(kv4_cache* cache, const uint32_t* sign_bits);

/*
 * kv4_set_value_rotation: store values in the keys' rotated basis too (a precision variant of the
 * rotation of KV4-RL, "Methodology in Plain English" paragraph 2, which rotates keys only;
 * default 0).  Not available with KV4_VALUES_BF16 (returns KV4_ERR_INVALID_ARG).  With 1 the append applies H diag(s) to V before quantising (INT4 and INT8 copies),
 * and the decode's merge returns every output to the original basis, out = diag(s) H o / h.  This
 * is part of the stored format: set it before the first append and keep it.  Returns
 * KV4_ERR_INVALID_ARG for a NULL or BF16 cache.
 */
kv4_status kv4_set_value_rotation(kv4_cache* cache, int enable);

/*
 * kv4_set_decode_overlap: how kv4_decode_attn of this cache starts (default 0).  Its kernel is
 * always launched as a programmatic dependent of the preceding kernel on the stream, and the
 * append kernel lets its dependent launch early.  With 0 the decode kernel reads nothing before
 * the preceding kernel has completed: stream order exactly.  With 1 it builds its work schedule
 * and first copy descriptors, reading lens and page_table only, while the preceding kernel runs,
 * then waits for it before reading q or the cache or writing any output; lens and page_table
 * must then not be written by the kernel that immediately precedes the decode on the stream
 * (writes earlier in stream order are fine).  Returns KV4_ERR_INVALID_ARG for a NULL or BF16
 * cache.
 */
kv4_status kv4_set_decode_overlap(kv4_cache* cache, int enable);

/*
 * kv4_debug_force_wait_timeout: a test hook for the device-side failure path (default 0, leave
 * it off in production).  With 1, every kv4_decode_attn of this cache makes each warp of the
 * split-K kernel wait, with a 1 ms limit, on a barrier that nothing arrives on: the wait runs
 * out, the warp sets KV4_DEVERR_WAIT_LIMIT, waits (bounded) for the bulk copies it already has
 * in flight, and returns.  The merge kernel then finds no fresh partial records: records that
 * point outside the workspace are skipped with KV4_DEVERR_RECORD.  That call's out and lse are
 * undefined; the context stays usable, and a call with 0 decodes normally.  The mixed
 * bit-width key cache takes the same path: each decode warp's first wait is on a barrier nothing
 * arrives on, runs out after 1 ms, sets KV4_DEVERR_WAIT_LIMIT, and the warp waits (bounded) for
 * its copies in flight and returns; that call's out and lse are undefined.  Returns
 * KV4_ERR_INVALID_ARG for a NULL or BF16 cache.
 */
kv4_status kv4_debug_force_wait_timeout(kv4_cache* cache, int enable);

/*
 * kv4_debug_mixed_row_copies: a test hook for the mixed bit-width key cache (default 0).  Key rows
 * whose word count is a multiple of 16 (4- and 8-bit keys at D = 128, 8-bit at D = 64) are
 * padded in shared memory and normally arrive by one tensor copy per 16-position slice; that
 * copy needs a tensor map from the driver's encoder.  With 1, kv4_decode_attn takes the path used
 * when the encoder is missing or refuses: one bulk copy per key row.  Results are the same either
 * way.  Returns KV4_ERR_INVALID_ARG for a NULL cache or one of another format.
 */
kv4_status kv4_debug_mixed_row_copies(kv4_cache* cache, int enable);

/*
 * Mixed bit-width keys (KV4_KEYS_MIXED): the block allocation of one layer.  "RoPE-Aware Bit
 * Allocation for KV-Cache Quantization" (searcharxiv abstract): under RoPE a key's share of a
 * later logit is a sum over its two-dimensional frequency blocks, so for every layer and KV head a
 * label-free energy score is taken per RoPE block and integer bit widths are handed out greedily
 * by marginal gain under the key budget.  Conventions: block b of a head is the rotate-half pair
 * of coordinates (b, b + D/2); its score E_b is the fp64 sum of k[b]^2 + k[b + D/2]^2 over the
 * given keys in order; its scale is sigma_b = sqrt(E_b / 2T) rounded to fp32 (1 when E_b = 0);
 * starting from 0 bits, one bit at a time goes to the block of largest E_b 4^-w_b below 8 bits
 * (lowest block on ties) until the blocks hold key_bits * D / 2 bits.
 *
 * kv4_allocate_key_bits scores the T keys K [T][Hkv][D] (KV4_F32, KV4_BF16 or KV4_F16, device
 * memory) and writes the allocation of every KV head of the layer, all on the device (one
 * kernel, one thread block per KV head summing in key order: about T * 10 ns).  Later appends of
 * the layer quantise with it; re-allocating does not re-encode what is already stored.
 * kv4_set_key_allocation copies a caller's allocation (host arrays widths [Hkv][D/2], each <= 8
 * with D/2-sums of key_bits * D / 2, and sigma [Hkv][D/2], positive and finite) to the device;
 * kv4_get_key_allocation copies the layer's allocation back to host arrays and synchronises the
 * stream.  Append and decode of a layer without an allocation return KV4_ERR_NO_ALLOCATION.
 */
kv4_status kv4_allocate_key_bits(kv4_cache* cache, int layer, int T, const void* K, kv4_dtype k_dtype, void* stream);
kv4_status kv4_set_key_allocation(kv4_cache* cache, int layer, const uint8_t* widths, const float* sigma, void* stream);
kv4_status kv4_get_key_allocation(kv4_cache* cache, int layer, uint8_t* widths, float* sigma, void* stream);

/*
 * BF16-KV baseline (KV4-RL, "Main Findings", quotes its speed-ups against BF16 KV) with the same
 * page table and conventions, no quantisation and no rotation:
 * a page holds Hkv head blocks of P * 4D bytes (bf16 K and V).  Used to measure the INT4
 * speed-up on the same GPU.  kv4_bf16_query_sizes returns num_layers * max_pages * Hkv * P * 4D.
 */
kv4_status kv4_bf16_query_sizes(const kv4_config* cfg, size_t* page_pool_bytes);
kv4_status kv4_bf16_cache_init(const kv4_config* cfg, void* page_pool, kv4_cache** out);
kv4_status kv4_bf16_append(kv4_cache* cache, int layer, int T, const void* K, kv4_dtype k_dtype,
                           const void* V, kv4_dtype v_dtype, const int32_t* seq_slot, const int32_t* pos,
                           const int32_t* page_table, int stride, void* stream);
kv4_status kv4_bf16_decode_workspace_bytes(const kv4_cache* cache, int B, size_t* bytes);
kv4_status kv4_bf16_decode_attn(kv4_cache* cache, int layer, int B, const void* q, kv4_dtype q_dtype,
                                const int32_t* page_table, int stride, const int32_t* lens,
                                int max_len_hint, float* out, float* lse, void* workspace,
                                size_t ws_bytes, void* stream);

/*
 * kv4_decode_attn_static: kv4_decode_attn for callers that cannot allocate device memory -- code
 * running inside another runtime's memory pool that forbids foreign allocations, a serving
 * process that reserved all device memory up front for its page pools, or a caller that has no
 * allocator of its own to size and keep a workspace.  The method pages have no counterpart; this
 * is a deployment variant of the same decode.
 * The split-K partials live in a static device array of KV4_STATIC_SCRATCH_BYTES per GPU, part of
 * the library image and held by every GPU that loads libkv4.so until the process exits.  The
 * call allocates and frees nothing.  Arguments and results are those of kv4_decode_attn minus the
 * workspace.  The limit: a call is accepted when kv4_decode_workspace_bytes(cache, B) <=
 * KV4_STATIC_SCRATCH_BYTES, else it returns KV4_ERR_WORKSPACE and launches nothing.  That size
 * holds one 16-byte record per (sequence slot, KV head) of the cache (max_seqs * Hkv * 16 bytes,
 * so the limit shrinks as max_seqs grows) plus the split partials of B sequences; for 8 KV heads,
 * head_dim 128, 4 q heads per KV head on 148 SMs and max_seqs = B it admits B <= 347.
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress) with that
 * device current; make that first call before any stream capture.  All calls on one GPU share
 * the array; every call writes every partial its merge reads, so nothing needs clearing between
 * calls.  Calls that overlap on the
 * GPU (different streams, or another thread) race on the array and must be serialised by the
 * caller.
 */
#define KV4_STATIC_SCRATCH_BYTES (16u << 20)
kv4_status kv4_decode_attn_static(kv4_cache* cache, int layer, int B, const void* q, kv4_dtype q_dtype,
                                  const int32_t* page_table, int stride, const int32_t* lens, int max_len_hint,
                                  float* out, float* lse, void* stream);

/* Read and clear the device error word of the current device (synchronises the device). */
kv4_status kv4_get_device_error(uint32_t* bits);

/* Number of kernels the library has launched since load (all devices). */
uint64_t kv4_launch_count(void);

const char* kv4_status_string(kv4_status status);
int kv4_version(void);

#ifdef __cplusplus
}
#endif
#endif /* KV4_H */
