// kv4_api.cu -- the C ABI of libkv4.so (declared in include/kv4.h): argument validation on the
// host, grid sizing from the SM count, and the launches.  No device memory is allocated here
// except the library's one static per-device error word.
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "../../include/kv4.h"
#include "kv4_internal.h"

namespace {

__device__ uint32_t g_kv4_device_error;

constexpr int kMaxDevices = 64;
std::mutex g_mu;
uint32_t* g_err_ptr[kMaxDevices] = {};
int g_sm_count[kMaxDevices] = {};
std::atomic<uint64_t> g_launches{0};

enum Format { FMT_INT4 = 1, FMT_BF16 = 2, FMT_MIXED = 3 };

}  // namespace

struct kv4_cache {
  kv4_config cfg;
  int format;
  uint8_t* pool;
  uint8_t* side;
  size_t page_bytes;       // one page, all KV heads
  size_t pool_layer_bytes;
  size_t side_slot_bytes;  // one sequence slot, all KV heads
  size_t side_layer_bytes;
  int nt8;
  int overlap;        // kv4_set_decode_overlap
  uint32_t signs[4];  // kv4_set_rotation_signs
  int rotate_v;       // kv4_set_value_rotation
  int stall_test;     // kv4_debug_force_wait_timeout
  int mixed_rows;     // kv4_debug_mixed_row_copies
  // mixed bit-width keys: per-layer block-allocation records after the pages, and which layers
  // have one
  uint8_t* alloc_base;
  size_t alloc_layer_bytes;
  std::vector<uint8_t> allocated;
};

namespace kv4 {
void note_launches(int n) { g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed); }
}  // namespace kv4

namespace {

bool device_info(uint32_t** err, int* sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_kv4_device_error) != cudaSuccess) return false;
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return false;
    g_err_ptr[dev] = static_cast<uint32_t*>(p);
    g_sm_count[dev] = n;
  }
  if (err) *err = g_err_ptr[dev];
  if (sms) *sms = g_sm_count[dev];
  return true;
}

bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }
bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

kv4_status check_config(const kv4_config* c) {
  if (!c) return KV4_ERR_INVALID_ARG;
  if (c->num_layers <= 0 || c->num_q_heads <= 0 || c->num_kv_heads <= 0 || c->max_seqs <= 0 || c->max_pages <= 0 ||
      c->page_size <= 0 || c->num_sinks < 0 || c->recent_window < 0 || c->head_dim <= 0 || c->hadamard_block <= 0)
    return KV4_ERR_INVALID_ARG;
  if (c->num_q_heads % c->num_kv_heads) return KV4_ERR_INVALID_ARG;
  const int G = c->num_q_heads / c->num_kv_heads;
  if (G != 1 && G != 2 && G != 4) return KV4_ERR_UNSUPPORTED;
  if (c->head_dim != 64 && c->head_dim != 128) return KV4_ERR_UNSUPPORTED;
  if (c->page_size % 16) return KV4_ERR_UNSUPPORTED;
  if (!pow2(c->hadamard_block) || c->head_dim % c->hadamard_block) return KV4_ERR_INVALID_ARG;
  if (c->num_sinks > (1 << 20) || c->recent_window > (1 << 20)) return KV4_ERR_UNSUPPORTED;
  if (c->value_format != KV4_VALUES_INT4 && c->value_format != KV4_VALUES_BF16 && c->value_format != KV4_KEYS_MIXED)
    return KV4_ERR_INVALID_ARG;
  if (c->value_format == KV4_KEYS_MIXED) {
    // the mixed bit-width key cache has no side cache and no rotation
    if (c->num_sinks != 0 || c->recent_window != 0 || c->hadamard_block != 1) return KV4_ERR_INVALID_ARG;
    if (c->key_bits < 1 || c->key_bits > 8) return KV4_ERR_INVALID_ARG;
    if (c->value_bits != 2 && c->value_bits != 3 && c->value_bits != 4 && c->value_bits != 8) return KV4_ERR_UNSUPPORTED;
  }
  return KV4_OK;
}

size_t mixed_alloc_layer_bytes(const kv4_config* c) {
  return static_cast<size_t>(c->num_kv_heads) * kv4::mixed_alloc_record_bytes(c->head_dim);
}

void sizes(const kv4_config* c, size_t* page_bytes, size_t* side_slot, int* nt8) {
  const size_t D = static_cast<size_t>(c->head_dim);
  if (c->value_format == KV4_KEYS_MIXED) {
    *page_bytes = static_cast<size_t>(c->num_kv_heads) * static_cast<size_t>(c->page_size) *
                  (static_cast<size_t>(c->key_bits + c->value_bits) * D / 8 + 8);
    *nt8 = 0;
    *side_slot = 0;
    return;
  }
  const bool vbf = c->value_format == KV4_VALUES_BF16;
  *page_bytes = static_cast<size_t>(c->num_kv_heads) * static_cast<size_t>(c->page_size) * (vbf ? D / 2 + 4 + 2 * D : D + 8);
  *nt8 = (c->num_sinks + c->recent_window + 15) / 16;
  *side_slot = static_cast<size_t>(c->num_kv_heads) * static_cast<size_t>(*nt8) * 16u * (vbf ? 3 * D + 2 : 2 * D + 4);
}

kv4_status dtype_ok_kv(kv4_dtype d) { return (d == KV4_F32 || d == KV4_BF16) ? KV4_OK : KV4_ERR_INVALID_ARG; }
kv4_status dtype_ok_q(kv4_dtype d) {
  return (d == KV4_F32 || d == KV4_BF16 || d == KV4_F16) ? KV4_OK : KV4_ERR_INVALID_ARG;
}

size_t align16(size_t x) { return (x + 15) & ~static_cast<size_t>(15); }

int decode_ctas_full(const kv4_cache* c, int sms) {
  if (c->format == FMT_INT4) return kv4::decode_ctas_per_sm() * sms;
  if (c->format == FMT_MIXED)
    return kv4::mixed_decode_ctas_per_sm(c->cfg.head_dim, c->cfg.num_q_heads / c->cfg.num_kv_heads, c->cfg.value_bits,
                                         c->cfg.key_bits) * sms;
  return sms;
}

int warps_per_cta(int format) {
  return format == FMT_INT4 ? kv4::decode_warps_per_cta()
                            : (format == FMT_MIXED ? kv4::mixed_decode_warps_per_cta() : kv4::bf16_decode_warps_per_cta());
}

// Workspace: per (sequence, KV head) a 16-byte record of where its partials are (max_seqs * Hkv
// records, INT4 format), then the split partials, one row group of G rows of (o[D], m, l) padded
// to D + 4 floats per possible partial index (warps of the grid + 2 * B * Hkv segments).
size_t meta_bytes(const kv4_cache* c) {
  return c->format == FMT_INT4 ? static_cast<size_t>(c->cfg.max_seqs) * c->cfg.num_kv_heads * 16 : 0;
}

size_t workspace_for(const kv4_cache* c, int B, int ctas) {
  const int G = c->cfg.num_q_heads / c->cfg.num_kv_heads;
  const int warps = ctas * warps_per_cta(c->format);
  const size_t segs = static_cast<size_t>(B) * c->cfg.num_kv_heads * (c->format == FMT_INT4 ? 2 : 1);
  return meta_bytes(c) + align16((static_cast<size_t>(warps) + segs) * G * (c->cfg.head_dim + 4) * sizeof(float));
}

// The format the INT4-cache entry points serve for this handle: the INT4 cache or the mixed
// bit-width key cache (a BF16 baseline handle maps to FMT_INT4 and is then rejected).
int own_format(const kv4_cache* c) { return (c && c->format == FMT_MIXED) ? FMT_MIXED : FMT_INT4; }

kv4_status append_common(kv4_cache* c, int fmt, int layer, int T, const void* K, kv4_dtype kd, const void* V,
                         kv4_dtype vd, const int32_t* seq_slot, const int32_t* pos, const int32_t* lens_after,
                         const int32_t* page_table, int stride, void* stream) {
  if (!c || c->format != fmt) return KV4_ERR_INVALID_ARG;
  if (layer < 0 || layer >= c->cfg.num_layers || T < 0 || stride <= 0) return KV4_ERR_INVALID_ARG;
  if (T == 0) return KV4_OK;
  if (!K || !V || !seq_slot || !pos || !page_table || (fmt == FMT_INT4 && !lens_after)) return KV4_ERR_INVALID_ARG;
  if (fmt == FMT_MIXED && !c->allocated[layer]) return KV4_ERR_NO_ALLOCATION;
  if (dtype_ok_kv(kd) != KV4_OK || dtype_ok_kv(vd) != KV4_OK) return KV4_ERR_INVALID_ARG;
  if (!aligned(K, kd == KV4_F32 ? 16 : 8) || !aligned(V, vd == KV4_F32 ? 16 : 8)) return KV4_ERR_INVALID_ARG;
  if (static_cast<long long>(T) * c->cfg.num_kv_heads > (1LL << 30)) return KV4_ERR_UNSUPPORTED;
  uint32_t* err = nullptr;
  if (!device_info(&err, nullptr)) return KV4_ERR_CUDA;
  kv4::AppendArgs a{};
  a.pool = c->pool + static_cast<size_t>(layer) * c->pool_layer_bytes;
  a.side = c->side ? c->side + static_cast<size_t>(layer) * c->side_layer_bytes : nullptr;
  a.K = K;
  a.V = V;
  a.k_dtype = kd;
  a.v_dtype = vd;
  a.seq_slot = seq_slot;
  a.pos = pos;
  a.lens_after = lens_after;
  a.page_table = page_table;
  a.stride = stride;
  a.T = T;
  a.Hkv = c->cfg.num_kv_heads;
  a.P = c->cfg.page_size;
  a.s = c->cfg.num_sinks;
  a.w = c->cfg.recent_window;
  a.h = c->cfg.hadamard_block;
  a.max_seqs = c->cfg.max_seqs;
  a.max_pages = c->cfg.max_pages;
  a.nt8 = c->nt8;
  a.page_bytes = c->page_bytes;
  a.side_slot_bytes = c->side_slot_bytes;
  for (int i = 0; i < 4; ++i) a.signs[i] = fmt == FMT_INT4 ? c->signs[i] : 0u;
  a.rotate_v = fmt == FMT_INT4 ? c->rotate_v : 0;
  a.vbf = (fmt == FMT_INT4 && c->cfg.value_format == KV4_VALUES_BF16) ? 1 : 0;
  if (fmt == FMT_MIXED) {
    a.alloc = c->alloc_base + static_cast<size_t>(layer) * c->alloc_layer_bytes;
    a.kbits = c->cfg.key_bits;
    a.vbits = c->cfg.value_bits;
  }
  a.err = err;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const cudaError_t e = fmt == FMT_INT4    ? kv4::launch_append_int4(a, c->cfg.head_dim, st)
                        : fmt == FMT_MIXED ? kv4::launch_append_mixed(a, c->cfg.head_dim, st)
                                           : kv4::launch_append_bf16(a, c->cfg.head_dim, st);
  return e == cudaSuccess ? KV4_OK : KV4_ERR_CUDA;
}

kv4_status decode_common(kv4_cache* c, int fmt, int layer, int B, const void* q, kv4_dtype qd,
                         const int32_t* page_table, int stride, const int32_t* lens, int max_len_hint, float* out,
                         float* lse, void* ws, size_t ws_bytes, void* stream) {
  if (!c || c->format != fmt) return KV4_ERR_INVALID_ARG;
  if (layer < 0 || layer >= c->cfg.num_layers || B < 0 || B > c->cfg.max_seqs || stride <= 0 || max_len_hint < 0)
    return KV4_ERR_INVALID_ARG;
  if (B == 0) return KV4_OK;
  if (!q || !page_table || !lens || !out) return KV4_ERR_INVALID_ARG;
  if (dtype_ok_q(qd) != KV4_OK) return KV4_ERR_INVALID_ARG;
  if (!aligned(q, qd == KV4_F32 ? 4 : 2) || !aligned(out, 16)) return KV4_ERR_INVALID_ARG;
  if (!ws || !aligned(ws, 16)) return KV4_ERR_WORKSPACE;
  if (fmt == FMT_MIXED && !c->allocated[layer]) return KV4_ERR_NO_ALLOCATION;
  uint32_t* err = nullptr;
  int sms = 0;
  if (!device_info(&err, &sms)) return KV4_ERR_CUDA;
  const int full = decode_ctas_full(c, sms);
  int ctas = full;
  if (max_len_hint > 0) {
    // Enough CTAs that each warp gets at least ~16 slots of the hinted upper bound.
    const long long tiles = (static_cast<long long>(max_len_hint) + 15) / 16;
    const long long slots = static_cast<long long>(B) * c->cfg.num_kv_heads * (tiles + (fmt == FMT_INT4 ? 2LL * c->nt8 : 0));
    const int warps = warps_per_cta(fmt);
    long long want = (slots + 16LL * warps - 1) / (16LL * warps);
    if (want < 1) want = 1;
    if (want < ctas) ctas = static_cast<int>(want);
  }
  if (ws_bytes < workspace_for(c, B, ctas)) return KV4_ERR_WORKSPACE;
  {
    // work units are counted in 32 bits on the device: bound the worst case (every sequence at
    // the page-table capacity)
    const long long tiles = (static_cast<long long>(stride) * c->cfg.page_size + 15) / 16;
    const long long units = static_cast<long long>(B) * c->cfg.num_kv_heads * (tiles + 2LL * c->nt8);
    if (units >= (1LL << 31)) return KV4_ERR_UNSUPPORTED;
  }
  kv4::DecodeArgs a{};
  a.pool = c->pool + static_cast<size_t>(layer) * c->pool_layer_bytes;
  a.side = c->side ? c->side + static_cast<size_t>(layer) * c->side_layer_bytes : nullptr;
  a.q = q;
  a.q_dtype = qd;
  a.page_table = page_table;
  a.stride = stride;
  a.lens = lens;
  a.B = B;
  a.Hq = c->cfg.num_q_heads;
  a.Hkv = c->cfg.num_kv_heads;
  a.P = c->cfg.page_size;
  a.s = fmt == FMT_INT4 ? c->cfg.num_sinks : 0;
  a.w = fmt == FMT_INT4 ? c->cfg.recent_window : 0;
  a.h = fmt == FMT_INT4 ? c->cfg.hadamard_block : 1;
  a.max_pages = c->cfg.max_pages;
  a.nt8 = c->nt8;
  a.smw = a.w > 0 ? a.s % a.w : 0;
  a.page_bytes = c->page_bytes;
  a.side_slot_bytes = c->side_slot_bytes;
  a.meta = static_cast<unsigned int*>(ws);
  a.part = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + meta_bytes(c));
  a.out = out;
  a.lse = lse;
  a.qscale = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(c->cfg.head_dim)));
  a.err = err;
  a.early = (fmt == FMT_INT4 && c->overlap) ? 1 : 0;
  for (int i = 0; i < 4; ++i) a.signs[i] = c->signs[i];
  a.rotate_v = fmt == FMT_INT4 ? c->rotate_v : 0;
  a.vbf = (fmt == FMT_INT4 && c->cfg.value_format == KV4_VALUES_BF16) ? 1 : 0;
  const int tpp = c->cfg.page_size / 16;
  a.tp_shift = pow2(tpp) ? __builtin_ctz(static_cast<unsigned>(tpp)) : -1;
  // The wait-limit test runs every warp's first wait out after 1 ms; the normal limit is 2 s.
  a.stall_test = ((fmt == FMT_INT4 || fmt == FMT_MIXED) && c->stall_test) ? 1 : 0;
  a.wait_ns = a.stall_test ? 1000000ull : 2000000000ull;
  if (fmt == FMT_MIXED) {
    a.alloc = c->alloc_base + static_cast<size_t>(layer) * c->alloc_layer_bytes;
    a.kbits = c->cfg.key_bits;
    a.vbits = c->cfg.value_bits;
  }
  const int G = c->cfg.num_q_heads / c->cfg.num_kv_heads;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  const cudaError_t e = fmt == FMT_INT4    ? kv4::launch_decode_int4(a, c->cfg.head_dim, G, ctas, st)
                        : fmt == FMT_MIXED ? kv4::launch_decode_mixed(a, c->cfg.head_dim, G, ctas, st, c->mixed_rows != 0)
                                           : kv4::launch_decode_bf16(a, c->cfg.head_dim, G, ctas, st);
  return e == cudaSuccess ? KV4_OK : KV4_ERR_CUDA;
}

}  // namespace

extern "C" {

kv4_status kv4_query_sizes(const kv4_config* cfg, size_t* page_pool_bytes, size_t* side_cache_bytes) {
  const kv4_status st = check_config(cfg);
  if (st != KV4_OK) return st;
  size_t pb, ss;
  int nt8;
  sizes(cfg, &pb, &ss, &nt8);
  if (page_pool_bytes)
    *page_pool_bytes = static_cast<size_t>(cfg->num_layers) * cfg->max_pages * pb +
                       (cfg->value_format == KV4_KEYS_MIXED ? static_cast<size_t>(cfg->num_layers) * mixed_alloc_layer_bytes(cfg) : 0);
  if (side_cache_bytes) *side_cache_bytes = static_cast<size_t>(cfg->num_layers) * cfg->max_seqs * ss;
  return KV4_OK;
}

kv4_status kv4_cache_init(const kv4_config* cfg, void* page_pool, void* side_cache, kv4_cache** out) {
  const kv4_status st = check_config(cfg);
  if (st != KV4_OK) return st;
  if (!out || !page_pool || !aligned(page_pool, 16)) return KV4_ERR_INVALID_ARG;
  const bool need_side = cfg->num_sinks + cfg->recent_window > 0;
  if (need_side && (!side_cache || !aligned(side_cache, 16))) return KV4_ERR_INVALID_ARG;
  kv4_cache* c = new (std::nothrow) kv4_cache();
  if (!c) return KV4_ERR_INVALID_ARG;
  c->cfg = *cfg;
  c->format = cfg->value_format == KV4_KEYS_MIXED ? FMT_MIXED : FMT_INT4;
  c->pool = static_cast<uint8_t*>(page_pool);
  c->side = need_side ? static_cast<uint8_t*>(side_cache) : nullptr;
  sizes(cfg, &c->page_bytes, &c->side_slot_bytes, &c->nt8);
  c->pool_layer_bytes = c->page_bytes * static_cast<size_t>(cfg->max_pages);
  c->side_layer_bytes = c->side_slot_bytes * static_cast<size_t>(cfg->max_seqs);
  if (c->format == FMT_MIXED) {
    c->alloc_base = c->pool + c->pool_layer_bytes * static_cast<size_t>(cfg->num_layers);
    c->alloc_layer_bytes = mixed_alloc_layer_bytes(cfg);
    try {
      c->allocated.assign(static_cast<size_t>(cfg->num_layers), 0);
    } catch (...) {
      delete c;
      return KV4_ERR_INVALID_ARG;
    }
  }
  *out = c;
  return KV4_OK;
}

void kv4_cache_destroy(kv4_cache* cache) { delete cache; }

kv4_status kv4_append(kv4_cache* cache, int layer, int T, const void* K, kv4_dtype k_dtype, const void* V,
                      kv4_dtype v_dtype, const int32_t* seq_slot, const int32_t* pos, const int32_t* lens_after,
                      const int32_t* page_table, int stride, void* stream) {
  return append_common(cache, own_format(cache), layer, T, K, k_dtype, V, v_dtype, seq_slot, pos, lens_after, page_table,
                       stride, stream);
}

kv4_status kv4_decode_workspace_bytes(const kv4_cache* cache, int B, size_t* bytes) {
  if (!cache || own_format(cache) != cache->format || B < 0 || !bytes) return KV4_ERR_INVALID_ARG;
  int sms = 0;
  if (!device_info(nullptr, &sms)) return KV4_ERR_CUDA;
  *bytes = workspace_for(cache, B, decode_ctas_full(cache, sms));
  return KV4_OK;
}

kv4_status kv4_decode_attn(kv4_cache* cache, int layer, int B, const void* q, kv4_dtype q_dtype,
                           const int32_t* page_table, int stride, const int32_t* lens, int max_len_hint, float* out,
                           float* lse, void* workspace, size_t ws_bytes, void* stream) {
  return decode_common(cache, own_format(cache), layer, B, q, q_dtype, page_table, stride, lens, max_len_hint, out,
                       lse, workspace, ws_bytes, stream);
}

// No-allocation decode: the split-K partials go to this file-scope device array instead of a
// caller workspace.  In host code the name is only a stand-in, so its device address is looked
// up per device (cudaGetSymbolAddress, with that device current) and passed to the kernels.
static __device__ __align__(256) unsigned char g_kv4_static_scratch[KV4_STATIC_SCRATCH_BYTES];
static void* g_static_scratch_ptr[kMaxDevices] = {};

// First use on a device: look up the array's address (with that device current).
static bool static_scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_static_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_kv4_static_scratch) != cudaSuccess || !p) return false;
    g_static_scratch_ptr[dev] = p;
  }
  *out = g_static_scratch_ptr[dev];
  return true;
}

kv4_status kv4_set_rotation_signs(kv4_cache* cache, const uint32_t* sign_bits) {
  if (!cache || cache->format != FMT_INT4) return KV4_ERR_INVALID_ARG;
  const int words = (cache->cfg.head_dim + 31) / 32;
  for (int i = 0; i < 4; ++i) cache->signs[i] = (sign_bits && i < words) ? sign_bits[i] : 0u;
  return KV4_OK;
}

kv4_status kv4_set_value_rotation(kv4_cache* cache, int enable) {
  if (!cache || cache->format != FMT_INT4) return KV4_ERR_INVALID_ARG;
  if (enable && cache->cfg.value_format == KV4_VALUES_BF16) return KV4_ERR_INVALID_ARG;
  cache->rotate_v = enable ? 1 : 0;
  return KV4_OK;
}

kv4_status kv4_set_decode_overlap(kv4_cache* cache, int enable) {
  if (!cache || cache->format != FMT_INT4) return KV4_ERR_INVALID_ARG;
  cache->overlap = enable ? 1 : 0;
  return KV4_OK;
}

kv4_status kv4_debug_force_wait_timeout(kv4_cache* cache, int enable) {
  if (!cache || (cache->format != FMT_INT4 && cache->format != FMT_MIXED)) return KV4_ERR_INVALID_ARG;
  cache->stall_test = enable ? 1 : 0;
  return KV4_OK;
}

kv4_status kv4_debug_mixed_row_copies(kv4_cache* cache, int enable) {
  if (!cache || cache->format != FMT_MIXED) return KV4_ERR_INVALID_ARG;
  cache->mixed_rows = enable ? 1 : 0;
  return KV4_OK;
}

kv4_status kv4_allocate_key_bits(kv4_cache* cache, int layer, int T, const void* K, kv4_dtype k_dtype, void* stream) {
  if (!cache || cache->format != FMT_MIXED || layer < 0 || layer >= cache->cfg.num_layers || T < 0)
    return KV4_ERR_INVALID_ARG;
  if (T > 0 && (!K || dtype_ok_q(k_dtype) != KV4_OK || !aligned(K, k_dtype == KV4_F32 ? 4 : 2))) return KV4_ERR_INVALID_ARG;
  if (!device_info(nullptr, nullptr)) return KV4_ERR_CUDA;
  kv4::ScoreArgs a{};
  a.K = K;
  a.k_dtype = k_dtype;
  a.T = T;
  a.Hkv = cache->cfg.num_kv_heads;
  a.kbits = cache->cfg.key_bits;
  a.alloc = cache->alloc_base + static_cast<size_t>(layer) * cache->alloc_layer_bytes;
  if (kv4::launch_mixed_score(a, cache->cfg.head_dim, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return KV4_ERR_CUDA;
  cache->allocated[layer] = 1;
  return KV4_OK;
}

kv4_status kv4_set_key_allocation(kv4_cache* cache, int layer, const uint8_t* widths, const float* sigma, void* stream) {
  if (!cache || cache->format != FMT_MIXED || layer < 0 || layer >= cache->cfg.num_layers || !widths || !sigma)
    return KV4_ERR_INVALID_ARG;
  const int Hkv = cache->cfg.num_kv_heads, NB = cache->cfg.head_dim / 2;
  const size_t rec = kv4::mixed_alloc_record_bytes(cache->cfg.head_dim);
  std::vector<uint8_t> host;
  try {
    host.assign(cache->alloc_layer_bytes, 0);
  } catch (...) {
    return KV4_ERR_INVALID_ARG;
  }
  for (int g = 0; g < Hkv; ++g) {
    int sum = 0;
    for (int b = 0; b < NB; ++b) {
      const uint8_t w = widths[static_cast<size_t>(g) * NB + b];
      const float sg = sigma[static_cast<size_t>(g) * NB + b];
      if (w > 8 || !(sg > 0.f) || !std::isfinite(sg)) return KV4_ERR_INVALID_ARG;
      sum += w;
      std::memcpy(host.data() + g * rec + 4 * static_cast<size_t>(b), &sg, 4);
      host[g * rec + 4 * static_cast<size_t>(NB) + b] = w;
    }
    if (sum != cache->cfg.key_bits * NB) return KV4_ERR_INVALID_ARG;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(cache->alloc_base + static_cast<size_t>(layer) * cache->alloc_layer_bytes, host.data(), host.size(),
                      cudaMemcpyHostToDevice, st) != cudaSuccess)
    return KV4_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return KV4_ERR_CUDA;  // host buffer freed on return
  cache->allocated[layer] = 1;
  return KV4_OK;
}

kv4_status kv4_get_key_allocation(kv4_cache* cache, int layer, uint8_t* widths, float* sigma, void* stream) {
  if (!cache || cache->format != FMT_MIXED || layer < 0 || layer >= cache->cfg.num_layers || !widths || !sigma)
    return KV4_ERR_INVALID_ARG;
  if (!cache->allocated[layer]) return KV4_ERR_NO_ALLOCATION;
  const int Hkv = cache->cfg.num_kv_heads, NB = cache->cfg.head_dim / 2;
  const size_t rec = kv4::mixed_alloc_record_bytes(cache->cfg.head_dim);
  std::vector<uint8_t> host;
  try {
    host.assign(cache->alloc_layer_bytes, 0);
  } catch (...) {
    return KV4_ERR_INVALID_ARG;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(host.data(), cache->alloc_base + static_cast<size_t>(layer) * cache->alloc_layer_bytes, host.size(),
                      cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return KV4_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return KV4_ERR_CUDA;
  for (int g = 0; g < Hkv; ++g)
    for (int b = 0; b < NB; ++b) {
      std::memcpy(&sigma[static_cast<size_t>(g) * NB + b], host.data() + g * rec + 4 * static_cast<size_t>(b), 4);
      widths[static_cast<size_t>(g) * NB + b] = host[g * rec + 4 * static_cast<size_t>(NB) + b];
    }
  return KV4_OK;
}

kv4_status kv4_decode_attn_static(kv4_cache* cache, int layer, int B, const void* q, kv4_dtype q_dtype,
                                  const int32_t* page_table, int stride, const int32_t* lens, int max_len_hint,
                                  float* out, float* lse, void* stream) {
  if (!cache || own_format(cache) != cache->format || B < 0 || B > cache->cfg.max_seqs) return KV4_ERR_INVALID_ARG;
  if (B == 0) return KV4_OK;
  int sms = 0;
  if (!device_info(nullptr, &sms)) return KV4_ERR_CUDA;
  if (workspace_for(cache, B, decode_ctas_full(cache, sms)) > KV4_STATIC_SCRATCH_BYTES) return KV4_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (!static_scratch_address(&scratch)) return KV4_ERR_CUDA;
  return decode_common(cache, cache->format, layer, B, q, q_dtype, page_table, stride, lens, max_len_hint, out, lse,
                       scratch, KV4_STATIC_SCRATCH_BYTES, stream);
}

kv4_status kv4_bf16_query_sizes(const kv4_config* cfg, size_t* page_pool_bytes) {
  const kv4_status st = check_config(cfg);
  if (st != KV4_OK) return st;
  if (page_pool_bytes)
    *page_pool_bytes = static_cast<size_t>(cfg->num_layers) * cfg->max_pages * cfg->num_kv_heads * cfg->page_size * 4 *
                       static_cast<size_t>(cfg->head_dim);
  return KV4_OK;
}

kv4_status kv4_bf16_cache_init(const kv4_config* cfg, void* page_pool, kv4_cache** out) {
  const kv4_status st = check_config(cfg);
  if (st != KV4_OK) return st;
  if (!out || !page_pool || !aligned(page_pool, 16)) return KV4_ERR_INVALID_ARG;
  kv4_cache* c = new (std::nothrow) kv4_cache();
  if (!c) return KV4_ERR_INVALID_ARG;
  c->cfg = *cfg;
  c->cfg.value_format = KV4_VALUES_INT4;  // the baseline pool stores K and V in bf16 whatever the field says
  c->format = FMT_BF16;
  c->pool = static_cast<uint8_t*>(page_pool);
  c->side = nullptr;
  c->page_bytes = static_cast<size_t>(cfg->num_kv_heads) * cfg->page_size * 4 * static_cast<size_t>(cfg->head_dim);
  c->pool_layer_bytes = c->page_bytes * static_cast<size_t>(cfg->max_pages);
  c->side_slot_bytes = 0;
  c->side_layer_bytes = 0;
  c->nt8 = 0;
  *out = c;
  return KV4_OK;
}

kv4_status kv4_bf16_append(kv4_cache* cache, int layer, int T, const void* K, kv4_dtype k_dtype, const void* V,
                           kv4_dtype v_dtype, const int32_t* seq_slot, const int32_t* pos, const int32_t* page_table,
                           int stride, void* stream) {
  return append_common(cache, FMT_BF16, layer, T, K, k_dtype, V, v_dtype, seq_slot, pos, nullptr, page_table, stride,
                       stream);
}

kv4_status kv4_bf16_decode_workspace_bytes(const kv4_cache* cache, int B, size_t* bytes) {
  if (!cache || cache->format != FMT_BF16 || B < 0 || !bytes) return KV4_ERR_INVALID_ARG;
  int sms = 0;
  if (!device_info(nullptr, &sms)) return KV4_ERR_CUDA;
  *bytes = workspace_for(cache, B, decode_ctas_full(cache, sms));
  return KV4_OK;
}

kv4_status kv4_bf16_decode_attn(kv4_cache* cache, int layer, int B, const void* q, kv4_dtype q_dtype,
                                const int32_t* page_table, int stride, const int32_t* lens, int max_len_hint,
                                float* out, float* lse, void* workspace, size_t ws_bytes, void* stream) {
  return decode_common(cache, FMT_BF16, layer, B, q, q_dtype, page_table, stride, lens, max_len_hint, out, lse,
                       workspace, ws_bytes, stream);
}

kv4_status kv4_get_device_error(uint32_t* bits) {
  if (!bits) return KV4_ERR_INVALID_ARG;
  if (!device_info(nullptr, nullptr)) return KV4_ERR_CUDA;
  if (cudaDeviceSynchronize() != cudaSuccess) return KV4_ERR_CUDA;
  uint32_t v = 0;
  if (cudaMemcpyFromSymbol(&v, g_kv4_device_error, sizeof(v)) != cudaSuccess) return KV4_ERR_CUDA;
  const uint32_t zero = 0;
  if (cudaMemcpyToSymbol(g_kv4_device_error, &zero, sizeof(zero)) != cudaSuccess) return KV4_ERR_CUDA;
  *bits = v;
  return KV4_OK;
}

uint64_t kv4_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char* kv4_status_string(kv4_status s) {
  switch (s) {
    case KV4_OK: return "ok";
    case KV4_ERR_INVALID_ARG: return "invalid argument";
    case KV4_ERR_UNSUPPORTED: return "unsupported geometry";
    case KV4_ERR_WORKSPACE: return "workspace missing or too small";
    case KV4_ERR_CUDA: return "CUDA error";
    case KV4_ERR_DEVICE: return "device-side guard fired";
    case KV4_ERR_NO_ALLOCATION: return "layer has no key bit allocation";
  }
  return "unknown status";
}

int kv4_version(void) { return 100; }

}  // extern "C"
