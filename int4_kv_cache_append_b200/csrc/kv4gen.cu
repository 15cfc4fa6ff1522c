// kv4gen.cu -- GPU twin of the seeded input generator in workload.py (libkv4gen.so).
//
// Inputs only: no rotation, quantisation or attention.  SplitMix64 (Steele, Lea and Flood,
// OOPSLA 2014; Vigna's reference form) gives output k of the stream with state `key` as
// mix64(key + (k + 1) * 0x9E3779B97F4A7C15); a normal deviate for element i is the centred sum
// of the twelve 16-bit fields of outputs 3i, 3i+1, 3i+2, divided by 65536 (exact in fp32).
// Integer arithmetic throughout, so the values equal the NumPy generator's bit for bit.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ float normal_at(uint64_t key, uint64_t i) {
  int64_t s = 0;
#pragma unroll
  for (int j = 0; j < 3; ++j) {
    const uint64_t u = mix64(key + (3 * i + j + 1) * 0x9E3779B97F4A7C15ull);
    s += (int64_t)(u & 0xffff) + (int64_t)((u >> 16) & 0xffff) + (int64_t)((u >> 32) & 0xffff) + (int64_t)(u >> 48);
  }
  return (float)(s - 393210) * (1.0f / 65536.0f);
}

__device__ __forceinline__ uint16_t to_bf16_bits(float x) {
  const uint32_t u = __float_as_uint(x);
  return (uint16_t)((u + 0x7fffu + ((u >> 16) & 1u)) >> 16);
}

// out[t][g][d] for token (b[t], pos[t]): element index ((b * 2^20 + pos) * Hkv + g) * D + d.
__global__ void tokens_kernel(void* out, int bf16, uint64_t key, const int32_t* b, const int32_t* pos, int T, int Hkv,
                              int D, const float* factor) {
  const long long n = (long long)T * Hkv * D;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < n; idx += (long long)gridDim.x * blockDim.x) {
    const int d = (int)(idx % D);
    const long long r = idx / D;
    const int g = (int)(r % Hkv);
    const int t = (int)(r / Hkv);
    const uint64_t e = (((uint64_t)b[t] * (1ull << 20) + (uint64_t)pos[t]) * (uint64_t)Hkv + (uint64_t)g) * (uint64_t)D + (uint64_t)d;
    const float v = normal_at(key, e) * factor[g * D + d];
    if (bf16)
      reinterpret_cast<uint16_t*>(out)[idx] = to_bf16_bits(v);
    else
      reinterpret_cast<float*>(out)[idx] = v;
  }
}

__global__ void normal_kernel(void* out, long long n, uint64_t key, long long start, int bf16) {
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < n; idx += (long long)gridDim.x * blockDim.x) {
    const float v = normal_at(key, (uint64_t)(start + idx));
    if (bf16)
      reinterpret_cast<uint16_t*>(out)[idx] = to_bf16_bits(v);
    else
      reinterpret_cast<float*>(out)[idx] = v;
  }
}

}  // namespace

extern "C" {

int kv4gen_tokens(void* out, int bf16, uint64_t key, const int32_t* b, const int32_t* pos, int T, int Hkv, int D,
                  const float* factor, void* stream) {
  if (T <= 0) return 0;
  if (!out || !b || !pos || !factor || Hkv <= 0 || D <= 0) return 1;
  tokens_kernel<<<1184, 256, 0, (cudaStream_t)stream>>>(out, bf16, key, b, pos, T, Hkv, D, factor);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

int kv4gen_normal(void* out, long long n, uint64_t key, long long start, int bf16, void* stream) {
  if (n <= 0) return 0;
  if (!out) return 1;
  normal_kernel<<<1184, 256, 0, (cudaStream_t)stream>>>(out, n, key, start, bf16);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

}  // extern "C"
