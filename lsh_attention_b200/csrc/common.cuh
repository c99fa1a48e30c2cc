// Shared device helpers for the LSH-attention kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace lsh {

constexpr float kSelfLogit = -1.0e5f;  // logit of a token against itself
// ||x||^2 is summed in this many interleaved partial sums over a row's 16-byte
// pieces, by the tensor-core hash and by the attention's norm pass alike
constexpr int kNormParts = 2;

// Workspace header: status word and counters, 256 bytes at the start of the
// caller's workspace. Field order matches lsh_attn_diag.
struct WsHeader {
  uint32_t status;
  uint32_t hash_refined;
  uint32_t bad_bucket_ids;
  uint32_t reserved;
  uint32_t pad[60];
};
static_assert(sizeof(WsHeader) == 256, "header is 256 bytes");

// Keep the first error a kernel reports.
__device__ __forceinline__ void record_status(WsHeader* h, uint32_t code) {
  atomicCAS(&h->status, 0u, code);
}

template <typename T>
struct Elem;
template <>
struct Elem<float> {
  static __device__ __forceinline__ float to_f(float v) { return v; }
  static __device__ __forceinline__ double to_d(float v) { return (double)v; }
  static __device__ __forceinline__ float from_f(float v) { return v; }
};
template <>
struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
  static __device__ __forceinline__ double to_d(__nv_bfloat16 v) {
    return (double)__bfloat162float(v);
  }
  static __device__ __forceinline__ __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
};

// Unpack a 16-byte vector of elements into fp32.
template <typename T>
struct Vec16;
template <>
struct Vec16<float> {
  static constexpr int N = 4;
  static __device__ __forceinline__ void unpack(const uint4& u, float* f) {
    f[0] = __uint_as_float(u.x);
    f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z);
    f[3] = __uint_as_float(u.w);
  }
};
template <>
struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  static __device__ __forceinline__ void unpack(const uint4& u, float* f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
  }
};

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace lsh
