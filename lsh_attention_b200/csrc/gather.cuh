// Row gather into sorted order, output-stationary: slot s of segment seg
// takes the x and v rows of position perm[seg][s], and 1/||x|| of that row
// ("Reformer summary" (ttnews.xyz), §局部敏感哈希注意力: the attention runs on
// the tokens in bucket order).
//
// The ranks (perm) come first, from the counting sort; this kernel then
// writes xs and vs strictly in slot order, so every store stream is
// sequential, and reads whole rows at scattered positions. CTAs are ordered
// (batch, head) first and round fastest, so the rounds of one (batch, head),
// which read the same rows, run together and share them through L2.
// A group of L = D * sizeof(T) / 16 lanes moves one row (16 bytes per lane);
// a warp keeps kGatherUnroll groups of rows in flight.
#pragma once

#include "common.cuh"

namespace lsh {

constexpr int kGatherWarps = 8;
constexpr int kGatherSlots = 256;  // slots per CTA
constexpr int kGatherUnroll = 4;

// grid BH * ceil(n / kGatherSlots) * rounds, block 256.
// perm, invnorm [seg][n]; x, v [BH][n][D] (position order); xs, vs [seg][n][D].
template <typename T, int D>
__global__ void __launch_bounds__(kGatherWarps * 32)
    k_gather_rows(const int32_t* __restrict__ perm, const T* __restrict__ x,
                  const T* __restrict__ v, T* __restrict__ xs, T* __restrict__ vs,
                  float* __restrict__ invnorm, int n, int rounds) {
  constexpr int L = D * (int)sizeof(T) / 16;  // lanes per row: 8, 16 or 32
  constexpr int RPI = 32 / L;                 // rows per warp instruction
  constexpr int EPV = 16 / (int)sizeof(T);    // elements per lane
  constexpr int STEP = RPI * kGatherUnroll;   // rows per warp iteration
  static_assert(L == 8 || L == 16 || L == 32, "a row is 128, 256 or 512 bytes");
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int blocks_per_seq = (n + kGatherSlots - 1) / kGatherSlots;
  const int r = blockIdx.x % rounds;
  const int rest = blockIdx.x / rounds;
  const int blk = rest % blocks_per_seq;
  const int64_t bh = rest / blocks_per_seq;
  const int64_t seg = bh * rounds + r;
  const int s_end = min(n, (blk + 1) * kGatherSlots);
  const int gl = lane % L;
  const T* xb = x + bh * (int64_t)n * D + gl * EPV;
  const T* vb = v + bh * (int64_t)n * D + gl * EPV;
  T* xo = xs + seg * (int64_t)n * D + gl * EPV;
  T* vo = vs + seg * (int64_t)n * D + gl * EPV;
  const int32_t* pm = perm + seg * (int64_t)n;

  for (int s0 = blk * kGatherSlots + warp * STEP; s0 < s_end; s0 += kGatherWarps * STEP) {
    int slot[kGatherUnroll];
    uint4 xa[kGatherUnroll], va[kGatherUnroll];
#pragma unroll
    for (int u = 0; u < kGatherUnroll; ++u) {
      slot[u] = s0 + u * RPI + lane / L;
      if (slot[u] < s_end) {
        const int64_t p = pm[slot[u]];
        xa[u] = *reinterpret_cast<const uint4*>(xb + p * D);
        va[u] = *reinterpret_cast<const uint4*>(vb + p * D);
      }
    }
#pragma unroll
    for (int u = 0; u < kGatherUnroll; ++u) {
      const bool ok = slot[u] < s_end;
      float ss = 0.f;
      if (ok) {
        *reinterpret_cast<uint4*>(xo + (int64_t)slot[u] * D) = xa[u];
        *reinterpret_cast<uint4*>(vo + (int64_t)slot[u] * D) = va[u];
        float f[EPV];
        Vec16<T>::unpack(xa[u], f);
#pragma unroll
        for (int e = 0; e < EPV; ++e) ss = fmaf(f[e], f[e], ss);
      }
      // the row's lanes are aligned groups of L: the xor stays inside
#pragma unroll
      for (int o = L / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (ok && gl == 0) invnorm[seg * n + slot[u]] = ss > 0.f ? 1.0f / sqrtf(ss) : 0.f;
    }
  }
}

}  // namespace lsh
