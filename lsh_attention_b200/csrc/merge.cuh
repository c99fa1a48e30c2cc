// Un-sort and round merge.
//
// "Reformer summary" (ttnews.xyz), §多輪LSH哈希 leaves the combination of
// rounds to the paper; the reading taken: with lse_r the log-normaliser of
// round r at a position, LSE = logsumexp_r lse_r and
//   out = sum_r exp(lse_r - LSE) * o_r,
// i.e. one softmax over the union of the rounds' candidate lists.
// One warp per (batch, head, position): the lanes fetch each round's slot and
// lse, then stream the rounds' fp32 rows and write the output row once.
#pragma once

#include "common.cuh"

namespace lsh {

constexpr int kMergeWarps = 8;

// grid ceil(BH * n / 8), block 256.
// inv, lse_s [BH][rounds][n]; out_s [BH][rounds][n][D] fp32 in slot order;
// out [BH][n][D] in T; lse [BH][rounds][n] fp32 in position order.
template <typename T, int D>
__global__ void __launch_bounds__(kMergeWarps * 32)
    k_merge(const int32_t* __restrict__ inv, const float* __restrict__ lse_s,
            const float* __restrict__ out_s, T* __restrict__ out, float* __restrict__ lse, int n,
            int rounds, int64_t total) {
  const int lane = threadIdx.x & 31;
  const int64_t item = (int64_t)blockIdx.x * kMergeWarps + (threadIdx.x >> 5);
  if (item >= total) return;
  const int64_t bh = item / n;
  const int pos = (int)(item % n);

  // lane r < rounds: slot and lse of round r
  int slot = 0;
  float l = -INFINITY;
  if (lane < rounds) {
    const int64_t seg = bh * rounds + lane;
    slot = inv[seg * n + pos];
    l = lse_s[seg * n + slot];
    lse[seg * n + pos] = l;
  }
  // w_r = exp(lse_r - mx) / sum_r' exp(lse_r' - mx). Forming logsumexp
  // first would round it to the fp32 grid near |lse| = 1e5 (self-only rows),
  // where the spacing is 1/128.
  const float mx = warp_max(l);
  const float e = lane < rounds ? expf(l - mx) : 0.f;
  const float w = e / warp_sum(e);

  constexpr int DL = D / 32;  // dims per lane: 2 or 4
  float acc[DL];
#pragma unroll
  for (int k = 0; k < DL; ++k) acc[k] = 0.f;
  for (int r = 0; r < rounds; ++r) {
    const float wr = __shfl_sync(0xffffffffu, w, r);
    const int sr = __shfl_sync(0xffffffffu, slot, r);
    const float* row = out_s + ((bh * rounds + r) * n + sr) * (int64_t)D + lane * DL;
    if constexpr (DL == 4) {
      const float4 a = *reinterpret_cast<const float4*>(row);
      acc[0] = fmaf(wr, a.x, acc[0]);
      acc[1] = fmaf(wr, a.y, acc[1]);
      acc[2] = fmaf(wr, a.z, acc[2]);
      acc[3] = fmaf(wr, a.w, acc[3]);
    } else {
      const float2 a = *reinterpret_cast<const float2*>(row);
      acc[0] = fmaf(wr, a.x, acc[0]);
      acc[1] = fmaf(wr, a.y, acc[1]);
    }
  }
  T* o = out + item * D + lane * DL;
#pragma unroll
  for (int k = 0; k < DL; ++k) o[k] = Elem<T>::from_f(acc[k]);
}

}  // namespace lsh
