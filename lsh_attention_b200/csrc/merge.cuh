// Un-sort and round merge. The attention writes each round's lse at the
// query's position and its output row at the query's slot; inv maps a
// position to its slot.
//
// "Reformer summary" (ttnews.xyz), §多輪LSH哈希 leaves the combination of
// rounds to the paper; the reading taken: with lse_r the log-normaliser of
// round r at a position, LSE = logsumexp_r lse_r and
//   out = sum_r exp(lse_r - LSE) * o_r,
// i.e. one softmax over the union of the rounds' candidate lists.
// One warp per (batch, head, position): lane r reads lse_r and slot_r (two
// independent loads), the weights come from a warp max and sum, then every
// round's fp32 row is loaded (four loads in flight before the sums) and the
// output row is written once.
#pragma once

#include "common.cuh"

namespace lsh {

constexpr int kMergeWarps = 8;

// grid ceil(BH * n / 8), block 256.
// inv, lse [BH][rounds][n] in position order; out_r [BH][rounds][n][D] in
// slot order; out [BH][n][D] in T.
template <typename T, int D>
__global__ void __launch_bounds__(kMergeWarps * 32)
    k_merge(const int32_t* __restrict__ inv, const float* __restrict__ lse,
            const float* __restrict__ out_r, T* __restrict__ out, int n, int rounds,
            int64_t total) {
  const int lane = threadIdx.x & 31;
  const int64_t item = (int64_t)blockIdx.x * kMergeWarps + (threadIdx.x >> 5);
  if (item >= total) return;
  const int64_t bh = item / n;
  const int pos = (int)(item % n);
  const float* segs = out_r + bh * rounds * (int64_t)n * D;  // round 0 of this (b, h)

  // w_r = exp(lse_r - mx) / sum_r' exp(lse_r' - mx). Forming logsumexp
  // first would round it to the fp32 grid near |lse| = 1e5 (self-only rows),
  // where the spacing is 1/128.
  float l = -INFINITY;
  int slot = 0;
  if (lane < rounds) {
    l = lse[(bh * rounds + lane) * (int64_t)n + pos];
    slot = inv[(bh * rounds + lane) * (int64_t)n + pos];
  }
  const float mx = warp_max(l);
  const float e = lane < rounds ? expf(l - mx) : 0.f;
  const float w = e / warp_sum(e);

  constexpr int DL = D / 32;  // dims per lane: 2 or 4
  float acc[DL];
#pragma unroll
  for (int k = 0; k < DL; ++k) acc[k] = 0.f;
  for (int r0 = 0; r0 < rounds; r0 += 4) {
    float v[4][DL];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int sr = __shfl_sync(0xffffffffu, slot, (r0 + i) & 31);
      const float* row = segs + ((int64_t)(r0 + i) * n + sr) * D + lane * DL;
      if (r0 + i < rounds) {
        if constexpr (DL == 4) {
          const float4 a = *reinterpret_cast<const float4*>(row);
          v[i][0] = a.x; v[i][1] = a.y; v[i][2] = a.z; v[i][3] = a.w;
        } else {
          const float2 a = *reinterpret_cast<const float2*>(row);
          v[i][0] = a.x; v[i][1] = a.y;
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float wr = __shfl_sync(0xffffffffu, w, (r0 + i) & 31);
      if (r0 + i < rounds) {
#pragma unroll
        for (int k = 0; k < DL; ++k) acc[k] = fmaf(wr, v[i][k], acc[k]);
      }
    }
  }
  T* o = out + item * D + lane * DL;
#pragma unroll
  for (int k = 0; k < DL; ++k) o[k] = Elem<T>::from_f(acc[k]);
}

}  // namespace lsh
