// Un-sort and round merge. The attention writes each round's lse at the
// query's position and its output row at the query's slot; inv maps a
// position to its slot.
//
// "Reformer summary" (ttnews.xyz), §多輪LSH哈希 leaves the combination of
// rounds to the paper; the reading taken: with lse_r the log-normaliser of
// round r at a position, LSE = logsumexp_r lse_r and
//   out = sum_r exp(lse_r - LSE) * o_r,
// i.e. one softmax over the union of the rounds' candidate lists.
// A group of G = D * sizeof(T) / 16 lanes merges one (batch, head,
// position): lane j of the group owns the 16-byte piece j of every row. The
// group's lanes read the rounds' lse (by position) and slots (inv) (lane j
// takes rounds j, j + G, ...), the weights come from shuffles inside the
// group, every round's row piece is loaded (four in flight before the sums)
// and the output piece is written once.
#pragma once

#include "common.cuh"

namespace lsh {

constexpr int kMergeWarps = 8;

template <int G>
__device__ __forceinline__ float group_max(float v) {
#pragma unroll
  for (int o = G / 2; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
template <int G>
__device__ __forceinline__ float group_sum(float v) {
#pragma unroll
  for (int o = G / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// 16 bytes of T as fp32.
template <typename T>
__device__ __forceinline__ void unpack16(const uint4& a, float (&f)[16 / sizeof(T)]) {
  if constexpr (sizeof(T) == 4) {
    f[0] = __uint_as_float(a.x); f[1] = __uint_as_float(a.y);
    f[2] = __uint_as_float(a.z); f[3] = __uint_as_float(a.w);
  } else {  // bf16: the high half of each 32-bit word is the later element
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      f[2 * k] = __uint_as_float(w[k] << 16);
      f[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
    }
  }
}

// CTAs per SM the merge is launched with (grid-stride loop over positions).
constexpr int kMergeCtasPerSm = 4;

template <int G, int RPL>
__device__ __forceinline__ void merge_meta(const int32_t* __restrict__ inv,
                                           const float* __restrict__ lse, bool valid, int64_t bh,
                                           int pos, int n, int rounds, int gl, float (&l)[RPL],
                                           int (&slot)[RPL]) {
#pragma unroll
  for (int k = 0; k < RPL; ++k) {
    const int r = gl + k * G;
    l[k] = -INFINITY;
    slot[k] = 0;
    if (valid && r < rounds) {
      l[k] = lse[(bh * rounds + r) * (int64_t)n + pos];
      slot[k] = inv[(bh * rounds + r) * (int64_t)n + pos];
    }
  }
}

// grid min(ceil(BH * n / (8 * 32 / G)), kMergeCtasPerSm * SMs), block 256.
// inv, lse [BH][rounds][n] in position order; out_r [BH][rounds][n][D] in
// slot order and out [BH][n][D], both in T. Each lane group walks positions
// with the grid's stride; the next position's lse and slots are loaded
// while the current position's rows are in flight.
template <typename T, int D>
__global__ void __launch_bounds__(kMergeWarps * 32, kMergeCtasPerSm)
    k_merge(const int32_t* __restrict__ inv, const float* __restrict__ lse,
            const T* __restrict__ out_r, T* __restrict__ out, int n, int rounds,
            int64_t total) {
  constexpr int G = D * (int)sizeof(T) / 16;  // lanes per position: 8, 16 or 32
  constexpr int EPV = 16 / (int)sizeof(T);    // elements per lane
  constexpr int RPL = (16 + G - 1) / G;       // rounds per lane (rounds <= 16)
  static_assert(G == 8 || G == 16 || G == 32, "a row is 128, 256 or 512 bytes");
  static_assert(RPL <= 2, "the shuffles below pick one of at most two rounds per lane");
  const int lane = threadIdx.x & 31, gl = lane % G, g0 = lane - gl;
  const int64_t stride = (int64_t)gridDim.x * kMergeWarps * (32 / G);
  const int64_t first =
      ((int64_t)blockIdx.x * kMergeWarps + (threadIdx.x >> 5)) * (32 / G) + lane / G;
  // the same count for every lane of the CTA: all of a warp's lanes run the
  // group shuffles of every iteration
  const int64_t iters = (total + stride - 1) / stride;

  // (batch-head, position) of the current and the next item, stepped by the
  // stride's quotient and remainder (no 64-bit division in the loop)
  const int64_t sq = stride / n;
  const int sr_ = (int)(stride % n);
  int64_t bh = first / n;
  int pos = (int)(first % n);
  int64_t bhn = bh + sq;
  int posn = pos + sr_;
  if (posn >= n) {
    posn -= n;
    ++bhn;
  }
  float ln[RPL];
  int sn[RPL];
  merge_meta<G, RPL>(inv, lse, first < total, bh, pos, n, rounds, gl, ln, sn);
  for (int64_t it = 0; it < iters; ++it) {
    const int64_t item = first + it * stride;
    const bool valid = item < total;
    float l[RPL];
    int slot[RPL];
#pragma unroll
    for (int k = 0; k < RPL; ++k) {
      l[k] = ln[k];
      slot[k] = sn[k];
    }
    merge_meta<G, RPL>(inv, lse, item + stride < total, bhn, posn, n, rounds, gl, ln, sn);

    // w_r = exp(lse_r - mx) / sum_r' exp(lse_r' - mx). Forming logsumexp
    // first would round it to the fp32 grid near |lse| = 1e5 (self-only
    // rows), where the spacing is 1/128.
    float mx = -INFINITY;
#pragma unroll
    for (int k = 0; k < RPL; ++k) mx = fmaxf(mx, l[k]);
    mx = group_max<G>(mx);
    float e[RPL], es = 0.f;
#pragma unroll
    for (int k = 0; k < RPL; ++k) {
      e[k] = gl + k * G < rounds ? expf(l[k] - mx) : 0.f;
      es += e[k];
    }
    const float rs = 1.0f / group_sum<G>(es);

    const T* segs = out_r + bh * rounds * (int64_t)n * D + gl * EPV;  // round 0 of this (b, h)
    float acc[EPV];
#pragma unroll
    for (int k = 0; k < EPV; ++k) acc[k] = 0.f;
    for (int r0 = 0; r0 < rounds; r0 += 4) {
      uint4 v[4];
      float wr[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = r0 + i;  // uniform over the warp
        const int k = r / G, src = g0 + r % G;
        const int sr = __shfl_sync(0xffffffffu, k == 0 ? slot[0] : slot[RPL - 1], src);
        wr[i] = __shfl_sync(0xffffffffu, k == 0 ? e[0] : e[RPL - 1], src) * rs;
        if (valid && r < rounds)
          v[i] = *reinterpret_cast<const uint4*>(segs + ((int64_t)r * n + sr) * D);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (valid && r0 + i < rounds) {
          float f[EPV];
          unpack16<T>(v[i], f);
#pragma unroll
          for (int k = 0; k < EPV; ++k) acc[k] = fmaf(wr[i], f[k], acc[k]);
        }
      }
    }
    if (valid) {
      T* o = out + item * D + gl * EPV;
      if constexpr (sizeof(T) == 4) {
        *reinterpret_cast<float4*>(o) = make_float4(acc[0], acc[1], acc[2], acc[3]);
      } else {
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const __nv_bfloat162 h = __floats2bfloat162_rn(acc[2 * k], acc[2 * k + 1]);
          w[k] = *reinterpret_cast<const uint32_t*>(&h);
        }
        *reinterpret_cast<uint4*>(o) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    bh = bhn;
    pos = posn;
    bhn += sq;
    posn += sr_;
    if (posn >= n) {
      posn -= n;
      ++bhn;
    }
  }
}

}  // namespace lsh
