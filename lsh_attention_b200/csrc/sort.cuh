// Stable counting sort of every (batch, head, round) by bucket, then position,
// fused with the gather of x and v rows into sorted order.
//
// "Reformer summary" (ttnews.xyz), §局部敏感哈希注意力: order the tokens by
// bucket, and inside a bucket by position. Positions are already in order, so
// slot(i) = #{j : b_j < b_i} + #{j < i : b_j = b_i}. Three kernels compute it
// without a global sort:
//   k_sort_hist   per-(segment, tile) bucket histograms, warp-aggregated
//   k_sort_scan   exclusive scan of each segment's [bucket][tile] counts
//   k_sort_rank   per-warp counts inside the tile, stable ranks from
//                 __match_any_sync, perm/inv writes
// (the rows follow in slot order: k_gather_rows). A segment is one (batch,
// head, round); a tile is sort_warps(nb) warps of kSortSub tokens each.
#pragma once

#include "common.cuh"

namespace lsh {

constexpr int kSortSub = 256;  // tokens per warp sub-range

// Warps per tile: per-warp counters take warps * nb * 4 bytes of shared memory
// (at most 32 KB, so two gathering CTAs share an SM).
__host__ __device__ inline int sort_warps(int nb) {
  int w = 8192 / nb;
  return w < 1 ? 1 : (w > 8 ? 8 : w);
}
__host__ __device__ inline int sort_tile(int nb) { return sort_warps(nb) * kSortSub; }

__device__ __forceinline__ int clamp_bucket(int b, int nb) { return b < 0 ? 0 : (b >= nb ? nb - 1 : b); }

// grid (tiles, segments), block 256. hist [seg][nb][tiles].
__global__ void __launch_bounds__(256)
    k_sort_hist(const int32_t* __restrict__ buckets, int n, int nb, int tile, int tiles,
                int32_t* __restrict__ hist, WsHeader* hdr) {
  extern __shared__ int32_t cnt[];
  const int seg = blockIdx.y, tl = blockIdx.x;
  for (int b = threadIdx.x; b < nb; b += blockDim.x) cnt[b] = 0;
  __syncthreads();
  const int start = tl * tile, end = min(n, start + tile);
  const int32_t* bk = buckets + (int64_t)seg * n;
  const int lane = threadIdx.x & 31;
  // every id of the tile is loaded before the first is counted (a tile is at
  // most kSortSub * 8 = 2048 tokens, 8 per thread of the 256)
  constexpr int kPer = 8;
  int raw[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int t = start + i * 256 + threadIdx.x;
    raw[i] = t < end ? bk[t] : 0;
  }
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int t = start + i * 256 + threadIdx.x;
    int b = -1;
    if (t < end) {
      b = clamp_bucket(raw[i], nb);
      if (b != raw[i]) {
        atomicAdd(&hdr->bad_bucket_ids, 1u);
        record_status(hdr, 6u /* LSH_ERR_DEVICE */);
      }
    }
    const uint32_t peers = __match_any_sync(0xffffffffu, b);
    if (b >= 0 && lane == __ffs(peers) - 1) atomicAdd(&cnt[b], __popc(peers));
  }
  __syncthreads();
  int32_t* h = hist + (int64_t)seg * nb * tiles + tl;
  for (int b = threadIdx.x; b < nb; b += blockDim.x) h[(int64_t)b * tiles] = cnt[b];
}

// grid (segments), block 1024: in-place exclusive scan of len ints per segment.
// Each thread scans a contiguous run of kScanPer counts, all loaded before
// any is used (sixteen-byte loads when the segment is 16-byte aligned), so a
// segment of up to 32K counts costs one load round trip and one block scan.
constexpr int kScanPer = 32;
__global__ void __launch_bounds__(1024) k_sort_scan(int32_t* __restrict__ hist, int len) {
  __shared__ int32_t wsum[32];
  int32_t* h = hist + (int64_t)blockIdx.x * len;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const bool vec = (len & 3) == 0;  // then every run of 4 starts 16-byte aligned
  int32_t carry = 0;
  for (int base = 0; base < len; base += kScanPer * 1024) {
    const int i0 = base + kScanPer * threadIdx.x;
    int32_t v[kScanPer];
    if (vec && i0 + kScanPer <= len) {
#pragma unroll
      for (int k = 0; k < kScanPer; k += 4) {
        const int4 q = *reinterpret_cast<const int4*>(h + i0 + k);
        v[k] = q.x; v[k + 1] = q.y; v[k + 2] = q.z; v[k + 3] = q.w;
      }
    } else {
#pragma unroll
      for (int k = 0; k < kScanPer; ++k) v[k] = (i0 + k < len) ? h[i0 + k] : 0;
    }
    int32_t local = 0;
#pragma unroll
    for (int k = 0; k < kScanPer; ++k) local += v[k];
    int32_t incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int32_t s = wsum[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, s, o);
        if (lane >= o) s += y;
      }
      wsum[lane] = s;  // inclusive over warps
    }
    __syncthreads();
    int32_t run = carry + (warp > 0 ? wsum[warp - 1] : 0) + incl - local;
#pragma unroll
    for (int k = 0; k < kScanPer; ++k) {
      const int32_t c = v[k];
      v[k] = run;
      run += c;
    }
    if (vec && i0 + kScanPer <= len) {
#pragma unroll
      for (int k = 0; k < kScanPer; k += 4)
        *reinterpret_cast<int4*>(h + i0 + k) = make_int4(v[k], v[k + 1], v[k + 2], v[k + 3]);
    } else {
#pragma unroll
      for (int k = 0; k < kScanPer; ++k)
        if (i0 + k < len) h[i0 + k] = v[k];
    }
    carry += wsum[31];
    __syncthreads();
  }
}

// Shared memory of k_sort_rank: the tile's offset of every bucket (int32)
// and each warp's running count in the bucket inside the tile (16 bits: a
// tile holds at most 2048 tokens).
__host__ __device__ inline size_t sort_rank_smem(int nb) {
  return sizeof(int32_t) * (size_t)nb + sizeof(uint16_t) * (size_t)sort_warps(nb) * nb;
}

// grid (tiles, segments), block sort_warps(nb) * 32, shared sort_rank_smem(nb).
// hist: scanned offsets [seg][nb][tiles]. perm, inv: [seg][n].
// Eight CTAs of 256 threads fit an SM, so a long-sequence launch is one wave.
__global__ void __launch_bounds__(256, 8)
    k_sort_rank(const int32_t* __restrict__ buckets, const int32_t* __restrict__ hist,
                int32_t* __restrict__ perm, int32_t* __restrict__ inv, int n, int nb, int tiles) {
  extern __shared__ int32_t toff[];  // [nb], then uint16 [warps][nb]
  const int seg = blockIdx.y, tl = blockIdx.x;
  const int nw = blockDim.x >> 5, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint16_t* cnt = reinterpret_cast<uint16_t*>(toff + nb);
  uint32_t* cnt32 = reinterpret_cast<uint32_t*>(cnt);  // nb is even
  for (int i = threadIdx.x; i < nw * nb / 2; i += blockDim.x) cnt32[i] = 0u;
  __syncthreads();

  const int tile = nw * kSortSub;
  const int wstart = tl * tile + warp * kSortSub;
  const int wend = min(n, wstart + kSortSub);
  const int32_t* bk = buckets + (int64_t)seg * n;
  uint16_t* mycnt = cnt + warp * nb;

  // this warp's ids, loaded once for both passes (-1 past the end)
  constexpr int kSteps = kSortSub / 32;
  int bks[kSteps];
#pragma unroll
  for (int i = 0; i < kSteps; ++i) {
    const int t = wstart + 32 * i + lane;
    bks[i] = t < wend ? clamp_bucket(bk[t], nb) : -1;
  }
  // 1) per-warp counts of its sub-range
#pragma unroll
  for (int i = 0; i < kSteps; ++i) {
    const int b = bks[i];
    const uint32_t peers = __match_any_sync(0xffffffffu, b);
    if (b >= 0 && lane == __ffs(peers) - 1) mycnt[b] = (uint16_t)(mycnt[b] + __popc(peers));
    __syncwarp();
  }
  __syncthreads();
  // 2) the tile's offset per bucket, and an exclusive scan over the warps
  const int32_t* h = hist + (int64_t)seg * nb * tiles + tl;
  for (int b = threadIdx.x; b < nb; b += blockDim.x) {
    toff[b] = h[(int64_t)b * tiles];
    uint32_t run = 0;
    for (int w = 0; w < nw; ++w) {
      const uint32_t c = cnt[w * nb + b];
      cnt[w * nb + b] = (uint16_t)run;
      run += c;
    }
  }
  __syncthreads();
  // 3) stable ranks, perm / inv
  const int64_t so = (int64_t)seg * n;
#pragma unroll
  for (int i = 0; i < kSteps; ++i) {
    const int t = wstart + 32 * i + lane;
    const int b = bks[i];
    const uint32_t peers = __match_any_sync(0xffffffffu, b);
    int slot = 0;
    if (b >= 0) slot = toff[b] + mycnt[b] + __popc(peers & lanemask_lt());
    __syncwarp();
    if (b >= 0 && lane == __ffs(peers) - 1) mycnt[b] = (uint16_t)(mycnt[b] + __popc(peers));
    __syncwarp();
    if (b >= 0) {
      perm[so + slot] = t;
      inv[so + t] = slot;
    }
  }
}

}  // namespace lsh
