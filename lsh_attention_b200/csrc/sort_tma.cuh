// Stable counting sort fused with the gather of x and v rows into sorted
// order, the rows streamed by TMA ("Reformer summary" (ttnews.xyz),
// §局部敏感哈希注意力: order the tokens by bucket, then by position). Two CTAs
// share an SM, so one's ranking overlaps the other's copying.
//
// Same ranks as k_sort_scatter (per-warp counts, scan over warps seeded by
// the tile's offsets, stable ranks from __match_any_sync); the slots of the
// whole tile go to shared memory first. The tile's rows are contiguous in x
// and v (position order), so a TMA ring (2 stages of 32 KB, issued before
// the ranks are computed) streams them into shared memory, and the warps
// copy each row to its slot with row-coalesced 16-byte stores, summing the
// squares of x on the way for 1/||x||. Each warp's 256 bucket ids are loaded
// once, up front, for both ranking passes.
#pragma once

#include "common.cuh"
#include "sm100.cuh"
#include "sort.cuh"

namespace lsh {

constexpr int kGatherStages = 2;
constexpr int kGatherStageBytes = 32768;  // x and v rows of one chunk

struct SortGatherPlan {
  int nw, tile;      // warps per CTA, tokens per tile
  int row_bytes;     // d * element size
  int chunk_rows;    // rows per TMA chunk (x and v each)
  size_t smem;
};

inline SortGatherPlan sort_gather_plan(int nb, int d, int esize) {
  SortGatherPlan p;
  p.nw = sort_warps(nb);
  p.tile = p.nw * kSortSub;
  p.row_bytes = d * esize;
  p.chunk_rows = kGatherStageBytes / (2 * p.row_bytes);
  p.smem = 1024 + (size_t)kGatherStages * kGatherStageBytes + sizeof(int32_t) * p.nw * nb +
           sizeof(int32_t) * p.tile + 256;
  return p;
}

// grid (tiles, segments), block nw * 32. hist: scanned offsets [seg][nb][tiles];
// perm, inv, invnorm [seg][n]; xs, vs [seg][n][d]. tmx / tmv: x, v as
// [BH * n][d] with boxes of chunk_rows x d, no swizzle.
template <typename T>
__global__ void __launch_bounds__(256, 2)
    k_sort_gather_tma(const __grid_constant__ CUtensorMap tmx,
                      const __grid_constant__ CUtensorMap tmv, const int32_t* __restrict__ buckets,
                      const int32_t* __restrict__ hist, int32_t* __restrict__ perm,
                      int32_t* __restrict__ inv, T* __restrict__ xs, T* __restrict__ vs,
                      float* __restrict__ invnorm, int n, int d, int nb, int rounds, int tiles,
                      int chunk_rows, WsHeader* hdr) {
  using namespace sm100;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* sbase = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* ring = sbase;  // [stage][x rows | v rows]
  const int nw = blockDim.x >> 5, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int32_t* base = reinterpret_cast<int32_t*>(ring + kGatherStages * kGatherStageBytes);  // [nw][nb]
  const int tile = nw * kSortSub;
  int32_t* slots = base + nw * nb;                                   // [tile]
  uint64_t* full = reinterpret_cast<uint64_t*>(slots + tile);        // [stages]
  uint64_t* empty = full + kGatherStages;                            // [stages]

  const int seg = blockIdx.y, tl = blockIdx.x;
  const int64_t bh = seg / rounds;
  const int t0 = tl * tile;
  const int tend = min(n, t0 + tile);
  const int row_bytes = d * (int)sizeof(T);
  const int half_stage = kGatherStageBytes / 2;
  const int nchunks = (tend - t0 + chunk_rows - 1) / chunk_rows;
  const uint32_t chunk_tx = 2u * chunk_rows * row_bytes;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGatherStages; ++s) {
      mbar_init(full + s, 1);
      mbar_init(empty + s, nw);
    }
    fence_mbar_init();
  }
  __syncthreads();
  auto issue = [&](int k) {  // thread 0: rows of chunk k into stage k % stages
    const int s = k % kGatherStages;
    const int row = (int)(bh * n) + t0 + k * chunk_rows;
    mbar_expect_tx(full + s, chunk_tx);
    tma_load_2d(ring + s * kGatherStageBytes, &tmx, full + s, 0, row);
    tma_load_2d(ring + s * kGatherStageBytes + half_stage, &tmv, full + s, 0, row);
  };
  if (threadIdx.x == 0)
    for (int k = 0; k < kGatherStages && k < nchunks; ++k) issue(k);

  // ---- ranks (as k_sort_scatter): per-warp counts, scan, stable ranks
  for (int i = threadIdx.x; i < nw * nb; i += blockDim.x) base[i] = 0;
  __syncthreads();
  const int wstart = t0 + warp * kSortSub;
  const int wend = min(n, wstart + kSortSub);
  const int32_t* bk = buckets + (int64_t)seg * n;
  int32_t* mybase = base + warp * nb;
  constexpr int kSteps = kSortSub / 32;
  int bks[kSteps];  // this warp's bucket ids, -1 past the end
#pragma unroll
  for (int i = 0; i < kSteps; ++i) {
    const int t = wstart + 32 * i + lane;
    bks[i] = t < wend ? clamp_bucket(bk[t], nb) : -1;
  }
#pragma unroll
  for (int i = 0; i < kSteps; ++i) {
    const int b = bks[i];
    const uint32_t peers = __match_any_sync(0xffffffffu, b);
    if (b >= 0 && lane == __ffs(peers) - 1) mybase[b] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  const int32_t* h = hist + (int64_t)seg * nb * tiles + tl;
  for (int b = threadIdx.x; b < nb; b += blockDim.x) {
    int32_t run = h[(int64_t)b * tiles];
    for (int w = 0; w < nw; ++w) {
      const int32_t c = base[w * nb + b];
      base[w * nb + b] = run;
      run += c;
    }
  }
  __syncthreads();
  const int64_t so = (int64_t)seg * n;
#pragma unroll
  for (int i = 0; i < kSteps; ++i) {
    const int t = wstart + 32 * i + lane;
    const int b = bks[i];
    const uint32_t peers = __match_any_sync(0xffffffffu, b);
    int slot = 0;
    if (b >= 0) slot = mybase[b] + __popc(peers & lanemask_lt());
    __syncwarp();
    if (b >= 0 && lane == __ffs(peers) - 1) mybase[b] += __popc(peers);
    __syncwarp();
    if (b >= 0) {
      perm[so + slot] = t;
      inv[so + t] = slot;
      slots[t - t0] = slot;
    }
  }
  __syncthreads();

  // ---- gather: every chunk's rows to their slots
  const int lpr = row_bytes / 16 < 32 ? row_bytes / 16 : 32;  // lanes per row
  const int rpi = 32 / lpr;                                    // rows per instruction
  const int ipr = row_bytes / 16 / lpr;                        // 16-byte pieces per lane
  T* xd = xs + so * d;
  T* vd = vs + so * d;
  bool ok = true;
  for (int k = 0; k < nchunks; ++k) {
    const int s = k % kGatherStages;
    if (!mbar_wait(full + s, (k / kGatherStages) & 1)) {
      ok = false;
      break;
    }
    const unsigned char* xr = ring + s * kGatherStageBytes;
    const unsigned char* vr = xr + half_stage;
    for (int r0 = warp * rpi; r0 < chunk_rows; r0 += nw * rpi) {
      const int r = r0 + lane / lpr;
      const int t = t0 + k * chunk_rows + r;
      const bool valid = r < chunk_rows && t < tend;
      const int slot = valid ? slots[t - t0] : 0;
      float ss = 0.f;
      for (int it = 0; it < ipr; ++it) {
        const int off = (lane % lpr + it * lpr) * 16;
        if (valid) {
          const uint4 a = *reinterpret_cast<const uint4*>(xr + r * row_bytes + off);
          const uint4 c = *reinterpret_cast<const uint4*>(vr + r * row_bytes + off);
          *reinterpret_cast<uint4*>(reinterpret_cast<unsigned char*>(xd + (int64_t)slot * d) + off) = a;
          *reinterpret_cast<uint4*>(reinterpret_cast<unsigned char*>(vd + (int64_t)slot * d) + off) = c;
          float f[Vec16<T>::N];
          Vec16<T>::unpack(a, f);
#pragma unroll
          for (int e = 0; e < Vec16<T>::N; ++e) ss = fmaf(f[e], f[e], ss);
        }
      }
      for (int o = lpr / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (valid && lane % lpr == 0) invnorm[so + slot] = ss > 0.f ? 1.0f / sqrtf(ss) : 0.f;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty + s);
    if (threadIdx.x == 0 && k + kGatherStages < nchunks) {
      if (!mbar_wait(empty + s, (k / kGatherStages) & 1)) {
        ok = false;
        break;
      }
      issue(k + kGatherStages);
    }
  }
  if (!ok) record_status(hdr, 5u /* LSH_ERR_TIMEOUT */);
}

}  // namespace lsh
