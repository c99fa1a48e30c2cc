// The in-bucket top-k variant of LSH attention described in "Reformer
// re-reading" (2kiu.com), §2.2 (SimHash codes mod K over several rounds,
// in-bucket ranking of keys, the top k per query, the union over rounds),
// as a second workload beside the chunked attention.
//
//   k_tk_hash    per (token, round): m bits [proj_t . x > 0] in fp64, the code
//                sum_t bit_t 2^t mod K (Horner); one thread per (token, round)
//   (the counting sort of sort.cuh orders every (batch, head, round) by bucket)
//   k_tk_select  one warp per (query, round): scores of the query against the
//                keys of its bucket in fp64 (causal: positions <= the query's),
//                kept as a sorted top-k (higher score first, lower position on
//                ties) by warp-wide bitonic merges of 32-candidate batches
//   k_tk_attend  one warp per query: the union of its rounds' top-k (a
//                position in an earlier round's list is not counted again),
//                fp32 logits, one softmax, out and lse
// Membership decisions (bucket bits and top-k sets) are taken in fp64 with
// the sums in increasing k, products and sums rounded separately (no fused
// multiply-add), the norm's square root and the two divisions correctly
// rounded, so they are the exact decisions of that fp64 evaluation.
#pragma once

#include "common.cuh"

namespace lsh {

constexpr int kTopkMaxK = 32;     // candidates kept per query and round
constexpr int kTopkMaxBits = 32;
constexpr int kTopkMaxRounds = 8;

// grid-stride over (bh, round, token). x [BH][n][D], proj [L][D][m] (bf16),
// bucket [BH][L][n].
template <int D>
__global__ void __launch_bounds__(256)
    k_tk_hash(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ proj,
              int32_t* __restrict__ bucket, int n, int L, int m, int K, int64_t total) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int i = (int)(e % n);
    const int64_t rest = e / n;
    const int l = (int)(rest % L);
    const int64_t bh = rest / L;
    const __nv_bfloat16* xr = x + (bh * n + i) * D;
    const __nv_bfloat16* pr = proj + (int64_t)l * D * m;
    double xv[D];
#pragma unroll
    for (int k = 0; k < D; ++k) xv[k] = (double)__bfloat162float(xr[k]);
    uint32_t bits = 0;
    for (int t = 0; t < m; ++t) {
      double p = 0.0;
#pragma unroll 8
      for (int k = 0; k < D; ++k)
        p = __dadd_rn(p, __dmul_rn(xv[k], (double)__bfloat162float(pr[(int64_t)k * m + t])));
      bits |= (p > 0.0 ? 1u : 0u) << t;
    }
    int code = 0;
    for (int t = m - 1; t >= 0; --t) code = (2 * code + (int)((bits >> t) & 1u)) % K;
    bucket[e] = code;
  }
}

// fp64 score of query i against key j (rows of one (batch, head)), in the
// fixed order described above; the query itself scores -1e5.
template <int D>
__device__ __forceinline__ double tk_score(const __nv_bfloat16* __restrict__ xb, const double* q,
                                           int i, int j) {
  if (j == i) return (double)kSelfLogit;
  const __nv_bfloat16* kr = xb + (int64_t)j * D;
  double dot = 0.0, nn = 0.0;
#pragma unroll 8
  for (int k = 0; k < D; ++k) {
    const double kv = (double)__bfloat162float(kr[k]);
    dot = __dadd_rn(dot, __dmul_rn(q[k], kv));
    nn = __dadd_rn(nn, __dmul_rn(kv, kv));
  }
  const double nrm = __dsqrt_rn(nn);
  return nrm > 0.0 ? __ddiv_rn(__ddiv_rn(dot, nrm), __dsqrt_rn((double)D)) : 0.0;
}

// a better than b: higher score, then lower position
__device__ __forceinline__ bool tk_better(double sa, int pa, double sb, int pb) {
  return sa > sb || (sa == sb && pa < pb);
}

// Compare-exchange with the lane `lane ^ j` inside a bitonic network: the
// lane keeps the better entry iff `keep_better`.
__device__ __forceinline__ void tk_cx(double& s, int& p, int j, bool keep_better) {
  const double os = __shfl_xor_sync(0xffffffffu, s, j);
  const int op = __shfl_xor_sync(0xffffffffu, p, j);
  const bool other_better = tk_better(os, op, s, p);
  if (other_better == keep_better) {
    s = os;
    p = op;
  }
}

// Sort 32 entries (one per lane) descending (best first) in lane order.
__device__ __forceinline__ void tk_sort32(double& s, int& p, int lane) {
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1)
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      // descending blocks where (lane & k) == 0, and the lower lane keeps the better
      const bool up = (lane & k) == 0;
      const bool lower = (lane & j) == 0;
      tk_cx(s, p, j, up == lower);
    }
}

// grid-stride over warps = (bh, round, query). perm, bucket [BH][L][n];
// cand [BH][L][n][k] positions, best first, -1 past the kept ones.
template <int D>
__global__ void __launch_bounds__(256)
    k_tk_select(const __nv_bfloat16* __restrict__ x, const int32_t* __restrict__ bucket,
                const int32_t* __restrict__ perm, int32_t* __restrict__ cand, int n, int L,
                int topk, int causal, int64_t total) {
  const int lane = threadIdx.x & 31;
  for (int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; w < total;
       w += ((int64_t)gridDim.x * blockDim.x) >> 5) {
    const int i = (int)(w % n);
    const int64_t seg = w / n;  // (bh, round)
    const int64_t bh = seg / L;
    const int32_t* bk = bucket + seg * n;
    const int32_t* pm = perm + seg * n;
    const int b = bk[i];
    // the bucket's slots [lo, hi) in the sorted order: bucket[perm[s]] is
    // non-decreasing in s
    int lo = 0, hi = n;
    {
      int a0 = 0, a1 = n;  // first slot with bucket >= b
      while (a0 < a1) {
        const int mid = (a0 + a1) >> 1;
        if (bk[pm[mid]] < b) a0 = mid + 1; else a1 = mid;
      }
      lo = a0;
      a1 = n;  // first slot with bucket > b
      while (a0 < a1) {
        const int mid = (a0 + a1) >> 1;
        if (bk[pm[mid]] <= b) a0 = mid + 1; else a1 = mid;
      }
      hi = a0;
    }
    const __nv_bfloat16* xb = x + bh * (int64_t)n * D;
    double q[D];
#pragma unroll
    for (int k = 0; k < D; ++k) q[k] = (double)__bfloat162float(xb[(int64_t)i * D + k]);
    double ts = -INFINITY;  // the kept entries, best first across lanes
    int tp = 0x7fffffff;
    for (int s0 = lo; s0 < hi; s0 += 32) {
      double cs = -INFINITY;
      int cp = 0x7fffffff;
      if (s0 + lane < hi) {
        const int j = pm[s0 + lane];  // slots of a bucket hold increasing positions
        if (!causal || j <= i) {
          cs = tk_score<D>(xb, q, i, j);
          cp = j;
        }
      }
      tk_sort32(cs, cp, lane);
      // merge: the better of kept[lane] and batch[31 - lane] are the best 32 of
      // the 64 (a bitonic sequence), then sort them
      const double rs = __shfl_sync(0xffffffffu, cs, 31 - lane);
      const int rp = __shfl_sync(0xffffffffu, cp, 31 - lane);
      if (tk_better(rs, rp, ts, tp)) {
        ts = rs;
        tp = rp;
      }
#pragma unroll
      for (int j = 16; j > 0; j >>= 1) tk_cx(ts, tp, j, (lane & j) == 0);
    }
    if (lane < topk)
      cand[(seg * n + i) * topk + lane] = (tp == 0x7fffffff) ? -1 : tp;
  }
}

// grid-stride over warps = (bh, query). cand [BH][L][n][k]; out [BH][n][D]
// (bf16), lse [BH][n].
template <int D>
__global__ void __launch_bounds__(256)
    k_tk_attend(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ v,
                const int32_t* __restrict__ cand, __nv_bfloat16* __restrict__ out,
                float* __restrict__ lse, int n, int L, int topk, int64_t total) {
  constexpr int PER = D / 32;
  __shared__ int32_t spos[8][kTopkMaxRounds * kTopkMaxK];
  __shared__ float sw[8][kTopkMaxRounds * kTopkMaxK];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  const float inv_sqrt_d = 1.0f / sqrtf((float)D);
  for (int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; w < total;
       w += ((int64_t)gridDim.x * blockDim.x) >> 5) {
    const int i = (int)(w % n);
    const int64_t bh = w / n;
    const int ne = L * topk;
    // entries (round l, rank r); a position already listed by an earlier
    // round is dropped (each round's list holds distinct positions)
    for (int e = lane; e < ne; e += 32) {
      const int l = e / topk;
      int p = cand[((bh * L + l) * n + i) * topk + e % topk];
      for (int l2 = 0; p >= 0 && l2 < l; ++l2)
        for (int r2 = 0; r2 < topk; ++r2)
          if (cand[((bh * L + l2) * n + i) * topk + r2] == p) { p = -1; break; }
      spos[wib][e] = p;
    }
    __syncwarp();
    const __nv_bfloat16* xb = x + bh * (int64_t)n * D;
    float qv[PER];
#pragma unroll
    for (int k = 0; k < PER; ++k) qv[k] = __bfloat162float(xb[(int64_t)i * D + lane + 32 * k]);
    // logits, one candidate at a time across the warp (lanes own features)
    float mx = -INFINITY;
    for (int e = 0; e < ne; ++e) {
      const int p = spos[wib][e];
      if (p < 0) continue;  // uniform across the warp
      float l;
      if (p == i) {
        l = kSelfLogit;
      } else {
        float dot = 0.f, nn = 0.f;
#pragma unroll
        for (int k = 0; k < PER; ++k) {
          const float kv = __bfloat162float(xb[(int64_t)p * D + lane + 32 * k]);
          dot = fmaf(qv[k], kv, dot);
          nn = fmaf(kv, kv, nn);
        }
        dot = warp_sum(dot);
        nn = warp_sum(nn);
        l = nn > 0.f ? dot / sqrtf(nn) * inv_sqrt_d : 0.f;
      }
      if (lane == 0) sw[wib][e] = l;
      mx = fmaxf(mx, l);
    }
    __syncwarp();
    float acc[PER];
#pragma unroll
    for (int k = 0; k < PER; ++k) acc[k] = 0.f;
    float z = 0.f;
    const __nv_bfloat16* vb = v + bh * (int64_t)n * D;
    for (int e = 0; e < ne; ++e) {
      const int p = spos[wib][e];
      if (p < 0) continue;
      const float wgt = expf(sw[wib][e] - mx);
      z += wgt;
#pragma unroll
      for (int k = 0; k < PER; ++k)
        acc[k] = fmaf(wgt, __bfloat162float(vb[(int64_t)p * D + lane + 32 * k]), acc[k]);
    }
    const float rz = 1.0f / z;
#pragma unroll
    for (int k = 0; k < PER; ++k)
      out[(bh * n + i) * D + lane + 32 * k] = __float2bfloat16_rn(acc[k] * rz);
    if (lane == 0) lse[bh * n + i] = mx + logf(z);
    __syncwarp();  // spos / sw are rewritten for the next query
  }
}

}  // namespace lsh
