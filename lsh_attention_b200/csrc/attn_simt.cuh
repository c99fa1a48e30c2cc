// Chunked shared-QK attention on the CUDA cores (fp32 arithmetic).
//
// "Reformer summary" (ttnews.xyz), §局部敏感哈希注意力 and §共享QK中的自掩碼;
// "Reformer: LSH attention and reversible layers" (dtcms.com), §二.1.
// For the query at sorted slot s in chunk c = s / m, the keys are the slots of
// chunks c-1 and c (chunk 0: itself only). Logit against key slot j:
//   causal and pos_j > pos_s  -> removed
//   j == s                    -> -1e5 (self)
//   otherwise                 -> (x_s . x_j) * invnorm_j / sqrt(d)
// The window is swept in blocks of 64 keys with a running max and sum, so
// any chunk length up to 128 fits. This kernel serves fp32 inputs and chunk
// lengths the tensor-core kernel does not take. Each round's output row is
// written at the query's slot, in the input type, and its lse at the query's
// position.
#pragma once

#include "common.cuh"

namespace lsh {

constexpr int kSimtWarps = 8;
constexpr int kSimtKeys = 64;  // keys per block of the window sweep

// grid (n / m, segments), block 256.
// xs, vs [seg][n][d] sorted rows; perm, invnorm [seg][n];
// out_r [seg][n][d] in T, slot order; lse [seg][n] fp32 in position order.
template <typename T, int D, int QPW>
__global__ void __launch_bounds__(kSimtWarps * 32)
    k_attn_simt(const T* __restrict__ xs, const T* __restrict__ vs,
                const int32_t* __restrict__ perm, const float* __restrict__ invnorm,
                T* __restrict__ out_r, float* __restrict__ lse, int n, int m, int causal) {
  constexpr int DP = D + 1;     // padded fp32 row: conflict-free per-lane key rows
  constexpr int DL = D / 32;    // output dims per lane
  extern __shared__ __align__(16) float sm[];
  float* Q = sm;                       // [m][DP]
  float* K = Q + 128 * DP;             // [64][DP]
  float* V = K + kSimtKeys * DP;       // [64][D]
  float* kin = V + kSimtKeys * D;      // [64]
  int* kpos = reinterpret_cast<int*>(kin + kSimtKeys);  // [64]

  const int seg = blockIdx.y, c = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t so = (int64_t)seg * n;
  const int q0 = c * m;
  const int lo = (c > 0 ? c - 1 : 0) * m, hi = q0 + m;
  const float scale = 1.0f / sqrtf((float)D);

  for (int e = threadIdx.x; e < m * D; e += blockDim.x)
    Q[(e / D) * DP + e % D] = Elem<T>::to_f(xs[(so + q0) * D + e]);

  float mrun[QPW], lrun[QPW], acc[QPW][DL];
  int qpos[QPW];
#pragma unroll
  for (int i = 0; i < QPW; ++i) {
    mrun[i] = -INFINITY;
    lrun[i] = 0.f;
#pragma unroll
    for (int k = 0; k < DL; ++k) acc[i][k] = 0.f;
    const int q = warp + i * kSimtWarps;
    qpos[i] = q < m ? perm[so + q0 + q] : 0;
  }

  for (int kb = lo; kb < hi; kb += kSimtKeys) {
    const int nk = min(kSimtKeys, hi - kb);
    __syncthreads();
    for (int e = threadIdx.x; e < nk * D; e += blockDim.x) {
      K[(e / D) * DP + e % D] = Elem<T>::to_f(xs[(so + kb) * D + e]);
      V[e] = Elem<T>::to_f(vs[(so + kb) * D + e]);
    }
    for (int j = threadIdx.x; j < nk; j += blockDim.x) {
      kin[j] = invnorm[so + kb + j];
      kpos[j] = perm[so + kb + j];
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < QPW; ++i) {
      const int q = warp + i * kSimtWarps;
      if (q >= m) break;
      const float* qr = Q + q * DP;
      float l[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int j = lane + 32 * h;
        l[h] = -INFINITY;
        if (j < nk) {
          const bool self = (kb + j) == (q0 + q);
          if (self) {
            l[h] = kSelfLogit;
          } else if (!(causal && kpos[j] > qpos[i])) {
            const float* kr = K + j * DP;
            float dot = 0.f;
#pragma unroll 16
            for (int k = 0; k < D; ++k) dot = fmaf(qr[k], kr[k], dot);
            l[h] = dot * kin[j] * scale;
          }
        }
      }
      const float bmax = warp_max(fmaxf(l[0], l[1]));
      if (bmax == -INFINITY) continue;  // nothing of this block is visible
      const float mnew = fmaxf(mrun[i], bmax);
      const float corr = expf(mrun[i] - mnew);  // 0 when mrun was -inf
      float p[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) p[h] = (l[h] == -INFINITY) ? 0.f : expf(l[h] - mnew);
      lrun[i] = lrun[i] * corr + warp_sum(p[0] + p[1]);
      mrun[i] = mnew;
#pragma unroll
      for (int k = 0; k < DL; ++k) acc[i][k] *= corr;
      for (int j = 0; j < nk; ++j) {
        const float pj = __shfl_sync(0xffffffffu, p[j >> 5], j & 31);
#pragma unroll
        for (int k = 0; k < DL; ++k) acc[i][k] = fmaf(pj, V[j * D + lane + 32 * k], acc[i][k]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < QPW; ++i) {
    const int q = warp + i * kSimtWarps;
    if (q >= m) break;
    const float inv = 1.0f / lrun[i];
    T* o = out_r + (so + q0 + q) * D;
#pragma unroll
    for (int k = 0; k < DL; ++k) o[lane + 32 * k] = Elem<T>::from_f(acc[i][k] * inv);
    if (lane == 0) lse[so + qpos[i]] = mrun[i] + logf(lrun[i]);
  }
}

inline size_t attn_simt_smem(int D) {
  return sizeof(float) * (128 * (D + 1) + kSimtKeys * (D + 1) + kSimtKeys * D + kSimtKeys) +
         sizeof(int) * kSimtKeys;
}

}  // namespace lsh
