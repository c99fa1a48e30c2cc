// Angular LSH hash evaluated exactly in fp64 on the CUDA cores.
//
// "Reformer summary" (ttnews.xyz), §局部敏感哈希: with R of size
// [dimension, b/2], h(x) = argmax([xR ; -xR]); ties take the first index.
//
// Every product of two fp32 (or two bf16) values is exact in fp64, and the
// sum runs over k = 0..d-1 in order, so p_j is the same fp64 number a plain
// sequential evaluation gives. This kernel is the whole hash for fp32 inputs
// and the tie-breaker that the tensor-core hash defers near ties to.
#pragma once

#include "common.cuh"

namespace lsh {

constexpr int kHashExactTokens = 128;  // tokens (threads) per CTA
constexpr int kHashExactCols = 32;     // columns of R staged per pass

// Ordering of candidates of [p ; -p]: larger value first, then lower index.
__device__ __forceinline__ void argmax_update(double v, int idx, double& bv, int& bi) {
  if (v > bv || (v == bv && idx < bi)) {
    bv = v;
    bi = idx;
  }
}

// p_j for one token, exact fp64, for every column j; returns the bucket.
// xrow: token's row in shared memory (stride 1), Rs: [d][kHashExactCols]
// doubles in shared memory for columns [j0, j0 + cols).
template <typename T>
__device__ __forceinline__ void hash_exact_cols(const T* xrow, const double* Rs, int d, int j0,
                                                int cols, int half, double& bv, int& bi) {
  double acc[kHashExactCols];
#pragma unroll
  for (int jj = 0; jj < kHashExactCols; ++jj) acc[jj] = 0.0;
  for (int k = 0; k < d; ++k) {
    const double xk = Elem<T>::to_d(xrow[k]);
    const double* Rk = Rs + k * kHashExactCols;
#pragma unroll
    for (int jj = 0; jj < kHashExactCols; ++jj) acc[jj] = fma(xk, Rk[jj], acc[jj]);
  }
#pragma unroll
  for (int jj = 0; jj < kHashExactCols; ++jj) {
    if (jj < cols) {
      argmax_update(acc[jj], j0 + jj, bv, bi);
      argmax_update(-acc[jj], half + j0 + jj, bv, bi);
    }
  }
}

// grid (ceil(n / 128), B*H, rounds), block 128.
// x [BH][n][d], R [rounds][d][half], buckets [BH][rounds][n].
template <typename T>
__global__ void __launch_bounds__(kHashExactTokens)
    k_hash_exact(const T* __restrict__ x, const T* __restrict__ R, int32_t* __restrict__ buckets,
                 int n, int d, int nb, int rounds) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int half = nb / 2;
  const int xstride = d + (sizeof(T) == 4 ? 1 : 2);  // padded rows: conflict-free column reads
  double* Rs = reinterpret_cast<double*>(smem_raw);
  T* xs = reinterpret_cast<T*>(smem_raw + sizeof(double) * d * kHashExactCols);

  const int t0 = blockIdx.x * kHashExactTokens;
  const int64_t bh = blockIdx.y;
  const int r = blockIdx.z;
  const int tid = threadIdx.x;
  const int ntok = min(kHashExactTokens, n - t0);

  const T* xg = x + (bh * n + t0) * (int64_t)d;
  for (int e = tid; e < ntok * d; e += kHashExactTokens) xs[(e / d) * xstride + e % d] = xg[e];

  const T* Rr = R + (int64_t)r * d * half;
  double bv = -INFINITY;
  int bi = 0x7fffffff;
  for (int j0 = 0; j0 < half; j0 += kHashExactCols) {
    const int cols = min(kHashExactCols, half - j0);
    __syncthreads();
    for (int e = tid; e < d * kHashExactCols; e += kHashExactTokens) {
      const int k = e / kHashExactCols, jj = e % kHashExactCols;
      Rs[e] = (jj < cols) ? Elem<T>::to_d(Rr[(int64_t)k * half + j0 + jj]) : 0.0;
    }
    __syncthreads();
    if (tid < ntok) hash_exact_cols<T>(xs + tid * xstride, Rs, d, j0, cols, half, bv, bi);
  }
  if (tid < ntok) buckets[(bh * rounds + r) * n + t0 + tid] = bi;
}

}  // namespace lsh
