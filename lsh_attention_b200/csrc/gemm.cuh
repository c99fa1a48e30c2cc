// Dense bf16 GEMM on the 5th-generation tensor cores with a fused epilogue,
// for the layers around the attention: the projections into and out of the
// heads and the chunked feed-forward layer of a reversible block
// ("Reformer: LSH attention and reversible layers" (dtcms.com), §二.2 and
// §二.3).
//
//   C[m][n] = R[m][n] + sign * act(sum_k A[m][k] B[n][k] + bias[n])
//
// A [M][K] and B [N][K] are K-major bf16 (B is a weight stored out x in);
// act is the identity or max(., 0); the residual R is optional; C is bf16.
// A may instead be read, and C written, in the head-split layout
// [batch][heads][n][d] of the attention (rows m = batch * n + position,
// columns = head * d + feature), through 4D tensor maps.
//
// One persistent CTA per SM walks 128 x 128 output tiles (m-tile major, so
// neighbouring CTAs share A rows and every CTA streams the weights from L2):
//   warp 0      TMA: 64-wide K steps of A and B into a 4-stage ring
//   warp 1      tcgen05.mma (M 128, N 128, K 16 per instruction) into one of
//               two TMEM accumulators, so a tile's epilogue overlaps the next
//               tile's products
//   warps 2-5   epilogue: the accumulator by 32-column slices, bias,
//               activation and residual in fp32, bf16, staged in swizzled
//               shared memory, TMA stores
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace lsh {

constexpr int kGemmBM = 128, kGemmBN = 128, kGemmBK = 64, kGemmStages = 4;
constexpr int kGemmWarps = 6;

struct GemmArgs {
  const float* bias;            // [N] fp32 or null
  const __nv_bfloat16* res;     // [M][N] or null
  int M, N, K;
  int relu;                     // 0 / 1
  float sign;                   // +1: R + (...), -1: R - (...)
  // head-split layouts: rows per batch (n) and features per head (d); 0 = plain 2D
  int a_split_n, a_split_d;
  int c_split_n, c_split_d;
  WsHeader* hdr;
};

__host__ __device__ constexpr size_t gemm_smem() {
  return 1024 + (size_t)kGemmStages * (kGemmBM + kGemmBN) * 128 + 4 * 32 * 128 + 256;
}

// 3D/4D-aware tile loads: a plain 2D map takes (k, row); a head-split 4D map
// [batch][heads][n][d] takes (feature, position, head, batch).
__device__ __forceinline__ void gemm_load_a(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int k, int row, int split_n, int split_d) {
  if (split_n == 0) {
    sm100::tma_load_2d(dst, map, bar, k, row);
  } else {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(sm100::smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(sm100::smem_u32(bar)), "r"(k % split_d),
        "r"(row % split_n), "r"(k / split_d), "r"(row / split_n)
        : "memory");
  }
}

__device__ __forceinline__ void gemm_store_c(const CUtensorMap* map, const void* src, int col,
                                             int row, int split_n, int split_d) {
  if (split_n == 0) {
    sm100::tma_store_2d(map, src, col, row);
  } else {
    asm volatile(
        "cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(sm100::smem_u32(src)), "r"(col % split_d), "r"(row % split_n), "r"(col / split_d),
        "r"(row / split_n)
        : "memory");
  }
}

__global__ void __launch_bounds__(kGemmWarps * 32, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tma, const __grid_constant__ CUtensorMap tmb,
              const __grid_constant__ CUtensorMap tmc, GemmArgs a) {
  using namespace sm100;
  constexpr uint32_t ABYTES = kGemmBM * 128, BBYTES = kGemmBN * 128;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* as = base;                                  // [stages][128 rows][128 B]
  unsigned char* bs = base + kGemmStages * ABYTES;           // [stages][128 rows][128 B]
  unsigned char* ostage = bs + kGemmStages * BBYTES;         // [4 warps][32][128 B]
  uint64_t* bars = reinterpret_cast<uint64_t*>(ostage + 4 * 32 * 128);
  uint64_t* full = bars;                       // [stages]
  uint64_t* empty = bars + kGemmStages;        // [stages]
  uint64_t* acc_full = empty + kGemmStages;    // [2]
  uint64_t* acc_empty = acc_full + 2;          // [2] 4 epilogue warps
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(drain + 2);
  volatile int* drain_fail = reinterpret_cast<volatile int*>(drain + 3);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mt = (a.M + kGemmBM - 1) / kGemmBM, ntn = (a.N + kGemmBN - 1) / kGemmBN;
  const int tiles = mt * ntn, ksteps = (a.K + kGemmBK - 1) / kGemmBK;
  if ((int)blockIdx.x >= tiles) return;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kGemmStages; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(acc_full + i, 1);
      mbar_init(acc_empty + i, 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    *drain_fail = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 2 * kGemmBN);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto fail = [&]() {
    record_status(a.hdr, 5u /* LSH_ERR_TIMEOUT */);
    *abort_flag = 1;
  };

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tensormap(&tma);
      prefetch_tensormap(&tmb);
      int it = 0;
      int last[kGemmStages];
      for (int s = 0; s < kGemmStages; ++s) last[s] = -1;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x) {
        const int m0 = (t / ntn) * kGemmBM, n0 = (t % ntn) * kGemmBN;
        for (int kb = 0; kb < ksteps; ++kb, ++it) {
          const int s = it % kGemmStages, k = it / kGemmStages;
          if (k > 0 && !mbar_wait(empty + s, (k - 1) & 1)) { ok = false; break; }
          if (*abort_flag) { ok = false; break; }
          mbar_expect_tx(full + s, ABYTES + BBYTES);
          gemm_load_a(as + s * ABYTES, &tma, full + s, kb * kGemmBK, m0, a.a_split_n, a.a_split_d);
          tma_load_2d(bs + s * BBYTES, &tmb, full + s, kb * kGemmBK, n0);
          last[s] = k;
        }
      }
      if (!ok && !*abort_flag) fail();
      for (int s = 0; s < kGemmStages; ++s)
        if (last[s] >= 0 && !mbar_wait(full + s, last[s] & 1)) *drain_fail = 1;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kGemmBM, kGemmBN);
      int it = 0, u = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++u) {
        const int ab = u & 1, uk = u >> 1;
        if (uk > 0 && !mbar_wait(acc_empty + ab, (uk - 1) & 1)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem + ab * kGemmBN;
        for (int kb = 0; kb < ksteps; ++kb, ++it) {
          const int s = it % kGemmStages, k = it / kGemmStages;
          if (!mbar_wait(full + s, k & 1) || *abort_flag) { ok = false; break; }
          tc_fence_after();
          const uint32_t aa = smem_u32(as + s * ABYTES), ba = smem_u32(bs + s * BBYTES);
#pragma unroll
          for (int ks = 0; ks < kGemmBK / 16; ++ks)
            mma_bf16_ss(d, desc_kmajor_sw128(aa + ks * 32), desc_kmajor_sw128(ba + ks * 32), idesc,
                        (kb > 0 || ks > 0) ? 1u : 0u);
          mma_commit(empty + s);
        }
        if (ok) mma_commit(acc_full + ab);
      }
      if (!ok && !*abort_flag) fail();
      mma_commit(drain);
      if (!mbar_wait(drain, 0)) *drain_fail = 1;
    }
  } else {
    const int q = warp & 3;  // TMEM lane quadrant: rows 32 q .. 32 q + 31
    const uint32_t tl = (uint32_t)(q * 32) << 16;
    unsigned char* stg = ostage + (warp - 2) * 32 * 128;
    int u = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++u) {
      const int ab = u & 1, uk = u >> 1;
      if (!mbar_wait(acc_full + ab, uk & 1)) {
        fail();
        break;
      }
      tc_fence_after();
      const int m0 = (t / ntn) * kGemmBM, n0 = (t % ntn) * kGemmBN;
      const int row = m0 + q * 32 + lane;
      uint32_t pk[kGemmBN / 2];
#pragma unroll
      for (int c = 0; c < kGemmBN / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tmem + tl + ab * kGemmBN + c * 32, v);
        tmem_wait_ld();
        float r[32];
        if (a.res != nullptr && row < a.M) {
          const uint4* rp = reinterpret_cast<const uint4*>(a.res + (int64_t)row * a.N + n0 + c * 32);
#pragma unroll
          for (int j = 0; j < 4; ++j) Vec16<__nv_bfloat16>::unpack(rp[j], r + 8 * j);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) r[j] = 0.f;
        }
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          float y[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int col = n0 + c * 32 + j + h;
            float acc = __uint_as_float(v[j + h]);
            if (a.bias != nullptr) acc += __ldg(a.bias + col);
            if (a.relu) acc = fmaxf(acc, 0.f);
            y[h] = fmaf(a.sign, acc, r[j + h]);
          }
          const __nv_bfloat162 p2 = __floats2bfloat162_rn(y[0], y[1]);
          pk[c * 16 + j / 2] = *reinterpret_cast<const uint32_t*>(&p2);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty + ab);
      if (m0 + q * 32 < a.M) {
#pragma unroll
        for (int b = 0; b < kGemmBN / 64; ++b) {  // 64 columns (128 bytes) per store
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
          unsigned char* line = stg + lane * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(line + ((c ^ (lane & 7)) << 4)) =
                make_uint4(pk[b * 32 + 4 * c], pk[b * 32 + 4 * c + 1], pk[b * 32 + 4 * c + 2],
                           pk[b * 32 + 4 * c + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            gemm_store_c(&tmc, stg, n0 + b * 64, m0 + q * 32, a.c_split_n, a.c_split_d);
            bulk_commit();
          }
        }
      }
    }
    if (lane == 0) bulk_wait_all();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1 && !*drain_fail) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * kGemmBN);
  }
}

}  // namespace lsh
