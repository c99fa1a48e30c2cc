// Chunked shared-QK attention on the 5th-generation tensor cores (bf16 in,
// fp32 accumulate), for chunks of m = 64 sorted slots.
//
// "Reformer summary" (ttnews.xyz), §局部敏感哈希注意力 (chunks of m in the
// sorted order), §共享QK中的自掩碼 (self-mask); "Reformer: LSH attention and
// reversible layers" (dtcms.com), §二.1 (unit-length keys, 1/sqrt(d_k)).
// A query in chunk c sees the keys of chunks c-1 and c.
//
// One work unit is a pair of chunks (c0, c0+1) of one (batch, head, round):
// its 128 queries are slots [64 c0, 64 c0 + 128) and its 192-key window is
// slots [64 (c0 - 1), 64 (c0 + 2)); the queries are rows 64..191 of the key
// tile, so Q needs no load of its own. Per unit:
//   TMA     sorted x and v rows of the window (2 x 192 rows), key norms and
//           positions (bulk copies) -> shared memory
//   MMA 1   S = Q K^T (M 128, N 192, K d) -> TMEM columns [0, 192)
//   softmax thread i owns query row i: reads its 128 in-window logits with
//           tcgen05.ld, applies 1/||k_j|| / sqrt(d), the causal mask and the
//           -1e5 self logit, and writes P (bf16, zero outside the window)
//           back to TMEM columns [0, 96) with tcgen05.st
//   MMA 2   O = P V (A = P from TMEM, B = V, MN-major) -> TMEM [128, 128 + d)
//   store   O / sum and lse, fp32, in slot order
// X is re-loaded as soon as MMA 1 completes and V as soon as MMA 2 does, and
// two CTAs share each SM (256 TMEM columns, < 114 KB shared memory each), so
// one CTA's loads overlap the other's math.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace lsh {

constexpr int kAttnM = 64;      // chunk length served by this kernel
constexpr int kAttnKeys = 192;  // key window of a pair of chunks
constexpr int kAttnTmemCols = 256;

struct AttnTcArgs {
  const float* invnorm;  // [S][n]
  const int32_t* perm;   // [S][n]
  float* out_s;          // [S][n][d] fp32, slot order
  float* lse_s;          // [S][n]
  WsHeader* hdr;
  int n, causal, pairs_per_seg;
  int64_t pairs;         // S * pairs_per_seg
  int64_t pairs_per_cta;
};

__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes,
                                              uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(sm100::smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(sm100::smem_u32(bar))
      : "memory");
}

// 32 lanes x 32 consecutive 32-bit TMEM columns.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
// D[tmem] (+)= A[tmem] * B[smem], kind::f16.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Shared-memory descriptor of an MN-major operand with the 128-byte swizzle:
// 64-element MN blocks `lbo` bytes apart, 8-row K groups 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_mnmajor_sw128(uint32_t saddr, uint32_t lbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // .x = lo (low half)
  return *reinterpret_cast<const uint32_t*>(&h);
}

// P row of one query: 192 keys packed two per 32-bit column, zero outside the
// 128 in-window keys starting at column WCOL; written to TMEM columns [0, 96).
template <int WCOL>
__device__ __forceinline__ void store_p_row(const float (&e)[128], uint32_t taddr) {
#pragma unroll
  for (int b = 0; b < 3; ++b) {
    uint32_t pk[32];
#pragma unroll
    for (int k = 0; k < 32; ++k) {
      const int i = b * 64 + 2 * k - WCOL;
      const float e0 = (i >= 0 && i < 128) ? e[(i >= 0 && i < 128) ? i : 0] : 0.f;
      const float e1 = (i + 1 >= 0 && i + 1 < 128) ? e[(i + 1 >= 0 && i + 1 < 128) ? i + 1 : 0] : 0.f;
      pk[k] = pack_bf16x2(e0, e1);
    }
    tmem_st32(taddr + b * 32, pk);
  }
}

template <int D>
__global__ void __launch_bounds__(128, 2)
    k_attn_tc(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmv,
              AttnTcArgs a) {
  using namespace sm100;
  constexpr int KH = D / 64;
  constexpr uint32_t BOX = kAttnKeys * 128;  // one 64-column box of 192 rows
  constexpr uint32_t TILE = KH * BOX;        // x (or v) tile of the window
  constexpr float kLog2e = 1.4426950408889634f;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* xt = base;            // [KH][192 rows][128 B]
  unsigned char* vt = base + TILE;     // [KH][192 rows][128 B]
  float* kinv = reinterpret_cast<float*>(base + 2 * TILE);  // [2][192]
  int32_t* kpos = reinterpret_cast<int32_t*>(kinv + 2 * kAttnKeys);  // [2][192]
  uint64_t* bars = reinterpret_cast<uint64_t*>(kpos + 2 * kAttnKeys);
  uint64_t* x_full = bars + 0;
  uint64_t* v_full = bars + 1;
  uint64_t* s_done = bars + 2;
  uint64_t* o_done = bars + 3;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t p_begin = blockIdx.x * a.pairs_per_cta;
  const int64_t p_end = min(a.pairs, p_begin + a.pairs_per_cta);
  if (p_begin >= p_end) return;  // uniform across the CTA

  if (tid == 0) {
    mbar_init(x_full, 1);
    mbar_init(v_full, 1);
    mbar_init(s_done, 1);
    mbar_init(o_done, 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, kAttnTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tm_s = tmem;        // S [0, 192), then P [0, 96)
  const uint32_t tm_o = tmem + 128;  // O [128, 128 + D): S is dead by then

  // Issue the loads of x rows, key norms and positions (x_full) or of v rows
  // (v_full) for unit p into meta buffer `mb`.
  auto load_x = [&](int64_t p, int mb) {
    const int64_t seg = p / a.pairs_per_seg;
    const int c0 = (int)(p % a.pairs_per_seg) * 2;
    const int k0 = (c0 - 1) * kAttnM;  // first key slot of the window (may be < 0)
    const int lo = max(0, k0), hi = min(a.n, k0 + kAttnKeys);
    const uint32_t mbytes = (uint32_t)(hi - lo) * 4;
    mbar_expect_tx(x_full, TILE + 2 * mbytes);
    const int row = (int)(seg * a.n) + k0;
    for (int kh = 0; kh < KH; ++kh) tma_load_2d(xt + kh * BOX, &tmx, x_full, kh * 64, row);
    bulk_copy_g2s(kinv + mb * kAttnKeys + (lo - k0), a.invnorm + seg * a.n + lo, mbytes, x_full);
    bulk_copy_g2s(kpos + mb * kAttnKeys + (lo - k0), a.perm + seg * a.n + lo, mbytes, x_full);
  };
  auto load_v = [&](int64_t p) {
    const int64_t seg = p / a.pairs_per_seg;
    const int c0 = (int)(p % a.pairs_per_seg) * 2;
    const int row = (int)(seg * a.n) + (c0 - 1) * kAttnM;
    mbar_expect_tx(v_full, TILE);
    for (int kh = 0; kh < KH; ++kh) tma_load_2d(vt + kh * BOX, &tmv, v_full, kh * 64, row);
  };

  if (tid == 0) {
    prefetch_tensormap(&tmx);
    prefetch_tensormap(&tmv);
    load_x(p_begin, 0);
    load_v(p_begin);
  }

  const uint32_t idesc_s = idesc_bf16_f32(128, kAttnKeys);
  const uint32_t idesc_o = idesc_bf16_f32(128, D) | (1u << 16);  // B (= V) MN-major
  const float qk_scale = 1.0f / sqrtf((float)D);
  const int row = warp * 32 + lane;         // query row of the unit = TMEM lane
  const int wcol = warp < 2 ? 0 : kAttnM;   // first in-window key column of this warp
  const uint32_t tl = (uint32_t)(warp * 32) << 16;
  bool ok = true;

  int it = 0;
  for (int64_t p = p_begin; p < p_end; ++p, ++it) {
    const int mb = it & 1;
    const uint32_t ph = it & 1;
    const int64_t seg = p / a.pairs_per_seg;
    const int c0 = (int)(p % a.pairs_per_seg) * 2;
    const int k0 = (c0 - 1) * kAttnM;

    // ---- MMA 1: S = Q K^T
    if (tid == 0) {
      if (mbar_wait(x_full, ph)) {
        tc_fence_after();
        const uint32_t xa = smem_u32(xt);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int kh = kk >> 2, ks = kk & 3;
          const uint64_t ad = desc_kmajor_sw128(xa + kh * BOX + kAttnM * 128 + ks * 32);
          const uint64_t bd = desc_kmajor_sw128(xa + kh * BOX + ks * 32);
          mma_bf16_ss(tm_s, ad, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(s_done);
      } else {
        ok = false;
      }
    }
    if (!__syncthreads_and(ok)) break;
    if (!mbar_wait(s_done, ph)) ok = false;
    tc_fence_after();
    // x tile is free again: prefetch the next unit's rows and metadata
    if (tid == 0 && ok && p + 1 < p_end) load_x(p + 1, mb ^ 1);

    // ---- softmax of query `row` over its 128 in-window keys
    const int qs = c0 * kAttnM + row;  // query slot
    const bool qvalid = qs < a.n;
    const float* ki = kinv + mb * kAttnKeys;
    const int32_t* kp = kpos + mb * kAttnKeys;
    const int qpos = kp[row + kAttnM];
    float l[128];
    float mx = -INFINITY;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      uint32_t v[32];
      tmem_ld32(tm_s + tl + wcol + b * 32, v);
      tmem_wait_ld();
#pragma unroll
      for (int k = 0; k < 32; ++k) {
        const int j = wcol + b * 32 + k;  // key column in the window
        const int ks = k0 + j;            // key slot
        float x = __uint_as_float(v[k]) * ki[j] * qk_scale;
        if (j == row + kAttnM) x = kSelfLogit;
        const bool keep = ks >= 0 && ks < a.n && !(a.causal && kp[j] > qpos);
        x = keep ? x : -INFINITY;
        l[b * 32 + k] = x;
        mx = fmaxf(mx, x);
      }
    }
    // the query's own slot is always in its window, so mx is finite
    float sum = 0.f;
    const float mx2 = mx * kLog2e;
#pragma unroll
    for (int k = 0; k < 128; ++k) {
      const float e = exp2f(fmaf(l[k], kLog2e, -mx2));  // 0 for removed keys (-inf)
      l[k] = e;
      sum += e;
    }
    if (warp < 2)
      store_p_row<0>(l, tm_s + tl);
    else
      store_p_row<kAttnM>(l, tm_s + tl);
    tmem_wait_st();
    tc_fence_before();
    if (!__syncthreads_and(ok)) break;

    // ---- MMA 2: O = P V
    if (tid == 0) {
      tc_fence_after();
      if (mbar_wait(v_full, ph)) {
        const uint32_t va = smem_u32(vt);
#pragma unroll
        for (int kk = 0; kk < kAttnKeys / 16; ++kk) {
          const uint64_t bd = desc_mnmajor_sw128(va + kk * 16 * 128, BOX);
          mma_bf16_ts(tm_o, tm_s + kk * 8, bd, idesc_o, kk > 0 ? 1u : 0u);
        }
        mma_commit(o_done);
      } else {
        ok = false;
      }
    }
    if (!__syncthreads_and(ok)) break;
    if (!mbar_wait(o_done, ph)) ok = false;
    tc_fence_after();
    if (tid == 0 && ok && p + 1 < p_end) load_v(p + 1);  // v tile is free again

    // ---- O / sum and lse
    if (qvalid) {
      const float inv = 1.0f / sum;
      float* orow = a.out_s + (seg * a.n + qs) * (int64_t)D;
#pragma unroll
      for (int b = 0; b < D / 32; ++b) {
        uint32_t v[32];
        tmem_ld32(tm_o + tl + b * 32, v);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; k += 4) {
          float4 o;
          o.x = __uint_as_float(v[k]) * inv;
          o.y = __uint_as_float(v[k + 1]) * inv;
          o.z = __uint_as_float(v[k + 2]) * inv;
          o.w = __uint_as_float(v[k + 3]) * inv;
          *reinterpret_cast<float4*>(orow + b * 32 + k) = o;
        }
      }
      a.lse_s[seg * a.n + qs] = mx + logf(sum);
    } else {
      // keep the warp's tcgen05.ld calls uniform
#pragma unroll
      for (int b = 0; b < D / 32; ++b) {
        uint32_t v[32];
        tmem_ld32(tm_o + tl + b * 32, v);
        tmem_wait_ld();
      }
    }
    tc_fence_before();
    if (!__syncthreads_and(ok)) break;
  }
  if (!ok && tid == 0) record_status(a.hdr, 5u /* LSH_ERR_TIMEOUT */);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kAttnTmemCols);
  }
}

inline size_t attn_tc_smem(int D) {
  const size_t tile = (size_t)(D / 64) * kAttnKeys * 128;
  size_t s = 1024 + 2 * tile + 2 * kAttnKeys * 4 * 2 + 64;
  // at most two CTAs per SM: each holds 256 of the 512 TMEM columns
  return s < 80 * 1024 ? 80 * 1024 : s;
}

}  // namespace lsh
