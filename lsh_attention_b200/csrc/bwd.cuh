// Backward pass of the LSH-attention forward (bf16, chunk 64), on the
// 5th-generation tensor cores.
//
// The forward is "Reformer summary" (ttnews.xyz), §局部敏感哈希注意力 and
// §多輪LSH哈希, with the logit of "Reformer: LSH attention and reversible
// layers" (dtcms.com), §二.1; the pages train it end to end ("Reformer
// re-reading" (2kiu.com), §2.2). Bucket ids are an input (the hash is
// piecewise constant), so the sort is recomputed from them.
//
// Derivation (upstream g = dL/dout, optional dlse_in = dL/dlse): with
// w_r = exp(lse_r - LSE) the merge weights and o_r each round's output,
//   dL/do_r = w_r g,   dL/dlse_r = w_r g.(o_r - out) + dlse_in_r.
// Per round, for query i and key j of its window, P_ij = exp(l_ij - lse_r,i),
//   dS_ij = P_ij (dP_ij - D_i + dL/dlse_r,i),  dP_ij = w_i g_i . v_j,
//   D_i = rowsum(P_i dP_i) = w_i g_i . o_r,i,
// and D_i cancels against the w_i g_i . o_r,i inside dL/dlse_r,i:
//   dS_ij = P_ij (w_i g_i . v_j + c_i),   c_i = dlse_in_r,i - w_i g_i . out_i,
// so no round's output is needed. The self logit and masked keys carry no
// gradient (dS = 0 there). With l_ij = x_i . x_j kinv_j / sqrt(d) and
// kd_j = kinv_j / sqrt(d), dS'_ij = dS_ij kd_j:
//   dx_i (query role)  = sum_j dS'_ij x_j
//   G_j = sum_i dS'_ij x_i,   dx_j (key role) = G_j - x_j kinv_j^2 (x_j . G_j)
//   dv_j = sum_i P_ij w_i g_i
// and each position sums its query and key roles over the rounds.
//
// Kernels:
//   k_bwd_prep_pos   per position: LSE over rounds and g . out
//   k_bwd_prep_slot  per (round, slot): (position, lse log2(e), w, c) and the
//                    key's (logit scale, kd, kinv)
//   k_bwd_dq         query-stationary, a pair of chunks per unit (128 queries,
//                    192 keys as in the forward): S = Q K^T and dPraw = G V^T
//                    into TMEM, dS' written over S in bf16, dQ = dS' X_window
//                    (A read from TMEM); dQ rows out, fp32, slot order
//   k_bwd_dkv        key-stationary, a pair of chunks of keys per unit (128
//                    keys, the 192 queries that see them, in two passes: the
//                    middle chunk, then the first and the last): S^T = K Q^T
//                    and dPraw^T = V G^T into TMEM,
//                    P w and dS' written over them in bf16, dV += (P w) G_q and
//                    G += dS' X_q (A read from TMEM); after both passes the key
//                    rows of dx and dv out, fp32, slot order
//   k_bwd_unsort     per position: dx = sum_r (dQ + dXk)[inv_r], dv = sum_r dV[inv_r]
// Each unit runs in phases separated by CTA barriers (loads, MMAs, the
// elementwise step, MMAs, write-out); TMEM holds [0, 512) for one unit.
#pragma once

#include <type_traits>

#include "attn_tc.cuh"
#include "common.cuh"
#include "merge.cuh"
#include "sm100.cuh"

namespace lsh {

constexpr int kBwdWarps = 8;  // warps 0-3 own TMEM lane quadrants; all 8 load
constexpr float kBwdLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------------------
// grid-stride over (bh, position); block 256, D * sizeof(T) / 16 lanes per
// position. lse [BH][R][n] (natural log), out, g [BH][n][D] in T; pos_tab
// [BH][n] float2 (LSE, g . out).
template <typename T, int D>
__global__ void __launch_bounds__(256)
    k_bwd_prep_pos(const float* __restrict__ lse, const T* __restrict__ out,
                   const T* __restrict__ g, float2* __restrict__ pos_tab, int n, int rounds,
                   int64_t total) {
  // a group of G lanes per position, lane j of the group one 16-byte piece of
  // the rows of g and out
  constexpr int G = D * (int)sizeof(T) / 16;
  constexpr int EPV = 16 / (int)sizeof(T);
  const int lane = threadIdx.x & 31, gl = lane % G;
  const int64_t stride = (int64_t)gridDim.x * (blockDim.x / 32) * (32 / G);
  const int64_t first = (((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5) * (32 / G) + lane / G;
  // the same count for every lane: all of a warp's lanes run every shuffle
  const int64_t iters = (total + stride - 1) / stride;
  for (int64_t it = 0; it < iters; ++it) {
    const int64_t r = first + it * stride;
    const bool valid = r < total;
    float dot = 0.f, mx = -INFINITY;
    int bh = 0, i = 0;
    if (valid) {
      bh = (int)(r / n);  // BH * n < 2^31
      i = (int)(r - (int64_t)bh * n);
      const uint4 ga = *reinterpret_cast<const uint4*>(g + r * D + gl * EPV);
      const uint4 oa = *reinterpret_cast<const uint4*>(out + r * D + gl * EPV);
      float fg[EPV], fo[EPV];
      unpack16<T>(ga, fg);
      unpack16<T>(oa, fo);
#pragma unroll
      for (int e = 0; e < EPV; ++e) dot = fmaf(fg[e], fo[e], dot);
      for (int q = gl; q < rounds; q += G) mx = fmaxf(mx, lse[((int64_t)bh * rounds + q) * n + i]);
    }
    dot = group_sum<G>(dot);
    mx = group_max<G>(mx);
    float z = 0.f;
    if (valid)
      for (int q = gl; q < rounds; q += G) z += expf(lse[((int64_t)bh * rounds + q) * n + i] - mx);
    z = group_sum<G>(z);
    if (valid && gl == 0) pos_tab[r] = make_float2(mx + logf(z), dot);
  }
}

// grid-stride over (seg, slot). perm [S][n]; lse, dlse (nullable) [S][n] by
// position; pinv [BH][n]; qtab [S][n] float4 (position bits, lse log2(e), w,
// c); ktab [S][n] float4 (logit scale kinv log2(e) / sqrt(d), kd, kinv, 0).
__global__ void __launch_bounds__(256)
    k_bwd_prep_slot(const int32_t* __restrict__ perm, const float* __restrict__ lse,
                    const float* __restrict__ dlse, const float2* __restrict__ pos_tab,
                    const float* __restrict__ pinv, float4* __restrict__ qtab,
                    float4* __restrict__ ktab, int n, int rounds, float inv_sqrt_d,
                    int64_t total) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t seg = e / n;
    const int64_t bh = seg / rounds;
    const int pos = perm[e];
    const int64_t at = seg * n + pos;
    const float l = lse[at];
    const float2 pt = pos_tab[bh * n + pos];
    const float w = expf(l - pt.x);
    const float c = (dlse ? dlse[at] : 0.f) - w * pt.y;
    const float kinv = pinv[bh * n + pos];
    qtab[e] = make_float4(__int_as_float(pos), l * kBwdLog2e, w, c);
    ktab[e] = make_float4(kinv * inv_sqrt_d * kBwdLog2e, kinv * inv_sqrt_d, kinv, 0.f);
  }
}

// ---------------------------------------------------------------------------
struct BwdArgs {
  const __nv_bfloat16* x;  // [BH][n][d] position order
  const __nv_bfloat16* v;
  const __nv_bfloat16* g;  // dL/dout [BH][n][d]
  const float4* qtab;      // [S][n] per slot (position, lse2, w, c)
  const float4* ktab;      // [S][n] per slot (ks, kd, kinv, 0)
  float* dq;               // k_bwd_dq: [S][n][d] query-role dx, slot order
  float* dxk;              // k_bwd_dkv: [S][n][d] key-role dx, slot order
  float* dv;               // k_bwd_dkv: [S][n][d] dv, slot order
  WsHeader* hdr;
  int n, rounds, pairs_per_seg;
  int oob;                 // a row index past x, v and g (BH * n): reads as zero
  int64_t units;           // BH * pairs_per_seg * rounds
};

constexpr int kNoPos = 0x7fffffff;

// All threads gather ROWS rows of a [BH * n][D] tensor (row rbase + pos(r);
// zeros for kNoPos) into a swizzled K-major tile [KH][ROWS][128 B]: chunk c
// of a row's 128-byte line goes to slot c ^ (row % 8), the layout the
// 128-byte-swizzle descriptors read. Each thread copies one 16-byte piece of
// every RSTEP-th row with cp.async, all positions read first.
template <int D, int ROWS, typename PosFn>
__device__ __forceinline__ void bwd_gather(unsigned char* tile, const __nv_bfloat16* src,
                                           int64_t rbase, PosFn pos) {
  constexpr int KH = D / 64, PPR = KH * 8;  // 16-byte pieces per row
  constexpr int RSTEP = kBwdWarps * 32 / PPR;
  constexpr int N = ROWS / RSTEP;
  static_assert(ROWS % RSTEP == 0, "rows split evenly over the threads");
  const int piece = threadIdx.x % PPR, kh = piece >> 3, c = piece & 7;
  const int r0 = threadIdx.x / PPR;
  int p[N];
#pragma unroll
  for (int k = 0; k < N; ++k) p[k] = pos(r0 + k * RSTEP);
  const unsigned char* s0 = reinterpret_cast<const unsigned char*>(src);
#pragma unroll
  for (int k = 0; k < N; ++k) {
    const int row = r0 + k * RSTEP;
    const bool valid = p[k] != kNoPos;
    sm100::cp_async16_zfill(tile + kh * ROWS * 128 + row * 128 + ((c ^ (row & 7)) << 4),
                            valid ? s0 + ((rbase + p[k]) * D + kh * 64 + c * 8) * 2 : s0, valid);
  }
}

// The gathers issued by this thread have landed; with a CTA barrier after
// it, every thread's have, for the tensor cores too.
__device__ __forceinline__ void bwd_gather_done() {
  sm100::cp_async_commit();
  sm100::cp_async_wait_all();
  sm100::fence_proxy_async_smem();
}

// (batch-head, segment, first chunk) of unit u (numbered (batch, head), pair, round)
__device__ __forceinline__ void bwd_unit(const BwdArgs& a, int64_t u, int64_t& bh, int64_t& seg,
                                         int& c0) {
  const int64_t per_bh = (int64_t)a.pairs_per_seg * a.rounds;
  bh = u / per_bh;
  const int rem = (int)(u - bh * per_bh);
  const int pair = rem / a.rounds;
  seg = bh * a.rounds + (rem - pair * a.rounds);
  c0 = 2 * pair;
}

template <int D>
inline size_t bwd_dq_smem() {
  constexpr size_t KH = D / 64;
  return 1024 + KH * 192 * 128 /* x window */ + KH * 192 * 128 /* v window */ +
         KH * 128 * 128 /* g queries */ + 192 * 16 /* key table */ + 128 * 16 /* query table */ +
         256;
}

// Query-stationary: dQ of the 128 queries of a chunk pair.
// TMEM: S [0, 192) (dS' bf16 over [0, 96)), dPraw [192, 384), dQ [384, 384 + d).
template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kBwdWarps * 32, 1)
    k_bwd_dq(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmv,
             const __grid_constant__ CUtensorMap tmg, BwdArgs a) {
  using namespace sm100;
  constexpr int KH = D / 64;
  constexpr uint32_t XBOX = 192 * 128, GBOX = 128 * 128;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* xt = base;                 // [KH][192][128 B] key window (queries: rows 64..191)
  unsigned char* vt = xt + KH * XBOX;       // [KH][192][128 B]
  unsigned char* gt = vt + KH * XBOX;       // [KH][128][128 B] g rows of the queries
  float4* kt = reinterpret_cast<float4*>(gt + KH * GBOX);  // [192] (ks, kd, kinv, pos bits)
  float4* qt = kt + 192;                                   // [128] (pos, lse2, w, c)
  uint64_t* bars = reinterpret_cast<uint64_t*>(qt + 128);
  uint64_t* bar_sp = bars;      // S and dP MMAs done
  uint64_t* bar_q = bars + 1;   // dQ MMA done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
  volatile int* bad = reinterpret_cast<volatile int*>(bars + 3);
  uint64_t* bar_ld = bars + 4;  // the unit's rows landed (tx)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    mbar_init(bar_sp, 1);
    mbar_init(bar_q, 1);
    mbar_init(bar_ld, 1);
    *bad = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tm_dp = tmem + 192, tm_dq = tmem + 384;

  // Table entry tid (< 192) of a unit, loaded a unit ahead: the loads read
  // a valid address and validity comes from the slot number.
  float4 pk = make_float4(0.f, 0.f, 0.f, 0.f), pq = pk;
  bool pvalid = false;
  auto fetch = [&](int64_t uu) {
    if (uu >= a.units || tid >= 192) return;
    int64_t bh_, seg_;
    int c0_;
    bwd_unit(a, uu, bh_, seg_, c0_);
    const int ks = (c0_ - 1) * kAttnM + tid;
    pvalid = ks >= 0 && ks < a.n;
    const int64_t at = seg_ * a.n + (pvalid ? ks : 0);
    pk = a.ktab[at];
    pq = a.qtab[at];
  };
  fetch(blockIdx.x);
  int it = 0;
  for (int64_t u = blockIdx.x; u < a.units; u += gridDim.x, ++it) {
    int64_t bh, seg;
    int c0;
    bwd_unit(a, u, bh, seg, c0);
    const int64_t so = seg * a.n;
    // ---- tables (key slots (c0 - 1) 64 + j; the queries are j >= 64) and rows
    if (tid < 192) {
      kt[tid] = pvalid ? make_float4(pk.x, pk.y, pk.z, pq.x)
                       : make_float4(0.f, 0.f, 0.f, __int_as_float(kNoPos));
      if (tid >= kAttnM)
        qt[tid - kAttnM] = pvalid ? pq : make_float4(__int_as_float(kNoPos), 0.f, 0.f, 0.f);
    }
    __syncthreads();
    {
      const int64_t rb = bh * a.n;
      auto kpos = [&](int r) { return __float_as_int(kt[r].w); };
      bwd_gather<D, 192>(xt, a.x, rb, kpos);
      bwd_gather<D, 192>(vt, a.v, rb, kpos);
      bwd_gather<D, 128>(gt, a.g, rb, [&](int r) { return __float_as_int(qt[r].x); });
      fetch(u + gridDim.x);  // the next unit's tables, while this one computes
      bwd_gather_done();
    }
    tc_fence_before();
    __syncthreads();
    // ---- S = Q K^T, dPraw = G_q V^T
    if (tid == 0) {
      tc_fence_after();
      const uint32_t xa = smem_u32(xt), va = smem_u32(vt), ga = smem_u32(gt);
      const uint32_t idesc = idesc_bf16_f32(128, 192);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int kh = kk >> 2, ks = kk & 3;
        mma_bf16_ss(tmem, desc_kmajor_sw128(xa + kh * XBOX + kAttnM * 128 + ks * 32),
                    desc_kmajor_sw128(xa + kh * XBOX + ks * 32), idesc, kk > 0 ? 1u : 0u);
      }
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const int kh = kk >> 2, ks = kk & 3;
        mma_bf16_ss(tm_dp, desc_kmajor_sw128(ga + kh * GBOX + ks * 32),
                    desc_kmajor_sw128(va + kh * XBOX + ks * 32), idesc, kk > 0 ? 1u : 0u);
      }
      mma_commit(bar_sp);
    }
    // ---- dS' = P (w dPraw + c) kd, over the S columns in bf16; warps w and
    // w + 4 share TMEM lane quadrant w and take alternate 32-column batches
    {
      if (!mbar_wait(bar_sp, it & 1)) *bad = 1;
      tc_fence_after();
      const int wq = warp & 3, half = warp >> 2;
      const int row = wq * 32 + lane;
      const uint32_t tl = (uint32_t)(wq * 32) << 16;
      const float4 me = qt[row];
      const int qpos = __float_as_int(me.x);
      const float lse2 = me.y, w = me.z, c = me.w;
      const int wlo = wq < 2 ? 0 : kAttnM;  // the row's window: keys [wlo, wlo + 128)
#pragma unroll 1
      for (int b = half; b < 6; b += 2) {
        if (b * 32 < wlo || b * 32 >= wlo + 128) {  // keys outside the row's window: dS' = 0
          uint32_t z[16];
#pragma unroll
          for (int c = 0; c < 16; ++c) z[c] = 0u;
          tmem_st16(tmem + tl + b * 16, z);
          continue;
        }
        uint32_t sv[32], dv_[32];
        tmem_ld32(tmem + tl + b * 32, sv);
        tmem_ld32(tm_dp + tl + b * 32, dv_);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int cc = 0; cc < 32; cc += 2) {
          float o2[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const float4 k = kt[b * 32 + cc + h];
            const int kp = __float_as_int(k.w);
            const bool in_window = kp != kNoPos;  // the batch lies in the row's window
            const bool live = in_window && kp != qpos && (!CAUSAL || kp < qpos);
            const float p = ex2_approx(fmaf(__uint_as_float(sv[cc + h]), k.x, -lse2));
            const float ds = p * fmaf(w, __uint_as_float(dv_[cc + h]), c) * k.y;
            o2[h] = live ? ds : 0.f;
          }
          pk[cc >> 1] = pack_bf16x2(o2[0], o2[1]);
        }
        tmem_st16(tmem + tl + b * 16, pk);
      }
      tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();
    // ---- dQ = dS' X_window (A from TMEM, B = x window MN-major)
    if (tid == 0) {
      tc_fence_after();
      const uint32_t xa = smem_u32(xt);
      const uint32_t idesc = idesc_bf16_f32(128, D) | (1u << 16);
#pragma unroll
      for (int kk = 0; kk < 192 / 16; ++kk)
        mma_bf16_ts(tm_dq, tmem + kk * 8, desc_mnmajor_sw128(xa + kk * 16 * 128, XBOX), idesc,
                    kk > 0 ? 1u : 0u);
      mma_commit(bar_q);
    }
    {  // dQ rows out: warps w and w + 4 each write one half of the columns,
       // staged per warp in shared memory (the v and g tiles are free) and
       // written as contiguous row runs
      if (!mbar_wait(bar_q, it & 1)) *bad = 1;
      tc_fence_after();
      const int wq = warp & 3, half = warp >> 2;
      const uint32_t tl = (uint32_t)(wq * 32) << 16;
      constexpr int CW = D / 2;     // columns of a half
      constexpr int RS = CW + 4;    // staged row stride in floats (conflict-free)
      constexpr int LPR = CW / 4;   // lanes per row when writing out
      constexpr int RPI = 32 / LPR; // rows per write instruction
      float* stg = reinterpret_cast<float*>(vt) + warp * 32 * RS;
#pragma unroll
      for (int bb = 0; bb < CW / 32; ++bb) {
        uint32_t o[32];
        tmem_ld32(tm_dq + tl + (half * (CW / 32) + bb) * 32, o);
        tmem_wait_ld();
        float4* d4 = reinterpret_cast<float4*>(stg + lane * RS + bb * 32);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          d4[k] = make_float4(__uint_as_float(o[4 * k]), __uint_as_float(o[4 * k + 1]),
                              __uint_as_float(o[4 * k + 2]), __uint_as_float(o[4 * k + 3]));
      }
      __syncwarp();
#pragma unroll 4
      for (int r0 = 0; r0 < 32; r0 += RPI) {
        const int rr = r0 + lane / LPR, c4 = lane % LPR;
        const int qs = c0 * kAttnM + wq * 32 + rr;
        if (qs < a.n)
          *reinterpret_cast<float4*>(a.dq + (so + qs) * D + half * CW + c4 * 4) =
              *reinterpret_cast<const float4*>(stg + rr * RS + c4 * 4);
      }
    }
    tc_fence_before();
    __syncthreads();  // TMEM and the tiles are reused by the next unit
    if (*bad) break;  // uniform: read after the barrier
  }
  if (tid == 0 && *bad) record_status(a.hdr, 5u /* LSH_ERR_TIMEOUT */);
  __syncthreads();
  if (warp == 0 && !*bad) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D>
inline size_t bwd_dkv_smem() {
  constexpr size_t KH = D / 64;
  return 1024 + KH * 192 * 128 /* x rows of the queries (keys: rows 0..127) */ +
         KH * 128 * 128 /* v rows of the keys */ + KH * 192 * 128 /* g rows of the queries */ +
         128 * 16 /* key table */ + 192 * 16 /* query table */ + 256;
}

// Key-stationary: dv and the key-role dx of the 128 keys of a chunk pair.
// Keys: slots [64 c0, 64 c0 + 128); queries: slots [64 c0, 64 c0 + 192).
// TMEM: S^T [0, 128) (P w bf16 over [0, 64)), dPraw^T [128, 256) (dS' bf16
// over [128, 192)), dV [256, 256 + d), G [384, 384 + d).
template <int D, bool CAUSAL>
__global__ void __launch_bounds__(kBwdWarps * 32, 1)
    k_bwd_dkv(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmv,
              const __grid_constant__ CUtensorMap tmg, BwdArgs a) {
  using namespace sm100;
  constexpr int KH = D / 64;
  constexpr uint32_t XBOX = 192 * 128, VBOX = 128 * 128;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* xt = base;                 // [KH][192][128 B] x of the queries
  unsigned char* vt = xt + KH * XBOX;       // [KH][128][128 B] v of the keys
  unsigned char* gt = vt + KH * VBOX;       // [KH][192][128 B] g of the queries
  float4* kt = reinterpret_cast<float4*>(gt + KH * XBOX);  // [128] (ks, kd, kinv, pos bits)
  float4* qt = kt + 128;                                   // [192] (pos, lse2, w, c)
  uint64_t* bars = reinterpret_cast<uint64_t*>(qt + 192);
  uint64_t* bar_sp = bars;     // S^T and dP^T MMAs of a pass done
  uint64_t* bar_acc = bars + 1;  // dV and G MMAs of a pass done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
  volatile int* bad = reinterpret_cast<volatile int*>(bars + 3);
  uint64_t* bar_ld = bars + 4;  // the unit's rows landed (tx)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    mbar_init(bar_sp, 1);
    mbar_init(bar_acc, 1);
    mbar_init(bar_ld, 1);
    *bad = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tm_dp = tmem + 128, tm_dv = tmem + 256, tm_g = tmem + 384;

  // Table entry tid (< 192) of a unit, loaded a unit ahead: the loads read
  // a valid address and validity comes from the slot number.
  float4 pk = make_float4(0.f, 0.f, 0.f, 0.f), pq = pk;
  bool pvalid = false;
  auto fetch = [&](int64_t uu) {
    if (uu >= a.units || tid >= 192) return;
    int64_t bh_, seg_;
    int c0_;
    bwd_unit(a, uu, bh_, seg_, c0_);
    const int s = c0_ * kAttnM + tid;
    pvalid = s < a.n;
    const int64_t at = seg_ * a.n + (pvalid ? s : 0);
    pq = a.qtab[at];
    pk = a.ktab[at];
  };
  fetch(blockIdx.x);
  int phase = 0;  // completions of bar_sp and bar_acc so far (twice per unit)
  for (int64_t u = blockIdx.x; u < a.units; u += gridDim.x) {
    int64_t bh, seg;
    int c0;
    bwd_unit(a, u, bh, seg, c0);
    const int s0 = c0 * kAttnM;  // first key slot and first query slot
    const int64_t so = seg * a.n;
    if (tid < 192) {  // queries s0 + j; the keys are j < 128
      const float4 q = pvalid ? pq : make_float4(__int_as_float(kNoPos), 0.f, 0.f, 0.f);
      qt[tid] = q;
      if (tid < 128)
        kt[tid] = pvalid ? make_float4(pk.x, pk.y, pk.z, q.x) : make_float4(0.f, 0.f, 0.f, q.x);
    }
    __syncthreads();
    {
      const int64_t rb = bh * a.n;
      auto qpos = [&](int r) { return __float_as_int(qt[r].x); };
      bwd_gather<D, 192>(xt, a.x, rb, qpos);
      bwd_gather<D, 128>(vt, a.v, rb, [&](int r) { return __float_as_int(kt[r].w); });
      bwd_gather<D, 192>(gt, a.g, rb, qpos);
      fetch(u + gridDim.x);  // the next unit's tables, while this one computes
      bwd_gather_done();
    }
    tc_fence_before();
    __syncthreads();
    // Pass 0 takes the middle query chunk (64 queries), which both key chunks
    // see; pass 1 the first and the last (128 queries), each of which one key
    // chunk sees: every warp then computes one 32-query batch per pass and
    // writes zeros for the other. Column c of a pass is query row qrow(c).
    for (int pass = 0; pass < 2; ++pass, ++phase) {
      const int N = pass == 0 ? 64 : 128;
      auto qrow = [&](int c) { return pass == 0 ? kAttnM + c : (c < kAttnM ? c : kAttnM + c); };
      // ---- S^T = K Q^T, dPraw^T = V_k G_q^T, 64 query columns per MMA
      if (tid == 0) {
        tc_fence_after();
        const uint32_t xa = smem_u32(xt), va = smem_u32(vt), ga = smem_u32(gt);
        const uint32_t idesc = idesc_bf16_f32(128, kAttnM);
        for (int part = 0; part < N / kAttnM; ++part) {
          const int r0 = qrow(part * kAttnM);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int kh = kk >> 2, ks = kk & 3;
            mma_bf16_ss(tmem + part * kAttnM, desc_kmajor_sw128(xa + kh * XBOX + ks * 32),
                        desc_kmajor_sw128(xa + kh * XBOX + r0 * 128 + ks * 32), idesc,
                        kk > 0 ? 1u : 0u);
          }
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int kh = kk >> 2, ks = kk & 3;
            mma_bf16_ss(tm_dp + part * kAttnM, desc_kmajor_sw128(va + kh * VBOX + ks * 32),
                        desc_kmajor_sw128(ga + kh * XBOX + r0 * 128 + ks * 32), idesc,
                        kk > 0 ? 1u : 0u);
          }
        }
        mma_commit(bar_sp);
      }
      // ---- P w and dS' for key row j (thread), the pass's queries; warps w
      // and w + 4 share lane quadrant w and take alternate 32-query batches
      {
        if (!mbar_wait(bar_sp, phase & 1)) *bad = 1;
        tc_fence_after();
        const int wq = warp & 3, half = warp >> 2;
        const int j = wq * 32 + lane;
        const uint32_t tl = (uint32_t)(wq * 32) << 16;
        const float4 k = kt[j];
        const int kp = __float_as_int(k.w);
        const int kc = j / kAttnM;  // key chunk within the unit (0 or 1)
#pragma unroll 1
        for (int b = half; b < N / 32; b += 2) {
          const int qcb = qrow(b * 32) / kAttnM;  // the batch's query chunk (0, 1 or 2)
          if (kc != qcb && kc != qcb - 1) {       // the key's chunk is outside its window
            uint32_t z[16];
#pragma unroll
            for (int c = 0; c < 16; ++c) z[c] = 0u;
            tmem_st16(tmem + tl + b * 16, z);
            tmem_st16(tm_dp + tl + b * 16, z);
            continue;
          }
          uint32_t sv[32], dv_[32];
          tmem_ld32(tmem + tl + b * 32, sv);
          tmem_ld32(tm_dp + tl + b * 32, dv_);
          tmem_wait_ld();
          uint32_t pw[16], pd[16];
          const float4* qb = qt + qrow(b * 32);  // the batch's 32 queries, one chunk
          const bool kvalid = kp != kNoPos;
#pragma unroll
          for (int cc = 0; cc < 32; cc += 2) {
            float ow[2], od[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const float4 q = qb[cc + h];
              const int qp = __float_as_int(q.x);
              // the batch's chunk sees this key's chunk (tested above)
              const bool window = kvalid && qp != kNoPos;
              const bool self = window && kp == qp;
              const bool live = window && kp != qp && (!CAUSAL || kp < qp);
              // the self logit is -1e5: weight 1 for a row that sees only
              // itself (its lse is -1e5), 0 otherwise; no gradient through it
              const float l2 = self ? kSelfLogit * kBwdLog2e : __uint_as_float(sv[cc + h]) * k.x;
              const float p = ex2_approx(l2 - q.y);
              const float pv = (live || self) ? p : 0.f;
              ow[h] = pv * q.z;
              od[h] = live ? p * fmaf(q.z, __uint_as_float(dv_[cc + h]), q.w) * k.y : 0.f;
            }
            pw[cc >> 1] = pack_bf16x2(ow[0], ow[1]);
            pd[cc >> 1] = pack_bf16x2(od[0], od[1]);
          }
          tmem_st16(tmem + tl + b * 16, pw);
          tmem_st16(tm_dp + tl + b * 16, pd);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      __syncthreads();
      // ---- dV += (P w) G_q, G += dS' X_q (A from TMEM; B MN-major, K = queries)
      if (tid == 0) {
        tc_fence_after();
        const uint32_t xa = smem_u32(xt), ga = smem_u32(gt);
        const uint32_t idesc = idesc_bf16_f32(128, D) | (1u << 16);
        for (int kk = 0; kk < N / 16; ++kk) {
          const uint32_t acc = (pass > 0 || kk > 0) ? 1u : 0u;
          const int r = qrow(kk * 16);  // 16 queries of one chunk
          mma_bf16_ts(tm_dv, tmem + kk * 8, desc_mnmajor_sw128(ga + r * 128, XBOX), idesc, acc);
          mma_bf16_ts(tm_g, tm_dp + kk * 8, desc_mnmajor_sw128(xa + r * 128, XBOX), idesc, acc);
        }
        mma_commit(bar_acc);
      }
      if (!mbar_wait(bar_acc, phase & 1)) *bad = 1;
      tc_fence_after();
      tc_fence_before();
      __syncthreads();  // S^T / dP^T columns are rewritten by the next pass
    }
    // ---- key rows out: dv, and dx_key = G - x kinv^2 (x . G); warps w and
    // w + 4 both form x . G for lane quadrant w and each write one half of the
    // columns. A warp stages its 32 rows of a half in shared memory (the v and
    // g tiles are free now) and writes them row by row, so the global stores
    // are whole contiguous runs.
    {
      tc_fence_after();
      const int wq = warp & 3, half = warp >> 2;
      const int j = wq * 32 + lane;
      const uint32_t tl = (uint32_t)(wq * 32) << 16;
      const float4 k = kt[j];
      // the key's own x row is row j of the query tile (keys are its first
      // 128 rows): 16-byte chunk c of each 64-column half at slot c ^ (j % 8)
      auto xrow8 = [&](int e8, float (&f)[8]) {  // elements 8 e8 .. 8 e8 + 7
        const unsigned char* line = xt + (e8 >> 3) * XBOX + j * 128;
        Vec16<__nv_bfloat16>::unpack(
            *reinterpret_cast<const uint4*>(line + (((e8 & 7) ^ (j & 7)) << 4)), f);
      };
      float xg = 0.f;
#pragma unroll
      for (int b = 0; b < D / 32; ++b) {
        uint32_t gv[32];
        tmem_ld32(tm_g + tl + b * 32, gv);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float f[8];
          xrow8(b * 4 + q, f);
#pragma unroll
          for (int e = 0; e < 8; ++e) xg = fmaf(f[e], __uint_as_float(gv[8 * q + e]), xg);
        }
      }
      const float fk = k.z * k.z * xg;
      constexpr int CW = D / 2;     // columns of a half
      constexpr int RS = CW + 4;    // staged row stride in floats (conflict-free)
      constexpr int LPR = CW / 4;   // lanes per row when writing out
      constexpr int RPI = 32 / LPR; // rows per write instruction
      float* stg = reinterpret_cast<float*>(vt) + warp * 32 * RS;
      // which = 0: dx_key, 1: dv
      for (int which = 0; which < 2; ++which) {
#pragma unroll
        for (int bb = 0; bb < CW / 32; ++bb) {
          const int b = half * (CW / 32) + bb;
          uint32_t tv[32];
          tmem_ld32((which == 0 ? tm_g : tm_dv) + tl + b * 32, tv);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float o[8];
            if (which == 0) {
              float f[8];
              xrow8(b * 4 + q, f);
#pragma unroll
              for (int e = 0; e < 8; ++e) o[e] = __uint_as_float(tv[8 * q + e]) - f[e] * fk;
            } else {
#pragma unroll
              for (int e = 0; e < 8; ++e) o[e] = __uint_as_float(tv[8 * q + e]);
            }
            float4* dst = reinterpret_cast<float4*>(stg + lane * RS + bb * 32 + 8 * q);
            dst[0] = make_float4(o[0], o[1], o[2], o[3]);
            dst[1] = make_float4(o[4], o[5], o[6], o[7]);
          }
        }
        __syncwarp();
        float* gdst = (which == 0 ? a.dxk : a.dv) + half * CW;
#pragma unroll 4
        for (int r0 = 0; r0 < 32; r0 += RPI) {
          const int rr = r0 + lane / LPR, c4 = lane % LPR;
          const int sj = s0 + wq * 32 + rr;
          if (sj < a.n)
            *reinterpret_cast<float4*>(gdst + (so + sj) * D + c4 * 4) =
                *reinterpret_cast<const float4*>(stg + rr * RS + c4 * 4);
        }
        __syncwarp();  // the staging rows are rewritten by the next array
      }
    }
    tc_fence_before();
    __syncthreads();
    if (*bad) break;
  }
  if (tid == 0 && *bad) record_status(a.hdr, 5u /* LSH_ERR_TIMEOUT */);
  __syncthreads();
  if (warp == 0 && !*bad) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------
// grid-stride over (bh, position), a warp per position, lane j owning the
// d / 32 consecutive elements from (d / 32) j: sums the query and key roles of
// every round through inv, in round order. The slots of every round are
// loaded first (one lane per round), then the rows of up to four rounds at a
// time, all in flight together.
template <typename T, int D>
__global__ void __launch_bounds__(256)
    k_bwd_unsort(const int32_t* __restrict__ inv, const float* __restrict__ dq,
                 const float* __restrict__ dxk, const float* __restrict__ dvs,
                 T* __restrict__ dx, T* __restrict__ dv, int n, int rounds, int64_t total) {
  constexpr int EPL = D / 32;  // elements per lane: 2 or 4
  using V = typename std::conditional<EPL == 4, float4, float2>::type;
  constexpr int RB = 4;        // rounds in flight
  const int lane = threadIdx.x & 31;
  auto vget = [](const V& a, int e) {
    if constexpr (EPL == 4) return e == 0 ? a.x : e == 1 ? a.y : e == 2 ? a.z : a.w;
    else return e == 0 ? a.x : a.y;
  };
  for (int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < total;
       r += ((int64_t)gridDim.x * blockDim.x) >> 5) {
    const int64_t bh = r / n;
    const int i = (int)(r - bh * n);
    const int my_slot = lane < rounds ? inv[(bh * rounds + lane) * n + i] : 0;
    float ax[EPL], av[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) ax[e] = av[e] = 0.f;
    for (int q0 = 0; q0 < rounds; q0 += RB) {
      V a[RB], b[RB], c[RB];
#pragma unroll
      for (int t = 0; t < RB; ++t) {
        const int q = q0 + t;
        const int slot = __shfl_sync(0xffffffffu, my_slot, q & 31);
        if (q < rounds) {
          const int64_t row = ((bh * rounds + q) * n + slot) * D + lane * EPL;
          a[t] = *reinterpret_cast<const V*>(dq + row);
          b[t] = *reinterpret_cast<const V*>(dxk + row);
          c[t] = *reinterpret_cast<const V*>(dvs + row);
        }
      }
#pragma unroll
      for (int t = 0; t < RB; ++t)
        if (q0 + t < rounds) {
#pragma unroll
          for (int e = 0; e < EPL; ++e) {
            ax[e] += vget(a[t], e) + vget(b[t], e);
            av[e] += vget(c[t], e);
          }
        }
    }
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      dx[r * D + lane * EPL + e] = Elem<T>::from_f(ax[e]);
      dv[r * D + lane * EPL + e] = Elem<T>::from_f(av[e]);
    }
  }
}

}  // namespace lsh
