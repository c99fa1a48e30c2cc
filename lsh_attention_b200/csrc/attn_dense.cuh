// Dense shared-QK attention on the 5th-generation tensor cores: every query
// against every key (causal: every key at an earlier position), under the
// same rules as the chunked LSH attention -- keys scaled to unit length,
// logits scaled by 1/sqrt(d), the -1e5 self logit, causal masking. It is the
// full-attention baseline the pages measure LSH attention against
// ("Reformer: LSH attention and reversible layers" (dtcms.com), §三.3, speed
// against full attention; §二.1 for the logit). With one round and one chunk
// covering the sequence, LSH attention computes exactly this.
//
// Work unit: a tile of 128 queries of one (batch, head). Its key tiles are
// 128 keys each: every tile, or (causal) the tiles up to the diagonal. Units
// are numbered heaviest first (the last query tiles have the most key tiles
// under the causal mask) and CTA c of G takes units c, c + G, ...
//
// One persistent CTA per SM, 10 warps:
//   warp 0      TMA: the unit's query tile (two buffers, so the next unit's
//               loads overlap this unit), then per key tile the K tile (rows of
//               x: queries and keys are the same vectors) with its 128 key
//               scales (bulk copy into a 4-deep ring) and the V tile, in an
//               NST-deep ring.
//   warp 1      tcgen05.mma: S(t+1) = Q K(t+1)^T into TMEM S[(t+1) & 1] ahead
//               of O += P(t) V(t) with P read from TMEM; O accumulates over the
//               unit's key tiles in TMEM.
//   warps 2-5   softmax, one query row per thread. Keys have unit length, so
//               ||q|| log2(e) / sqrt(d) bounds every logit of the row: with it
//               as the stabiliser every probability is exp2(l - bound) <= 1
//               and the pass needs no rescaling of O. Masks: keys past n,
//               (causal) keys at later positions, and the diagonal element
//               (the -1e5 self logit, whose weight is exp(-1e5) = 0 unless the
//               row sees nothing else). A row whose bound is too large for
//               that (kAttnBoundMax) is queued and recomputed exactly by
//               k_dense_fixup.
//   warps 6-9   epilogue: O from TMEM, divided by the row sum, packed to bf16,
//               staged in swizzled shared memory and written by TMA stores
//               in position order; a row that sees only itself outputs its own
//               v row.
// TMEM: S[0] = [0, 128), S[1] = [128, 256), O = [256, 256 + d).
#pragma once

#include "attn_tc.cuh"
#include "common.cuh"
#include "sm100.cuh"

namespace lsh {

constexpr int kDenseTile = 128;  // queries per unit, keys per tile
constexpr int kDenseWarps = 10;
constexpr int kDenseRing = 4;    // key-scale ring depth

struct DenseArgs {
  const float* kscale;     // [BH][kstride] log2(e) / (sqrt(d) ||x||) by position, 0 past n
  const __nv_bfloat16* v;  // [BH][n][d] (rows that see only themselves copy theirs)
  float* lse;              // [BH][n]
  int32_t* fix_queue;      // [BH * n] rows (bh * n + position) for k_dense_fixup
  WsHeader* hdr;           // queue length in hdr->pad[32]
  int n, BH, qtiles, kstride;
  int64_t units;           // BH * qtiles
};

constexpr int kDenseFixSlot = 32;  // hdr->pad index of the fixup queue's length

template <int D, int NST>
inline size_t dense_smem() {
  constexpr size_t tile = (size_t)(D / 64) * kDenseTile * 128;
  return 1024 + (2 + 2 * NST) * tile + 4 * 32 * 128 + kDenseRing * kDenseTile * 4 +
         4 * kDenseTile * 4 + 512;
}

template <int D, bool CAUSAL, int NST>
__global__ void __launch_bounds__(kDenseWarps * 32, 1)
    k_attn_dense(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmv,
                 const __grid_constant__ CUtensorMap tmo, DenseArgs a) {
  using namespace sm100;
  constexpr int KH = D / 64;
  constexpr uint32_t BOX = kDenseTile * 128;  // one 64-column box of a 128-row tile
  constexpr uint32_t TILE = KH * BOX;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* qs_ = base;                         // [2][KH][128][128 B]
  unsigned char* ks_ = base + 2 * TILE;              // [NST][KH][128][128 B]
  unsigned char* vs_ = ks_ + NST * TILE;             // [NST][KH][128][128 B]
  unsigned char* ostage = vs_ + NST * TILE;          // [4 warps][32][128 B]
  float* kscl = reinterpret_cast<float*>(ostage + 4 * 32 * 128);  // [ring][128]
  float* rstat = kscl + kDenseRing * kDenseTile;                   // [4][128] 1/sum
  uint64_t* bars = reinterpret_cast<uint64_t*>(rstat + 4 * kDenseTile);
  uint64_t* qfull = bars;               // [2] query tile landed
  uint64_t* qfree = bars + 2;           // [2] last S MMA of the unit done
  uint64_t* kfull = bars + 4;           // [NST] K tile + key scales landed
  uint64_t* kfree = kfull + NST;        // [NST] S MMA done with the K tile
  uint64_t* vfull = kfree + NST;        // [NST]
  uint64_t* vfree = vfull + NST;        // [NST] PV MMA done with the V tile
  uint64_t* sfull = vfree + NST;        // [2] S MMA done
  uint64_t* pready = sfull + 2;         // [2] P written (4 softmax warps)
  uint64_t* sfree = pready + 2;         // [2] PV MMA done with P
  uint64_t* ofull = sfree + 2;          // the unit's last PV MMA done
  uint64_t* ofree = ofull + 1;          // 4 epilogue warps done reading O
  uint64_t* statf = ofree + 1;          // [4] row sums written (4 softmax warps)
  uint64_t* mfull = statf + 4;          // [ring] key scales landed
  uint64_t* mfree = mfull + kDenseRing; // [ring] key-scale slot read (4 softmax warps)
  uint64_t* drain = mfree + kDenseRing;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(drain + 2);
  volatile int* drain_fail = reinterpret_cast<volatile int*>(drain + 3);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if ((int64_t)blockIdx.x >= a.units) return;  // uniform across the CTA
  const int nu = (int)((a.units - 1 - blockIdx.x) / gridDim.x) + 1;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(qfull + i, 1);
      mbar_init(qfree + i, 1);
      mbar_init(sfull + i, 1);
      mbar_init(pready + i, 4);
      mbar_init(sfree + i, 1);
    }
    for (int i = 0; i < NST; ++i) {
      mbar_init(kfull + i, 1);
      mbar_init(kfree + i, 1);
      mbar_init(vfull + i, 1);
      mbar_init(vfree + i, 1);
    }
    mbar_init(ofull, 1);
    mbar_init(ofree, 4);
    for (int i = 0; i < 4; ++i) mbar_init(statf + i, 4);
    for (int i = 0; i < kDenseRing; ++i) {
      mbar_init(mfull + i, 1);
      mbar_init(mfree + i, 4);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    *drain_fail = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tm_o = tmem + 256;

  auto fail = [&]() {
    record_status(a.hdr, 5u /* LSH_ERR_TIMEOUT */);
    *abort_flag = 1;
  };
  // (batch-head, query tile, key tiles) of this CTA's unit i
  auto unit_of = [&](int i, int& bh, int& qt, int& nt) {
    const int64_t u = (int64_t)blockIdx.x + (int64_t)i * gridDim.x;
    qt = a.qtiles - 1 - (int)(u / a.BH);
    bh = (int)(u % a.BH);
    nt = CAUSAL ? qt + 1 : a.qtiles;
  };

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&tmx);
      prefetch_tensormap(&tmv);
      bool ok = true;
      int lastq[2] = {-1, -1}, lastk[NST], lastv[NST], lastm[kDenseRing];
      for (int j = 0; j < NST; ++j) lastk[j] = lastv[j] = -1;
      for (int j = 0; j < kDenseRing; ++j) lastm[j] = -1;
      int g = 0;
      for (int i = 0; ok && i < nu && !*abort_flag; ++i) {
        int bh, qt, nt;
        unit_of(i, bh, qt, nt);
        const int qb = i & 1, kq = i >> 1;
        if (kq > 0 && !mbar_wait(qfree + qb, (kq - 1) & 1)) { ok = false; break; }
        mbar_expect_tx(qfull + qb, TILE);
        for (int kh = 0; kh < KH; ++kh)
          tma_load_3d(qs_ + qb * TILE + kh * BOX, &tmx, qfull + qb, kh * 64, qt * kDenseTile, bh);
        lastq[qb] = kq;
        for (int t = 0; t < nt; ++t, ++g) {
          const int s = g % NST, k = g / NST, m = g % kDenseRing, km = g / kDenseRing;
          if (k > 0 && !mbar_wait(kfree + s, (k - 1) & 1)) { ok = false; break; }
          if (km > 0 && !mbar_wait(mfree + m, (km - 1) & 1)) { ok = false; break; }
          mbar_expect_tx(kfull + s, TILE);
          for (int kh = 0; kh < KH; ++kh)
            tma_load_3d(ks_ + s * TILE + kh * BOX, &tmx, kfull + s, kh * 64, t * kDenseTile, bh);
          lastk[s] = k;
          mbar_expect_tx(mfull + m, kDenseTile * 4);
          bulk_copy_g2s(kscl + m * kDenseTile, a.kscale + (int64_t)bh * a.kstride + t * kDenseTile,
                        kDenseTile * 4, mfull + m);
          lastm[m] = km;
          if (k > 0 && !mbar_wait(vfree + s, (k - 1) & 1)) { ok = false; break; }
          mbar_expect_tx(vfull + s, TILE);
          for (int kh = 0; kh < KH; ++kh)
            tma_load_3d(vs_ + s * TILE + kh * BOX, &tmv, vfull + s, kh * 64, t * kDenseTile, bh);
          lastv[s] = k;
        }
      }
      if (!ok) fail();
      // no copy may still be writing this CTA's shared memory when it exits
      for (int j = 0; j < 2; ++j)
        if (lastq[j] >= 0 && !mbar_wait(qfull + j, lastq[j] & 1)) *drain_fail = 1;
      for (int j = 0; j < NST; ++j)
        if ((lastk[j] >= 0 && !mbar_wait(kfull + j, lastk[j] & 1)) ||
            (lastv[j] >= 0 && !mbar_wait(vfull + j, lastv[j] & 1)))
          *drain_fail = 1;
      for (int j = 0; j < kDenseRing; ++j)
        if (lastm[j] >= 0 && !mbar_wait(mfull + j, lastm[j] & 1)) *drain_fail = 1;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(128, kDenseTile);
      const uint32_t idesc_o = idesc_bf16_f32(128, D) | (1u << 16);  // B = V, MN-major
      // (unit, tile) of the flattened tile index, walked forward by both streams
      struct Cursor {
        int i = 0, t = 0, g = 0, nt = 0;
      };
      Cursor cs, cp;  // next S to issue, next PV to issue
      auto load_nt = [&](Cursor& c) {
        int bh, qt;
        if (c.i < nu) unit_of(c.i, bh, qt, c.nt);
      };
      auto advance = [&](Cursor& c) {
        ++c.g;
        if (++c.t == c.nt) {
          c.t = 0;
          ++c.i;
          load_nt(c);
        }
      };
      auto issue_s = [&](const Cursor& c) {
        const int s = c.g % NST, k = c.g / NST, sb = c.g & 1, kb = c.g >> 1;
        const int qb = c.i & 1;
        if (!mbar_wait(qfull + qb, (c.i >> 1) & 1)) return false;
        if (!mbar_wait(kfull + s, k & 1)) return false;
        if (kb > 0 && !mbar_wait(sfree + sb, (kb - 1) & 1)) return false;
        tc_fence_after();
        const uint32_t qa = smem_u32(qs_ + qb * TILE);
        const uint32_t ka = smem_u32(ks_ + s * TILE);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const int kh = kk >> 2, ks = kk & 3;
          mma_bf16_ss(tmem + sb * kDenseTile, desc_kmajor_sw128(qa + kh * BOX + ks * 32),
                      desc_kmajor_sw128(ka + kh * BOX + ks * 32), idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(sfull + sb);
        mma_commit(kfree + s);
        if (c.t == c.nt - 1) mma_commit(qfree + qb);
        return true;
      };
      auto issue_pv = [&](const Cursor& c) {
        const int s = c.g % NST, k = c.g / NST, sb = c.g & 1, kb = c.g >> 1;
        if (!mbar_wait(pready + sb, kb & 1)) return false;
        if (!mbar_wait(vfull + s, k & 1)) return false;
        if (c.t == 0 && c.i > 0 && !mbar_wait(ofree, (c.i - 1) & 1)) return false;
        tc_fence_after();
        const uint32_t va = smem_u32(vs_ + s * TILE);
#pragma unroll
        for (int kk = 0; kk < kDenseTile / 16; ++kk) {
          const uint64_t bd = desc_mnmajor_sw128(va + kk * 16 * 128, BOX);
          mma_bf16_ts(tm_o, tmem + sb * kDenseTile + kk * 8, bd, idesc_o,
                      (c.t > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(vfree + s);
        mma_commit(sfree + sb);
        if (c.t == c.nt - 1) mma_commit(ofull);
        return true;
      };
      load_nt(cs);
      load_nt(cp);
      bool ok = issue_s(cs);
      advance(cs);
      while (ok && cp.i < nu && !*abort_flag) {
        ok = (cs.i >= nu || issue_s(cs)) && issue_pv(cp);
        if (cs.i < nu) advance(cs);
        advance(cp);
      }
      if (!ok) fail();
      mma_commit(drain);  // TMEM is freed below: every MMA issued must have completed
      if (!mbar_wait(drain, 0)) *drain_fail = 1;
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ softmax
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const uint32_t tl = (uint32_t)(q * 32) << 16;
    int g = 0;
    bool stop = false;
    for (int i = 0; i < nu && !stop; ++i) {
      int bh, qt, nt;
      unit_of(i, bh, qt, nt);
      const int qpos = qt * kDenseTile + row;
      const float qs = qpos < a.n ? a.kscale[(int64_t)bh * a.kstride + qpos] : 0.f;
      // ||q|| log2(e) / sqrt(d) from the row's own scale c / ||q|| (c = log2(e) / sqrt(d))
      const float c_scale = 1.4426950408889634f / sqrtf((float)D);
      const float bound = qs > 0.f ? c_scale * c_scale / qs : 0.f;
      float sum0 = 0.f, sum1 = 0.f;
      for (int t = 0; t < nt; ++t, ++g) {
        const int sb = g & 1, kb = g >> 1, m = g % kDenseRing, km = g / kDenseRing;
        const bool got = mbar_wait(sfull + sb, kb & 1) && mbar_wait(mfull + m, km & 1);
        if (!got) fail();
        tc_fence_after();
        if (bar_sync_any(1, 128, !got || *abort_flag)) {
          stop = true;
          break;
        }
        const float* ks = kscl + m * kDenseTile;
        const uint32_t ts = tmem + tl + sb * kDenseTile;
        const int lim = min(kDenseTile, a.n - t * kDenseTile);  // keys before n
        const bool diag = t == qt;
        const bool plain = !diag && lim == kDenseTile;  // every key of the tile visible
        constexpr int BPW = D == 64 ? 2 : 1;
#pragma unroll 1
        for (int b2 = 0; b2 < 4; b2 += BPW) {
          uint32_t v[BPW][32];
#pragma unroll
          for (int h = 0; h < BPW; ++h) tmem_ld32(ts + (b2 + h) * 32, v[h]);
          tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < BPW; ++h) {
            const int b = b2 + h;
            uint32_t pk[16];
            const float4* ks4 = reinterpret_cast<const float4*>(ks + b * 32);
            if (plain) {
#pragma unroll
              for (int c = 0; c < 32; c += 4) {
                const float4 sc = ks4[c >> 2];
                const float e0 = ex2_approx(fmaf(__uint_as_float(v[h][c]), sc.x, -bound));
                const float e1 = ex2_approx(fmaf(__uint_as_float(v[h][c + 1]), sc.y, -bound));
                const float e2 = ex2_approx(fmaf(__uint_as_float(v[h][c + 2]), sc.z, -bound));
                const float e3 = ex2_approx(fmaf(__uint_as_float(v[h][c + 3]), sc.w, -bound));
                sum0 += e0 + e2;
                sum1 += e1 + e3;
                pk[c >> 1] = pack_bf16x2(e0, e1);
                pk[(c >> 1) + 1] = pack_bf16x2(e2, e3);
              }
            } else {
#pragma unroll
              for (int c = 0; c < 32; c += 4) {
                const float4 sc = ks4[c >> 2];
                const float scv[4] = {sc.x, sc.y, sc.z, sc.w};
                float e[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                  const int kj = b * 32 + c + u;
                  const bool vis = kj < lim && (!diag || (CAUSAL ? kj < row : kj != row));
                  const float ex = ex2_approx(fmaf(__uint_as_float(v[h][c + u]), scv[u], -bound));
                  e[u] = vis ? ex : 0.f;
                }
                sum0 += e[0] + e[2];
                sum1 += e[1] + e[3];
                pk[c >> 1] = pack_bf16x2(e[0], e[1]);
                pk[(c >> 1) + 1] = pack_bf16x2(e[2], e[3]);
              }
            }
            tmem_st16(ts + b * 16, pk);  // P over S columns already read
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(pready + sb);
          mbar_arrive(mfree + m);
        }
      }
      if (stop) break;
      const float sum = sum0 + sum1;
      if (qpos < a.n) {
        a.lse[(int64_t)bh * a.n + qpos] =
            sum > 0.f ? (bound + log2f(sum)) * 0.6931471805599453f : kSelfLogit;
        if (bound > kAttnBoundMax) {  // recomputed exactly afterwards
          const uint32_t k = atomicAdd(&a.hdr->pad[kDenseFixSlot], 1u);
          a.fix_queue[k] = bh * a.n + qpos;
        }
      }
      rstat[(i & 3) * kDenseTile + row] = sum > 0.f ? 1.0f / sum : -1.f;
      __syncwarp();
      if (lane == 0) mbar_arrive(statf + (i & 3));
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const uint32_t tl = (uint32_t)(q * 32) << 16;
    for (int i = 0; i < nu; ++i) {
      if (!mbar_wait(ofull, i & 1) || !mbar_wait(statf + (i & 3), (i >> 2) & 1)) {
        fail();
        break;
      }
      tc_fence_after();
      int bh, qt, nt;
      unit_of(i, bh, qt, nt);
      const float inv = rstat[(i & 3) * kDenseTile + row];
      uint32_t pk[D / 2];
#pragma unroll
      for (int b = 0; b < D / 64; ++b) {
        uint32_t o[2][32];
        tmem_ld32(tm_o + tl + b * 64, o[0]);
        tmem_ld32(tm_o + tl + b * 64 + 32, o[1]);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int c = 0; c < 32; c += 2)
            pk[b * 32 + h * 16 + c / 2] =
                pack_bf16x2(__uint_as_float(o[h][c]) * inv, __uint_as_float(o[h][c + 1]) * inv);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(ofree);
      const int q0 = qt * kDenseTile + q * 32;  // first query position of this warp
      if (q0 < a.n) {
        const int qpos = q0 + lane;
        const uint4* vr = nullptr;
        if (inv <= 0.f && qpos < a.n)  // the row sees only itself: its own value row
          vr = reinterpret_cast<const uint4*>(a.v + ((int64_t)bh * a.n + qpos) * D);
        unsigned char* stg = ostage + (warp - 6) * 32 * 128;
#pragma unroll
        for (int b = 0; b < D / 64; ++b) {
          if (lane == 0) bulk_wait_read_all();  // the previous store has read the buffer
          __syncwarp();
          unsigned char* line = stg + lane * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 val = vr ? vr[b * 8 + c]
                                 : make_uint4(pk[b * 32 + 4 * c], pk[b * 32 + 4 * c + 1],
                                              pk[b * 32 + 4 * c + 2], pk[b * 32 + 4 * c + 3]);
            *reinterpret_cast<uint4*>(line + ((c ^ (lane & 7)) << 4)) = val;
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {  // rows past n are clipped by the tensor map
            tma_store_3d(&tmo, stg, b * 64, q0, bh);
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
    tmem_dealloc(tmem, 512);
  }
}

// Key scales log2(e) / (sqrt(d) ||x||) of every position of x [BH][n][D]
// (bf16) into [BH][kstride], zero for a zero row and past n: a group of D / 8
// lanes per position.
template <int D>
__global__ void __launch_bounds__(256)
    k_dense_kscale(const __nv_bfloat16* __restrict__ x, float* __restrict__ kscale, int n,
                   int kstride, int64_t total /* BH * kstride */) {
  constexpr int L = D / 8;
  const int gl = threadIdx.x % L;
  const float c = 1.4426950408889634f / sqrtf((float)D);
  const int64_t stride = (int64_t)gridDim.x * (blockDim.x / L);
  const int64_t warp_first = ((int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31)) / L;
  for (int64_t r0 = warp_first; r0 < total; r0 += stride) {
    const int64_t r = r0 + (threadIdx.x & 31) / L;
    const int64_t bh = r / kstride;
    const int p = (int)(r - bh * kstride);
    float ss = 0.f;
    if (r < total && p < n) {
      const uint4 u = *reinterpret_cast<const uint4*>(x + (bh * n + p) * D + gl * 8);
      float f[8];
      Vec16<__nv_bfloat16>::unpack(u, f);
#pragma unroll
      for (int e = 0; e < 8; ++e) ss = fmaf(f[e], f[e], ss);
    }
#pragma unroll
    for (int o = L / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if (r < total && gl == 0) kscale[r] = ss > 0.f ? c / sqrtf(ss) : 0.f;
  }
}

// Exact recomputation of queued rows (their stabiliser was too far above the
// logits for one pass): one warp per row, two passes over the visible keys in
// fp32 -- the row maximum, then the exponent sums and the weighted v rows.
template <int D, bool CAUSAL>
__global__ void __launch_bounds__(256)
    k_dense_fixup(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ v,
                  const float* __restrict__ kscale, __nv_bfloat16* __restrict__ out,
                  float* __restrict__ lse, const int32_t* __restrict__ queue,
                  const WsHeader* __restrict__ hdr, int n, int kstride) {
  constexpr int PER = D / 32;  // elements per lane
  const uint32_t count = hdr->pad[kDenseFixSlot];
  const int lane = threadIdx.x & 31;
  const int wg = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  for (uint32_t e = wg; e < count; e += nw) {
    const int row = queue[e];
    const int bh = row / n, i = row % n;
    const __nv_bfloat16* xb = x + (int64_t)bh * n * D;
    const __nv_bfloat16* vb = v + (int64_t)bh * n * D;
    const float* ks = kscale + (int64_t)bh * kstride;
    float qv[PER];
#pragma unroll
    for (int k = 0; k < PER; ++k) qv[k] = __bfloat162float(xb[(int64_t)i * D + lane + 32 * k]);
    const int jend = CAUSAL ? i : n;
    auto logit = [&](int j) {  // log2 units
      float dot = 0.f;
#pragma unroll
      for (int k = 0; k < PER; ++k) dot = fmaf(qv[k], __bfloat162float(xb[(int64_t)j * D + lane + 32 * k]), dot);
      return warp_sum(dot) * ks[j];
    };
    float mx = -INFINITY;
    for (int j = 0; j < jend; ++j)
      if (j != i) mx = fmaxf(mx, logit(j));
    float o[PER], z = 0.f;
#pragma unroll
    for (int k = 0; k < PER; ++k) o[k] = 0.f;
    if (mx == -INFINITY) {  // nothing but itself
#pragma unroll
      for (int k = 0; k < PER; ++k) o[k] = __bfloat162float(vb[(int64_t)i * D + lane + 32 * k]);
      z = 1.f;
    } else {
      for (int j = 0; j < jend; ++j) {
        if (j == i) continue;
        const float w = exp2f(logit(j) - mx);
        z += w;
#pragma unroll
        for (int k = 0; k < PER; ++k) o[k] = fmaf(w, __bfloat162float(vb[(int64_t)j * D + lane + 32 * k]), o[k]);
      }
    }
#pragma unroll
    for (int k = 0; k < PER; ++k)
      out[((int64_t)bh * n + i) * D + lane + 32 * k] = __float2bfloat16_rn(o[k] / z);
    if (lane == 0)
      lse[(int64_t)bh * n + i] = mx == -INFINITY ? kSelfLogit : (mx + log2f(z)) * 0.6931471805599453f;
  }
}

}  // namespace lsh
